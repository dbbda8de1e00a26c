"""Host-side checks of the Python binding that need no GPU: every entry
point refuses host tensors before reaching the library, so there is no
silent CPU path, and the pairing rules of optional arguments hold."""
import pytest
import torch

from sparse_attention_sigma_b200 import build as _build

_build.build()                      # the library loads without a GPU
from sparse_attention_sigma_b200 import had  # noqa: E402

x = torch.zeros(1, 1, 8, 64)
bits = torch.zeros(1, 1, 8, 2, dtype=torch.int32)
idx = torch.zeros(1, 1, 8, 2, dtype=torch.int32)
lg16 = torch.zeros(1, 1, 8, 2, dtype=torch.int16)
lg32 = torch.zeros(1, 1, 8, 2)
s = torch.ones(1)

CALLS = {
    "had_binarize_pack": lambda: had.had_binarize_pack(x, s),
    "had_hamming_topn": lambda: had.had_hamming_topn(bits, bits, 64, 2),
    "had_hamming_topn_causal": lambda: had.had_hamming_topn_causal(bits, bits, 64, 2),
    "had_sparse_softmax_av": lambda: had.had_sparse_softmax_av(idx, lg16, x, 0.1),
    "had_attention_fwd": lambda: had.had_attention_fwd(x, x, x, s, s, 2, 0.1),
    "had_attention_causal_fwd": lambda: had.had_attention_causal_fwd(x, x, x, s, s, 2, 0.1),
    "had_topn_mass": lambda: had.had_topn_mass(bits, bits, 64, 0.1, [0.9]),
    "had_soft_binarize": lambda: had.had_soft_binarize(x, s, 1.0),
    "had_soft_topn": lambda: had.had_soft_topn(x, x, 2),
    "had_soft_softmax_av": lambda: had.had_soft_softmax_av(idx, lg32, x, 0.1),
    "had_soft_attention_fwd": lambda: had.had_soft_attention_fwd(x, x, x, s, s, 1.0, 2, 0.1),
    "had_attention_bwd": lambda: had.had_attention_bwd(x, x, x, s, s, x, 2, 0.1),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_host_tensors_are_refused(name):
    with pytest.raises(ValueError, match="no CPU path"):
        CALLS[name]()


# entry points that take no tensors or that the tests above reach through
# another wrapper (prepare + core and the allocation-free call share the
# fused path's argument checks)
HELPERS = {"had_status_string", "had_workspace_bytes", "had_launch_count",
           "had_noalloc_scratch_bytes", "had_attention_prepare", "had_attention_core",
           "had_attention_fwd_noalloc", "had_set_wait_limit_ns",
           "had_attention_window_misses"}


def test_every_wrapper_is_covered():
    public = {n for n in dir(had) if n.startswith("had_") and callable(getattr(had, n))}
    assert public <= set(CALLS) | HELPERS, public - set(CALLS) - HELPERS
