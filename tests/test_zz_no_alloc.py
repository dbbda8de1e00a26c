"""The allocation-free entry point against the workspace entry point.

had_attention_fwd_noalloc serves callers that cannot call cudaMalloc (code
running under another runtime's allocator, plugins handed only their input
and output buffers, processes whose device memory is reserved up front): it
runs the same kernels as had_attention_fwd but in a fixed device array
inside the library.  The kernels are deterministic, so its output must equal
the workspace entry point's bit for bit, call after call; and after its first
call on a device its calls must not change the device's free memory.  This
file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3


def _close(got, ref):
    got = got.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS
    assert np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30) <= REL_L2


def _inputs(B, H, n, d, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, n, d, generator=g).to(dtype) for _ in range(3))
    return (q.cuda(), k.cuda(), v.cuda(), synth.per_head_sigma(q).cuda(),
            synth.per_head_sigma(k).cuda())


@pytest.mark.parametrize("B,H,n,d,N,dtype", [
    (2, 3, 700, 64, 90, torch.bfloat16),
    (1, 2, 260, 128, 33, torch.float32),
])
def test_noalloc_matches_workspace_entry_point_twice(B, H, n, d, N, dtype):
    from sparse_attention_sigma_b200 import had
    q, k, v, sq, sk = _inputs(B, H, n, d, 21, dtype)
    tau = 1 / math.sqrt(d)
    ref = had.had_attention_fwd(q, k, v, sq, sk, N, tau)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = [torch.full((B, H, n, d), float("nan"), device="cuda") for _ in range(3)]
    # the first call looks the array's address up; later calls allocate nothing
    had.had_attention_fwd_noalloc(q, k, v, sq, sk, N, tau, outs[0], dev_status=status)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for out in outs[1:]:
        had.had_attention_fwd_noalloc(q, k, v, sq, sk, N, tau, out, dev_status=status)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert status.item() == 0
    for out in outs:
        _close(out, ref)
        assert torch.equal(out, ref)


def test_noalloc_long_workload_fits_and_matches():
    from sparse_attention_sigma_b200 import had
    cfg = synth.CONFIGS["long"]
    need = had.had_workspace_bytes(had.HAD_OP_ATTENTION_FWD, cfg.B, cfg.H, cfg.n, cfg.d, cfg.N)
    assert 0 < need <= had.had_noalloc_scratch_bytes()
    q, k, v, sq, sk = (t.cuda() for t in synth.make_inputs(cfg))
    ref = had.had_attention_fwd(q, k, v, sq, sk, cfg.N, cfg.tau)
    for _ in range(2):
        out = torch.empty_like(ref)
        had.had_attention_fwd_noalloc(q, k, v, sq, sk, cfg.N, cfg.tau, out)
        torch.cuda.synchronize()
        _close(out, ref)
        assert torch.equal(out, ref)


def test_noalloc_rejects_sizes_beyond_its_array():
    from sparse_attention_sigma_b200 import had
    lib = had._lib
    fake = ctypes.c_void_p(4096)     # never dereferenced: the size check fails first
    st = lib.had_attention_fwd_noalloc(fake, fake, fake, had.HAD_BF16, fake, fake,
                                       1, 32, 16384, 128, 2048, ctypes.c_float(0.088),
                                       fake, None, None)
    assert st == had.HAD_ERR_WORKSPACE
