"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bit-exact for packed bits, kept indices and integer logits; fp32 outputs
within max |err| <= 2e-3 and ||err||_2 / ||ref||_2 <= 1e-3 (the tolerance
the forward pass is specified to, on bf16 inputs).  Small cases compare
every row; the five full-size workloads compare every packed bit and a
seeded sample of rows, in the launch configuration the benchmark times.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _golden

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3


@pytest.fixture(scope="module")
def had():
    from sparse_attention_sigma_b200 import had as _had
    return _had


def assert_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= REL_L2, f"{what}: rel L2 err {rel:.3e}"


class Case:
    """Inputs on the CPU and the GPU plus the oracle's signs."""

    def __init__(self, q, k, v, sgq, sgk, N, tau):
        self.q, self.k, self.v, self.sgq, self.sgk = q, k, v, sgq, sgk
        self.B, self.H, self.n, self.d = q.shape
        self.N, self.tau = N, tau
        self.sq = oracle.binarize(synth.to_oracle_array(q), sgq.numpy())
        self.sk = oracle.binarize(synth.to_oracle_array(k), sgk.numpy())
        self.v_or = synth.to_oracle_array(v)
        self.gq, self.gk, self.gv = q.cuda(), k.cuda(), v.cuda()
        self.gsq, self.gsk = sgq.cuda(), sgk.cuda()

    def oracle_rows(self, rows):
        return oracle.attention_rows(self.sq, self.sk, self.v_or, self.tau, self.N, rows)


_cases = {}


def config_case(name):
    if name not in _cases:
        cfg = synth.CONFIGS[name]
        q, k, v, sgq, sgk = synth.make_inputs(cfg)
        _cases[name] = Case(q, k, v, sgq, sgk, cfg.N, cfg.tau)
    return _cases[name]


def random_case(B, H, n, d, N, seed, dtype=torch.bfloat16, tau=None):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, n, d, generator=g).to(dtype)
    k = torch.randn(B, H, n, d, generator=g).to(dtype)
    v = torch.randn(B, H, n, d, generator=g).to(dtype)
    return Case(q, k, v, synth.per_head_sigma(q), synth.per_head_sigma(k), N,
                1 / math.sqrt(d) if tau is None else tau)


def all_rows(c):
    return np.arange(c.B * c.H * c.n)


SMALL = [
    # (B, H, n, d, N, seed, dtype): several 128-row tiles and ragged tails
    (1, 2, 128, 64, 16, 1, torch.float32),
    (2, 3, 300, 64, 40, 2, torch.bfloat16),
    (1, 2, 700, 64, 90, 3, torch.bfloat16),
    (1, 2, 260, 128, 33, 4, torch.bfloat16),
    (2, 1, 129, 128, 129, 5, torch.float32),        # N = n: dense softmax
    (1, 1, 1, 64, 1, 6, torch.bfloat16),            # a single row and key
    (1, 3, 97, 64, 1, 7, torch.bfloat16),           # N = 1
    # ragged last tiles in each way of finding the quota tile's kept ties:
    # from the key signs in shared memory (4 .. 32 key tiles at d 64, odd n
    # too), masked from S in pass 2 (fewer key tiles, or d 128 with more than
    # 16 KB of key signs and at most 12 tiles), gathered after pass 2 (d 128,
    # more key tiles)
    (1, 2, 2000, 64, 300, 8, torch.bfloat16),
    (1, 1, 1999, 64, 250, 9, torch.float32),
    (1, 1, 1100, 128, 150, 11, torch.bfloat16),
    (1, 1, 1700, 128, 200, 10, torch.bfloat16),
]


def _check_bits(had, c):
    gb = had.had_binarize_pack(c.gq, c.gsq).cpu().numpy().view(np.uint32)
    assert np.array_equal(gb, oracle.pack(c.sq))
    kb = had.had_binarize_pack(c.gk, c.gsk)
    assert np.array_equal(kb.cpu().numpy().view(np.uint32), oracle.pack(c.sk))
    return had.had_binarize_pack(c.gq, c.gsq), kb


def _check_unfused(had, c, rows):
    qb, kb = _check_bits(had, c)
    idx, lg = had.had_hamming_topn(qb, kb, c.d, c.N)
    out, p = had.had_sparse_softmax_av(idx, lg, c.gv, c.tau, want_p=True)
    torch.cuda.synchronize()
    o_idx, o_lg, o_p, o_out = c.oracle_rows(rows)
    flat = lambda t: t.reshape(-1, t.shape[-1]).cpu().numpy()[rows]
    assert np.array_equal(flat(idx), o_idx)
    assert np.array_equal(flat(lg), o_lg)
    assert_close(flat(p), o_p, "p")
    assert_close(flat(out), o_out, "out")


def _check_fused(had, c, rows):
    dbg_idx = torch.empty((c.B, c.H, c.n, c.N), dtype=torch.int32, device="cuda")
    dbg_lg = torch.empty((c.B, c.H, c.n, c.N), dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau,
                                dbg_idx=dbg_idx, dbg_logits=dbg_lg, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_idx, o_lg, o_p, o_out = c.oracle_rows(rows)
    sel = torch.as_tensor(np.asarray(rows), device="cuda")
    flat = lambda t: t.reshape(-1, t.shape[-1])[sel].cpu().numpy()
    assert np.array_equal(flat(dbg_idx), o_idx)
    assert np.array_equal(flat(dbg_lg), o_lg)
    assert_close(flat(out), o_out, "fused out (debug outputs on)")
    # the same through the split calls, whose core writes the kept set from
    # the 128-key kernel (had_attention_fwd takes the 64-key one for it)
    ws = had.workspace(c.B, c.H, c.n, c.d, c.N)
    had.had_attention_prepare(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, ws)
    dbg_idx.fill_(-7)
    dbg_lg.fill_(-7)
    out_s = had.had_attention_core(c.gv, c.N, c.tau, ws, dbg_idx=dbg_idx, dbg_logits=dbg_lg)
    torch.cuda.synchronize()
    assert np.array_equal(flat(dbg_idx), o_idx)
    assert np.array_equal(flat(dbg_lg), o_lg)
    assert_close(flat(out_s), o_out, "fused out (split calls, debug outputs on)")
    # Without the debug outputs every full key tile takes the table path and
    # the kept ties of a row's quota tile are added afterwards in fp32, so the
    # rounding differs from the key-by-key debug path: both must match the
    # oracle on their own.
    out2 = had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau)
    torch.cuda.synchronize()
    got = flat(out2)
    assert_close(got, o_out, "fused out")
    err = np.abs(got.astype(np.float64) - o_out)
    rel = np.linalg.norm(got.astype(np.float64) - o_out) / max(np.linalg.norm(o_out), 1e-30)
    return float(err.max()), float(rel)


@pytest.mark.parametrize("B,H,n,d,N,seed,dtype", SMALL)
def test_small_unfused_all_rows(had, B, H, n, d, N, seed, dtype):
    c = random_case(B, H, n, d, N, seed, dtype)
    _check_unfused(had, c, all_rows(c))


@pytest.mark.parametrize("B,H,n,d,N,seed,dtype", SMALL)
def test_small_fused_all_rows(had, B, H, n, d, N, seed, dtype):
    c = random_case(B, H, n, d, N, seed, dtype)
    _check_fused(had, c, all_rows(c))


@pytest.mark.parametrize("name", ["tiny", "bert", "vit", "long", "vlong"])
def test_workload_bits_full(had, name):
    _check_bits(had, config_case(name))


@pytest.mark.parametrize("name,count", [("tiny", 0), ("bert", 384), ("vit", 384),
                                        ("long", 256), ("vlong", 96)])
def test_workload_unfused_sampled(had, name, count):
    c = config_case(name)
    rows = all_rows(c) if count == 0 else synth.sample_rows(synth.CONFIGS[name], count)
    _check_unfused(had, c, rows)


def _head_rows(cfg, heads):
    return np.concatenate([np.arange(h * cfg.n, (h + 1) * cfg.n) for h in heads])


# Rows compared with the oracle: every row of the small workloads; two whole
# heads (the first and the last) of long and one of vlong, plus a seeded
# sample across all heads.
FUSED_ROWS = {
    "tiny": lambda cfg: None,
    "bert": lambda cfg: None,
    "vit": lambda cfg: None,
    "long": lambda cfg: np.union1d(_head_rows(cfg, [0, cfg.B * cfg.H - 1]),
                                   synth.sample_rows(cfg, 256)),
    "vlong": lambda cfg: np.union1d(_head_rows(cfg, [cfg.B * cfg.H - 1]),
                                    synth.sample_rows(cfg, 96)),
}


@pytest.mark.parametrize("name", ["tiny", "bert", "vit", "long", "vlong"])
def test_workload_fused(had, name):
    c = config_case(name)
    rows = FUSED_ROWS[name](synth.CONFIGS[name])
    rows = all_rows(c) if rows is None else rows
    max_abs, rel = _check_fused(had, c, rows)
    # the margin left by fp16 P in the value product (run with -s to see it)
    print(f"\nfused error {name}: {len(rows)} rows, max abs {max_abs:.3e} "
          f"(bound {MAX_ABS:.0e}), rel L2 {rel:.3e} (bound {REL_L2:.0e})")


@pytest.mark.parametrize("name", ["bert", "vit", "long"])
def test_workload_fused_equals_unfused_on_every_row(had, name):
    """Every row, on the GPU: the fused kernels' kept sets (their debug
    outputs) are bit-identical to the unfused top-N kernel's, whichever path
    (window or exact fix-up) the row took.  had_attention_fwd writes the kept
    set from the 64-key kernel, had_attention_core from the 128-key one (its
    window, threshold and fix-up logic, shared with the production call)."""
    c = config_case(name)
    qb = had.had_binarize_pack(c.gq, c.gsq)
    kb = had.had_binarize_pack(c.gk, c.gsk)
    idx, lg = had.had_hamming_topn(qb, kb, c.d, c.N)
    dbg_idx = torch.empty_like(idx)
    dbg_lg = torch.empty_like(lg)
    had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau,
                          dbg_idx=dbg_idx, dbg_logits=dbg_lg)
    torch.cuda.synchronize()
    assert torch.equal(dbg_idx, idx)
    assert torch.equal(dbg_lg, lg)
    ws = had.workspace(c.B, c.H, c.n, c.d, c.N)
    had.had_attention_prepare(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, ws)
    dbg_idx.fill_(-7)
    dbg_lg.fill_(-7)
    had.had_attention_core(c.gv, c.N, c.tau, ws, dbg_idx=dbg_idx, dbg_logits=dbg_lg)
    torch.cuda.synchronize()
    assert torch.equal(dbg_idx, idx)
    assert torch.equal(dbg_lg, lg)


def test_all_keys_equal(had):
    c = random_case(1, 2, 300, 64, 17, 11)
    c.k[:] = c.k[:, :, :1]
    c = Case(c.q, c.k, c.v, c.sgq, synth.per_head_sigma(c.k), c.N, c.tau)
    dbg = torch.empty((1, 2, 300, 17), dtype=torch.int32, device="cuda")
    out = had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau, dbg_idx=dbg)
    torch.cuda.synchronize()
    assert (dbg.cpu() == torch.arange(17, dtype=torch.int32)).all()
    mean = c.v[:, :, :17].double().mean(dim=2, keepdim=True).expand(-1, -1, 300, -1)
    assert_close(out.cpu().numpy(), mean.numpy(), "mean of first N")


@pytest.mark.parametrize("n,N", [(2048, 300), (2047, 300), (2048, 356), (1700, 356)])
def test_all_keys_equal_many_tiles(had, n, N):
    """Every key a tie at the threshold, over 14-16 key tiles: the quota
    tile is the third (keys 256 .. 383) and keeps its first N - 256 keys, on
    the production path (the key-sign scan).  44 kept of 128 ties: the kept
    ones are set in P; 100 kept: the 28 dropped ones are cleared instead."""
    c = random_case(1, 2, n, 64, N, 13)
    c.k[:] = c.k[:, :, :1]
    c = Case(c.q, c.k, c.v, c.sgq, synth.per_head_sigma(c.k), c.N, c.tau)
    out = had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau)
    torch.cuda.synchronize()
    mean = c.v[:, :, :N].double().mean(dim=2, keepdim=True).expand(-1, -1, n, -1)
    assert_close(out.cpu().numpy(), mean.numpy(), "mean of first N")


def test_golden_handworked(had):
    case = _golden.load()
    q, k, v, sgq, sgk = (torch.from_numpy(a) for a in _golden.tensors(case))
    c = Case(q, k, v, sgq, sgk, case["N"], case["tau"])
    dbg = torch.empty((1, 1, 4, 2), dtype=torch.int32, device="cuda")
    out = had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau, dbg_idx=dbg)
    torch.cuda.synchronize()
    exp = case["expected"]
    kb = had.had_binarize_pack(c.gk, c.gsk).cpu().numpy().view(np.uint32)
    assert kb[0, 0].tolist() == exp["k_bits"]
    for key in ("row0", "row1", "row2", "row3"):
        r = int(key[3:])
        assert dbg[0, 0, r].tolist() == exp[key]["idx"]
        want = np.zeros(case["d"])
        for col, ex in exp[key]["out_nonzero"].items():
            want[int(col)] = _golden.closed_form(ex)
        # P enters the value product as fp16: within the output tolerance
        assert_close(out[0, 0, r].cpu().numpy(), want, f"golden {key}")
    # the causal form of the fused kernel on the same hand-worked rows
    dbg_c = torch.empty((1, 1, 4, 2), dtype=torch.int32, device="cuda")
    lg_c = torch.empty((1, 1, 4, 2), dtype=torch.int16, device="cuda")
    out_c = had.had_attention_causal_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau,
                                         dbg_idx=dbg_c, dbg_logits=lg_c)
    torch.cuda.synchronize()
    for key, e in case["expected_causal"].items():
        r = int(key[3:])
        assert dbg_c[0, 0, r].tolist() == e["idx"]
        assert lg_c[0, 0, r].tolist() == e["logits"]
        want = np.zeros(case["d"])
        for col, ex in e["out_nonzero"].items():
            want[int(col)] = _golden.closed_form(ex)
        assert_close(out_c[0, 0, r].cpu().numpy(), want, f"golden causal {key}")


def test_sign_edge_values_on_device(had):
    vals = [0.0, -0.0, float("nan"), float("inf"), float("-inf"), 1e-45, -1e-45,
            -1.1754944e-38, -1e-30, 3.0, -3.0]
    x = torch.ones(1, 3, 1, 64)
    for i, v in enumerate(vals):
        x[0, :, 0, i] = v
    sigma = torch.tensor([1.0, 3.0, 1e9])
    got = had.had_binarize_pack(x.cuda(), sigma.cuda()).cpu().numpy().view(np.uint32)
    ref = oracle.pack(oracle.binarize(x.numpy(), sigma.numpy()))
    assert np.array_equal(got, ref)


# Values whose sign after the fp32 division is decided at an edge: -0, the
# tiny magnitudes (bf16 keeps the fp32 exponent range, down to 2^-133) whose
# quotient rounds to -0 under a large sigma, infinities and NaN.
BF16_SIGN_VALS = [0.0, -0.0, float("nan"), float("inf"), float("-inf"), -9.2e-41, 9.2e-41,
                  -1.1754944e-38, -1e-37, -1e-30, -1e-22, -1e-20, -1e-10, 3.0, -3.0]
BF16_SIGMAS = [1.0, 3.0, 1e9, 1e30, 1e-30]


def test_sign_edge_values_on_device_bf16(had):
    """bf16 signs on their raw bits (pack kernel), edges against the oracle."""
    H = len(BF16_SIGMAS)
    x = (torch.randn(1, H, 2, 64, generator=torch.Generator().manual_seed(21)) * 1e-21)
    for i, v in enumerate(BF16_SIGN_VALS):
        x[0, :, 0, i] = v
    x = x.to(torch.bfloat16)
    sigma = torch.tensor(BF16_SIGMAS)
    got = had.had_binarize_pack(x.cuda(), sigma.cuda()).cpu().numpy().view(np.uint32)
    ref = oracle.pack(oracle.binarize(synth.to_oracle_array(x), sigma.numpy()))
    assert np.array_equal(got, ref)


def test_fused_sign_edge_values_bf16(had):
    """The same edges in Q and K through the fused path's operand
    preparation: indices and logits must equal the oracle's exactly."""
    H, n, d, N = len(BF16_SIGMAS), 130, 64, 20
    g = torch.Generator().manual_seed(22)
    q = torch.randn(1, H, n, d, generator=g)
    k = torch.randn(1, H, n, d, generator=g)
    v = torch.randn(1, H, n, d, generator=g).to(torch.bfloat16)
    for t in (q, k):
        for i, val in enumerate(BF16_SIGN_VALS):
            t[0, :, (7 * i) % n, (5 * i) % d] = val
            t[0, :, (11 * i + 3) % n, :: 9] = val * (1 if i % 2 else 1e-25)
    sigma = torch.tensor(BF16_SIGMAS)
    case = Case(q.to(torch.bfloat16), k.to(torch.bfloat16), v, sigma, sigma, N, 0.125)
    _check_fused(had, case, all_rows(case))


def test_bad_sigma_is_flagged(had):
    c = random_case(1, 2, 64, 64, 8, 12)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    had.had_binarize_pack(c.gq, torch.tensor([1.0, -1.0], device="cuda"), dev_status=status)
    torch.cuda.synchronize()
    assert status.item() & (1 << had.HAD_ERR_BAD_SIGMA)
    status.zero_()
    had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, torch.tensor([float("nan"), 1.0], device="cuda"),
                          c.N, c.tau, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() & (1 << had.HAD_ERR_BAD_SIGMA)


def test_invalid_arguments_rejected_before_launch(had):
    c = random_case(1, 1, 64, 64, 8, 13)
    with pytest.raises(had.HadError) as e:
        had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, 65, c.tau)
    assert e.value.status == had.HAD_ERR_INVALID_ARG
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(had.HadError) as e:
        had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, 8, c.tau, ws=small)
    assert e.value.status == had.HAD_ERR_WORKSPACE
    x = torch.randn(1, 1, 8, 96, device="cuda")
    with pytest.raises(had.HadError) as e:
        had.had_binarize_pack(x, torch.ones(1, device="cuda"))
    assert e.value.status == had.HAD_ERR_UNSUPPORTED


def test_out_of_range_index_flagged(had):
    c = random_case(1, 1, 40, 64, 4, 14)
    idx = torch.zeros((1, 1, 40, 4), dtype=torch.int32, device="cuda")
    idx[0, 0, 3, 2] = 40
    lg = torch.zeros((1, 1, 40, 4), dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    had.had_sparse_softmax_av(idx, lg, c.gv, c.tau, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() & (1 << had.HAD_ERR_INVALID_ARG)


def test_prepare_then_core_equals_fwd(had):
    c = random_case(2, 3, 700, 64, 90, 15)
    ref = had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau)
    ws = had.workspace(c.B, c.H, c.n, c.d, c.N)
    had.had_attention_prepare(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, ws)
    out = had.had_attention_core(c.gv, c.N, c.tau, ws)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    # the core stage may run again on the same prepared operands
    for _ in range(3):
        again = had.had_attention_core(c.gv, c.N, c.tau, ws)
        torch.cuda.synchronize()
        assert torch.equal(again, ref)


def test_tau_zero_is_uniform_over_kept(had):
    c = random_case(1, 2, 300, 64, 40, 16, tau=0.0)
    idx = torch.empty((1, 2, 300, 40), dtype=torch.int32, device="cuda")
    out = had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, 0.0, dbg_idx=idx)
    torch.cuda.synchronize()
    v = c.v.double()
    ii = idx.long().cpu()
    mean = torch.stack([torch.stack([v[0, h, ii[0, h, i]].mean(0) for i in range(300)])
                        for h in range(2)])[None]
    assert_close(out.cpu().numpy(), mean.numpy(), "tau = 0")


def test_negative_tau_rejected(had):
    c = random_case(1, 1, 64, 64, 8, 17)
    with pytest.raises(had.HadError) as e:
        had.had_attention_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, -0.1)
    assert e.value.status == had.HAD_ERR_INVALID_ARG


def _window_estimate(lev, d, N):
    """Host restatement of where the fused kernel centres a row's threshold
    window: the exact mean level over all keys plus z times the spread of the
    first 128 keys, z the standard normal quantile at N / n."""
    from statistics import NormalDist
    n = lev.shape[1]
    z = NormalDist().inv_cdf(min(max(N / n, 1e-9), 1 - 1e-9))
    first = lev[:, :min(128, n)].astype(np.float64)
    return np.rint(lev.mean(axis=1) + z * first.std(axis=1)).astype(int)


def test_window_misses_take_the_exact_fixup(had):
    """Every row misses its window: the first key tile holds keys far from
    all queries, so its spread is small and the window sits well away from
    the true threshold level; the fix-up kernel recomputes each row."""
    B, H, n, d, N = 1, 2, 1024, 64, 64
    g = torch.Generator().manual_seed(77)
    c = torch.randn(1, H, 1, d, generator=g)
    q = (c + 0.3 * torch.randn(B, H, n, d, generator=g)).to(torch.bfloat16)
    k = torch.randn(B, H, n, d, generator=g)
    k[:, :, :256] = -c + 0.3 * torch.randn(B, H, 256, d, generator=g)
    k = k.to(torch.bfloat16)
    v = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    case = Case(q, k, v, synth.per_head_sigma(q), synth.per_head_sigma(k), N, 1 / math.sqrt(d))
    rows = all_rows(case)
    # on the host: the window misses the threshold level by more than one
    s = oracle.logits_rows(case.sq, case.sk, rows)
    lev = (d - s) // 2
    t = np.sort(lev, axis=1)[:, N - 1]
    est = _window_estimate(lev, d, N)
    assert np.mean(np.abs(t - est) > 1) > 0.9
    _check_fused(had, case, rows)
    # the diagnostic reports those rows
    ws = had.workspace(B, H, n, d, N)
    had.had_attention_fwd(case.gq, case.gk, case.gv, case.gsq, case.gsk, N, case.tau, ws=ws)
    misses = had.had_attention_window_misses(ws, B, H, n, d, N)
    assert misses >= 0.9 * len(rows)
    assert misses <= len(rows)


def _mass_check(had, c, p, rows):
    """Kernel vs oracle, exact except where the fp64 sums put p Z within
    rounding of a boundary (then the two may differ by one key)."""
    qb = had.had_binarize_pack(c.gq, c.gsq)
    kb = had.had_binarize_pack(c.gk, c.gsk)
    got = had.had_topn_mass(qb, kb, c.d, c.tau, p).reshape(-1, len(p)).cpu().numpy()[rows]
    tau32 = float(np.float32(c.tau))           # the C ABI takes tau as fp32
    want = oracle.topn_mass_rows(c.sq, c.sk, tau32, p, rows)
    diff = np.argwhere(got != want)
    if len(diff):
        s = oracle.logits_rows(c.sq, c.sk, rows).astype(np.float64)
        w = np.exp(tau32 * (s - s.max(axis=1, keepdims=True)))
        cum = np.cumsum(-np.sort(-w, axis=1), axis=1)
        for r, k in diff:
            assert abs(int(got[r, k]) - int(want[r, k])) == 1
            lo = min(got[r, k], want[r, k]) - 1
            tgt = p[k] * cum[r, -1]
            assert abs(cum[r, lo] - tgt) <= 1e-12 * cum[r, -1], (r, k)
    return got


@pytest.mark.parametrize("B,H,n,d,seed", [(1, 2, 300, 64, 11), (2, 1, 257, 128, 12),
                                          (1, 1, 1, 64, 13)])
def test_topn_mass_small_all_rows(had, B, H, n, d, seed):
    c = random_case(B, H, n, d, max(1, n // 8), seed)
    p = [0.5, 0.9, 0.95, 0.99, 1.0]
    got = _mass_check(had, c, p, all_rows(c))
    assert (np.diff(got, axis=1) >= 0).all()


def test_topn_mass_long_workload_sampled(had):
    c = config_case("long")
    rows = synth.sample_rows(synth.CONFIGS["long"], 256, seed=21)
    _mass_check(had, c, [0.9, 0.95, 0.99], rows)


def _check_causal(had, c, rows):
    """Causal top-N and softmax-V against the oracle: kept indices and logits
    (empty slots included) bit-exact, probabilities and output within the
    tolerance; the one-call forward equals the three-call composition."""
    qb, kb = _check_bits(had, c)
    idx, lg = had.had_hamming_topn_causal(qb, kb, c.d, c.N)
    out, p = had.had_sparse_softmax_av(idx, lg, c.gv, c.tau, want_p=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dbg_idx = torch.empty((c.B, c.H, c.n, c.N), dtype=torch.int32, device="cuda")
    dbg_lg = torch.empty((c.B, c.H, c.n, c.N), dtype=torch.int16, device="cuda")
    fused = had.had_attention_causal_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau,
                                         dbg_idx=dbg_idx, dbg_logits=dbg_lg, dev_status=status)
    plain = had.had_attention_causal_fwd(c.gq, c.gk, c.gv, c.gsq, c.gsk, c.N, c.tau,
                                         dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(fused, plain)      # the debug outputs change nothing
    o_idx, o_lg, o_p, o_out = oracle.attention_causal_rows(c.sq, c.sk, c.v_or, c.tau, c.N, rows)
    flat = lambda t: t.reshape(-1, t.shape[-1]).cpu().numpy()[rows]
    # unfused building blocks
    assert np.array_equal(flat(idx), o_idx)
    assert np.array_equal(flat(lg), o_lg)
    assert_close(flat(p), o_p, "causal p")
    assert_close(flat(out), o_out, "causal out")
    # fused tensor-core path
    assert np.array_equal(flat(dbg_idx), o_idx)
    assert np.array_equal(flat(dbg_lg), o_lg)
    assert_close(flat(fused), o_out, "causal fused out")


@pytest.mark.parametrize("B,H,n,d,N,seed", [(1, 2, 300, 64, 40, 31), (2, 1, 257, 128, 33, 32),
                                            (1, 1, 1, 64, 1, 33), (1, 2, 130, 64, 130, 34),
                                            (1, 3, 200, 64, 1, 35), (1, 2, 1100, 64, 200, 36),
                                            (1, 1, 1000, 128, 100, 37)])
def test_causal_small_all_rows(had, B, H, n, d, N, seed):
    c = random_case(B, H, n, d, N, seed)
    _check_causal(had, c, all_rows(c))


def test_causal_window_misses_take_the_exact_fixup(had):
    """As the non-causal case: the first 256 keys are far from every query,
    so for rows past them the sampled window misses and the causal fix-up
    recomputes the row on its visible keys."""
    B, H, n, d, N = 1, 2, 1024, 64, 64
    g = torch.Generator().manual_seed(79)
    c = torch.randn(1, H, 1, d, generator=g)
    q = (c + 0.3 * torch.randn(B, H, n, d, generator=g)).to(torch.bfloat16)
    k = torch.randn(B, H, n, d, generator=g)
    k[:, :, :256] = -c + 0.3 * torch.randn(B, H, 256, d, generator=g)
    k = k.to(torch.bfloat16)
    v = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    case = Case(q, k, v, synth.per_head_sigma(q), synth.per_head_sigma(k), N, 1 / math.sqrt(d))
    rows = all_rows(case)
    # on the host, rows 768.. of the first head: the estimate from the first
    # 256 keys misses the causal threshold level by more than one level
    s = oracle.logits_rows(case.sq, case.sk, np.arange(768, 1024))
    lev = (d - s) // 2
    miss = 0
    for t, i in enumerate(range(768, 1024)):
        vis = lev[t, :i + 1]
        thr = np.sort(vis)[N - 1]
        est = np.sort(vis[:256])[max(1, round(N * 256 / (i + 1))) - 1]
        miss += abs(int(thr) - int(est)) > 1
    assert miss > 0.9 * 256
    _check_causal(had, case, rows)


def test_causal_long_workload_sampled(had):
    c = config_case("long")
    cfg = synth.CONFIGS["long"]
    # the diagonal region (rows that see fewer than N keys, and the first
    # CTA boundaries) in two heads, plus a seeded sample of the rest
    early = np.array([0, 1, 2, 127, 128, 129, 255, 510, 511, 512, 513, 4095])
    heads = np.array([0, cfg.B * cfg.H - 1])
    rows = np.unique(np.concatenate([(heads[:, None] * cfg.n + early[None, :]).ravel(),
                                     synth.sample_rows(cfg, 128, seed=41)]))
    _check_causal(had, c, rows)


def test_empty_slots_give_zeros_without_error(had):
    c = random_case(1, 1, 64, 64, 8, 36)
    idx = torch.full((1, 1, 64, 8), -1, dtype=torch.int32, device="cuda")
    idx[0, 0, 1::2, 3] = 5          # odd rows keep one key
    lg = torch.zeros((1, 1, 64, 8), dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, p = had.had_sparse_softmax_av(idx, lg, c.gv, c.tau, want_p=True, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.count_nonzero(out[0, 0, 0::2]) == 0 and torch.count_nonzero(p[0, 0, 0::2]) == 0
    v5 = c.gv[0, 0, 5].float()
    assert torch.equal(out[0, 0, 1::2], v5.expand(32, -1))
    assert torch.all(p[0, 0, 1::2, 3] == 1) and p[0, 0, 1::2].sum() == 32


# ------------------------------------------------------ soft (tanh) codes


def _soft_inputs(B, H, n, d, seed, dtype=torch.bfloat16, dup=0, min_abs=0.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, n, d, generator=g)
    k = torch.randn(B, H, n, d, generator=g)
    v = torch.randn(B, H, n, d, generator=g)
    if min_abs:                    # move small entries out to +-min_abs
        away = lambda x: torch.where(x.abs() < min_abs,
                                     torch.where(x >= 0, min_abs, -min_abs), x)
        q, k = away(q), away(k)
    if dup:
        k[:, :, dup:2 * dup] = k[:, :, :dup]
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    return q, k, v, synth.per_head_sigma(q), synth.per_head_sigma(k)


def _ulps(got, want):
    got = np.asarray(got, np.float32)
    want = np.asarray(want, np.float32)
    return np.abs(got.astype(np.float64) - want) / np.spacing(np.maximum(np.abs(want), 1e-30))


def _soft_error_bound(o_tq, o_tk, rows, n, d):
    """Bound on |GPU logit - oracle logit| per (row, key): codes within 2 ulp
    (tanhf) and fp32 accumulation of d products, from sum_k |tq_k| |tk_k|."""
    tq = np.abs(o_tq.reshape(-1, d)).astype(np.float64)
    tk = np.abs(o_tk.reshape(-1, n, d)).astype(np.float64)
    A = np.stack([tq[r] @ tk[r // n].T for r in rows])
    return (2.0 ** -20 + d * 2.0 ** -23) * A + 1e-30


def _check_soft_rule_on_gpu_logits(had, tq, tk, N, rows, g_idx, g_lg):
    """The kept set follows the selection rule exactly on the GPU's own fp32
    logits: nothing dropped lies above the smallest kept logit, and among
    keys equal to it the lower indices are the kept ones.  The logits are
    read from the scratch of a one-head had_soft_topn call, which holds that
    head's [n][ceil(n/4)*4] fp32 logit matrix; that call must also reproduce
    the full call's kept set."""
    B, H, n, d = tq.shape
    ld = (n + 3) // 4 * 4
    heads = sorted({int(r) // n for r in rows})
    for h in heads:
        b_, h_ = divmod(h, H)
        q1 = tq[b_:b_ + 1, h_:h_ + 1].contiguous()
        k1 = tk[b_:b_ + 1, h_:h_ + 1].contiguous()
        ws = torch.empty(had.had_workspace_bytes(had.HAD_OP_SOFT_TOPN, 1, 1, n, d, N),
                         dtype=torch.uint8, device="cuda")
        idx1, lg1 = had.had_soft_topn(q1, k1, N, ws=ws)
        torch.cuda.synchronize()
        sel = np.nonzero(np.asarray(rows) // n == h)[0]
        local = torch.tensor(np.asarray(rows)[sel] % n, device="cuda")
        S_rows = ws[:n * ld * 4].view(torch.float32).reshape(n, ld)[local, :n].cpu().numpy()
        idx1, lg1 = idx1[0, 0].cpu().numpy(), lg1[0, 0].cpu().numpy()
        for u, t in enumerate(sel):
            i = int(rows[t]) % n
            srow = S_rows[u]
            gi = g_idx[t]
            assert np.array_equal(idx1[i], gi)
            assert np.array_equal(lg1[i], g_lg[t])
            assert np.array_equal(srow[gi], g_lg[t])
            kept = np.zeros(n, bool)
            kept[gi] = True
            T = srow[kept].min()
            assert (srow[~kept] <= T).all()
            tie_kept = np.nonzero(kept & (srow == T))[0]
            tie_drop = np.nonzero(~kept & (srow == T))[0]
            if len(tie_drop):
                assert tie_kept.max() < tie_drop.min()


def _check_soft(had, q, k, v, sgq, sgk, c, N, tau, rows):
    """Soft forward against the oracle on every listed row.

    Codes within 2 ulp.  Every row: the kept set is valid (ascending, no
    dropped key seen above a kept one beyond the logit error bound, kept
    logits within that bound), and out and p match the oracle's softmax and
    value product over the GPU's kept set within the tolerance.  Rows whose
    oracle threshold is isolated beyond the bound (the kept set is fixed by
    the arithmetic) must also keep exactly the oracle's set.  The selection
    rule is checked exactly on the GPU's own logits."""
    B, H, n, d = q.shape
    gq, gk, gv = q.cuda(), k.cuda(), v.cuda()
    gsq, gsk = sgq.cuda(), sgk.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq = had.had_soft_binarize(gq, gsq, c, dev_status=status)
    tk = had.had_soft_binarize(gk, gsk, c, dev_status=status)
    idx, lg = had.had_soft_topn(tq, tk, N)
    out, p = had.had_soft_softmax_av(idx, lg, gv, tau, want_p=True, dev_status=status)
    out1 = had.had_soft_attention_fwd(gq, gk, gv, gsq, gsk, c, N, tau, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(out, out1)

    o_tq = oracle.soft_binarize(synth.to_oracle_array(q), sgq.numpy(), c)
    o_tk = oracle.soft_binarize(synth.to_oracle_array(k), sgk.numpy(), c)
    assert _ulps(tq.cpu().numpy(), o_tq).max() <= 2
    assert _ulps(tk.cpu().numpy(), o_tk).max() <= 2

    v_or = synth.to_oracle_array(v)
    o_idx, o_lg, o_p, o_out = oracle.soft_attention_rows(o_tq, o_tk, v_or, tau, N, rows)
    s_or = oracle.soft_logits_rows(o_tq, o_tk, rows)
    eps = _soft_error_bound(o_tq, o_tk, rows, n, d)
    flat = lambda t: t.reshape(-1, t.shape[-1]).cpu().numpy()[rows]
    g_idx, g_lg, g_p, g_out = flat(idx), flat(lg), flat(p), flat(out)
    # every row: the oracle's softmax and value product over the GPU's set
    gp_ref, gout_ref = oracle.soft_attention_given(o_tq, o_tk, v_or, tau, g_idx, rows)
    assert_close(g_out, gout_ref, "soft out (GPU kept set)")
    assert_close(g_p, gp_ref, "soft p (GPU kept set)")
    for t in range(len(rows)):
        gi = g_idx[t]
        assert (np.diff(gi) > 0).all() and gi[0] >= 0 and gi[-1] < n
        assert (np.abs(g_lg[t].astype(np.float64) - s_or[t, gi]) <= eps[t, gi]).all()
        kept = np.zeros(n, bool)
        kept[gi] = True
        if N < n:
            # no dropped key can have been seen above a kept one
            assert (s_or[t, kept] + eps[t, kept]).min() >= (s_or[t, ~kept] - eps[t, ~kept]).max()
        ok = np.zeros(n, bool)
        ok[o_idx[t]] = True
        # The oracle's kept set is fixed beyond rounding when its threshold
        # value T (with any exact ties at T, which equal codes reproduce
        # exactly on both sides) is separated from every other value by
        # more than the error bounds.
        vals, e = s_or[t], eps[t]
        T = vals[ok].min()
        at = vals == T
        e_T = e[at].max()
        above = ok & ~at
        below = ~ok & ~at
        isolated = ((vals[above] - e[above]).min(initial=np.inf) > T + e_T and
                    T - e_T > (vals[below] + e[below]).max(initial=-np.inf))
        if N == n or isolated:
            assert np.array_equal(gi, o_idx[t])
            assert_close(g_out[t], o_out[t], "soft out")
            assert_close(g_p[t], o_p[t], "soft p")
    assert np.allclose(g_p.sum(axis=1), 1.0, atol=1e-5)
    _check_soft_rule_on_gpu_logits(had, tq, tk, N, rows, g_idx, g_lg)


SOFT_SMALL = [
    # (B, H, n, d, N, seed, c, dtype)
    (1, 2, 300, 64, 40, 51, 1.0, torch.bfloat16),
    (2, 1, 257, 128, 33, 52, 2.0, torch.bfloat16),
    (1, 1, 1, 64, 1, 53, 1.0, torch.bfloat16),
    (1, 2, 130, 64, 130, 54, 0.5, torch.float32),      # N = n: dense softmax
    (1, 3, 200, 64, 1, 55, 1.5, torch.float32),        # N = 1
    (1, 1, 700, 64, 90, 56, 0.2, torch.bfloat16),
]


@pytest.mark.parametrize("B,H,n,d,N,seed,c,dtype", SOFT_SMALL)
def test_soft_small_all_rows(had, B, H, n, d, N, seed, c, dtype):
    q, k, v, sgq, sgk = _soft_inputs(B, H, n, d, seed, dtype)
    _check_soft(had, q, k, v, sgq, sgk, c, N, 1 / math.sqrt(d), np.arange(B * H * n))


def test_soft_exact_ties_keep_the_lower_index(had):
    q, k, v, sgq, sgk = _soft_inputs(1, 2, 160, 64, 57, dup=40)
    _check_soft(had, q, k, v, sgq, sgk, 1.0, 24, 0.125, np.arange(320))
    # all keys equal: every logit of a row ties, the first N keys are kept
    k_all = k[:, :, :1].expand(-1, -1, 160, -1).contiguous()
    tq = had.had_soft_binarize(q.cuda(), sgq.cuda(), 1.0)
    tk = had.had_soft_binarize(k_all.cuda(), synth.per_head_sigma(k_all).cuda(), 1.0)
    idx, _ = had.had_soft_topn(tq, tk, 24)
    assert (idx.cpu() == torch.arange(24, dtype=torch.int32)).all()


def test_soft_at_large_c_is_the_binarized_path(had):
    # with |x / sigma| >= 0.01 and c = 1e4 every code is exactly +-1, so the
    # soft path must give the binarized path's kept set, ties included
    q, k, v, sgq, sgk = _soft_inputs(1, 2, 300, 64, 58, torch.float32, min_abs=0.05)
    tq = had.had_soft_binarize(q.cuda(), sgq.cuda(), 1e4)
    tk = had.had_soft_binarize(k.cuda(), sgk.cuda(), 1e4)
    assert torch.equal(tq.abs(), torch.ones_like(tq))
    idx, lg = had.had_soft_topn(tq, tk, 37)
    out, _ = had.had_soft_softmax_av(idx, lg, v.cuda(), 0.125)
    sq = oracle.binarize(synth.to_oracle_array(q), sgq.numpy())
    sk = oracle.binarize(synth.to_oracle_array(k), sgk.numpy())
    o_idx, o_lg, _, o_out = oracle.attention_rows(sq, sk, synth.to_oracle_array(v), 0.125, 37,
                                                  np.arange(600))
    assert np.array_equal(idx.reshape(600, 37).cpu().numpy(), o_idx)
    assert np.array_equal(lg.reshape(600, 37).cpu().numpy(), o_lg.astype(np.float32))
    assert_close(out.reshape(600, 64).cpu().numpy(), o_out, "soft large-c out")


def test_soft_long_workload_sampled(had):
    cfg = synth.CONFIGS["long"]
    c = config_case("long")
    rows = synth.sample_rows(cfg, 192, seed=61)
    _check_soft(had, c.q, c.k, c.v, c.sgq, c.sgk, 1.0, cfg.N, cfg.tau, rows)


# ------------------------------------------- straight-through backward


def _bwd_inputs(B, H, n, d, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, n, d, generator=g).to(dtype) for _ in range(3))
    dout = torch.randn(B, H, n, d, generator=g)
    return q, k, v, dout, synth.per_head_sigma(q), synth.per_head_sigma(k)


def _check_bwd(had, q, k, v, dout, sgq, sgk, N, tau, clip, heads=None):
    """GPU backward on the whole tensor; oracle on the listed (b, h) heads."""
    dq, dk, dv = had.had_attention_bwd(q.cuda(), k.cuda(), v.cuda(), sgq.cuda(), sgk.cuda(),
                                       dout.cuda(), N, tau, clip)
    torch.cuda.synchronize()
    B, H = q.shape[:2]
    heads = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in heads:
        sl = lambda t: t[b:b + 1, h:h + 1].contiguous()
        oq, ok_, ov = oracle.attention_bwd(
            synth.to_oracle_array(sl(q)), synth.to_oracle_array(sl(k)),
            synth.to_oracle_array(sl(v)), sgq[h:h + 1].numpy(), sgk[h:h + 1].numpy(),
            sl(dout).numpy(), tau, N, clip)
        for got, want, name in ((dq, oq, "dq"), (dk, ok_, "dk"), (dv, ov, "dv")):
            assert_close(got[b, h].cpu().numpy(), want[0, 0], f"{name} head {b},{h}")
    return dq, dk, dv


BWD_SMALL = [
    # (B, H, n, d, N, seed, dtype, clip)
    (1, 2, 300, 64, 40, 71, torch.bfloat16, 1.0),
    (2, 1, 257, 128, 33, 72, torch.bfloat16, 1.0),
    (1, 1, 1, 64, 1, 73, torch.bfloat16, 1.0),
    (1, 2, 130, 64, 130, 74, torch.float32, float("inf")),   # N = n
    (1, 3, 200, 64, 1, 75, torch.float32, 1.0),              # N = 1: dq = dk = 0
    (1, 1, 700, 64, 90, 76, torch.bfloat16, 0.5),
]


@pytest.mark.parametrize("B,H,n,d,N,seed,dtype,clip", BWD_SMALL)
def test_bwd_small_all_heads(had, B, H, n, d, N, seed, dtype, clip):
    q, k, v, dout, sgq, sgk = _bwd_inputs(B, H, n, d, seed, dtype)
    dq, dk, _ = _check_bwd(had, q, k, v, dout, sgq, sgk, N, 1 / math.sqrt(d), clip)
    if N == 1:
        assert not dq.any() and not dk.any()


def test_bwd_with_the_forward_kept_set(had):
    # the kept set from the fused forward's debug outputs gives the same dq
    # (row gathers are deterministic) and the same dk, dv within rounding
    q, k, v, dout, sgq, sgk = _bwd_inputs(1, 2, 520, 64, 78)
    N, tau = 64, 0.125
    g = [t.cuda() for t in (q, k, v, sgq, sgk)]
    idx = torch.empty((1, 2, 520, N), dtype=torch.int32, device="cuda")
    lg = torch.empty((1, 2, 520, N), dtype=torch.int16, device="cuda")
    had.had_attention_fwd(*g, N, tau, dbg_idx=idx, dbg_logits=lg)
    a = had.had_attention_bwd(*g, dout.cuda(), N, tau, idx=idx, logits=lg)
    b = had.had_attention_bwd(*g, dout.cuda(), N, tau)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0])
    for x, y, name in zip(a[1:], b[1:], ("dk", "dv")):
        assert_close(x.cpu().numpy(), y.cpu().numpy(), name)
    _check_bwd(had, q, k, v, dout, sgq, sgk, N, tau, 1.0)


def test_bwd_long_workload_two_heads(had):
    cfg = synth.CONFIGS["long"]
    c = config_case("long")
    dout = torch.randn(c.q.shape, generator=torch.Generator().manual_seed(77))
    _check_bwd(had, c.q, c.k, c.v, dout, c.sgq, c.sgk, cfg.N, cfg.tau, 1.0,
               heads=[(0, 0), (cfg.B - 1, cfg.H - 1)])
