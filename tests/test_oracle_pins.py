"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

Each test ties one step of the oracle to something other than the oracle
itself: IEEE edge values, a library routine (numpy float64 matrix product,
numpy/Python sorts, torch softmax), an independent algorithm (histogram
threshold selection), a closed form, or the hand-worked fixture under
tests/golden/.  The steps follow the pith.science review of "Hamming
Attention Distillation" (arXiv 2502.01770), "What carries the argument":
standardize by sigma, sign to +/-1 (Eqs. 4-5), Hamming logits (Eq. 5),
top-N mask (Eq. 6), softmax over the kept logits (Eq. 7), value product.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _golden


def _signs_np(x, sigma):
    """Library route to the signs: numpy float32 division, then < 0."""
    z = np.asarray(x, np.float32) / np.asarray(sigma, np.float32)[None, :, None, None]
    return np.where(z < 0, -1, 1).astype(np.int8)


def _popcount32(a):
    a = a.astype(np.uint64)
    return np.array([int(x).bit_count() for x in a.reshape(-1)], np.int64).reshape(a.shape)


def _rand_case(B, H, n, d, seed, dist="normal"):
    g = np.random.default_rng(seed)
    x = g.standard_normal((B, H, n, d)).astype(np.float32)
    return x


# ----------------------------------------------------------------- step 1


SIGN_EDGES = [
    # (x, sigma, expected sign) -- sign is -1 iff x/sigma < 0 in IEEE fp32
    (0.0, 1.0, 1),
    (-0.0, 1.0, 1),                          # -0 is not < 0
    (float("nan"), 1.0, 1),                  # comparisons with NaN are false
    (float("inf"), 2.0, 1),
    (float("-inf"), 2.0, -1),
    (1e-45, 1.0, 1),                         # smallest subnormal
    (-1e-45, 1.0, -1),
    (-1e-45, 3.0, 1),                        # quotient rounds to -0
    (-1e-45, 0.5, -1),                       # quotient is a subnormal, kept
    (-1.1754944e-38, 1.0, -1),               # smallest normal
    (np.nextafter(np.float32(0), np.float32(1)), 1e10, 1),
    (-np.nextafter(np.float32(0), np.float32(1)), 1e10, 1),   # underflow to -0
    (-1e-30, 1e9, -1),                       # subnormal quotient, no flush
    (3.0, 7.0, 1),
    (-3.0, 7.0, -1),
]


@pytest.mark.parametrize("x,sigma,expected", SIGN_EDGES)
def test_sign_edge_values(x, sigma, expected):
    arr = np.full((1, 1, 1, 32), 1.0, np.float32)
    arr[0, 0, 0, 3] = np.float32(x)
    s = oracle.binarize(arr, np.asarray([sigma], np.float32))
    assert s[0, 0, 0, 3] == expected
    assert (np.delete(s.reshape(-1), 3) == 1).all()


def test_sign_bf16_path_matches_widened_fp32():
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(2, 3, 16, 64, generator=g) * 1e-3).to(torch.bfloat16)
    x[0, 0, 0, :4] = torch.tensor([0.0, -0.0, 1e-40, -1e-40]).to(torch.bfloat16)
    sigma = np.asarray([0.7, 1.3, 2.0], np.float32)
    a = oracle.binarize(synth.to_oracle_array(x), sigma)
    b = oracle.binarize(x.float().numpy(), sigma)
    assert np.array_equal(a, b)
    assert np.array_equal(a, _signs_np(x.float().numpy(), sigma))


def test_sign_matches_numpy_division():
    g = np.random.default_rng(1)
    x = g.standard_normal((2, 4, 33, 64)).astype(np.float32)
    x *= np.float32(10.0) ** g.integers(-40, 5, size=x.shape).astype(np.float32)
    sigma = np.asarray([0.3, 1.0, 7.5, 1e-3], np.float32)
    assert np.array_equal(oracle.binarize(x, sigma), _signs_np(x, sigma))


def test_sigma_positive_scale_does_not_change_bits():
    x = _rand_case(2, 3, 40, 64, 2)
    s1 = oracle.binarize(x, np.asarray([1.0, 2.0, 3.0], np.float32))
    s2 = oracle.binarize(x, np.asarray([0.01, 50.0, 3e4], np.float32))
    assert np.array_equal(s1, s2)


# ----------------------------------------------------------------- packing


def test_pack_bit_order_lsb_first():
    sg = np.ones((4, 64), np.int8)
    sg[1, 0] = -1            # word 0, bit 0
    sg[2, 33] = -1           # word 1, bit 1
    sg[3, 31] = -1           # word 0, bit 31
    sg[3, 63] = -1           # word 1, bit 31
    bits = oracle.pack(sg)
    assert bits.tolist() == [[0, 0], [1, 0], [0, 2], [1 << 31, 1 << 31]]


def test_pack_popcount_counts_negatives():
    g = np.random.default_rng(3)
    sg = np.where(g.random((50, 128)) < 0.3, -1, 1).astype(np.int8)
    bits = oracle.pack(sg)
    assert np.array_equal(_popcount32(bits).sum(axis=1), (sg < 0).sum(axis=1))
    # unpack by shifting and compare element by element
    unpacked = ((bits[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(50, 128)
    assert np.array_equal(unpacked == 1, sg < 0)


# ----------------------------------------------------------------- step 2


def _head_logits(sq, sk, b, h):
    B, H, n, d = sq.shape
    rows = (b * H + h) * n + np.arange(n)
    return oracle.logits_rows(sq, sk, rows)


@pytest.mark.parametrize("d", [64, 128])
def test_logits_popcount_identity(d):
    """q.k = d - 2*Hamming(q, k) for +/-1 vectors (the Eq. 5 identity)."""
    x = _rand_case(1, 2, 37, d, 4)
    y = _rand_case(1, 2, 37, d, 5)
    sg = np.asarray([1.0, 1.0], np.float32)
    sq, sk = oracle.binarize(x, sg), oracle.binarize(y, sg)
    bq, bk = oracle.pack(sq), oracle.pack(sk)
    for h in range(2):
        s = _head_logits(sq, sk, 0, h)
        xor = bq[0, h][:, None, :] ^ bk[0, h][None, :, :]
        ham = _popcount32(xor).sum(axis=-1)
        assert np.array_equal(s, d - 2 * ham)


def test_logits_match_float64_matmul():
    x = _rand_case(2, 3, 29, 64, 6)
    y = _rand_case(2, 3, 29, 64, 7)
    sg = np.asarray([0.5, 1.0, 2.0], np.float32)
    sq, sk = oracle.binarize(x, sg), oracle.binarize(y, sg)
    for b in range(2):
        for h in range(3):
            ref = sq[b, h].astype(np.float64) @ sk[b, h].astype(np.float64).T
            assert np.array_equal(_head_logits(sq, sk, b, h), ref.astype(np.int32))


def test_logits_not_transposed():
    """Row i of the logits uses query i against all keys (asymmetric case)."""
    sq = np.ones((1, 1, 3, 64), np.int8)
    sk = np.ones((1, 1, 3, 64), np.int8)
    sq[0, 0, 0, :10] = -1          # query 0 differs from every key in 10 places
    sk[0, 0, 2, :] = -1            # key 2 is the negation of the all-ones key
    s = _head_logits(sq, sk, 0, 0)
    assert s.tolist() == [[44, 44, -44], [64, 64, -64], [64, 64, -64]]


def test_logits_invariants():
    x = _rand_case(1, 2, 50, 64, 8)
    y = _rand_case(1, 2, 50, 64, 9)
    sg = np.ones(2, np.float32)
    sq, sk = oracle.binarize(x, sg), oracle.binarize(y, sg)
    s = _head_logits(sq, sk, 0, 1)
    assert np.abs(s).max() <= 64 and (s % 2 == 0).all()            # s = d mod 2
    assert np.array_equal(_head_logits(sq, -sk, 0, 1), -s)         # K -> -K
    assert np.array_equal(_head_logits(-sq, -sk, 0, 1), s)         # both flipped
    assert (np.diag(_head_logits(sq, sq, 0, 1)) == 64).all()       # Q == K


# ----------------------------------------------------------------- step 3


def _binarized(cfg_or_shape, seed=10, offset=0.0):
    B, H, n, d = cfg_or_shape
    x = _rand_case(B, H, n, d, seed) + np.float32(offset)
    y = _rand_case(B, H, n, d, seed + 1) + np.float32(offset)
    v = _rand_case(B, H, n, d, seed + 2)
    sg = np.ones(H, np.float32)
    return oracle.binarize(x, sg), oracle.binarize(y, sg), v


def _threshold_select(s_row, N, d):
    """Histogram-threshold top-N (a different algorithm from a sort).

    Count each logit value; walk values from the largest down until the
    running count reaches N; keep all larger values and the first q keys
    (in index order) at the threshold value."""
    counts = {}
    for v in s_row.tolist():
        counts[v] = counts.get(v, 0) + 1
    above = 0
    for t in range(d, -d - 1, -2):
        c = counts.get(t, 0)
        if above + c >= N:
            break
        above += c
    q = N - above
    keep = []
    for j, v in enumerate(s_row.tolist()):
        if v > t:
            keep.append(j)
        elif v == t and q > 0:
            keep.append(j)
            q -= 1
    return keep


@pytest.mark.parametrize("shape,N,offset", [((1, 2, 64, 64), 8, 0.0),
                                            ((1, 2, 197, 64), 32, 0.3),
                                            ((1, 1, 96, 128), 20, 0.0)])
def test_topn_against_sorts_and_threshold(shape, N, offset):
    sq, sk, v = _binarized(shape, offset=offset)
    B, H, n, d = shape
    idx, lg, p, out = oracle.attention(sq, sk, v, 0.125, N)
    for h in range(H):
        s = _head_logits(sq, sk, 0, h)
        for i in range(n):
            py = sorted(sorted(range(n), key=lambda j: (-s[i, j], j))[:N])
            lx = np.sort(np.lexsort((np.arange(n), -s[i]))[:N])
            th = _threshold_select(s[i], N, d)
            assert idx[0, h, i].tolist() == py == lx.tolist() == th
            assert np.array_equal(lg[0, h, i], s[i, idx[0, h, i]])


def test_topn_all_keys_equal_keeps_first_N():
    sq, sk, v = _binarized((1, 1, 40, 64), seed=20)
    sk[:] = sk[0, 0, 0]                     # every key identical -> all ties
    idx, lg, p, out = oracle.attention(sq, sk, v, 0.125, 7)
    assert (idx == np.arange(7)).all()
    assert np.allclose(p, 1.0 / 7, rtol=0, atol=1e-15)
    mean = v[0, 0, :7].astype(np.float64).mean(axis=0)
    assert np.allclose(out[0, 0], mean[None, :], rtol=0, atol=2e-7)


def test_topn_N_equals_n_is_dense_softmax():
    sq, sk, v = _binarized((1, 2, 48, 64), seed=30)
    tau = 0.125
    idx, lg, p, out = oracle.attention(sq, sk, v, tau, 48)
    for h in range(2):
        assert (idx[0, h] == np.arange(48)).all()
        s = torch.from_numpy(_head_logits(sq, sk, 0, h)).double()
        pd = torch.softmax(tau * s, dim=-1)
        od = pd @ torch.from_numpy(v[0, h]).double()
        assert np.allclose(p[0, h], pd.numpy(), rtol=1e-12, atol=1e-15)
        assert np.allclose(out[0, h], od.numpy(), rtol=0, atol=1e-6)


def test_N1_is_first_argmax():
    sq, sk, v = _binarized((1, 2, 77, 64), seed=40)
    idx, lg, p, out = oracle.attention(sq, sk, v, 0.125, 1)
    for h in range(2):
        s = _head_logits(sq, sk, 0, h)
        am = np.argmax(s, axis=1)          # numpy returns the first maximum
        assert np.array_equal(idx[0, h, :, 0], am)
        assert np.array_equal(out[0, h], v[0, h, am])
        assert (p == 1.0).all()


def test_rows_of_p_sum_to_one_with_N_nonzeros():
    sq, sk, v = _binarized((2, 2, 130, 128), seed=50)
    N = 37
    idx, lg, p, out = oracle.attention(sq, sk, v, 1 / math.sqrt(128), N)
    assert np.allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-12)
    assert (p > 0).all() and p.shape[-1] == N
    assert (np.diff(idx, axis=-1) > 0).all()           # ascending, distinct


def test_softmax_uses_tau_times_logit_difference():
    """p_k / p_l = exp(tau * (s_k - s_l)) within a row (Eq. 7)."""
    sq, sk, v = _binarized((1, 1, 60, 64), seed=60)
    tau = float(np.float32(0.3))          # tau crosses the C boundary as fp32
    idx, lg, p, out = oracle.attention(sq, sk, v, tau, 12)
    r = p[0, 0, 5]
    s = lg[0, 0, 5].astype(np.float64)
    assert np.allclose(r / r[0], np.exp(tau * (s - s[0])), rtol=1e-12)


# ----------------------------------------------------------------- fixture


def test_golden_handworked():
    case = _golden.load()
    q, k, v, sgq, sgk = _golden.tensors(case)
    sq, sk = oracle.binarize(q, sgq), oracle.binarize(k, sgk)
    exp = case["expected"]
    assert oracle.pack(sk)[0, 0].tolist() == exp["k_bits"]
    assert _head_logits(sq, sk, 0, 0)[0].tolist() == exp["logits_row0_all"]
    idx, lg, p, out = oracle.attention(sq, sk, v, case["tau"], case["N"])
    for key in ("row0", "row1", "row2", "row3"):
        r = int(key[3:])
        e = exp[key]
        assert idx[0, 0, r].tolist() == e["idx"]
        assert lg[0, 0, r].tolist() == e["logits"]
        assert np.allclose(p[0, 0, r], [_golden.closed_form(x) for x in e["p"]],
                           rtol=1e-14, atol=0)
        want = np.zeros(case["d"])
        for c, ex in e["out_nonzero"].items():
            want[int(c)] = _golden.closed_form(ex)
        assert np.allclose(out[0, 0, r], want, rtol=1e-7, atol=1e-9)


def test_golden_handworked_causal():
    case = _golden.load()
    q, k, v, sgq, sgk = _golden.tensors(case)
    sq, sk = oracle.binarize(q, sgq), oracle.binarize(k, sgk)
    idx, lg, p, out = oracle.attention_causal_rows(sq, sk, v, case["tau"], case["N"],
                                                   np.arange(case["n"]))
    for key, e in case["expected_causal"].items():
        r = int(key[3:])
        assert idx[r].tolist() == e["idx"]
        assert lg[r].tolist() == e["logits"]
        assert np.allclose(p[r], [_golden.closed_form(x) for x in e["p"]], rtol=1e-14, atol=0)
        want = np.zeros(case["d"])
        for c, ex in e["out_nonzero"].items():
            want[int(c)] = _golden.closed_form(ex)
        assert np.allclose(out[r], want, rtol=1e-7, atol=1e-9)


# ----------------------------------------------------------------- plumbing


def test_threads_deterministic():
    sq, sk, v = _binarized((2, 2, 100, 64), seed=70)
    a = oracle.attention(sq, sk, v, 0.125, 10, threads=1)
    b = oracle.attention(sq, sk, v, 0.125, 10, threads=4)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_rows_subset_matches_full():
    sq, sk, v = _binarized((1, 3, 50, 64), seed=80)
    full = oracle.attention(sq, sk, v, 0.125, 9)
    rows = np.array([0, 49, 50, 77, 149])
    sub = oracle.attention_rows(sq, sk, v, 0.125, 9, rows)
    for f, s in zip(full, sub):
        assert np.array_equal(f.reshape(-1, f.shape[-1])[rows], s)


@pytest.mark.parametrize("N", [0, 51])
def test_oracle_rejects_bad_N(N):
    sq, sk, v = _binarized((1, 1, 50, 64), seed=90)
    with pytest.raises(ValueError):
        oracle.attention(sq, sk, v, 0.125, N)


# ------------------------------------------------------ top-N mass retention
# The smallest N whose N largest softmax weights (full softmax over all keys)
# reach a fraction p of the row's total; pinned by closed forms and by an
# independent numpy brute force.


def test_mass_all_keys_equal_is_ceil_p_n():
    # equal logits: every weight is 1, so N = ceil(p n)
    sq, sk, _ = _binarized((1, 1, 40, 64), seed=100)
    sk[...] = sk[:, :, :1]
    p = [0.1, 0.25, 0.5, 0.9, 1.0]
    got = oracle.topn_mass_rows(sq, sk, 0.125, p, np.arange(40))
    assert (got == np.array([math.ceil(x * 40) for x in p])[None, :]).all()


def test_mass_two_levels_closed_form():
    # k1 keys equal to the query (logit d) and the rest its negation (-d):
    # weights 1 and e = exp(-2 tau d); Z = k1 + (n - k1) e
    n, d, k1, tau = 64, 64, 5, 0.03
    rng = np.random.default_rng(3)
    q = np.where(rng.random(d) < 0.5, -1, 1).astype(np.int8)
    sq = np.broadcast_to(q, (1, 1, n, d)).copy()
    sk = np.broadcast_to(-q, (1, 1, n, d)).copy()
    sk[0, 0, 7:7 + k1] = q
    e = math.exp(-2 * tau * d)
    Z = k1 + (n - k1) * e
    p = [0.2, k1 / Z - 1e-9, 0.9, 0.99]
    got = oracle.topn_mass_rows(sq, sk, tau, p, [0])[0]
    for pk, g in zip(p, got):
        t = pk * Z
        want = math.ceil(t - 1e-12) if t <= k1 else k1 + math.ceil((t - k1) / e - 1e-9)
        assert g == want, (pk, g, want)


def test_mass_matches_numpy_brute_force():
    sq, sk, _ = _binarized((1, 2, 300, 64), seed=110)
    p = np.array([0.5, 0.9, 0.95, 0.99])
    tau = 0.125
    got = oracle.topn_mass_rows(sq, sk, tau, p, np.arange(600))
    s = np.einsum("hik,hjk->hij", sq[0].astype(np.float64), sk[0].astype(np.float64))
    w = np.exp(tau * (s - s.max(axis=-1, keepdims=True))).reshape(600, 300)
    cum = np.cumsum(-np.sort(-w, axis=1), axis=1)
    want = np.stack([np.argmax(cum >= pk * cum[:, -1:], axis=1) + 1 for pk in p], axis=1)
    # equal up to fp64 rounding at an exact boundary (none is expected here)
    assert np.array_equal(got, want)


def test_mass_monotone_in_p_and_bounded():
    sq, sk, _ = _binarized((1, 1, 200, 64), seed=120)
    p = np.linspace(0.05, 1.0, 20)
    got = oracle.topn_mass_rows(sq, sk, 0.125, p, np.arange(200))
    assert (np.diff(got, axis=1) >= 0).all()
    assert (got >= 1).all() and (got <= 200).all()


@pytest.mark.parametrize("p", [0.0, -0.5, 1.5])
def test_mass_rejects_bad_p(p):
    sq, sk, _ = _binarized((1, 1, 10, 64), seed=130)
    with pytest.raises(ValueError):
        oracle.topn_mass_rows(sq, sk, 0.125, [p], [0])


# --------------------------------------------------------------- causal variant
# Query i sees keys 0..i and keeps min(N, i+1) of them; empty slots hold
# idx -1, logit 0, p 0.


def test_causal_last_row_is_the_full_row():
    sq, sk, v = _binarized((1, 2, 60, 64), seed=140)
    rows = np.array([59, 119])                    # last position of each head
    a = oracle.attention_causal_rows(sq, sk, v, 0.125, 12, rows)
    b = oracle.attention_rows(sq, sk, v, 0.125, 12, rows)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_causal_row_is_the_truncated_problem():
    # row i equals the non-causal answer on keys 0..i with N_i = min(N, i+1)
    sq, sk, v = _binarized((1, 1, 50, 64), seed=150)
    N = 9
    for i in (0, 3, 8, 9, 20, 49):
        idx, lg, p, out = oracle.attention_causal_rows(sq, sk, v, 0.125, N, [i])
        Ni = min(N, i + 1)
        sub = oracle.attention_rows(sq[:, :, :i + 1], sk[:, :, :i + 1], v[:, :, :i + 1],
                                    0.125, Ni, [i])
        assert np.array_equal(idx[0, :Ni], sub[0][0]) and (idx[0, Ni:] == -1).all()
        assert np.array_equal(lg[0, :Ni], sub[1][0]) and (lg[0, Ni:] == 0).all()
        assert np.array_equal(p[0, :Ni], sub[2][0]) and (p[0, Ni:] == 0).all()
        assert np.array_equal(out[0], sub[3][0])


def test_causal_dense_rows_match_masked_softmax():
    # with N = n every row keeps all visible keys: a dense masked softmax
    sq, sk, v = _binarized((1, 1, 40, 64), seed=160)
    tau = 0.2
    idx, lg, p, out = oracle.attention_causal_rows(sq, sk, v, tau, 40, np.arange(40))
    s = torch.tensor(sq[0, 0], dtype=torch.float64) @ torch.tensor(sk[0, 0], dtype=torch.float64).T
    mask = torch.tril(torch.ones(40, 40, dtype=torch.bool))
    w = torch.softmax((tau * s).masked_fill(~mask, float("-inf")), dim=-1)
    ref = (w @ torch.tensor(v[0, 0], dtype=torch.float64)).numpy()
    assert np.allclose(out, ref, rtol=1e-6, atol=1e-6)
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-12)
    assert (idx[0] == [0] + [-1] * 39).all() and out[0].tolist() == v[0, 0, 0].tolist()


# ------------------------------------------------- soft (tanh) codes, stages 1-2


def _soft_codes(shape, c, seed, min_abs=0.0, dup_keys=0):
    g = np.random.default_rng(seed)
    q = g.standard_normal(shape).astype(np.float32)
    k = g.standard_normal(shape).astype(np.float32)
    if min_abs:
        q = np.where(np.abs(q) < min_abs, np.float32(min_abs) * np.sign(q + 1e-30), q)
        k = np.where(np.abs(k) < min_abs, np.float32(min_abs) * np.sign(k + 1e-30), k)
    if dup_keys:
        k[:, :, dup_keys:2 * dup_keys] = k[:, :, :dup_keys]   # exact logit ties
    v = g.standard_normal(shape).astype(np.float32)
    sg = np.ones(shape[1], np.float32)
    return q, k, v, sg, oracle.soft_binarize(q, sg, c), oracle.soft_binarize(k, sg, c)


@pytest.mark.parametrize("x,sigma,c,want", [
    (0.0, 1.0, 1.0, 0.0),
    (math.log(2.0), 1.0, 1.0, 0.6),              # tanh(ln 2) = 3/5
    (0.5 * math.log(3.0), 1.0, 1.0, 0.5),        # tanh(ln sqrt 3) = 1/2
    (math.log(3.0), 1.0, 1.0, 0.8),              # tanh(ln 3) = 4/5
    (-math.log(3.0), 1.0, 1.0, -0.8),            # odd
    (0.3, 0.6, 2.0, math.tanh(1.0)),             # c * x / sigma = 1
    (1e-20, 1.0, 1.0, 1e-20),                    # tanh(u) = u below fp32 resolution
    (20.0, 1.0, 1.0, 1.0),                       # saturates to exactly +1 in fp32
    (-3.0, 1.0, 100.0, -1.0),
])
def test_soft_code_closed_forms(x, sigma, c, want):
    t = oracle.soft_binarize(np.full((1, 1, 1, 32), x, np.float32),
                             np.array([sigma], np.float32), c)
    # the argument is rounded to fp32 (slope of tanh <= 1) and so is the result
    assert np.all(np.abs(t.astype(np.float64) - want) <= 1.2e-7 * max(abs(want), 1e-13))


def test_soft_codes_bf16_path_matches_widened_fp32():
    x = torch.randn(1, 2, 8, 64, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    sg = np.array([0.7, 1.9], np.float32)
    a = oracle.soft_binarize(synth.to_oracle_array(x), sg, 1.5)
    b = oracle.soft_binarize(x.float().numpy(), sg, 1.5)
    assert np.array_equal(a, b)


def test_soft_codes_become_signs_at_large_c():
    q, _, _, sg, tq, _ = _soft_codes((1, 2, 20, 64), 1e4, seed=170, min_abs=0.01)
    assert np.array_equal(tq, oracle.binarize(q, sg).astype(np.float32))


def test_soft_attention_at_large_c_is_the_binarized_path():
    q, k, v, sg, tq, tk = _soft_codes((1, 2, 70, 64), 1e4, seed=171, min_abs=0.01)
    sq, sk = oracle.binarize(q, sg), oracle.binarize(k, sg)
    rows = np.arange(140)
    a = oracle.soft_attention_rows(tq, tk, v, 0.125, 9, rows)
    b = oracle.attention_rows(sq, sk, v, 0.125, 9, rows)
    assert np.array_equal(a[0], b[0])                     # same kept keys, same tie rule
    assert np.array_equal(a[1], b[1].astype(np.float64))
    assert np.allclose(a[2], b[2], rtol=0, atol=1e-14)
    assert np.array_equal(a[3], b[3])


def test_soft_logits_at_small_c_are_the_scaled_dot_product():
    # tanh(u) = u (1 - u^2/3 + ...): s / c^2 -> z_q . z_k as c -> 0
    q, k, _, sg, tq, tk = _soft_codes((1, 1, 30, 64), 1e-3, seed=172)
    s = oracle.soft_logits_rows(tq, tk, np.arange(30)) / 1e-6
    ref = q[0, 0].astype(np.float64) @ k[0, 0].astype(np.float64).T
    assert np.allclose(s, ref, rtol=1e-4, atol=1e-4)
    assert not np.allclose(s, ref.T, rtol=1e-2, atol=1e-2)     # orientation: row = query


def test_soft_logits_are_odd_in_the_keys():
    _, _, _, _, tq, tk = _soft_codes((1, 1, 16, 64), 0.8, seed=173)
    a = oracle.soft_logits_rows(tq, tk, np.arange(16))
    b = oracle.soft_logits_rows(tq, -tk, np.arange(16))
    assert np.array_equal(a, -b)
    assert np.all(np.abs(a) < 64)


def test_soft_topn_against_numpy_sort_with_exact_ties():
    _, _, v, _, tq, tk = _soft_codes((1, 2, 90, 64), 0.9, seed=174, dup_keys=30)
    rows = np.arange(180)
    N = 17
    idx, lg, p, _ = oracle.soft_attention_rows(tq, tk, v, 0.125, N, rows)
    s = oracle.soft_logits_rows(tq, tk, rows)
    for t in range(180):
        order = np.lexsort((np.arange(90), -s[t]))[:N]         # logit desc, index asc
        want = np.sort(order)
        assert np.array_equal(idx[t], want)
        assert np.array_equal(lg[t], s[t, want])
    # duplicated keys (j and j + 30) tie exactly; the lower index is kept first
    assert np.array_equal(s[:, :30], s[:, 30:60])
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-12)


def test_soft_N_equals_n_is_dense_softmax():
    _, _, v, _, tq, tk = _soft_codes((1, 1, 40, 64), 1.3, seed=175)
    tau = float(np.float32(0.3))                 # the oracle takes tau as fp32
    idx, lg, p, out = oracle.soft_attention_rows(tq, tk, v, tau, 40, np.arange(40))
    s = torch.tensor(oracle.soft_logits_rows(tq, tk, np.arange(40)))
    w = torch.softmax(tau * s, dim=-1)
    ref = (w @ torch.tensor(v[0, 0], dtype=torch.float64)).numpy()
    assert (idx == np.arange(40)).all()
    assert np.allclose(p, w.numpy(), rtol=1e-12, atol=1e-15)
    assert np.allclose(out, ref, rtol=1e-6, atol=1e-6)


def test_soft_given_set_is_a_softmax_over_exactly_those_keys():
    # any kept set, in any order: a library softmax of tau * s over the set
    # and a matrix product with the set's value rows
    _, _, v, _, tq, tk = _soft_codes((1, 2, 50, 64), 1.1, seed=176)
    g = np.random.default_rng(177)
    rows = np.arange(100)
    N = 11
    idx = np.stack([g.permutation(50)[:N] for _ in rows]).astype(np.int32)
    tau = float(np.float32(0.21))
    p, out = oracle.soft_attention_given(tq, tk, v, tau, idx, rows)
    s = oracle.soft_logits_rows(tq, tk, rows)
    for t, r in enumerate(rows):
        h = r // 50
        sel = torch.tensor(s[t, idx[t]])
        w = torch.softmax(tau * sel, dim=-1)
        ref = w @ torch.tensor(v[0, h][idx[t]], dtype=torch.float64)
        assert np.allclose(p[t], w.numpy(), rtol=1e-12, atol=1e-15)
        assert np.allclose(out[t], ref.numpy(), rtol=1e-12, atol=1e-12)
    # permuting a row's set permutes its weights and leaves its output
    perm = g.permutation(N)
    p2, out2 = oracle.soft_attention_given(tq, tk, v, tau, idx[:, perm], rows)
    assert np.allclose(p2, p[:, perm], rtol=1e-13, atol=1e-16)
    assert np.allclose(out2, out, rtol=1e-12, atol=1e-13)


def test_soft_given_oracle_set_reproduces_the_selecting_oracle():
    _, _, v, _, tq, tk = _soft_codes((1, 2, 90, 64), 0.9, seed=178, dup_keys=30)
    rows = np.arange(180)
    idx, _, p, out = oracle.soft_attention_rows(tq, tk, v, 0.125, 17, rows)
    p2, out2 = oracle.soft_attention_given(tq, tk, v, 0.125, idx, rows)
    assert np.array_equal(p2, p)
    assert np.array_equal(out2.astype(np.float32), out)


def test_soft_given_rejects_out_of_range_keys():
    _, _, v, _, tq, tk = _soft_codes((1, 1, 20, 64), 1.0, seed=179)
    bad = np.array([[0, 20]], np.int32)
    with pytest.raises(ValueError):
        oracle.soft_attention_given(tq, tk, v, 0.125, bad, np.arange(1))


# ------------------------------------------- straight-through backward


def _bwd_case(shape, seed):
    g = np.random.default_rng(seed)
    q, k, v, dout = (g.standard_normal(shape).astype(np.float32) for _ in range(4))
    sq = np.array([0.9, 1.3][:shape[1]], np.float32)
    sk = np.array([1.1, 0.7][:shape[1]], np.float32)
    return q, k, v, dout, sq, sk


def _autograd_bwd(q, k, v, dout, sgq, sgk, tau, N, clip):
    """The same gradients by torch autograd in float64: the sign replaced by
    its straight-through surrogate, the forward oracle's kept set as a
    fixed mask."""
    B, H, n, d = q.shape
    zq = q / sgq[None, :, None, None]                 # fp32, as the sign rule
    zk = k / sgk[None, :, None, None]
    idx = oracle.attention_rows(np.where(zq < 0, -1, 1).astype(np.int8),
                                np.where(zk < 0, -1, 1).astype(np.int8), v, tau, N,
                                np.arange(B * H * n))[0]
    kept = torch.zeros(B * H * n, n, dtype=torch.bool)
    kept[torch.arange(B * H * n)[:, None], torch.tensor(idx, dtype=torch.long)] = True
    kept = kept.reshape(B, H, n, n)

    def code(x, z, sg):
        xt = torch.tensor(x, dtype=torch.float64, requires_grad=True)
        zt = xt / torch.tensor(sg, dtype=torch.float64)[None, :, None, None]
        m = torch.tensor(np.abs(z) <= clip, dtype=torch.float64)
        sign = torch.tensor(np.where(z < 0, -1.0, 1.0))
        return xt, sign + (zt * m - (zt * m).detach())

    xq, bq = code(q, zq, sgq)
    xk, bk = code(k, zk, sgk)
    vt = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    s = (bq @ bk.transpose(-1, -2)).masked_fill(~kept, float("-inf"))
    o = torch.softmax(tau * s, dim=-1) @ vt
    (o * torch.tensor(dout, dtype=torch.float64)).sum().backward()
    return xq.grad.numpy(), xk.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("N,clip", [(7, 1.0), (40, 1.0), (5, float("inf")), (12, 0.4)])
def test_bwd_matches_torch_autograd(N, clip):
    q, k, v, dout, sgq, sgk = _bwd_case((1, 2, 40, 64), seed=180 + N)
    tau = float(np.float32(0.3))
    dq, dk, dv = oracle.attention_bwd(q, k, v, sgq, sgk, dout, tau, N, clip)
    aq, ak, av = _autograd_bwd(q, k, v, dout, sgq, sgk, tau, N, clip)
    assert np.allclose(dv, av, rtol=1e-10, atol=1e-12)
    assert np.allclose(dq, aq, rtol=1e-9, atol=1e-12)
    assert np.allclose(dk, ak, rtol=1e-9, atol=1e-12)
    assert np.abs(dq).max() > 1e-3 and np.abs(dk).max() > 1e-3      # not trivially zero


def test_bwd_dv_is_the_forward_difference_in_v():
    # the forward is linear in V: O(V + e E) - O(V) = e P E exactly
    q, k, v, dout, sgq, sgk = _bwd_case((1, 1, 30, 64), seed=190)
    sq, sk = oracle.binarize(q, sgq), oracle.binarize(k, sgk)
    _, _, dv = oracle.attention_bwd(q, k, v, sgq, sgk, dout, 0.25, 6)
    rows = np.arange(30)
    base = oracle.attention_rows(sq, sk, v, 0.25, 6, rows)[3].astype(np.float64)
    for j, c in [(0, 0), (7, 13), (29, 63)]:
        v2 = v.copy()
        v2[0, 0, j, c] += np.float32(0.5)
        o2 = oracle.attention_rows(sq, sk, v2, 0.25, 6, rows)[3].astype(np.float64)
        fd = ((o2 - base) * dout[0, 0].astype(np.float64)).sum() / 0.5
        assert abs(fd - dv[0, 0, j, c]) <= 1e-5 * max(1.0, abs(dv[0, 0, j, c]))


def test_bwd_closed_forms_N1_and_tau0():
    q, k, v, dout, sgq, sgk = _bwd_case((1, 2, 24, 64), seed=191)
    sq, sk = oracle.binarize(q, sgq), oracle.binarize(k, sgk)
    rows = np.arange(48)
    # N = 1: p = 1, so ds = 0 and dV_j sums dO of the rows whose one key is j
    dq, dk, dv = oracle.attention_bwd(q, k, v, sgq, sgk, dout, 0.3, 1)
    assert not dq.any() and not dk.any()
    idx = oracle.attention_rows(sq, sk, v, 0.3, 1, rows)[0][:, 0]
    want = np.zeros_like(dv)
    for r in rows:
        want[0, r // 24, idx[r]] += dout[0, r // 24, r % 24]
    assert np.allclose(dv, want, rtol=0, atol=1e-12)
    # tau = 0: uniform weights 1/N, again ds = 0
    dq, dk, dv = oracle.attention_bwd(q, k, v, sgq, sgk, dout, 0.0, 5)
    assert not dq.any() and not dk.any()
    idx = oracle.attention_rows(sq, sk, v, 0.0, 5, rows)[0]
    want = np.zeros_like(dv)
    for r in rows:
        for j in idx[r]:
            want[0, r // 24, j] += dout[0, r // 24, r % 24].astype(np.float64) / 5.0
    assert np.allclose(dv, want, rtol=0, atol=1e-12)


def test_bwd_clip_masks_exactly():
    q, k, v, dout, sgq, sgk = _bwd_case((1, 2, 30, 64), seed=192)
    a = oracle.attention_bwd(q, k, v, sgq, sgk, dout, 0.3, 8, clip=float("inf"))
    b = oracle.attention_bwd(q, k, v, sgq, sgk, dout, 0.3, 8, clip=0.5)
    zq = q / sgq[None, :, None, None]
    zk = k / sgk[None, :, None, None]
    assert np.array_equal(b[0], np.where(np.abs(zq) <= 0.5, a[0], 0.0))
    assert np.array_equal(b[1], np.where(np.abs(zk) <= 0.5, a[1], 0.0))
    assert np.array_equal(b[2], a[2])


def test_golden_handworked_soft():
    """Soft codes at tanh's closed forms (3/5, 4/5, 1/2): logits, kept set,
    weights and output of row 0 against the fixture's hand derivation."""
    import json
    import os
    case = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                       "handworked_soft_n4_d64.json")))
    n, d = case["n"], case["d"]
    val = {"ln(2)": math.log(2.0), "ln(3)": math.log(3.0), "-ln(3)": -math.log(3.0),
           "-ln(3)/2": -0.5 * math.log(3.0)}
    q = np.zeros((1, 1, n, d), np.float32)
    q[0, 0, 0] = val[case["q_row0"]]
    k = np.zeros((1, 1, n, d), np.float32)
    for r, spec in case["k_rows"].items():
        row = []
        for name, count in zip(spec[0::2], spec[1::2]):
            row += [val[name]] * count
        k[0, 0, int(r)] = row
    v = np.eye(n, d, dtype=np.float32)[None, None]
    sg = np.array(case["sigma"], np.float32)
    tq, tk = oracle.soft_binarize(q, sg, case["c"]), oracle.soft_binarize(k, sg, case["c"])
    exp = case["expected"]
    s = oracle.soft_logits_rows(tq, tk, [0])[0]
    assert np.allclose(s, [_golden.closed_form(e) for e in exp["logits_row0_all"]],
                       rtol=0, atol=1e-4)
    idx, lg, p, out = oracle.soft_attention_rows(tq, tk, v, case["tau"], case["N"], [0])
    assert idx[0].tolist() == exp["idx"]
    assert np.allclose(p[0], [_golden.closed_form(e) for e in exp["p"]], rtol=1e-5, atol=0)
    want = np.zeros(d)
    for col, e in exp["out_nonzero"].items():
        want[int(col)] = _golden.closed_form(e)
    assert np.allclose(out[0], want, rtol=1e-5, atol=1e-7)


def test_golden_handworked_bwd():
    """Straight-through backward of a two-key row worked by hand: the
    gradients are closed forms in a = 1/(1+e^-2), b = e^-2/(1+e^-2)."""
    import json
    import os
    case = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                       "handworked_bwd_n2_d64.json")))
    n, d = case["n"], case["d"]
    q = np.full((1, 1, n, d), 0.5, np.float32)
    q[0, 0, :, 3] = 1.5                              # past the clip; the sign is still +1
    k = np.full((1, 1, n, d), 0.5, np.float32)
    k[0, 0, 1, :8] = -0.5
    v = np.eye(n, d, dtype=np.float32)[None, None]
    dout = np.zeros((1, 1, n, d), np.float32)
    dout[0, 0, 0, 0] = 1.0
    one = np.ones(1, np.float32)
    dq, dk, dv = oracle.attention_bwd(q, k, v, one, one, dout, case["tau"], case["N"],
                                      case["clip"])
    e = {key: _golden.closed_form(x) for key, x in case["expected"].items()}
    want_q = np.zeros((n, d))
    want_q[0, :8] = e["dq_row0_first8_except3"]
    want_q[0, 3] = 0.0
    assert np.allclose(dq[0, 0], want_q, rtol=1e-12, atol=1e-15)
    assert np.allclose(dk[0, 0, 0], e["dk_row0"], rtol=1e-12, atol=0)
    assert np.allclose(dk[0, 0, 1], e["dk_row1"], rtol=1e-12, atol=0)
    want_v = np.zeros((n, d))
    want_v[0, 0], want_v[1, 0] = e["dv_row0_col0"], e["dv_row1_col0"]
    assert np.allclose(dv[0, 0], want_v, rtol=1e-12, atol=1e-15)
