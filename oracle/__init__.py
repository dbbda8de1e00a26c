"""CPU oracle for the HAD binarized top-N attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  It is a plain,
slow and obviously correct restatement of the method (C loops driven from
numpy), written from "Hamming Attention Distillation: Binarizing Keys and
Queries for Efficient Long-Context Transformers" (arXiv 2502.01770) as
summarised on its pith.science review page ("What carries the argument":
standardize by sigma_Q/sigma_K, sign-quantize, Hamming logits, top-N mask,
softmax over the kept logits, value product in full precision; Eqs. 4-7 and
Eq. 12).  It shares no code with the CUDA library.

Every function takes numpy arrays.  bf16 tensors are passed as their raw
16-bit patterns (``np.uint16``); fp32 tensors as ``np.float32``.

Pins (checked in ``tests/test_oracle_pins.py``): sign edge values, the
LSB-first bit order, the identity dot = d - 2*popcount(xor), logits against a
float64 matrix product of the signs, top-N against independent sorts and a
histogram-threshold selection, the N = n case against a dense library
softmax, closed forms (all keys equal, N = 1), and a hand-worked example
under ``tests/golden/``.  The soft (tanh) codes of the training stages are
pinned by tanh closed forms (tanh(ln 2) = 3/5, tanh(ln 3) = 4/5, ...), their
limits (signs at large c, the scaled dot product at small c), oddness, a
numpy sort with exact ties, and a dense library softmax at N = n; their
softmax over a GIVEN kept set by a library softmax and matrix product over
that set, and by the selecting oracle on its own set.  The
straight-through backward is pinned by torch autograd in float64 (the
surrogate sign, the kept set as a fixed mask), by finite differences of the
forward in V, and by closed forms (N = 1 and tau = 0 give dQ = dK = 0).  No
function is left unpinned.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lp, c_long, c_int = ctypes.c_void_p, ctypes.c_long, ctypes.c_int
        lib.had_oracle_binarize.argtypes = [lp, c_int, lp, c_long, c_long,
                                            c_long, c_long, lp]
        lib.had_oracle_binarize.restype = None
        lib.had_oracle_pack.argtypes = [lp, c_long, c_long, lp]
        lib.had_oracle_pack.restype = None
        lib.had_oracle_logits_rows.argtypes = [lp, lp, c_long, c_long, c_long,
                                               c_long, lp, c_long, lp, c_int]
        lib.had_oracle_logits_rows.restype = None
        lib.had_oracle_attention_rows.argtypes = [
            lp, lp, lp, c_int, c_long, c_long, c_long, c_long, c_long,
            ctypes.c_float, lp, c_long, lp, lp, lp, lp, c_int]
        lib.had_oracle_attention_rows.restype = c_int
        lib.had_oracle_attention_causal_rows.argtypes = [
            lp, lp, lp, c_int, c_long, c_long, c_long, c_long, c_long,
            ctypes.c_float, lp, c_long, lp, lp, lp, lp, c_int]
        lib.had_oracle_attention_causal_rows.restype = c_int
        lib.had_oracle_topn_mass_rows.argtypes = [
            lp, lp, c_long, c_long, c_long, c_long, ctypes.c_double, lp, c_int, lp,
            c_long, lp, c_int]
        lib.had_oracle_topn_mass_rows.restype = c_int
        lib.had_oracle_soft_binarize.argtypes = [lp, c_int, lp, ctypes.c_float, c_long,
                                                 c_long, c_long, c_long, lp]
        lib.had_oracle_soft_binarize.restype = None
        lib.had_oracle_soft_logits_rows.argtypes = [lp, lp, c_long, c_long, c_long,
                                                    c_long, lp, c_long, lp, c_int]
        lib.had_oracle_soft_logits_rows.restype = None
        lib.had_oracle_soft_attention_rows.argtypes = [
            lp, lp, lp, c_int, c_long, c_long, c_long, c_long, c_long,
            ctypes.c_float, lp, c_long, lp, lp, lp, lp, c_int]
        lib.had_oracle_soft_attention_rows.restype = c_int
        lib.had_oracle_soft_attention_given.argtypes = [
            lp, lp, lp, c_int, c_long, c_long, c_long, c_long, c_long,
            ctypes.c_float, lp, c_long, lp, lp, lp]
        lib.had_oracle_soft_attention_given.restype = c_int
        lib.had_oracle_attention_bwd.argtypes = [
            lp, lp, lp, c_int, lp, lp, lp, c_long, c_long, c_long, c_long, c_long,
            ctypes.c_float, ctypes.c_float, lp, lp, lp, c_int]
        lib.had_oracle_attention_bwd.restype = c_int
        lib.had_oracle_max_threads.argtypes = []
        lib.had_oracle_max_threads.restype = c_int
        _lib = lib
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def _is_bf16(x):
    if x.dtype == np.uint16:
        return 1
    if x.dtype == np.float32:
        return 0
    raise TypeError("oracle inputs are float32 or bf16 bit patterns (uint16), got %s" % x.dtype)


def max_threads() -> int:
    """OpenMP threads the oracle uses by default."""
    return int(_load().had_oracle_max_threads())


def binarize(x, sigma):
    """Signs (+1/-1, int8) of x / sigma[h] for x of shape [B,H,n,d]."""
    x = np.ascontiguousarray(x)
    sigma = np.ascontiguousarray(sigma, dtype=np.float32)
    B, H, n, d = x.shape
    assert sigma.shape == (H,)
    out = np.empty((B, H, n, d), dtype=np.int8)
    _load().had_oracle_binarize(_ptr(x), _is_bf16(x), _ptr(sigma), B, H, n, d, _ptr(out))
    return out


def pack(signs):
    """Pack +/-1 signs [..., d] into uint32 words [..., d/32], LSB first, 1 = -1."""
    signs = np.ascontiguousarray(signs, dtype=np.int8)
    d = signs.shape[-1]
    assert d % 32 == 0
    rows = signs.size // d
    out = np.empty(signs.shape[:-1] + (d // 32,), dtype=np.uint32)
    _load().had_oracle_pack(_ptr(signs), rows, d, _ptr(out))
    return out


def _rows_array(rows, total):
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    if rows.size and (rows.min() < 0 or rows.max() >= total):
        raise ValueError("row id out of range")
    return rows


def logits_rows(sq, sk, rows, threads=0):
    """Integer logits [len(rows), n] of the given flat query rows."""
    sq = np.ascontiguousarray(sq, dtype=np.int8)
    sk = np.ascontiguousarray(sk, dtype=np.int8)
    B, H, n, d = sq.shape
    rows = _rows_array(rows, B * H * n)
    out = np.empty((rows.size, n), dtype=np.int32)
    _load().had_oracle_logits_rows(_ptr(sq), _ptr(sk), B, H, n, d, _ptr(rows),
                                   rows.size, _ptr(out), int(threads))
    return out


def attention_rows(sq, sk, v, tau, N, rows, threads=0):
    """Top-N binarized attention for the given flat query rows.

    Returns (idx [R,N] int32 ascending, logits [R,N] int16, p [R,N] float64,
    out [R,d] float32) where R = len(rows) and a flat row id is
    (b*H + h)*n + i.
    """
    sq = np.ascontiguousarray(sq, dtype=np.int8)
    sk = np.ascontiguousarray(sk, dtype=np.int8)
    v = np.ascontiguousarray(v)
    B, H, n, d = sq.shape
    assert sk.shape == sq.shape and v.shape == sq.shape
    rows = _rows_array(rows, B * H * n)
    R = rows.size
    idx = np.empty((R, N), dtype=np.int32)
    lg = np.empty((R, N), dtype=np.int16)
    p = np.empty((R, N), dtype=np.float64)
    out = np.empty((R, d), dtype=np.float32)
    rc = _load().had_oracle_attention_rows(
        _ptr(sq), _ptr(sk), _ptr(v), _is_bf16(v), B, H, n, d, int(N),
        ctypes.c_float(float(tau)), _ptr(rows), R, _ptr(idx), _ptr(lg), _ptr(p),
        _ptr(out), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (N must be in [1, n])")
    return idx, lg, p, out


def attention_causal_rows(sq, sk, v, tau, N, rows, threads=0):
    """Causal top-N attention for the given flat query rows: query i of a head
    sees keys 0..i and keeps min(N, i+1) of them.  Same outputs as
    attention_rows; empty slots hold idx -1, logit 0, p 0."""
    sq = np.ascontiguousarray(sq, dtype=np.int8)
    sk = np.ascontiguousarray(sk, dtype=np.int8)
    v = np.ascontiguousarray(v)
    B, H, n, d = sq.shape
    assert sk.shape == sq.shape and v.shape == sq.shape
    rows = _rows_array(rows, B * H * n)
    R = rows.size
    idx = np.empty((R, N), dtype=np.int32)
    lg = np.empty((R, N), dtype=np.int16)
    p = np.empty((R, N), dtype=np.float64)
    out = np.empty((R, d), dtype=np.float32)
    rc = _load().had_oracle_attention_causal_rows(
        _ptr(sq), _ptr(sk), _ptr(v), _is_bf16(v), B, H, n, d, int(N),
        ctypes.c_float(float(tau)), _ptr(rows), R, _ptr(idx), _ptr(lg), _ptr(p),
        _ptr(out), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (N must be in [1, n])")
    return idx, lg, p, out


def topn_mass_rows(sq, sk, tau, p, rows, threads=0):
    """Top-N mass retention for the given flat query rows.

    Returns nmin [R, len(p)] int32: for each row and threshold p_k in (0, 1],
    the smallest N whose N largest weights of the full softmax over all keys
    (temperature tau, in fp64) hold at least p_k of the row's total.
    """
    sq = np.ascontiguousarray(sq, dtype=np.int8)
    sk = np.ascontiguousarray(sk, dtype=np.int8)
    B, H, n, d = sq.shape
    assert sk.shape == sq.shape
    rows = _rows_array(rows, B * H * n)
    pv = np.ascontiguousarray(p, dtype=np.float64).reshape(-1)
    out = np.empty((rows.size, pv.size), dtype=np.int32)
    rc = _load().had_oracle_topn_mass_rows(
        _ptr(sq), _ptr(sk), B, H, n, d, float(tau), _ptr(pv), int(pv.size), _ptr(rows),
        rows.size, _ptr(out), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (each p must be in (0, 1])")
    return out


def attention(sq, sk, v, tau, N, threads=0):
    """All rows: (idx, logits, p, out) shaped [B,H,n,N] / [B,H,n,d]."""
    B, H, n, d = sq.shape
    idx, lg, p, out = attention_rows(sq, sk, v, tau, N, np.arange(B * H * n), threads)
    return (idx.reshape(B, H, n, N), lg.reshape(B, H, n, N),
            p.reshape(B, H, n, N), out.reshape(B, H, n, d))


def lib_path() -> str:
    return os.path.abspath(_build.LIB)


def soft_binarize(x, sigma, c):
    """Soft codes tanh(c * x / sigma[h]) (fp32) for x of shape [B,H,n,d]:
    the forward pass of the tanh training stages."""
    x = np.ascontiguousarray(x)
    sigma = np.ascontiguousarray(sigma, dtype=np.float32)
    B, H, n, d = x.shape
    assert sigma.shape == (H,)
    out = np.empty((B, H, n, d), dtype=np.float32)
    _load().had_oracle_soft_binarize(_ptr(x), _is_bf16(x), _ptr(sigma), ctypes.c_float(c),
                                     B, H, n, d, _ptr(out))
    return out


def soft_logits_rows(tq, tk, rows, threads=0):
    """fp64 logits [len(rows), n] of the soft codes for the given flat query rows."""
    tq = np.ascontiguousarray(tq, dtype=np.float32)
    tk = np.ascontiguousarray(tk, dtype=np.float32)
    B, H, n, d = tq.shape
    assert tk.shape == tq.shape
    rows = _rows_array(rows, B * H * n)
    out = np.empty((rows.size, n), dtype=np.float64)
    _load().had_oracle_soft_logits_rows(_ptr(tq), _ptr(tk), B, H, n, d, _ptr(rows), rows.size,
                                        _ptr(out), int(threads))
    return out


def soft_attention_rows(tq, tk, v, tau, N, rows, threads=0):
    """Top-N attention on the soft codes for the given flat query rows.

    Returns (idx [R, N] int32 ascending, logits [R, N] float64,
    p [R, N] float64, out [R, d] float32)."""
    tq = np.ascontiguousarray(tq, dtype=np.float32)
    tk = np.ascontiguousarray(tk, dtype=np.float32)
    v = np.ascontiguousarray(v)
    B, H, n, d = tq.shape
    assert tk.shape == tq.shape and v.shape == tq.shape
    rows = _rows_array(rows, B * H * n)
    R = rows.size
    idx = np.empty((R, N), dtype=np.int32)
    lg = np.empty((R, N), dtype=np.float64)
    p = np.empty((R, N), dtype=np.float64)
    out = np.empty((R, d), dtype=np.float32)
    rc = _load().had_oracle_soft_attention_rows(
        _ptr(tq), _ptr(tk), _ptr(v), _is_bf16(v), B, H, n, d, int(N),
        ctypes.c_float(float(tau)), _ptr(rows), R, _ptr(idx), _ptr(lg), _ptr(p),
        _ptr(out), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (N must be in [1, n])")
    return idx, lg, p, out


def soft_attention_given(tq, tk, v, tau, idx, rows):
    """Softmax and value product on the soft codes over a GIVEN kept set.

    idx [R, N] int32 holds each listed row's kept keys; returns
    (p [R, N] float64 in idx's order, out [R, d] float64)."""
    tq = np.ascontiguousarray(tq, dtype=np.float32)
    tk = np.ascontiguousarray(tk, dtype=np.float32)
    v = np.ascontiguousarray(v)
    B, H, n, d = tq.shape
    assert tk.shape == tq.shape and v.shape == tq.shape
    rows = _rows_array(rows, B * H * n)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    R, N = idx.shape
    assert R == rows.size
    p = np.empty((R, N), dtype=np.float64)
    out = np.empty((R, d), dtype=np.float64)
    rc = _load().had_oracle_soft_attention_given(
        _ptr(tq), _ptr(tk), _ptr(v), _is_bf16(v), B, H, n, d, int(N),
        ctypes.c_float(float(tau)), _ptr(rows), R, _ptr(idx), _ptr(p), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (indices must lie in [0, n))")
    return p, out


def attention_bwd(q, k, v, sigma_q, sigma_k, dout, tau, N, clip=1.0, threads=0):
    """Straight-through backward of the binarized top-N forward.

    q, k, v are [B,H,n,d] (float32, or bf16 bit patterns as uint16, all the
    same); dout is float32 [B,H,n,d].  Returns (dq, dk, dv) as float64
    [B,H,n,d]: the sign passes the gradient where |x / sigma| <= clip."""
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    dout = np.ascontiguousarray(dout, dtype=np.float32)
    sigma_q = np.ascontiguousarray(sigma_q, dtype=np.float32)
    sigma_k = np.ascontiguousarray(sigma_k, dtype=np.float32)
    B, H, n, d = q.shape
    assert k.shape == q.shape and v.shape == q.shape and dout.shape == q.shape
    assert q.dtype == k.dtype == v.dtype
    dq = np.empty((B, H, n, d), dtype=np.float64)
    dk = np.empty_like(dq)
    dv = np.empty_like(dq)
    rc = _load().had_oracle_attention_bwd(
        _ptr(q), _ptr(k), _ptr(v), _is_bf16(q), _ptr(sigma_q), _ptr(sigma_k), _ptr(dout),
        B, H, n, d, int(N), ctypes.c_float(float(tau)), ctypes.c_float(float(clip)),
        _ptr(dq), _ptr(dk), _ptr(dv), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (N must be in [1, n])")
    return dq, dk, dv
