"""ctypes binding of the C ABI in include/had.h (argument marshalling only).

Each function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks that tensors are contiguous CUDA tensors of
the right shape and dtype, allocates missing outputs with torch (torch is
used for device memory and streams only), passes raw pointers and the current
CUDA stream, and raises ``HadError`` on a non-OK status.  Every step of the
forward pass runs in the CUDA kernels of ``libhad.so``; there is no CPU
fallback, and importing this module fails if the library cannot be loaded.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhad.so")

HAD_OK = 0
HAD_ERR_INVALID_ARG = 1
HAD_ERR_UNSUPPORTED = 2
HAD_ERR_WORKSPACE = 3
HAD_ERR_CUDA = 4
HAD_ERR_BAD_SIGMA = 5
HAD_ERR_TIMEOUT = 6

HAD_BF16 = 0
HAD_F32 = 1

HAD_OP_BINARIZE_PACK = 0
HAD_OP_HAMMING_TOPN = 1
HAD_OP_ATTENTION_FWD = 2
HAD_OP_SPARSE_SOFTMAX_AV = 3
HAD_OP_ATTENTION_PREPARE = 4
HAD_OP_ATTENTION_CORE = 5
HAD_OP_TOPN_MASS = 6
HAD_OP_ATTENTION_CAUSAL = 7
HAD_OP_SOFT_BINARIZE = 8
HAD_OP_SOFT_TOPN = 9
HAD_OP_SOFT_SOFTMAX_AV = 10
HAD_OP_SOFT_ATTENTION_FWD = 11
HAD_OP_ATTENTION_BWD = 12


class HadError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {had_status_string(status)} ({status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m sparse_attention_sigma_b200.build` "
            "(the HAD path has no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    sig = {
        "had_binarize_pack": [vp, i32, vp, i32, i32, i32, i32, vp, vp, vp],
        "had_hamming_topn": [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, sz, vp, vp],
        "had_sparse_softmax_av": [vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp, vp],
        "had_attention_fwd": [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, f32, vp, vp, vp,
                              vp, sz, vp, vp],
        "had_attention_fwd_noalloc": [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, f32, vp,
                                      vp, vp],
        "had_attention_prepare": [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, vp, sz, vp, vp],
        "had_attention_core": [vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp, vp, sz, vp, vp],
        "had_topn_mass": [vp, vp, i32, i32, i32, i32, f32, vp, i32, vp, vp, vp],
        "had_hamming_topn_causal": [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp],
        "had_attention_causal_fwd": [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, f32, vp,
                                     vp, vp, vp, sz, vp, vp],
        "had_soft_binarize": [vp, i32, vp, f32, i32, i32, i32, i32, vp, vp, vp],
        "had_soft_topn": [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, sz, vp, vp],
        "had_soft_softmax_av": [vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp, vp],
        "had_soft_attention_fwd": [vp, vp, vp, i32, vp, vp, f32, i32, i32, i32, i32, i32, f32,
                                   vp, vp, sz, vp, vp],
        "had_attention_bwd": [vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32,
                              f32, vp, vp, vp, vp, sz, vp, vp],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.had_workspace_bytes.argtypes = [i32] * 6
    lib.had_workspace_bytes.restype = ctypes.c_size_t
    lib.had_launch_count.argtypes = [i32] * 6
    lib.had_launch_count.restype = ctypes.c_int
    lib.had_attention_window_misses.argtypes = [vp, sz, i32, i32, i32, i32, i32, vp, vp]
    lib.had_attention_window_misses.restype = ctypes.c_int
    lib.had_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.had_set_wait_limit_ns.restype = ctypes.c_ulonglong
    lib.had_noalloc_scratch_bytes.argtypes = []
    lib.had_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.had_status_string.argtypes = [ctypes.c_int]
    lib.had_status_string.restype = ctypes.c_char_p
    return lib


_lib = _load()


def had_status_string(status: int) -> str:
    return _lib.had_status_string(int(status)).decode()


def had_workspace_bytes(op: int, B: int, H: int, n: int, d: int, N: int) -> int:
    v = _lib.had_workspace_bytes(op, B, H, n, d, N)
    return -1 if v == ctypes.c_size_t(-1).value else int(v)


def had_launch_count(op: int, B: int, H: int, n: int, d: int, N: int) -> int:
    return int(_lib.had_launch_count(op, B, H, n, d, N))


def _check(status, where):
    if status != HAD_OK:
        raise HadError(status, where)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _dev(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the HAD library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return HAD_BF16
    if t.dtype == torch.float32:
        return HAD_F32
    raise TypeError(f"Q/K/V must be bfloat16 or float32, got {t.dtype}")


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _shape4(x, name):
    if x.dim() != 4:
        raise ValueError(f"{name} must be [B, H, n, d]")
    return tuple(int(v) for v in x.shape)


def had_binarize_pack(x, sigma, bits=None, dev_status=None, stream=None):
    """Standardize by sigma[h], sign, pack to uint32 words; returns bits [B,H,n,d/32]."""
    _dev(x, "x")
    B, H, n, d = _shape4(x, "x")
    _dev(sigma, "sigma", torch.float32, (H,))
    if bits is None:
        bits = torch.empty((B, H, n, d // 32), dtype=torch.int32, device=x.device)
    _dev(bits, "bits", torch.int32, (B, H, n, d // 32))
    st = _lib.had_binarize_pack(_ptr(x), _dtype_code(x), _ptr(sigma), B, H, n, d, _ptr(bits),
                                _ptr(dev_status), _stream(stream))
    _check(st, "had_binarize_pack")
    return bits


def had_hamming_topn(qbits, kbits, d, N, idx=None, logits=None, ws=None, dev_status=None,
                     stream=None, want_logits=True):
    """Exact top-N of the Hamming logits; returns (idx [B,H,n,N] int32, logits int16 or None)."""
    _dev(qbits, "qbits", torch.int32)
    B, H, n, w = _shape4(qbits, "qbits")
    if w * 32 != d:
        raise ValueError("qbits last dimension must be d/32")
    _dev(kbits, "kbits", torch.int32, (B, H, n, w))
    if idx is None:
        idx = torch.empty((B, H, n, N), dtype=torch.int32, device=qbits.device)
    _dev(idx, "idx", torch.int32, (B, H, n, N))
    if logits is None and want_logits:
        logits = torch.empty((B, H, n, N), dtype=torch.int16, device=qbits.device)
    if logits is not None:
        _dev(logits, "logits", torch.int16, (B, H, n, N))
    need = had_workspace_bytes(HAD_OP_HAMMING_TOPN, B, H, n, d, N)
    if need < 0:
        raise HadError(HAD_ERR_UNSUPPORTED, "had_hamming_topn")
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=qbits.device)
    st = _lib.had_hamming_topn(_ptr(qbits), _ptr(kbits), B, H, n, d, N, _ptr(idx), _ptr(logits),
                               _ptr(ws), 0 if ws is None else ws.numel(), _ptr(dev_status),
                               _stream(stream))
    _check(st, "had_hamming_topn")
    return idx, logits


def had_hamming_topn_causal(qbits, kbits, d, N, idx=None, logits=None, dev_status=None,
                            stream=None, want_logits=True):
    """Causal top-N: query i keeps the min(N, i+1) best of keys 0..i, slots past
    that hold idx -1 / logit 0; returns (idx [B,H,n,N] int32, logits int16 or None)."""
    _dev(qbits, "qbits", torch.int32)
    B, H, n, w = _shape4(qbits, "qbits")
    if w * 32 != d:
        raise ValueError("qbits last dimension must be d/32")
    _dev(kbits, "kbits", torch.int32, (B, H, n, w))
    if idx is None:
        idx = torch.empty((B, H, n, N), dtype=torch.int32, device=qbits.device)
    _dev(idx, "idx", torch.int32, (B, H, n, N))
    if logits is None and want_logits:
        logits = torch.empty((B, H, n, N), dtype=torch.int16, device=qbits.device)
    if logits is not None:
        _dev(logits, "logits", torch.int16, (B, H, n, N))
    st = _lib.had_hamming_topn_causal(_ptr(qbits), _ptr(kbits), B, H, n, d, N, _ptr(idx),
                                      _ptr(logits), _ptr(dev_status), _stream(stream))
    _check(st, "had_hamming_topn_causal")
    return idx, logits


def had_attention_causal_fwd(Q, K, V, sigma_q, sigma_k, N, tau, out=None, dbg_idx=None,
                             dbg_logits=None, ws=None, dev_status=None, stream=None):
    """Causal binarized top-N attention forward on the fused path (query i sees
    keys 0..i, keeps min(N, i+1)); returns out [B,H,n,d] float32."""
    _dev(Q, "Q")
    B, H, n, d = _shape4(Q, "Q")
    _dev(K, "K", Q.dtype, (B, H, n, d))
    _dev(V, "V", Q.dtype, (B, H, n, d))
    _dev(sigma_q, "sigma_q", torch.float32, (H,))
    _dev(sigma_k, "sigma_k", torch.float32, (H,))
    if out is None:
        out = torch.empty((B, H, n, d), dtype=torch.float32, device=Q.device)
    _dev(out, "out", torch.float32, (B, H, n, d))
    if dbg_idx is not None:
        _dev(dbg_idx, "dbg_idx", torch.int32, (B, H, n, N))
    if dbg_logits is not None:
        _dev(dbg_logits, "dbg_logits", torch.int16, (B, H, n, N))
    need = had_workspace_bytes(HAD_OP_ATTENTION_CAUSAL, B, H, n, d, N)
    if need < 0:
        raise HadError(HAD_ERR_UNSUPPORTED if d not in (64, 128) else HAD_ERR_INVALID_ARG,
                       "had_attention_causal_fwd")
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=Q.device)
    st = _lib.had_attention_causal_fwd(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(sigma_q),
                                       _ptr(sigma_k), B, H, n, d, N, ctypes.c_float(tau),
                                       _ptr(out), _ptr(dbg_idx), _ptr(dbg_logits), _ptr(ws),
                                       ws.numel(), _ptr(dev_status), _stream(stream))
    _check(st, "had_attention_causal_fwd")
    return out


def had_soft_binarize(x, sigma, c, t=None, dev_status=None, stream=None):
    """Soft codes tanh(c * x / sigma[h]) as float32 [B,H,n,d] (tanh training stages)."""
    _dev(x, "x")
    B, H, n, d = _shape4(x, "x")
    _dev(sigma, "sigma", torch.float32, (H,))
    if t is None:
        t = torch.empty((B, H, n, d), dtype=torch.float32, device=x.device)
    _dev(t, "t", torch.float32, (B, H, n, d))
    st = _lib.had_soft_binarize(_ptr(x), _dtype_code(x), _ptr(sigma), ctypes.c_float(c), B, H,
                                n, d, _ptr(t), _ptr(dev_status), _stream(stream))
    _check(st, "had_soft_binarize")
    return t


def had_soft_topn(tq, tk, N, idx=None, logits=None, ws=None, dev_status=None, stream=None,
                  want_logits=True):
    """Top-N of the soft logits tq . tk; returns (idx int32, logits float32 or None)."""
    _dev(tq, "tq", torch.float32)
    B, H, n, d = _shape4(tq, "tq")
    _dev(tk, "tk", torch.float32, (B, H, n, d))
    if idx is None:
        idx = torch.empty((B, H, n, N), dtype=torch.int32, device=tq.device)
    _dev(idx, "idx", torch.int32, (B, H, n, N))
    if logits is None and want_logits:
        logits = torch.empty((B, H, n, N), dtype=torch.float32, device=tq.device)
    if logits is not None:
        _dev(logits, "logits", torch.float32, (B, H, n, N))
    need = had_workspace_bytes(HAD_OP_SOFT_TOPN, B, H, n, d, N)
    if need < 0:
        raise HadError(HAD_ERR_UNSUPPORTED if d not in (64, 128) else HAD_ERR_INVALID_ARG,
                       "had_soft_topn")
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=tq.device)
    st = _lib.had_soft_topn(_ptr(tq), _ptr(tk), B, H, n, d, N, _ptr(idx), _ptr(logits),
                            _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream))
    _check(st, "had_soft_topn")
    return idx, logits


def had_soft_softmax_av(idx, logits, V, tau, out=None, p=None, want_p=False, dev_status=None,
                        stream=None):
    """Softmax over kept fp32 logits and sparse product with V; returns (out, p or None)."""
    _dev(V, "V")
    B, H, n, d = _shape4(V, "V")
    _dev(idx, "idx", torch.int32)
    N = int(idx.shape[-1])
    _dev(idx, "idx", torch.int32, (B, H, n, N))
    _dev(logits, "logits", torch.float32, (B, H, n, N))
    if out is None:
        out = torch.empty((B, H, n, d), dtype=torch.float32, device=V.device)
    _dev(out, "out", torch.float32, (B, H, n, d))
    if p is None and want_p:
        p = torch.empty((B, H, n, N), dtype=torch.float32, device=V.device)
    if p is not None:
        _dev(p, "p", torch.float32, (B, H, n, N))
    st = _lib.had_soft_softmax_av(_ptr(idx), _ptr(logits), _ptr(V), _dtype_code(V), B, H, n, d,
                                  N, ctypes.c_float(tau), _ptr(out), _ptr(p), _ptr(dev_status),
                                  _stream(stream))
    _check(st, "had_soft_softmax_av")
    return out, p


def had_soft_attention_fwd(Q, K, V, sigma_q, sigma_k, c, N, tau, out=None, ws=None,
                           dev_status=None, stream=None):
    """Top-N attention on the soft codes tanh(c x / sigma); returns out [B,H,n,d] float32."""
    _dev(Q, "Q")
    B, H, n, d = _shape4(Q, "Q")
    _dev(K, "K", Q.dtype, (B, H, n, d))
    _dev(V, "V", Q.dtype, (B, H, n, d))
    _dev(sigma_q, "sigma_q", torch.float32, (H,))
    _dev(sigma_k, "sigma_k", torch.float32, (H,))
    if out is None:
        out = torch.empty((B, H, n, d), dtype=torch.float32, device=Q.device)
    _dev(out, "out", torch.float32, (B, H, n, d))
    need = had_workspace_bytes(HAD_OP_SOFT_ATTENTION_FWD, B, H, n, d, N)
    if need < 0:
        raise HadError(HAD_ERR_UNSUPPORTED if d not in (64, 128) else HAD_ERR_INVALID_ARG,
                       "had_soft_attention_fwd")
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=Q.device)
    st = _lib.had_soft_attention_fwd(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(sigma_q),
                                     _ptr(sigma_k), ctypes.c_float(c), B, H, n, d, N,
                                     ctypes.c_float(tau), _ptr(out), _ptr(ws), ws.numel(),
                                     _ptr(dev_status), _stream(stream))
    _check(st, "had_soft_attention_fwd")
    return out


def had_attention_bwd(Q, K, V, sigma_q, sigma_k, dout, N, tau, clip=1.0, idx=None, logits=None,
                      dq=None, dk=None, dv=None, ws=None, dev_status=None, stream=None):
    """Straight-through backward of had_attention_fwd; returns (dq, dk, dv) float32.
    idx/logits: the forward's kept set (e.g. had_attention_fwd's debug
    outputs), or None to recompute it."""
    _dev(Q, "Q")
    B, H, n, d = _shape4(Q, "Q")
    _dev(K, "K", Q.dtype, (B, H, n, d))
    _dev(V, "V", Q.dtype, (B, H, n, d))
    _dev(sigma_q, "sigma_q", torch.float32, (H,))
    _dev(sigma_k, "sigma_k", torch.float32, (H,))
    _dev(dout, "dout", torch.float32, (B, H, n, d))
    if (idx is None) != (logits is None):
        raise ValueError("give both idx and logits, or neither")
    if idx is not None:
        _dev(idx, "idx", torch.int32, (B, H, n, N))
        _dev(logits, "logits", torch.int16, (B, H, n, N))
    outs = []
    for t, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        if t is None:
            t = torch.empty((B, H, n, d), dtype=torch.float32, device=Q.device)
        _dev(t, name, torch.float32, (B, H, n, d))
        outs.append(t)
    need = had_workspace_bytes(HAD_OP_ATTENTION_BWD, B, H, n, d, N)
    if need < 0:
        raise HadError(HAD_ERR_UNSUPPORTED if d not in (64, 128) else HAD_ERR_INVALID_ARG,
                       "had_attention_bwd")
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=Q.device)
    st = _lib.had_attention_bwd(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(sigma_q),
                                _ptr(sigma_k), _ptr(dout), _ptr(idx), _ptr(logits), B, H, n,
                                d, N, ctypes.c_float(tau),
                                ctypes.c_float(clip), _ptr(outs[0]), _ptr(outs[1]),
                                _ptr(outs[2]), _ptr(ws), ws.numel(), _ptr(dev_status),
                                _stream(stream))
    _check(st, "had_attention_bwd")
    return tuple(outs)


def had_topn_mass(qbits, kbits, d, tau, p, nmin=None, dev_status=None, stream=None):
    """Top-N mass retention: nmin [B,H,n,len(p)] int32, the smallest N whose N
    largest softmax weights (over all keys) hold at least p[k] of a row's mass."""
    _dev(qbits, "qbits", torch.int32)
    B, H, n, w = _shape4(qbits, "qbits")
    if w * 32 != d:
        raise ValueError("qbits last dimension must be d/32")
    _dev(kbits, "kbits", torch.int32, (B, H, n, w))
    pv = (ctypes.c_double * len(p))(*[float(x) for x in p])
    if nmin is None:
        nmin = torch.empty((B, H, n, len(p)), dtype=torch.int32, device=qbits.device)
    _dev(nmin, "nmin", torch.int32, (B, H, n, len(p)))
    st = _lib.had_topn_mass(_ptr(qbits), _ptr(kbits), B, H, n, d, ctypes.c_float(tau),
                            ctypes.cast(pv, ctypes.c_void_p), len(p), _ptr(nmin),
                            _ptr(dev_status), _stream(stream))
    _check(st, "had_topn_mass")
    return nmin


def had_sparse_softmax_av(idx, logits, V, tau, out=None, p=None, want_p=False, dev_status=None,
                          stream=None):
    """Softmax over the kept logits and sparse product with V; returns (out, p or None)."""
    _dev(V, "V")
    B, H, n, d = _shape4(V, "V")
    _dev(idx, "idx", torch.int32)
    N = int(idx.shape[-1])
    _dev(idx, "idx", torch.int32, (B, H, n, N))
    _dev(logits, "logits", torch.int16, (B, H, n, N))
    if out is None:
        out = torch.empty((B, H, n, d), dtype=torch.float32, device=V.device)
    _dev(out, "out", torch.float32, (B, H, n, d))
    if p is None and want_p:
        p = torch.empty((B, H, n, N), dtype=torch.float32, device=V.device)
    if p is not None:
        _dev(p, "p", torch.float32, (B, H, n, N))
    st = _lib.had_sparse_softmax_av(_ptr(idx), _ptr(logits), _ptr(V), _dtype_code(V), B, H, n, d,
                                    N, ctypes.c_float(tau), _ptr(out), _ptr(p), _ptr(dev_status),
                                    _stream(stream))
    _check(st, "had_sparse_softmax_av")
    return out, p


def had_attention_fwd(Q, K, V, sigma_q, sigma_k, N, tau, out=None, dbg_idx=None,
                      dbg_logits=None, ws=None, dev_status=None, stream=None):
    """Fused binarized top-N attention forward; returns out [B,H,n,d] float32."""
    _dev(Q, "Q")
    B, H, n, d = _shape4(Q, "Q")
    _dev(K, "K", Q.dtype, (B, H, n, d))
    _dev(V, "V", Q.dtype, (B, H, n, d))
    _dev(sigma_q, "sigma_q", torch.float32, (H,))
    _dev(sigma_k, "sigma_k", torch.float32, (H,))
    if out is None:
        out = torch.empty((B, H, n, d), dtype=torch.float32, device=Q.device)
    _dev(out, "out", torch.float32, (B, H, n, d))
    if dbg_idx is not None:
        _dev(dbg_idx, "dbg_idx", torch.int32, (B, H, n, N))
    if dbg_logits is not None:
        _dev(dbg_logits, "dbg_logits", torch.int16, (B, H, n, N))
    need = had_workspace_bytes(HAD_OP_ATTENTION_FWD, B, H, n, d, N)
    if need < 0:
        raise HadError(HAD_ERR_UNSUPPORTED if d not in (64, 128) else HAD_ERR_INVALID_ARG,
                       "had_attention_fwd")
    if ws is None:
        ws = workspace(B, H, n, d, N, device=Q.device)
    st = _lib.had_attention_fwd(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(sigma_q),
                                _ptr(sigma_k), B, H, n, d, N, ctypes.c_float(tau), _ptr(out),
                                _ptr(dbg_idx), _ptr(dbg_logits), _ptr(ws), ws.numel(),
                                _ptr(dev_status), _stream(stream))
    _check(st, "had_attention_fwd")
    return out


def had_attention_prepare(Q, K, V, sigma_q, sigma_k, N, ws, dev_status=None, stream=None):
    """First stage of had_attention_fwd: operand tiles and packed bits into ws."""
    _dev(Q, "Q")
    B, H, n, d = _shape4(Q, "Q")
    _dev(K, "K", Q.dtype, (B, H, n, d))
    _dev(V, "V", Q.dtype, (B, H, n, d))
    _dev(sigma_q, "sigma_q", torch.float32, (H,))
    _dev(sigma_k, "sigma_k", torch.float32, (H,))
    _dev(ws, "ws", torch.uint8)
    st = _lib.had_attention_prepare(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(sigma_q),
                                    _ptr(sigma_k), B, H, n, d, N, _ptr(ws), ws.numel(),
                                    _ptr(dev_status), _stream(stream))
    _check(st, "had_attention_prepare")
    return ws


def had_attention_core(V, N, tau, ws, out=None, dbg_idx=None, dbg_logits=None, dev_status=None,
                       stream=None):
    """Second stage of had_attention_fwd: the fused kernel on the prepared ws."""
    _dev(V, "V")
    B, H, n, d = _shape4(V, "V")
    _dev(ws, "ws", torch.uint8)
    if out is None:
        out = torch.empty((B, H, n, d), dtype=torch.float32, device=V.device)
    _dev(out, "out", torch.float32, (B, H, n, d))
    if dbg_idx is not None:
        _dev(dbg_idx, "dbg_idx", torch.int32, (B, H, n, N))
    if dbg_logits is not None:
        _dev(dbg_logits, "dbg_logits", torch.int16, (B, H, n, N))
    st = _lib.had_attention_core(_ptr(V), _dtype_code(V), B, H, n, d, N, ctypes.c_float(tau),
                                 _ptr(out), _ptr(dbg_idx), _ptr(dbg_logits), _ptr(ws),
                                 ws.numel(), _ptr(dev_status), _stream(stream))
    _check(st, "had_attention_core")
    return out


def had_attention_fwd_noalloc(Q, K, V, sigma_q, sigma_k, N, tau, out, dev_status=None,
                              stream=None):
    """had_attention_fwd for callers that cannot allocate device memory.

    The library works in a fixed device array of had_noalloc_scratch_bytes()
    bytes instead of a workspace, so nothing is allocated here either: the
    caller passes every tensor, `out` included.  Sizes whose workspace
    exceeds the array raise HadError(HAD_ERR_WORKSPACE).  Calls that overlap
    on the GPU share the array and race.
    """
    _dev(Q, "Q")
    B, H, n, d = _shape4(Q, "Q")
    _dev(K, "K", Q.dtype, (B, H, n, d))
    _dev(V, "V", Q.dtype, (B, H, n, d))
    _dev(sigma_q, "sigma_q", torch.float32, (H,))
    _dev(sigma_k, "sigma_k", torch.float32, (H,))
    _dev(out, "out", torch.float32, (B, H, n, d))
    st = _lib.had_attention_fwd_noalloc(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(sigma_q),
                                        _ptr(sigma_k), B, H, n, d, N, ctypes.c_float(tau),
                                        _ptr(out), _ptr(dev_status), _stream(stream))
    _check(st, "had_attention_fwd_noalloc")
    return out


def had_noalloc_scratch_bytes() -> int:
    return int(_lib.had_noalloc_scratch_bytes())


def had_attention_window_misses(ws, B, H, n, d, N, stream=None) -> int:
    """Rows of the last fused call on ``ws`` that the exact fix-up kernel
    recomputed (their threshold fell outside the fused kernel's window).
    Synchronizes the stream to read the count."""
    _dev(ws, "ws", torch.uint8)
    dst = torch.zeros(1, dtype=torch.int32, device=ws.device)
    st = _lib.had_attention_window_misses(_ptr(ws), ws.numel(), B, H, n, d, N, _ptr(dst),
                                          _stream(stream))
    _check(st, "had_attention_window_misses")
    return int(dst.item())


def had_set_wait_limit_ns(ns: int) -> int:
    """Limit of the fused kernels' on-chip waits (0 = the 2 s default);
    returns the previous limit."""
    return int(_lib.had_set_wait_limit_ns(int(ns)))


def workspace(B, H, n, d, N, device="cuda"):
    """A workspace tensor big enough for had_attention_fwd at these sizes."""
    need = had_workspace_bytes(HAD_OP_ATTENTION_FWD, B, H, n, d, N)
    if need < 0:
        raise HadError(HAD_ERR_INVALID_ARG, "workspace")
    return torch.empty(max(need, 16), dtype=torch.uint8, device=device)
