// had_api.cu -- the C ABI of include/had.h: argument checks, workspace
// layout and kernel launches.  Every step of the forward pass runs in the
// kernels included below; this file only validates and enqueues.
#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

#include "had.h"
#include "had_common.cuh"
#include "had_pack.cuh"
#include "had_topn.cuh"
#include "had_av.cuh"

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape rules shared by every entry point.
had_status_t check_shape(int B, int H, int n, int d)
{
    if (B < 1 || H < 1 || n < 1 || d < 1) return HAD_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return HAD_ERR_UNSUPPORTED;
    const long long rows = (long long)B * H * n;
    if (rows > (1LL << 40) / d) return HAD_ERR_UNSUPPORTED;
    if ((long long)H * n > INT_MAX) return HAD_ERR_UNSUPPORTED;
    return HAD_OK;
}

had_status_t check_topn(int B, int H, int n, int d, int N)
{
    had_status_t s = check_shape(B, H, n, d);
    if (s != HAD_OK) return s;
    if (N < 1 || N > n) return HAD_ERR_INVALID_ARG;
    if ((long long)n * N >= (1LL << 31)) return HAD_ERR_UNSUPPORTED;
    return HAD_OK;
}

had_status_t launched()
{
    return cudaGetLastError() == cudaSuccess ? HAD_OK : HAD_ERR_CUDA;
}

int grid_for(long long work_items, int per_block)
{
    long long blocks = (work_items + per_block - 1) / per_block;
    const long long cap = 148LL * 32;        // enough resident work for 148 SMs
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

had_status_t launch_pack(const void *x, had_dtype_t dt, const float *sigma, int B, int H,
                         int n, int d, uint32_t *bits, int32_t *status, cudaStream_t st)
{
    const long long groups = (long long)B * H * n * d / 8;
    const int threads = 256;
    const int grid = grid_for(groups, threads);
    if (dt == HAD_BF16)
        had::pack_bits_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(x), sigma, H, n, d, groups, bits, status);
    else
        had::pack_bits_kernel<float><<<grid, threads, 0, st>>>(
            static_cast<const float *>(x), sigma, H, n, d, groups, bits, status);
    return launched();
}

template <int DW>
had_status_t launch_topn_dw(const uint32_t *qb, const uint32_t *kb, int B, int H, int n,
                            int N, int32_t *idx, int16_t *lg, cudaStream_t st)
{
    constexpr int smem = had::topn_smem_bytes<DW>();
    // Set on every call: the attribute belongs to the current device.
    if (cudaFuncSetAttribute(had::topn_simt_kernel<DW>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HAD_ERR_CUDA;
    const long long blocks = (long long)((n + had::kTopnRows - 1) / had::kTopnRows) * B * H;
    if (blocks > INT_MAX) return HAD_ERR_UNSUPPORTED;
    had::topn_simt_kernel<DW><<<(unsigned)blocks, had::kTopnRows, smem, st>>>(qb, kb, n, N, idx, lg);
    return launched();
}

had_status_t launch_topn(const uint32_t *qb, const uint32_t *kb, int B, int H, int n, int d,
                         int N, int32_t *idx, int16_t *lg, cudaStream_t st)
{
    return d == 64 ? launch_topn_dw<2>(qb, kb, B, H, n, N, idx, lg, st)
                   : launch_topn_dw<4>(qb, kb, B, H, n, N, idx, lg, st);
}

had_status_t launch_av(const int32_t *idx, const int16_t *lg, const void *V, had_dtype_t dt,
                       int B, int H, int n, int d, int N, float tau, float *out, float *p,
                       int32_t *status, cudaStream_t st)
{
    const long long rows = (long long)B * H * n;
    const int threads = 256;
    const long long blocks = (rows * 32 + threads - 1) / threads;
    if (blocks > INT_MAX) return HAD_ERR_UNSUPPORTED;
    const int grid = (int)blocks;
    if (dt == HAD_BF16) {
        const auto *v = static_cast<const __nv_bfloat16 *>(V);
        if (d == 64)
            had::sparse_softmax_av_kernel<__nv_bfloat16, 64><<<grid, threads, 0, st>>>(
                idx, lg, v, n, N, tau, rows, out, p, status);
        else
            had::sparse_softmax_av_kernel<__nv_bfloat16, 128><<<grid, threads, 0, st>>>(
                idx, lg, v, n, N, tau, rows, out, p, status);
    } else {
        const auto *v = static_cast<const float *>(V);
        if (d == 64)
            had::sparse_softmax_av_kernel<float, 64><<<grid, threads, 0, st>>>(
                idx, lg, v, n, N, tau, rows, out, p, status);
        else
            had::sparse_softmax_av_kernel<float, 128><<<grid, threads, 0, st>>>(
                idx, lg, v, n, N, tau, rows, out, p, status);
    }
    return launched();
}

// Workspace of the fused forward: packed Q and K bits, then the kept set.
struct FwdWorkspace {
    size_t qbits, kbits, idx, lg, total;
};

FwdWorkspace fwd_layout(int B, int H, int n, int d, int N)
{
    const size_t rows = (size_t)B * H * n;
    FwdWorkspace w;
    w.qbits = 0;
    w.kbits = w.qbits + round_up(rows * (d / 32) * 4);
    w.idx = w.kbits + round_up(rows * (d / 32) * 4);
    w.lg = w.idx + round_up(rows * (size_t)N * 4);
    w.total = w.lg + round_up(rows * (size_t)N * 2);
    return w;
}

}  // namespace

extern "C" {

had_status_t had_binarize_pack(const void *x, had_dtype_t dt, const float *sigma, int B, int H,
                               int n, int d, uint32_t *bits, int32_t *dev_status,
                               cudaStream_t stream)
{
    had_status_t s = check_shape(B, H, n, d);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!x || !sigma || !bits || !aligned16(x) || !aligned16(bits)) return HAD_ERR_INVALID_ARG;
    return launch_pack(x, dt, sigma, B, H, n, d, bits, dev_status, stream);
}

had_status_t had_hamming_topn(const uint32_t *qbits, const uint32_t *kbits, int B, int H, int n,
                              int d, int N, int32_t *idx, int16_t *logits, void *ws,
                              size_t ws_bytes, int32_t *dev_status, cudaStream_t stream)
{
    (void)ws;
    (void)ws_bytes;
    (void)dev_status;
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (!qbits || !kbits || !idx) return HAD_ERR_INVALID_ARG;
    if (!aligned16(qbits) || !aligned16(kbits) || !aligned16(idx) ||
        (logits && !aligned16(logits)))
        return HAD_ERR_INVALID_ARG;
    return launch_topn(qbits, kbits, B, H, n, d, N, idx, logits, stream);
}

had_status_t had_sparse_softmax_av(const int32_t *idx, const int16_t *logits, const void *V,
                                   had_dtype_t dt, int B, int H, int n, int d, int N, float tau,
                                   float *out, float *p, int32_t *dev_status,
                                   cudaStream_t stream)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!idx || !logits || !V || !out) return HAD_ERR_INVALID_ARG;
    if (!aligned16(idx) || !aligned16(logits) || !aligned16(V) || !aligned16(out) ||
        (p && !aligned16(p)))
        return HAD_ERR_INVALID_ARG;
    if (!(tau == tau) || tau > 3.0e38f || tau < -3.0e38f) return HAD_ERR_INVALID_ARG;
    return launch_av(idx, logits, V, dt, B, H, n, d, N, tau, out, p, dev_status, stream);
}

had_status_t had_attention_fwd(const void *Q, const void *K, const void *V, had_dtype_t dt,
                               const float *sigma_q, const float *sigma_k, int B, int H, int n,
                               int d, int N, float tau, float *out, int32_t *dbg_idx,
                               int16_t *dbg_logits, void *ws, size_t ws_bytes,
                               int32_t *dev_status, cudaStream_t stream)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!Q || !K || !V || !sigma_q || !sigma_k || !out) return HAD_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) ||
        (dbg_idx && !aligned16(dbg_idx)) || (dbg_logits && !aligned16(dbg_logits)))
        return HAD_ERR_INVALID_ARG;
    if (!(tau == tau) || tau > 3.0e38f || tau < -3.0e38f) return HAD_ERR_INVALID_ARG;
    const FwdWorkspace w = fwd_layout(B, H, n, d, N);
    if (!ws || ws_bytes < w.total || !aligned16(ws)) return HAD_ERR_WORKSPACE;
    char *base = static_cast<char *>(ws);
    auto *qb = reinterpret_cast<uint32_t *>(base + w.qbits);
    auto *kb = reinterpret_cast<uint32_t *>(base + w.kbits);
    int32_t *idx = dbg_idx ? dbg_idx : reinterpret_cast<int32_t *>(base + w.idx);
    int16_t *lg = dbg_logits ? dbg_logits : reinterpret_cast<int16_t *>(base + w.lg);
    if ((s = launch_pack(Q, dt, sigma_q, B, H, n, d, qb, dev_status, stream)) != HAD_OK) return s;
    if ((s = launch_pack(K, dt, sigma_k, B, H, n, d, kb, dev_status, stream)) != HAD_OK) return s;
    if ((s = launch_topn(qb, kb, B, H, n, d, N, idx, lg, stream)) != HAD_OK) return s;
    return launch_av(idx, lg, V, dt, B, H, n, d, N, tau, out, nullptr, dev_status, stream);
}

size_t had_workspace_bytes(int op, int B, int H, int n, int d, int N)
{
    switch (op) {
    case HAD_OP_BINARIZE_PACK:
        return check_shape(B, H, n, d) == HAD_OK ? 0 : (size_t)-1;
    case HAD_OP_HAMMING_TOPN:
    case HAD_OP_SPARSE_SOFTMAX_AV:
        return check_topn(B, H, n, d, N) == HAD_OK ? 0 : (size_t)-1;
    case HAD_OP_ATTENTION_FWD:
        if (check_topn(B, H, n, d, N) != HAD_OK) return (size_t)-1;
        return fwd_layout(B, H, n, d, N).total;
    default:
        return (size_t)-1;
    }
}

int had_launch_count(int op, int B, int H, int n, int d, int N)
{
    switch (op) {
    case HAD_OP_BINARIZE_PACK:
        return check_shape(B, H, n, d) == HAD_OK ? 1 : -1;
    case HAD_OP_HAMMING_TOPN:
    case HAD_OP_SPARSE_SOFTMAX_AV:
        return check_topn(B, H, n, d, N) == HAD_OK ? 1 : -1;
    case HAD_OP_ATTENTION_FWD:
        return check_topn(B, H, n, d, N) == HAD_OK ? 4 : -1;
    default:
        return -1;
    }
}

const char *had_status_string(had_status_t status)
{
    switch (status) {
    case HAD_OK: return "HAD_OK";
    case HAD_ERR_INVALID_ARG: return "HAD_ERR_INVALID_ARG";
    case HAD_ERR_UNSUPPORTED: return "HAD_ERR_UNSUPPORTED";
    case HAD_ERR_WORKSPACE: return "HAD_ERR_WORKSPACE";
    case HAD_ERR_CUDA: return "HAD_ERR_CUDA";
    case HAD_ERR_BAD_SIGMA: return "HAD_ERR_BAD_SIGMA";
    case HAD_ERR_TIMEOUT: return "HAD_ERR_TIMEOUT";
    }
    return "HAD_ERR_UNKNOWN";
}

}  // extern "C"
