// had_api.cu -- the C ABI of include/had.h: argument checks, workspace
// layout and kernel launches.  Every step of the forward pass runs in the
// kernels included below; this file only validates and enqueues.
#include <climits>
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cuda_runtime.h>

#include "had.h"
#include "had_common.cuh"
#include "had_pack.cuh"
#include "had_topn.cuh"
#include "had_av.cuh"
#include "had_fwd_launch.cuh"
#include "had_mass.cuh"
#include "had_soft.cuh"
#include "had_bwd.cuh"

namespace {

using had::fwdapi::FwdWorkspace;
using had::fwdapi::fwd_layout;
using had::fwdapi::launch_fused;
using had::fwdapi::prep_typed;
using had::fwdapi::core_typed;

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
    // one block row per (b, h) slab; two 1024-element steps per warp (half
    // the blocks of one step each: measured 12 % faster at n 4096, d 64)
    const long long slab = (long long)n * d, bh = (long long)B * H;
    const int threads = 256;
    const long long quads = (slab + 1023) / 1024;   // a warp's 1024-element steps
    const long long bx = (quads + 16 - 1) / 16;
    const dim3 grid((unsigned)(bx < 1 ? 1 : bx > 65535 ? 65535 : bx),
                    (unsigned)(bh > 65535 ? 65535 : bh));
    if (dt == HAD_BF16)
        had::pack_bits_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(x), sigma, H, slab, bh, bits, status);
    else
        had::pack_bits_kernel<float><<<grid, threads, 0, st>>>(
            static_cast<const float *>(x), sigma, H, slab, bh, bits, status);
    return launched();
}

template <int DW, bool kCausal>
had_status_t launch_topn_dw(const uint32_t *qb, const uint32_t *kb, int B, int H, int n,
                            int N, int32_t *idx, int16_t *lg, cudaStream_t st)
{
    constexpr int smem = had::topn_smem_bytes<DW>();
    // Set on every call: the attribute belongs to the current device.
    if (cudaFuncSetAttribute(had::topn_simt_kernel<DW, kCausal>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HAD_ERR_CUDA;
    const long long blocks = (long long)((n + had::kTopnRows - 1) / had::kTopnRows) * B * H;
    if (blocks > INT_MAX) return HAD_ERR_UNSUPPORTED;
    had::topn_simt_kernel<DW, kCausal><<<(unsigned)blocks, had::kTopnRows, smem, st>>>(
        qb, kb, n, N, idx, lg);
    return launched();
}

had_status_t launch_topn(const uint32_t *qb, const uint32_t *kb, int B, int H, int n, int d,
                         int N, int32_t *idx, int16_t *lg, bool causal, cudaStream_t st)
{
    if (causal)
        return d == 64 ? launch_topn_dw<2, true>(qb, kb, B, H, n, N, idx, lg, st)
                       : launch_topn_dw<4, true>(qb, kb, B, H, n, N, idx, lg, st);
    return d == 64 ? launch_topn_dw<2, false>(qb, kb, B, H, n, N, idx, lg, st)
                   : launch_topn_dw<4, false>(qb, kb, B, H, n, N, idx, lg, st);
}

template <typename L>
had_status_t launch_av(const int32_t *idx, const L *lg, const void *V, had_dtype_t dt,
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
            had::sparse_softmax_av_kernel<__nv_bfloat16, 64, L><<<grid, threads, 0, st>>>(
                idx, lg, v, n, N, tau, rows, out, p, status);
        else
            had::sparse_softmax_av_kernel<__nv_bfloat16, 128, L><<<grid, threads, 0, st>>>(
                idx, lg, v, n, N, tau, rows, out, p, status);
    } else {
        const auto *v = static_cast<const float *>(V);
        if (d == 64)
            had::sparse_softmax_av_kernel<float, 64, L><<<grid, threads, 0, st>>>(
                idx, lg, v, n, N, tau, rows, out, p, status);
        else
            had::sparse_softmax_av_kernel<float, 128, L><<<grid, threads, 0, st>>>(
                idx, lg, v, n, N, tau, rows, out, p, status);
    }
    return launched();
}

// Fixed scratch of had_attention_fwd_noalloc.  Some callers cannot call
// cudaMalloc at all (code running inside another runtime's allocator, a
// plugin that is handed only input and output buffers, or a process whose
// device memory is fully reserved up front), so this entry point takes its
// workspace from a statically sized device array instead.  The array is part
// of the module: every GPU that loads the library holds it until the process
// exits.
constexpr size_t kNoAllocScratchBytes = size_t(96) << 20;   // 96 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// In host code `g_noalloc_scratch` is only a stand-in symbol, never a device
// address.  Its device address belongs to the context the module was loaded
// in, so it is looked up with cudaGetSymbolAddress in the context current on
// the calling thread and cached under that context (a primary context and a
// context the caller created on the same device hold different copies).
using CtxGetCurrentFn = CUresult (*)(CUcontext *);

CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<CtxGetCurrentFn>(f);
    }();
    return fn;
}

constexpr int kMaxContexts = 64;
struct NoallocEntry {
    CUcontext ctx;
    void *ptr;
};
NoallocEntry g_noalloc_cache[kMaxContexts] = {};
int g_noalloc_entries = 0;
std::mutex g_noalloc_mutex;

had_status_t noalloc_scratch(void **ptr)
{
    CtxGetCurrentFn get = ctx_get_current();
    if (!get) return HAD_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return HAD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (ctx)
        for (int i = 0; i < g_noalloc_entries; ++i)
            if (g_noalloc_cache[i].ctx == ctx) {
                *ptr = g_noalloc_cache[i].ptr;
                return HAD_OK;
            }
    // First call in this context (or none current yet: the runtime makes the
    // device's primary context current while looking the symbol up).
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HAD_ERR_CUDA;
    if (!ctx && get(&ctx) != CUDA_SUCCESS) return HAD_ERR_CUDA;
    if (ctx && g_noalloc_entries < kMaxContexts)
        g_noalloc_cache[g_noalloc_entries++] = NoallocEntry{ctx, p};
    *ptr = p;
    return HAD_OK;
}

template <int DW>
had_status_t launch_mass_dw(const uint32_t *qb, const uint32_t *kb, int B, int H, int n,
                            float tau, const had::MassP &ps, int32_t *nmin, cudaStream_t st)
{
    constexpr int smem = had::mass_smem_bytes<DW>();
    if (cudaFuncSetAttribute(had::topn_mass_kernel<DW>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HAD_ERR_CUDA;
    const long long blocks = (long long)((n + had::kTopnRows - 1) / had::kTopnRows) * B * H;
    if (blocks > INT_MAX) return HAD_ERR_UNSUPPORTED;
    had::topn_mass_kernel<DW><<<(unsigned)blocks, had::kTopnRows, smem, st>>>(
        qb, kb, n, (double)tau, ps, nmin);
    return launched();
}

// Soft-code path: n is bounded by the select kernel's shared memory (one
// 4-byte key per column of a row).
constexpr int kSoftMaxN = 32768;
constexpr size_t kSoftScratchBytes = size_t(2) << 30;   // logits of one group of heads

had_status_t check_soft(int B, int H, int n, int d, int N)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    return n > kSoftMaxN ? HAD_ERR_UNSUPPORTED : HAD_OK;
}

long long soft_ld(int n) { return (n + 3LL) / 4 * 4; }

// Heads whose logit matrices share the scratch at one time.
long long soft_group(int B, int H, int n)
{
    const long long per = (long long)n * soft_ld(n) * 4;
    long long g = (long long)kSoftScratchBytes / per;
    const long long bh = (long long)B * H;
    if (g > bh) g = bh;
    if (g > 65535) g = 65535;
    return g < 1 ? 1 : g;
}

size_t soft_scratch_bytes(int B, int H, int n)
{
    return round_up((size_t)soft_group(B, H, n) * n * soft_ld(n) * 4);
}

int soft_passes(int B, int H, int n)
{
    const long long g = soft_group(B, H, n);
    return (int)(((long long)B * H + g - 1) / g);
}

had_status_t launch_soft_codes(const void *x, had_dtype_t dt, const float *sigma, float c, int B,
                               int H, int n, int d, float *t, int32_t *status, cudaStream_t st)
{
    const long long groups = (long long)B * H * n * d / 8;
    const int threads = 256;
    const int grid = grid_for(groups, threads);
    if (dt == HAD_BF16)
        had::soft_codes_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(x), sigma, c, H, n, d, groups, t, status);
    else
        had::soft_codes_kernel<float><<<grid, threads, 0, st>>>(
            static_cast<const float *>(x), sigma, c, H, n, d, groups, t, status);
    return launched();
}

template <int D>
had_status_t launch_soft_logits(const float *tq, const float *tk, int n, long long heads,
                                float *S, cudaStream_t st)
{
    constexpr int smem = had::soft_logits_smem_bytes<D>();
    if (cudaFuncSetAttribute(had::soft_logits_kernel<D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HAD_ERR_CUDA;
    const unsigned tiles = (unsigned)((n + had::kSoftTile - 1) / had::kSoftTile);
    had::soft_logits_kernel<D><<<dim3(tiles, tiles, (unsigned)heads), 256, smem, st>>>(
        tq, tk, n, soft_ld(n), S);
    return launched();
}

// Soft top-N over all heads, one group of heads at a time through the scratch.
had_status_t launch_soft_topn(const float *tq, const float *tk, int B, int H, int n, int d,
                              int N, int32_t *idx, float *lg, float *S, cudaStream_t st)
{
    const long long bh = (long long)B * H, g = soft_group(B, H, n);
    const int smem = (int)had::soft_select_smem_bytes(n);
    auto *select = d == 64 ? had::soft_select_kernel<64> : had::soft_select_kernel<128>;
    if (cudaFuncSetAttribute(select,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return HAD_ERR_CUDA;
    for (long long h0 = 0; h0 < bh; h0 += g) {
        const long long heads = bh - h0 < g ? bh - h0 : g;
        const long long off = h0 * n * (long long)d;
        had_status_t s = d == 64 ? launch_soft_logits<64>(tq + off, tk + off, n, heads, S, st)
                                 : launch_soft_logits<128>(tq + off, tk + off, n, heads, S, st);
        if (s != HAD_OK) return s;
        const long long rows = heads * n;
        if (rows > INT_MAX) return HAD_ERR_UNSUPPORTED;
        select<<<(unsigned)rows, had::kSelThreads, smem, st>>>(
            S, soft_ld(n), n, N, h0 * n, idx, lg);
        if ((s = launched()) != HAD_OK) return s;
    }
    return HAD_OK;
}

// Workspace of the soft forward: codes of Q and K, the kept set, the scratch.
struct SoftWorkspace {
    size_t tq, tk, idx, logits, scratch, total;
};

SoftWorkspace soft_layout(int B, int H, int n, int d, int N)
{
    const size_t rows = (size_t)B * H * n;
    SoftWorkspace w;
    w.tq = 0;
    w.tk = w.tq + round_up(rows * d * 4);
    w.idx = w.tk + round_up(rows * d * 4);
    w.logits = w.idx + round_up(rows * (size_t)N * 4);
    w.scratch = w.logits + round_up(rows * (size_t)N * 4);
    w.total = w.scratch + soft_scratch_bytes(B, H, n);
    return w;
}

bool finite_float(float x) { return x == x && x < 3.0e38f && x > -3.0e38f; }

// Workspace of the straight-through backward: the forward's packed codes and
// kept set, p and ds per kept pair, the per-key counts and offsets, and the
// key-ordered lists.
struct BwdWorkspace {
    size_t qbits, kbits, idx, logits, P, DS, cnt, off, cursor, rec, total;
};

BwdWorkspace bwd_layout(int B, int H, int n, int d, int N)
{
    const size_t rows = (size_t)B * H * n, pairs = rows * (size_t)N;
    BwdWorkspace w;
    w.qbits = 0;
    w.kbits = w.qbits + round_up(rows * (d / 8));
    w.idx = w.kbits + round_up(rows * (d / 8));
    w.logits = w.idx + round_up(pairs * 4);
    w.P = w.logits + round_up(pairs * 2);
    w.DS = w.P + round_up(pairs * 4);
    w.cnt = w.DS + round_up(pairs * 4);
    w.off = w.cnt + round_up(rows * 4);
    w.cursor = w.off + round_up(rows * 8);
    w.rec = w.cursor + round_up(rows * 4);
    w.total = w.rec + round_up(pairs * 16);
    return w;
}

template <typename T, int D>
had_status_t launch_bwd_typed(const T *Q, const T *K, const T *V, const float *sq,
                              const float *sk, const float *dout, const int32_t *kept_idx,
                              const int16_t *kept_lg, int B, int H, int n, int N, float tau,
                              float clip, float *dq, float *dk, float *dv,
                              const BwdWorkspace &w, char *base, int32_t *status,
                              cudaStream_t st)
{
    auto *qb = reinterpret_cast<uint32_t *>(base + w.qbits);
    auto *kb = reinterpret_cast<uint32_t *>(base + w.kbits);
    auto *idx = reinterpret_cast<int32_t *>(base + w.idx);
    auto *lg = reinterpret_cast<int16_t *>(base + w.logits);
    auto *P = reinterpret_cast<float *>(base + w.P);
    auto *DS = reinterpret_cast<float *>(base + w.DS);
    auto *cnt = reinterpret_cast<int32_t *>(base + w.cnt);
    auto *off = reinterpret_cast<long long *>(base + w.off);
    auto *cur = reinterpret_cast<uint32_t *>(base + w.cursor);
    auto *rec = reinterpret_cast<int4 *>(base + w.rec);
    const had_dtype_t dt = sizeof(T) == 2 ? HAD_BF16 : HAD_F32;
    had_status_t s;
    if ((s = launch_pack(Q, dt, sq, B, H, n, D, qb, status, st)) != HAD_OK) return s;
    if ((s = launch_pack(K, dt, sk, B, H, n, D, kb, status, st)) != HAD_OK) return s;
    if (kept_idx) {          // the forward's kept set, as given
        idx = const_cast<int32_t *>(kept_idx);
        lg = const_cast<int16_t *>(kept_lg);
    } else if ((s = launch_topn(qb, kb, B, H, n, D, N, idx, lg, false, st)) != HAD_OK) {
        return s;
    }
    const long long rows = (long long)B * H * n, pairs = rows * N;
    const long long warp_blocks = (rows * 32 + 255) / 256;
    if (warp_blocks > INT_MAX) return HAD_ERR_UNSUPPORTED;
    had::bwd_rows_kernel<T, D><<<(unsigned)warp_blocks, 256, 0, st>>>(
        idx, lg, V, dout, Q, sq, kb, H, n, N, tau, clip, rows, P, DS, dq, cnt, status);
    if ((s = launched()) != HAD_OK) return s;
    had::bwd_count_kernel<<<grid_for(pairs, 256), 256, 0, st>>>(idx, pairs, n, N, cnt);
    if ((s = launched()) != HAD_OK) return s;
    had::bwd_scan_kernel<<<(unsigned)(B * H), had::kScanThreads, 0, st>>>(cnt, n, N, off, cur);
    if ((s = launched()) != HAD_OK) return s;
    had::bwd_fill_kernel<<<grid_for(pairs, 256), 256, 0, st>>>(idx, P, DS, pairs, n, N, off,
                                                              cur, rec);
    if ((s = launched()) != HAD_OK) return s;
    had::bwd_keys_kernel<T, D><<<(unsigned)warp_blocks, 256, 0, st>>>(
        off, cnt, rec, dout, qb, K, sk, H, n, clip, rows, dk, dv);
    return launched();
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
    return launch_topn(qbits, kbits, B, H, n, d, N, idx, logits, false, stream);
}

had_status_t had_hamming_topn_causal(const uint32_t *qbits, const uint32_t *kbits, int B, int H,
                                     int n, int d, int N, int32_t *idx, int16_t *logits,
                                     int32_t *dev_status, cudaStream_t stream)
{
    (void)dev_status;
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (!qbits || !kbits || !idx) return HAD_ERR_INVALID_ARG;
    if (!aligned16(qbits) || !aligned16(kbits) || !aligned16(idx) ||
        (logits && !aligned16(logits)))
        return HAD_ERR_INVALID_ARG;
    return launch_topn(qbits, kbits, B, H, n, d, N, idx, logits, true, stream);
}

had_status_t had_attention_causal_fwd(const void *Q, const void *K, const void *V,
                                      had_dtype_t dt, const float *sigma_q, const float *sigma_k,
                                      int B, int H, int n, int d, int N, float tau, float *out,
                                      int32_t *dbg_idx, int16_t *dbg_logits, void *ws,
                                      size_t ws_bytes, int32_t *dev_status, cudaStream_t stream)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!Q || !K || !V || !sigma_q || !sigma_k || !out) return HAD_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) ||
        (dbg_idx && !aligned16(dbg_idx)) || (dbg_logits && !aligned16(dbg_logits)))
        return HAD_ERR_INVALID_ARG;
    if (!(tau >= 0.0f) || tau > 3.0e38f) return HAD_ERR_INVALID_ARG;
    const FwdWorkspace w = fwd_layout(B, H, n, d, N);
    if (!ws || ws_bytes < w.total || !aligned16(ws)) return HAD_ERR_WORKSPACE;
    if ((long long)B * H * w.qtiles > INT_MAX) return HAD_ERR_UNSUPPORTED;
    char *base = static_cast<char *>(ws);
    if (dt == HAD_BF16)
        return launch_fused<__nv_bfloat16>(Q, K, V, sigma_q, sigma_k, B, H, n, d, N, tau, out,
                                           dbg_idx, dbg_logits, base, w, dev_status, stream,
                                           true);
    return launch_fused<float>(Q, K, V, sigma_q, sigma_k, B, H, n, d, N, tau, out, dbg_idx,
                               dbg_logits, base, w, dev_status, stream, true);
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
    if (!(tau >= 0.0f) || tau > 3.0e38f) return HAD_ERR_INVALID_ARG;
    const FwdWorkspace w = fwd_layout(B, H, n, d, N);
    if (!ws || ws_bytes < w.total || !aligned16(ws)) return HAD_ERR_WORKSPACE;
    if ((long long)B * H * w.qtiles > INT_MAX) return HAD_ERR_UNSUPPORTED;
    char *base = static_cast<char *>(ws);
    if (dt == HAD_BF16)
        return launch_fused<__nv_bfloat16>(Q, K, V, sigma_q, sigma_k, B, H, n, d, N, tau, out,
                                           dbg_idx, dbg_logits, base, w, dev_status, stream);
    return launch_fused<float>(Q, K, V, sigma_q, sigma_k, B, H, n, d, N, tau, out, dbg_idx,
                               dbg_logits, base, w, dev_status, stream);
}

had_status_t had_attention_prepare(const void *Q, const void *K, const void *V, had_dtype_t dt,
                                   const float *sigma_q, const float *sigma_k, int B, int H,
                                   int n, int d, int N, void *ws, size_t ws_bytes,
                                   int32_t *dev_status, cudaStream_t stream)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!Q || !K || !V || !sigma_q || !sigma_k) return HAD_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V)) return HAD_ERR_INVALID_ARG;
    const FwdWorkspace w = fwd_layout(B, H, n, d, N);
    if (!ws || ws_bytes < w.total || !aligned16(ws)) return HAD_ERR_WORKSPACE;
    if ((long long)B * H * w.qtiles > INT_MAX) return HAD_ERR_UNSUPPORTED;
    char *base = static_cast<char *>(ws);
    if (dt == HAD_BF16) {
        const auto *q = static_cast<const __nv_bfloat16 *>(Q), *k = static_cast<const __nv_bfloat16 *>(K),
                   *v = static_cast<const __nv_bfloat16 *>(V);
        return d == 64 ? prep_typed<__nv_bfloat16, 64>(q, k, v, sigma_q, sigma_k, B, H, n, base, w,
                                                       dev_status, stream)
                       : prep_typed<__nv_bfloat16, 128>(q, k, v, sigma_q, sigma_k, B, H, n, base,
                                                        w, dev_status, stream);
    }
    const auto *q = static_cast<const float *>(Q), *k = static_cast<const float *>(K),
               *v = static_cast<const float *>(V);
    return d == 64 ? prep_typed<float, 64>(q, k, v, sigma_q, sigma_k, B, H, n, base, w,
                                           dev_status, stream)
                   : prep_typed<float, 128>(q, k, v, sigma_q, sigma_k, B, H, n, base, w,
                                            dev_status, stream);
}

had_status_t had_attention_core(const void *V, had_dtype_t dt, int B, int H, int n, int d, int N,
                                float tau, float *out, int32_t *dbg_idx, int16_t *dbg_logits,
                                void *ws, size_t ws_bytes, int32_t *dev_status,
                                cudaStream_t stream)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!V || !out || !aligned16(V) || !aligned16(out) || (dbg_idx && !aligned16(dbg_idx)) ||
        (dbg_logits && !aligned16(dbg_logits)))
        return HAD_ERR_INVALID_ARG;
    if (!(tau >= 0.0f) || tau > 3.0e38f) return HAD_ERR_INVALID_ARG;
    const FwdWorkspace w = fwd_layout(B, H, n, d, N);
    if (!ws || ws_bytes < w.total || !aligned16(ws)) return HAD_ERR_WORKSPACE;
    if ((long long)B * H * w.qtiles > INT_MAX) return HAD_ERR_UNSUPPORTED;
    char *base = static_cast<char *>(ws);
    if (dt == HAD_BF16) {
        const auto *v = static_cast<const __nv_bfloat16 *>(V);
        return d == 64 ? core_typed<__nv_bfloat16, 64>(v, B, H, n, N, tau, out, dbg_idx, dbg_logits,
                                                       base, w, dev_status, stream)
                       : core_typed<__nv_bfloat16, 128>(v, B, H, n, N, tau, out, dbg_idx,
                                                        dbg_logits, base, w, dev_status, stream);
    }
    const auto *v = static_cast<const float *>(V);
    return d == 64 ? core_typed<float, 64>(v, B, H, n, N, tau, out, dbg_idx, dbg_logits, base, w,
                                           dev_status, stream)
                   : core_typed<float, 128>(v, B, H, n, N, tau, out, dbg_idx, dbg_logits, base, w,
                                            dev_status, stream);
}

had_status_t had_attention_fwd_noalloc(const void *Q, const void *K, const void *V,
                                       had_dtype_t dt, const float *sigma_q,
                                       const float *sigma_k, int B, int H, int n, int d, int N,
                                       float tau, float *out, int32_t *dev_status,
                                       cudaStream_t stream)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!Q || !K || !V || !sigma_q || !sigma_k || !out) return HAD_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out))
        return HAD_ERR_INVALID_ARG;
    if (!(tau >= 0.0f) || tau > 3.0e38f) return HAD_ERR_INVALID_ARG;
    const FwdWorkspace w = fwd_layout(B, H, n, d, N);
    if (w.total > kNoAllocScratchBytes) return HAD_ERR_WORKSPACE;
    if ((long long)B * H * w.qtiles > INT_MAX) return HAD_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != HAD_OK) return s;
    char *base = static_cast<char *>(scratch);
    if (dt == HAD_BF16)
        return launch_fused<__nv_bfloat16>(Q, K, V, sigma_q, sigma_k, B, H, n, d, N, tau, out,
                                           nullptr, nullptr, base, w, dev_status, stream);
    return launch_fused<float>(Q, K, V, sigma_q, sigma_k, B, H, n, d, N, tau, out, nullptr,
                               nullptr, base, w, dev_status, stream);
}

had_status_t had_attention_window_misses(const void *ws, size_t ws_bytes, int B, int H, int n,
                                         int d, int N, int32_t *dst, cudaStream_t stream)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (!dst) return HAD_ERR_INVALID_ARG;
    const FwdWorkspace w = fwd_layout(B, H, n, d, N);
    if (!ws || ws_bytes < w.total) return HAD_ERR_WORKSPACE;
    const char *src = static_cast<const char *>(ws) + w.miss + 2 * sizeof(int32_t);
    return cudaMemcpyAsync(dst, src, sizeof(int32_t), cudaMemcpyDefault, stream) == cudaSuccess
               ? HAD_OK
               : HAD_ERR_CUDA;
}

size_t had_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

unsigned long long had_set_wait_limit_ns(unsigned long long ns)
{
    return had::fwdapi::wait_limit_ns().exchange(ns ? ns : had::fwdapi::kDefaultWaitNs);
}

had_status_t had_topn_mass(const uint32_t *qbits, const uint32_t *kbits, int B, int H, int n,
                           int d, float tau, const double *p, int np, int32_t *nmin,
                           int32_t *dev_status, cudaStream_t stream)
{
    (void)dev_status;
    had_status_t s = check_shape(B, H, n, d);
    if (s != HAD_OK) return s;
    if (!qbits || !kbits || !nmin || !p) return HAD_ERR_INVALID_ARG;
    if (!aligned16(qbits) || !aligned16(kbits) || !aligned16(nmin)) return HAD_ERR_INVALID_ARG;
    if (np < 1 || np > had::kMassMaxP || !(tau >= 0.0f) || !isfinite(tau)) return HAD_ERR_INVALID_ARG;
    had::MassP ps{};
    ps.np = np;
    for (int k = 0; k < np; ++k) {
        if (!(p[k] > 0.0) || p[k] > 1.0) return HAD_ERR_INVALID_ARG;
        ps.p[k] = p[k];
    }
    return d == 64 ? launch_mass_dw<2>(qbits, kbits, B, H, n, tau, ps, nmin, stream)
                   : launch_mass_dw<4>(qbits, kbits, B, H, n, tau, ps, nmin, stream);
}

had_status_t had_soft_binarize(const void *x, had_dtype_t dt, const float *sigma, float c, int B,
                               int H, int n, int d, float *t, int32_t *dev_status,
                               cudaStream_t stream)
{
    had_status_t s = check_shape(B, H, n, d);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!x || !sigma || !t) return HAD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(t)) return HAD_ERR_INVALID_ARG;
    if (!finite_float(c) || !(c > 0.0f)) return HAD_ERR_INVALID_ARG;
    return launch_soft_codes(x, dt, sigma, c, B, H, n, d, t, dev_status, stream);
}

had_status_t had_soft_topn(const float *tq, const float *tk, int B, int H, int n, int d, int N,
                           int32_t *idx, float *logits, void *ws, size_t ws_bytes,
                           int32_t *dev_status, cudaStream_t stream)
{
    (void)dev_status;
    had_status_t s = check_soft(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (!tq || !tk || !idx || !ws) return HAD_ERR_INVALID_ARG;
    if (!aligned16(tq) || !aligned16(tk) || !aligned16(idx) || !aligned16(ws) ||
        (logits && !aligned16(logits)))
        return HAD_ERR_INVALID_ARG;
    if (ws_bytes < soft_scratch_bytes(B, H, n)) return HAD_ERR_WORKSPACE;
    return launch_soft_topn(tq, tk, B, H, n, d, N, idx, logits, static_cast<float *>(ws), stream);
}

had_status_t had_soft_softmax_av(const int32_t *idx, const float *logits, const void *V,
                                 had_dtype_t dt, int B, int H, int n, int d, int N, float tau,
                                 float *out, float *p, int32_t *dev_status, cudaStream_t stream)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!idx || !logits || !V || !out) return HAD_ERR_INVALID_ARG;
    if (!aligned16(idx) || !aligned16(logits) || !aligned16(V) || !aligned16(out) ||
        (p && !aligned16(p)))
        return HAD_ERR_INVALID_ARG;
    if (!finite_float(tau)) return HAD_ERR_INVALID_ARG;
    return launch_av(idx, logits, V, dt, B, H, n, d, N, tau, out, p, dev_status, stream);
}

had_status_t had_soft_attention_fwd(const void *Q, const void *K, const void *V, had_dtype_t dt,
                                    const float *sigma_q, const float *sigma_k, float c, int B,
                                    int H, int n, int d, int N, float tau, float *out, void *ws,
                                    size_t ws_bytes, int32_t *dev_status, cudaStream_t stream)
{
    had_status_t s = check_soft(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!Q || !K || !V || !sigma_q || !sigma_k || !out || !ws) return HAD_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || !aligned16(ws))
        return HAD_ERR_INVALID_ARG;
    if (!finite_float(c) || !(c > 0.0f) || !finite_float(tau)) return HAD_ERR_INVALID_ARG;
    const SoftWorkspace w = soft_layout(B, H, n, d, N);
    if (ws_bytes < w.total) return HAD_ERR_WORKSPACE;
    char *base = static_cast<char *>(ws);
    auto *tq = reinterpret_cast<float *>(base + w.tq);
    auto *tk = reinterpret_cast<float *>(base + w.tk);
    auto *idx = reinterpret_cast<int32_t *>(base + w.idx);
    auto *lg = reinterpret_cast<float *>(base + w.logits);
    auto *S = reinterpret_cast<float *>(base + w.scratch);
    if ((s = launch_soft_codes(Q, dt, sigma_q, c, B, H, n, d, tq, dev_status, stream)) != HAD_OK)
        return s;
    if ((s = launch_soft_codes(K, dt, sigma_k, c, B, H, n, d, tk, dev_status, stream)) != HAD_OK)
        return s;
    if ((s = launch_soft_topn(tq, tk, B, H, n, d, N, idx, lg, S, stream)) != HAD_OK) return s;
    return launch_av(idx, lg, V, dt, B, H, n, d, N, tau, out, nullptr, dev_status, stream);
}

had_status_t had_attention_bwd(const void *Q, const void *K, const void *V, had_dtype_t dt,
                               const float *sigma_q, const float *sigma_k, const float *dout,
                               const int32_t *idx, const int16_t *logits, int B, int H, int n,
                               int d, int N, float tau, float clip, float *dq, float *dk,
                               float *dv, void *ws, size_t ws_bytes, int32_t *dev_status,
                               cudaStream_t stream)
{
    had_status_t s = check_topn(B, H, n, d, N);
    if (s != HAD_OK) return s;
    if ((long long)B * H > INT_MAX) return HAD_ERR_UNSUPPORTED;
    if (dt != HAD_BF16 && dt != HAD_F32) return HAD_ERR_INVALID_ARG;
    if (!Q || !K || !V || !sigma_q || !sigma_k || !dout || !dq || !dk || !dv || !ws)
        return HAD_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || !aligned16(ws))
        return HAD_ERR_INVALID_ARG;
    if (!finite_float(tau) || !(clip >= 0.0f)) return HAD_ERR_INVALID_ARG;
    if ((idx == nullptr) != (logits == nullptr)) return HAD_ERR_INVALID_ARG;
    if (idx && (!aligned16(idx) || !aligned16(logits))) return HAD_ERR_INVALID_ARG;
    const BwdWorkspace w = bwd_layout(B, H, n, d, N);
    if (ws_bytes < w.total) return HAD_ERR_WORKSPACE;
    char *base = static_cast<char *>(ws);
    if (dt == HAD_BF16) {
        const auto *q = static_cast<const __nv_bfloat16 *>(Q);
        const auto *k = static_cast<const __nv_bfloat16 *>(K);
        const auto *v = static_cast<const __nv_bfloat16 *>(V);
        return d == 64 ? launch_bwd_typed<__nv_bfloat16, 64>(q, k, v, sigma_q, sigma_k, dout, idx, logits, B,
                                                              H, n, N, tau, clip, dq, dk, dv, w,
                                                              base, dev_status, stream)
                       : launch_bwd_typed<__nv_bfloat16, 128>(q, k, v, sigma_q, sigma_k, dout, idx, logits, B,
                                                               H, n, N, tau, clip, dq, dk, dv, w,
                                                               base, dev_status, stream);
    }
    const auto *q = static_cast<const float *>(Q);
    const auto *k = static_cast<const float *>(K);
    const auto *v = static_cast<const float *>(V);
    return d == 64 ? launch_bwd_typed<float, 64>(q, k, v, sigma_q, sigma_k, dout, idx, logits, B, H, n, N,
                                                 tau, clip, dq, dk, dv, w, base, dev_status,
                                                 stream)
                   : launch_bwd_typed<float, 128>(q, k, v, sigma_q, sigma_k, dout, idx, logits, B, H, n, N,
                                                  tau, clip, dq, dk, dv, w, base, dev_status,
                                                  stream);
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
    case HAD_OP_ATTENTION_PREPARE:
    case HAD_OP_ATTENTION_CORE:
        if (check_topn(B, H, n, d, N) != HAD_OK) return (size_t)-1;
        return fwd_layout(B, H, n, d, N).total;
    case HAD_OP_TOPN_MASS:
        return check_shape(B, H, n, d) == HAD_OK ? 0 : (size_t)-1;
    case HAD_OP_ATTENTION_CAUSAL:
        return check_topn(B, H, n, d, N) == HAD_OK ? fwd_layout(B, H, n, d, N).total
                                                   : (size_t)-1;
    case HAD_OP_SOFT_BINARIZE:
        return check_shape(B, H, n, d) == HAD_OK ? 0 : (size_t)-1;
    case HAD_OP_SOFT_TOPN:
        return check_soft(B, H, n, d, N) == HAD_OK ? soft_scratch_bytes(B, H, n) : (size_t)-1;
    case HAD_OP_SOFT_SOFTMAX_AV:
        return check_topn(B, H, n, d, N) == HAD_OK ? 0 : (size_t)-1;
    case HAD_OP_SOFT_ATTENTION_FWD:
        return check_soft(B, H, n, d, N) == HAD_OK ? soft_layout(B, H, n, d, N).total
                                                   : (size_t)-1;
    case HAD_OP_ATTENTION_BWD:
        return check_topn(B, H, n, d, N) == HAD_OK ? bwd_layout(B, H, n, d, N).total
                                                   : (size_t)-1;
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
    case HAD_OP_ATTENTION_PREPARE:
        return check_topn(B, H, n, d, N) == HAD_OK ? 2 : -1;
    case HAD_OP_ATTENTION_CORE:
        return check_topn(B, H, n, d, N) == HAD_OK ? 2 : -1;
    case HAD_OP_TOPN_MASS:
        return check_shape(B, H, n, d) == HAD_OK ? 1 : -1;
    case HAD_OP_ATTENTION_CAUSAL:
        return check_topn(B, H, n, d, N) == HAD_OK ? 4 : -1;
    case HAD_OP_SOFT_BINARIZE:
        return check_shape(B, H, n, d) == HAD_OK ? 1 : -1;
    case HAD_OP_SOFT_TOPN:
        return check_soft(B, H, n, d, N) == HAD_OK ? 2 * soft_passes(B, H, n) : -1;
    case HAD_OP_SOFT_SOFTMAX_AV:
        return check_topn(B, H, n, d, N) == HAD_OK ? 1 : -1;
    case HAD_OP_SOFT_ATTENTION_FWD:
        return check_soft(B, H, n, d, N) == HAD_OK ? 3 + 2 * soft_passes(B, H, n) : -1;
    case HAD_OP_ATTENTION_BWD:
        return check_topn(B, H, n, d, N) == HAD_OK ? 8 : -1;
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
