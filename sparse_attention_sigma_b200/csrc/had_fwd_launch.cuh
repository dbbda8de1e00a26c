// had_fwd_launch.cuh -- host side of the fused forward: the workspace
// layout of had_attention_fwd / _prepare / _core and the launches of the
// operand preparation, the fused kernels and their exact fix-up.  Kept apart
// from the other entry points so that this file, with the kernels it
// launches, is the whole of the fused path.
#pragma once
#include <atomic>
#include <climits>
#include <cmath>
#include <cstddef>
#include <cuda_runtime.h>

#include "had.h"
#include "had_common.cuh"
#include "had_prep.cuh"
#include "had_fused.cuh"
#include "had_fwd_tc.cuh"

namespace had {
namespace fwdapi {

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

inline had_status_t launch_status()
{
    return cudaGetLastError() == cudaSuccess ? HAD_OK : HAD_ERR_CUDA;
}

// Limit of every wait of the fused kernels for another role of the same CTA
// (a copy, an MMA, an epilogue warp).  Far beyond any real wait by default.
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
inline std::atomic<unsigned long long> &wait_limit_ns()
{
    static std::atomic<unsigned long long> ns{kDefaultWaitNs};
    return ns;
}

// Workspace of the fused forward: tensor-core operand tiles of Q, K and V^T,
// packed signs, per-head V scale and key column sums, and the list of rows
// the fix-up kernel recomputes.
struct FwdWorkspace {
    size_t qop, qop2, kop, vop, qbits, kbits, vpart, miss, vexp, kpart, ksum, miss_rows, total;
    int qtiles, ktiles, kstride, vchunks;
};

inline FwdWorkspace fwd_layout(int B, int H, int n, int d, int N)
{
    (void)N;
    const size_t bh = (size_t)B * H;
    FwdWorkspace w;
    const int qt = d == 64 ? fused::Cfg<64>::QT : fused::Cfg<128>::QT;
    w.qtiles = (n + fused::kRows - 1) / fused::kRows;
    w.qtiles = (w.qtiles + qt - 1) / qt * qt;
    w.ktiles = (n + fused::kKeys - 1) / fused::kKeys;
    w.kstride = (w.ktiles + 1) / 2 * 2;                 // whole 128-key pairs
    // V chunks of 8192 elements for the per-head maximum
    w.vchunks = (int)(((size_t)n * d + 8191) / 8192);
    w.qop = 0;
    w.qop2 = w.qop + align256(bh * w.qtiles * fused::kRows * d);
    w.kop = w.qop2 + align256(bh * w.qtiles * fused::kRows * d);
    w.vop = w.kop + align256(bh * w.kstride * fused::kKeys * d);
    w.qbits = w.vop + align256(bh * w.kstride * fused::kKeys * d * 2);
    w.kbits = w.qbits + align256(bh * n * (d / 8));
    w.vpart = w.kbits + align256(bh * n * (d / 8));
    w.miss = w.vpart + align256(bh * w.vchunks * 4);
    w.vexp = w.miss + align256(8);                      // miss counter, fix-up done counter
    w.kpart = w.vexp + align256(bh * 4);
    w.ksum = w.kpart + align256(bh * w.kstride * d);
    w.miss_rows = w.ksum + align256(bh * d * 4);
    w.total = w.miss_rows + align256(bh * (size_t)w.qtiles * fused::kRows * 4);
    return w;
}

// Operand preparation: Q/K signs as tensor-core tiles and packed bits, the
// key column sums and the V chunk maxima in one launch, then V^T in fp16 with
// its per-head scale (and the per-head key sums).  The +/-64 copy of Q is
// written only for the 64-key kernel (qop2 = true), which reads it.
template <typename T, int D>
had_status_t prep_typed(const T *Q, const T *K, const T *V, const float *sq, const float *sk,
                        int B, int H, int n, char *ws, const FwdWorkspace &w, int32_t *status,
                        cudaStream_t st, bool qop2 = false)
{
    const long long bh = (long long)B * H;
    const long long blocks = bh * (w.qtiles + w.kstride + w.vchunks);
    if (blocks > INT_MAX || bh * w.kstride > INT_MAX) return HAD_ERR_UNSUPPORTED;
    auto *vpart = reinterpret_cast<float *>(ws + w.vpart);
    // Q as the negated signs (and, for the 64-key kernel, +/-64), K as +/-4:
    // the i8 MMA accumulates -4 s (or 256 s)
    prep::operands_kernel<T, D><<<(unsigned)blocks, 256, 0, st>>>(
        Q, K, V, sq, sk, H, n, (int)bh, w.qtiles, w.kstride, w.vchunks,
        reinterpret_cast<int8_t *>(ws + w.qop),
        qop2 ? reinterpret_cast<int8_t *>(ws + w.qop2) : nullptr,
        reinterpret_cast<int8_t *>(ws + w.kop), reinterpret_cast<uint16_t *>(ws + w.qbits),
        reinterpret_cast<uint16_t *>(ws + w.kbits), reinterpret_cast<int8_t *>(ws + w.kpart),
        vpart, reinterpret_cast<int *>(ws + w.miss), status);
    const int ctiles = (w.kstride + 256 / D - 1) / (256 / D);   // CTAs per head, 256 / D tiles each
    prep::v_operand_kernel<T, D><<<(unsigned)(bh * ctiles), 256, 0, st>>>(
        V, n, w.kstride, ctiles, vpart, w.vchunks, reinterpret_cast<__half *>(ws + w.vop),
        reinterpret_cast<int *>(ws + w.vexp), reinterpret_cast<const int8_t *>(ws + w.kpart),
        reinterpret_cast<int *>(ws + w.ksum));
    return launch_status();
}

// Standard normal quantile Phi^-1(p) by bisection on erfc (host, once per
// call); it only places the fused kernel's threshold window.
inline float normal_quantile(double p)
{
    p = std::fmin(std::fmax(p, 1e-9), 1.0 - 1e-9);
    double lo = -40.0, hi = 40.0;
    for (int i = 0; i < 100; ++i) {
        const double mid = 0.5 * (lo + hi);
        if (0.5 * std::erfc(-mid / std::sqrt(2.0)) < p) lo = mid;
        else hi = mid;
    }
    return (float)(0.5 * (lo + hi));
}

inline int sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms < 1)
        return 148;
    return sms;
}

// Non-causal core: the 128-key tensor-core kernel.
template <int D>
had_status_t core_tc(const void *V, bool v_f32, int B, int H, int n, int N, float tau,
                     float *out, int32_t *dbg_idx, int16_t *dbg_lg, char *ws,
                     const FwdWorkspace &w, int32_t *status, cudaStream_t st)
{
    using C = tcfwd::Cfg<D>;
    const long long bh = (long long)B * H;
    const bool dbg = dbg_idx != nullptr || dbg_lg != nullptr;
    // The quota tile's kept ties: found by a scan of the head's key signs in
    // shared memory where they fit and there are 4 key tiles or more (mode
    // 2, measured fastest at 4 and at 32 tiles; at 2 the scan costs more
    // than the mask); else, with few key tiles, a per-chunk mask in pass 2
    // (mode 1) costs less than gathering them after it (mode 0, a fixed
    // latency per CTA; measured crossover near 12 tiles).
    const int T = (n + tcfwd::kKeys - 1) / tcfwd::kKeys;
    const long long kb_bytes = (long long)n * (D / 8);
    // a head's signs start on a 16-byte boundary when their size is a
    // multiple of 16; otherwise the copy widens them by up to 30 bytes
    const long long kb_copy = kb_bytes % 16 == 0 ? kb_bytes : kb_bytes + 32;
    const bool kb = !dbg && T >= 4 && kb_copy <= C::KB_CAP && T <= C::STASH_CAP &&
                    (reinterpret_cast<uintptr_t>(ws + w.kbits) & 15u) == 0;
    const bool q2 = T <= 12;
    auto kernel = dbg  ? tcfwd::attention_tc_kernel<D, true, 0>
                  : kb ? tcfwd::attention_tc_kernel<D, false, 2>
                  : q2 ? tcfwd::attention_tc_kernel<D, false, 1>
                       : tcfwd::attention_tc_kernel<D, false, 0>;
    const int smem_bytes = kb ? C::SMEM_BYTES_KB : C::SMEM_BYTES;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_bytes) != cudaSuccess ||
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return HAD_ERR_CUDA;
    tcfwd::Params p;
    p.qop = reinterpret_cast<int8_t *>(ws + w.qop);
    p.kop = reinterpret_cast<int8_t *>(ws + w.kop);
    p.vop = reinterpret_cast<__half *>(ws + w.vop);
    p.vexp = reinterpret_cast<int *>(ws + w.vexp);
    p.qbits = reinterpret_cast<uint32_t *>(ws + w.qbits);
    p.kbits = reinterpret_cast<uint32_t *>(ws + w.kbits);
    p.v = V;
    p.v_f32 = v_f32 ? 1 : 0;

    p.ksum = reinterpret_cast<int *>(ws + w.ksum);
    p.out = out;
    p.dbg_idx = dbg_idx;
    p.dbg_logits = dbg_lg;
    p.status = status;
    p.miss_count = reinterpret_cast<int *>(ws + w.miss);
    p.miss_rows = reinterpret_cast<int *>(ws + w.miss_rows);
    p.miss_cap = (long long)bh * w.qtiles * fused::kRows;
    p.n = n;
    p.N = N;
    p.qtiles = w.qtiles;
    p.kstride = w.kstride;
    p.ctas_per_head = w.qtiles / C::QT;
    p.c2 = tau * 1.4426950408889634f;
    p.z = normal_quantile((double)N / (double)n);
    p.wait_ns = wait_limit_ns().load();
    const long long blocks = bh * p.ctas_per_head;
    kernel<<<(unsigned)blocks, C::THREADS, smem_bytes, st>>>(p);
    return launch_status();
}

// The 64-key fused kernel: the causal core, and the non-causal core that
// writes the kept set (its per-key path costs less there than the 128-key
// kernel's: 3.6 against 5.1 ms at n 4096, d 64, N 512).  Both read the
// +/-64 Q tiles (qop2), which the preparation writes for them.
template <int D>
had_status_t core_fused64(int B, int H, int n, int N, float tau, float *out, int32_t *dbg_idx,
                          int16_t *dbg_lg, char *ws, const FwdWorkspace &w, int32_t *status,
                          cudaStream_t st, bool causal)
{
    using C = fused::Cfg<D>;
    const long long bh = (long long)B * H;
    const bool dbg = dbg_idx != nullptr || dbg_lg != nullptr;
    auto kernel = !causal ? fused::attention_fwd_kernel<D, true, false>
                  : dbg   ? fused::attention_fwd_kernel<D, true, true>
                          : fused::attention_fwd_kernel<D, false, true>;
    // the CTA takes most of the unified L1 as shared memory
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return HAD_ERR_CUDA;
    fused::Params p;
    p.qop = reinterpret_cast<int8_t *>(ws + w.qop);
    p.qop2 = reinterpret_cast<int8_t *>(ws + w.qop2);
    p.kop = reinterpret_cast<int8_t *>(ws + w.kop);
    p.vop = reinterpret_cast<__half *>(ws + w.vop);
    p.vexp = reinterpret_cast<int *>(ws + w.vexp);
    p.out = out;
    p.dbg_idx = dbg_idx;
    p.dbg_logits = dbg_lg;
    p.status = status;
    p.miss_count = reinterpret_cast<int *>(ws + w.miss);
    p.miss_rows = reinterpret_cast<int *>(ws + w.miss_rows);
    p.miss_cap = (long long)bh * w.qtiles * fused::kRows;
    p.sample_tiles = w.ktiles / 16 > 4 ? w.ktiles / 16 : 4;
    p.n = n;
    p.N = N;
    p.qtiles = w.qtiles;
    p.ktiles = w.ktiles;
    p.kstride = w.kstride;
    p.ctas_per_head = w.qtiles / C::QT;
    p.c2 = tau * 1.4426950408889634f;
    const long long blocks = bh * p.ctas_per_head;
    kernel<<<(unsigned)blocks, C::THREADS, C::SMEM_BYTES, st>>>(p);
    return launch_status();
}

// The fused kernel on prepared operands, then the exact fix-up of the rows
// whose threshold fell outside their window.
// causal: query i sees keys 0 .. i and keeps min(N, i + 1) of them.
// qop2_ready: the preparation wrote the +/-64 Q tiles, so that a call that
// writes the kept set can take the 64-key kernel.
template <typename T, int D>
had_status_t core_typed(const T *V, int B, int H, int n, int N, float tau, float *out,
                        int32_t *dbg_idx, int16_t *dbg_lg, char *ws, const FwdWorkspace &w,
                        int32_t *status, cudaStream_t st, bool causal = false,
                        bool qop2_ready = false)
{
    const bool dbg = dbg_idx != nullptr || dbg_lg != nullptr;
    had_status_t s = causal || (dbg && qop2_ready)
                         ? core_fused64<D>(B, H, n, N, tau, out, dbg_idx, dbg_lg, ws, w, status,
                                           st, causal)
                         : core_tc<D>(V, sizeof(T) == 4, B, H, n, N, tau, out, dbg_idx, dbg_lg,
                                      ws, w, status, st);
    if (s != HAD_OK) return s;
    auto *qbits = reinterpret_cast<uint32_t *>(ws + w.qbits);
    auto *kbits = reinterpret_cast<uint32_t *>(ws + w.kbits);
    auto *miss_count = reinterpret_cast<int *>(ws + w.miss);
    auto *miss_rows = reinterpret_cast<int *>(ws + w.miss_rows);
    auto fixup = causal ? fused::fixup_rows_kernel<T, D, true> : fused::fixup_rows_kernel<T, D, false>;
    fixup<<<sm_count() * 4, 256, 0, st>>>(qbits, kbits, V, n, N, tau, miss_count, miss_count + 1,
                                          miss_rows, out, dbg_idx, dbg_lg);
    return launch_status();
}

template <typename T, int D>
had_status_t launch_fused_typed(const T *Q, const T *K, const T *V, const float *sq,
                                const float *sk, int B, int H, int n, int N, float tau,
                                float *out, int32_t *dbg_idx, int16_t *dbg_lg, char *ws,
                                const FwdWorkspace &w, int32_t *status, cudaStream_t st,
                                bool causal)
{
    // the +/-64 Q tiles for the 64-key kernel: causal, or writing the kept set
    const bool qop2 = causal || dbg_idx != nullptr || dbg_lg != nullptr;
    had_status_t s = prep_typed<T, D>(Q, K, V, sq, sk, B, H, n, ws, w, status, st, qop2);
    if (s != HAD_OK) return s;
    return core_typed<T, D>(V, B, H, n, N, tau, out, dbg_idx, dbg_lg, ws, w, status, st,
                            causal, qop2);
}

template <typename T>
had_status_t launch_fused(const void *Q, const void *K, const void *V, const float *sq,
                          const float *sk, int B, int H, int n, int d, int N, float tau,
                          float *out, int32_t *dbg_idx, int16_t *dbg_lg, char *ws,
                          const FwdWorkspace &w, int32_t *status, cudaStream_t st,
                          bool causal = false)
{
    const T *q = static_cast<const T *>(Q), *k = static_cast<const T *>(K),
            *v = static_cast<const T *>(V);
    return d == 64 ? launch_fused_typed<T, 64>(q, k, v, sq, sk, B, H, n, N, tau, out, dbg_idx,
                                               dbg_lg, ws, w, status, st, causal)
                   : launch_fused_typed<T, 128>(q, k, v, sq, sk, B, H, n, N, tau, out, dbg_idx,
                                                dbg_lg, ws, w, status, st, causal);
}

}  // namespace fwdapi
}  // namespace had
