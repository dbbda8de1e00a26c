// had_bwd.cuh -- backward pass of the binarized top-N forward for the
// straight-through training stage ("Hamming Attention Distillation",
// pith.science review: a straight-through estimator finishes the
// binarization after the tanh stages).
//
// The kept set is a fixed selection; softmax and value product are
// differentiated exactly, and the sign passes the gradient where
// |x / sigma| <= clip.  Per head, over the pairs (query i, kept key j):
//   dV_j  = sum_i p_ij dO_i              dp_ij = dO_i . V_j
//   ds_ij = tau p_ij (dp_ij - D_i)       D_i   = sum_j p_ij dp_ij
//   dQb_i = sum_j ds_ij Kb_j             dKb_j = sum_i ds_ij Qb_i
//   dQ = dQb [|zq| <= clip] / sigma_q,   dK likewise.
// Query-side sums gather along a row's kept list (bwd_rows_kernel).  The
// key-side sums need the transposed lists: a counting sort by key builds
// them (count, scan, fill) and bwd_keys_kernel gathers along each key's
// list.  The fill places a key's entries in the order the atomics hand out,
// so the key-side fp32 sums are not bitwise reproducible run to run.
#pragma once
#include "had_common.cuh"
#include "had_av.cuh"

namespace had {

// Signs of the D/8 elements that lane l8 of an 8-lane group owns, from the
// packed bits of one row: bit e of the result is element l8 * D/8 + e.
template <int D>
__device__ __forceinline__ uint32_t slice_bits(const uint32_t *row_bits, int l8)
{
    constexpr int EPL = D / 8;
    const int first = l8 * EPL;
    const uint32_t w = __ldg(row_bits + (first >> 5));
    return (w >> (first & 31)) & (EPL == 32 ? 0xffffffffu : ((1u << EPL) - 1u));
}

// acc[e] += (bit e ? -x : x)
template <int EPL>
__device__ __forceinline__ void add_signed(uint32_t bits, float x, float (&acc)[EPL])
{
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] += ((bits >> e) & 1u) ? -x : x;
}

// Sum over the four 8-lane groups; group g then holds elements
// l8 * EPL + g * EPL/4 .. + EPL/4 - 1 of the row in o[].
template <int EPL>
__device__ __forceinline__ void group_quarter(float (&acc)[EPL], int g, float (&o)[EPL / 4])
{
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        acc[e] += __shfl_xor_sync(kFullMask, acc[e], 8);
        acc[e] += __shfl_xor_sync(kFullMask, acc[e], 16);
    }
    constexpr int Q4 = EPL / 4;
#pragma unroll
    for (int e = 0; e < Q4; ++e) {
        float x = acc[e];
#pragma unroll
        for (int gg = 1; gg < 4; ++gg) x = (g == gg) ? acc[Q4 * gg + e] : x;
        o[e] = x;
    }
}

// Straight-through gradient of one element of x: dxb / sigma where
// |x / sigma| <= clip, else 0.
__device__ __forceinline__ float ste(float dxb, float x, float sigma, float clip)
{
    return fabsf(__fdiv_rn(x, sigma)) <= clip ? __fdiv_rn(dxb, sigma) : 0.0f;
}

template <typename T>
__device__ __forceinline__ float load_scalar(const T *p);
template <>
__device__ __forceinline__ float load_scalar<float>(const float *p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_scalar<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __bfloat162float(*p);
}

template <int Q4>
__device__ __forceinline__ void store_quarter(float *dst, const float (&o)[Q4])
{
    if constexpr (Q4 == 2)
        *reinterpret_cast<float2 *>(dst) = make_float2(o[0], o[1]);
    else
        *reinterpret_cast<float4 *>(dst) = make_float4(o[0], o[1], o[2], o[3]);
}

// One warp per query row.  Pass A gathers V rows (8-lane groups, as in the
// forward's softmax-V kernel) for dp and stores the unnormalised weights
// and dp; pass B turns them into p and ds and gathers the kept keys' sign
// bits into dQb.  Also clears cnt[row] for the counting sort that follows.
template <typename T, int D>
__global__ void __launch_bounds__(256)
bwd_rows_kernel(const int32_t *__restrict__ idx, const int16_t *__restrict__ logits,
                const T *__restrict__ V, const float *__restrict__ dout,
                const T *__restrict__ Q, const float *__restrict__ sigma_q,
                const uint32_t *__restrict__ kbits, int H, int n, int N, float tau, float clip,
                long long rows, float *__restrict__ P, float *__restrict__ DS,
                float *__restrict__ dq, int32_t *__restrict__ cnt, int32_t *status)
{
    using S = VSlice<T, D>;
    using F = VSlice<float, D>;
    constexpr int EPL = S::EPL;
    constexpr int VEC = S::VEC;
    constexpr int FV = F::VEC;
    constexpr int DW = D / 32;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 3;
    const int l8 = lane & 7;
    const long long row = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    if (row >= rows) return;
    if (lane == 0) cnt[row] = 0;
    const long long head = row / n;
    const int32_t *ir = idx + row * N;
    const int16_t *lr = logits + row * N;
    const T *vh = V + head * n * (long long)D;
    const uint32_t *kbh = kbits + head * n * (long long)DW;
    float *pr = P + row * N;
    float *dsr = DS + row * N;

    // this lane's slice of dO_i
    float go[EPL];
    {
        uint4 u[FV];
        F::load(dout + row * D, l8, u);
#pragma unroll
        for (int e = 0; e < EPL; ++e) go[e] = 0.0f;
        F::fma(u, 1.0f, go);
    }

    int m = -2147483647;
    for (int k = lane; k < N; k += 32)
        if (ir[k] != -1) m = max(m, (int)lr[k]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFullMask, m, o));

    // pass A: w = exp(tau (s - m)) and dp = dO_i . V_j
    float z = 0.0f, zd = 0.0f;
    for (int k0 = 0; k0 < N; k0 += 32) {
        const int k = k0 + lane;
        int j = -1;
        float w = 0.0f;
        if (k < N) {
            j = ir[k];
            if (j == -1) {
                w = 0.0f;
            } else if (j < 0 || j >= n) {
                flag(status, HAD_ERR_INVALID_ARG);
                j = -1;
            } else {
                w = expf(tau * (float)((int)lr[k] - m));
            }
        }
        float dp = 0.0f;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int t = r * 4 + g;
            const int jt = __shfl_sync(kFullMask, j, t);
            float part = 0.0f;
            if (jt != -1) {
                uint4 u[VEC];
                S::load(vh + (long long)jt * D, l8, u);
                float vv[EPL];
#pragma unroll
                for (int e = 0; e < EPL; ++e) vv[e] = 0.0f;
                S::fma(u, 1.0f, vv);
#pragma unroll
                for (int e = 0; e < EPL; ++e) part = fmaf(go[e], vv[e], part);
            }
            part += __shfl_xor_sync(kFullMask, part, 1);
            part += __shfl_xor_sync(kFullMask, part, 2);
            part += __shfl_xor_sync(kFullMask, part, 4);
            // key k0 + lane was handled in round lane / 4 by group lane % 4
            const float got = __shfl_sync(kFullMask, part, (lane & 3) * 8);
            if ((lane >> 2) == r) dp = got;
        }
        if (k < N) {
            pr[k] = w;
            dsr[k] = dp;
        }
        z += w;
        zd = fmaf(w, dp, zd);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        z += __shfl_xor_sync(kFullMask, z, o);
        zd += __shfl_xor_sync(kFullMask, zd, o);
    }
    const float inv = z > 0.0f ? 1.0f / z : 0.0f;
    const float Dm = zd * inv;

    // pass B: p, ds, and dQb = sum ds_ij Kb_j
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.0f;
    for (int k0 = 0; k0 < N; k0 += 32) {
        const int k = k0 + lane;
        int j = -1;
        float ds = 0.0f;
        if (k < N) {
            j = ir[k];
            if (j < 0 || j >= n) j = -1;
            const float p = pr[k] * inv;
            ds = tau * p * (dsr[k] - Dm);
            if (j == -1) ds = 0.0f;
            pr[k] = p;
            dsr[k] = ds;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int t = r * 4 + g;
            const int jt = __shfl_sync(kFullMask, j, t);
            const float dst = __shfl_sync(kFullMask, ds, t);
            if (jt != -1) add_signed<EPL>(slice_bits<D>(kbh + (long long)jt * DW, l8), dst, acc);
        }
    }
    float o[EPL / 4];
    group_quarter<EPL>(acc, g, o);
    const int c0 = l8 * EPL + g * (EPL / 4);
    const float sg = __ldg(sigma_q + (int)(head % H));
#pragma unroll
    for (int e = 0; e < EPL / 4; ++e) o[e] = ste(o[e], load_scalar<T>(Q + row * D + c0 + e), sg, clip);
    store_quarter<EPL / 4>(dq + row * D + c0, o);
}

// Kept pairs per key: cnt[head n + j] counts the rows of the head that keep j.
__global__ void __launch_bounds__(256)
bwd_count_kernel(const int32_t *__restrict__ idx, long long pairs, int n, int N,
                 int32_t *__restrict__ cnt)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < pairs; e += stride) {
        const int j = __ldg(idx + e);
        if (j < 0 || j >= n) continue;
        const long long head = e / N / n;
        atomicAdd(cnt + head * n + j, 1);
    }
}

// One CTA per head: exclusive scan of the head's n counts, offset by the
// head's first slot head n N, into off; the fill's per-key cursors (counts
// from the key's start) are cleared.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
bwd_scan_kernel(const int32_t *__restrict__ cnt, int n, int N, long long *__restrict__ off,
                uint32_t *__restrict__ cursor)
{
    __shared__ long long wsum[kScanThreads / 32];
    __shared__ long long carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long head = blockIdx.x;
    const int32_t *c = cnt + head * n;
    if (tid == 0) carry = head * n * (long long)N;
    __syncthreads();
    for (int j0 = 0; j0 < n; j0 += kScanThreads) {
        const int j = j0 + tid;
        const long long v = j < n ? __ldg(c + j) : 0;
        long long incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(kFullMask, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        long long before = carry;
        for (int w = 0; w < warp; ++w) before += wsum[w];
        if (j < n) {
            off[head * n + j] = before + incl - v;
            cursor[head * n + j] = 0u;
        }
        __syncthreads();
        if (tid == kScanThreads - 1) carry = before + incl;
        __syncthreads();
    }
}

// Every kept pair to its key's list as one 16-byte record (query row within
// the head, p, ds, unused): one store per pair.
__global__ void __launch_bounds__(256)
bwd_fill_kernel(const int32_t *__restrict__ idx, const float *__restrict__ P,
                const float *__restrict__ DS, long long pairs, int n, int N,
                const long long *__restrict__ off, uint32_t *__restrict__ cursor,
                int4 *__restrict__ rec)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < pairs; e += stride) {
        const int j = __ldg(idx + e);
        if (j < 0 || j >= n) continue;
        const long long row = e / N;
        const long long head = row / n;
        const long long key = head * n + j;
        const long long pos = __ldg(off + key) + atomicAdd(cursor + key, 1u);
        rec[pos] = make_int4((int)(row - head * n), __float_as_int(__ldg(P + e)),
                             __float_as_int(__ldg(DS + e)), 0);
    }
}

// One warp per key: dV_j and dKb_j along the key's list (8-lane groups, one
// entry per group per round), then the straight-through step for K.
template <typename T, int D>
__global__ void __launch_bounds__(256)
bwd_keys_kernel(const long long *__restrict__ off, const int32_t *__restrict__ cnt,
                const int4 *__restrict__ rec, const float *__restrict__ dout,
                const uint32_t *__restrict__ qbits, const T *__restrict__ K,
                const float *__restrict__ sigma_k, int H, int n, float clip, long long keys,
                float *__restrict__ dk, float *__restrict__ dv)
{
    using F = VSlice<float, D>;
    constexpr int EPL = F::EPL;
    constexpr int FV = F::VEC;
    constexpr int DW = D / 32;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 3;
    const int l8 = lane & 7;
    const long long key = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    if (key >= keys) return;
    const long long head = key / n;
    const long long start = __ldg(off + key);
    const int c = __ldg(cnt + key);
    const float *doh = dout + head * n * (long long)D;
    const uint32_t *qbh = qbits + head * n * (long long)DW;

    float av[EPL], ak[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) { av[e] = 0.0f; ak[e] = 0.0f; }
    for (int k0 = 0; k0 < c; k0 += 32) {
        const int k = k0 + lane;
        int i = -1;
        float p = 0.0f, ds = 0.0f;
        if (k < c) {
            const int4 e = __ldg(rec + start + k);
            i = e.x;
            p = __int_as_float(e.y);
            ds = __int_as_float(e.z);
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int t = r * 4 + g;
            const int it = __shfl_sync(kFullMask, i, t);
            const float pt = __shfl_sync(kFullMask, p, t);
            const float dst = __shfl_sync(kFullMask, ds, t);
            if (it != -1) {
                uint4 u[FV];
                F::load(doh + (long long)it * D, l8, u);
                F::fma(u, pt, av);
                add_signed<EPL>(slice_bits<D>(qbh + (long long)it * DW, l8), dst, ak);
            }
        }
    }
    float ov[EPL / 4], ok[EPL / 4];
    group_quarter<EPL>(av, g, ov);
    group_quarter<EPL>(ak, g, ok);
    const int c0 = l8 * EPL + g * (EPL / 4);
    const float sg = __ldg(sigma_k + (int)(head % H));
#pragma unroll
    for (int e = 0; e < EPL / 4; ++e) ok[e] = ste(ok[e], load_scalar<T>(K + key * D + c0 + e), sg, clip);
    store_quarter<EPL / 4>(dv + key * D + c0, ov);
    store_quarter<EPL / 4>(dk + key * D + c0, ok);
}

}  // namespace had
