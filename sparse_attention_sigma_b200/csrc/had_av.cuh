// had_av.cuh -- softmax over the kept logits and sparse product with V
// (Eq. 7 of "Hamming Attention Distillation", pith.science review, "What
// carries the argument": softmax and value accumulation on the sparse
// matrix; the referee report notes V stays in full precision).
//
// One warp per query row; the layout of the gather is described at the
// kernel.  Accumulation is fp32; the result is divided by Z at the end.
#pragma once
#include "had_common.cuh"

namespace had {

// Slice of one V row that a lane of an 8-lane group owns: d/8 consecutive
// elements, loaded as 16-byte vectors and widened to fp32.
template <typename T, int D>
struct VSlice {
    static constexpr int EPL = D / 8;                        // elements per lane
    static constexpr int VEC = EPL * (int)sizeof(T) / 16;    // 16-byte loads per lane
    __device__ __forceinline__ static void load(const T *row, int l8, uint4 (&u)[VEC])
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(row + l8 * EPL);
#pragma unroll
        for (int c = 0; c < VEC; ++c) u[c] = __ldg(src + c);
    }
    __device__ __forceinline__ static void fma(const uint4 (&u)[VEC], float w, float (&acc)[EPL])
    {
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
            const uint32_t x[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
            if constexpr (sizeof(T) == 2) {
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    acc[c * 8 + 2 * h] = fmaf(w, bf16_lo(x[h]), acc[c * 8 + 2 * h]);
                    acc[c * 8 + 2 * h + 1] = fmaf(w, bf16_hi(x[h]), acc[c * 8 + 2 * h + 1]);
                }
            } else {
#pragma unroll
                for (int h = 0; h < 4; ++h) acc[c * 4 + h] = fmaf(w, __uint_as_float(x[h]), acc[c * 4 + h]);
            }
        }
    }
};

// Logits arrive as int16 (binarized codes: integers in [-d, d]) or fp32
// (soft codes); the row maximum and the differences s - m take their type.
template <typename L>
struct LogitT;
template <>
struct LogitT<int16_t> {
    using M = int;
    __device__ __forceinline__ static M lowest() { return -2147483647; }
    __device__ __forceinline__ static float diff(int16_t s, M m) { return (float)((int)s - m); }
};
template <>
struct LogitT<float> {
    using M = float;
    __device__ __forceinline__ static M lowest() { return -__int_as_float(0x7f800000); }
    __device__ __forceinline__ static float diff(float s, M m) { return s - m; }
};

// One warp per query row, split into four 8-lane groups.  Kept entries are
// taken 32 at a time: lane l reads index and logit l of the chunk and
// computes its weight exp(tau (s - m)) once; then in 8 rounds each group
// takes one of the 32 keys (shuffled in), and its 8 lanes read that key's V
// row as 8 slices of d/8 elements.  One warp load instruction thus fetches 4
// whole V rows (coalesced 128-byte lines), and the unrolled rounds keep up to
// 32 rows in flight per warp: the gather is bound by L2 bandwidth, not by
// its latency.  The four groups' partial sums are added with two shuffles at
// the end, and each group stores a quarter of the row.
template <typename T, int D, typename L = int16_t>
__global__ void __launch_bounds__(256)
sparse_softmax_av_kernel(const int32_t *__restrict__ idx, const L *__restrict__ logits,
                         const T *__restrict__ V, int n, int N, float tau, long long rows,
                         float *__restrict__ out, float *__restrict__ p, int32_t *status)
{
    using S = VSlice<T, D>;
    constexpr int EPL = S::EPL;
    constexpr int VEC = S::VEC;
    constexpr int BATCH = VEC >= 4 ? 2 : (VEC == 2 ? 4 : 8);   // rounds whose loads fly together
    const int lane = threadIdx.x & 31;
    const int g = lane >> 3;
    const int l8 = lane & 7;
    const long long row = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    if (row >= rows) return;
    const long long head = row / n;
    const int32_t *ir = idx + row * N;
    const L *lr = logits + row * N;
    const T *vh = V + head * n * (long long)D;
    using LT = LogitT<L>;

    // an index of -1 marks an empty slot (rows of the causal form that see
    // fewer than N keys): it weighs nothing and takes no part in the max
    typename LT::M m = LT::lowest();
    for (int k = lane; k < N; k += 32)
        if (ir[k] != -1) m = max(m, (typename LT::M)lr[k]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFullMask, m, o));

    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.0f;
    float z = 0.0f;
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
                w = 0.0f;
            } else {
                w = expf(tau * LT::diff(lr[k], m));
            }
        }
        z += w;
        if (__all_sync(kFullMask, j == -1)) continue;   // a chunk of empty slots
#pragma unroll
        for (int r0 = 0; r0 < 8; r0 += BATCH) {
            uint4 u[BATCH][VEC];
            float wt[BATCH];
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                const int t = (r0 + b) * 4 + g;
                const int jt = __shfl_sync(kFullMask, j, t);
                wt[b] = __shfl_sync(kFullMask, w, t);
                if (jt != -1) {
                    S::load(vh + (long long)jt * D, l8, u[b]);
                } else {
#pragma unroll
                    for (int c = 0; c < VEC; ++c) u[b][c] = make_uint4(0u, 0u, 0u, 0u);
                    wt[b] = 0.0f;
                }
            }
#pragma unroll
            for (int b = 0; b < BATCH; ++b) S::fma(u[b], wt[b], acc);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFullMask, z, o);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        acc[e] += __shfl_xor_sync(kFullMask, acc[e], 8);
        acc[e] += __shfl_xor_sync(kFullMask, acc[e], 16);
    }
    // z >= 1 whenever the row keeps a key (its largest logit weighs 1); a
    // row of empty slots only gets zeros
    const float inv = z > 0.0f ? 1.0f / z : 0.0f;
    // every group holds the whole sum of slice l8; group g stores quarter g
    constexpr int Q4 = EPL / 4;
    float *orow = out + row * D + l8 * EPL + g * Q4;
    float o[Q4];
#pragma unroll
    for (int e = 0; e < Q4; ++e) {
        // acc[Q4 g + e], selected without dynamic register indexing
        float x = acc[e];
#pragma unroll
        for (int gg = 1; gg < 4; ++gg) x = (g == gg) ? acc[Q4 * gg + e] : x;
        o[e] = x * inv;
    }
    if constexpr (Q4 == 2)
        *reinterpret_cast<float2 *>(orow) = make_float2(o[0], o[1]);
    else
        *reinterpret_cast<float4 *>(orow) = make_float4(o[0], o[1], o[2], o[3]);
    if (p) {
        for (int k = lane; k < N; k += 32) {
            const int j = ir[k];
            const float w = (j < 0 || j >= n) ? 0.0f : expf(tau * LT::diff(lr[k], m));
            p[row * N + k] = w * inv;
        }
    }
}

}  // namespace had
