// had_av.cuh -- softmax over the kept logits and sparse product with V
// (Eq. 7 of "Hamming Attention Distillation", pith.science review, "What
// carries the argument": softmax and value accumulation on the sparse
// matrix; the referee report notes V stays in full precision).
//
// One warp per query row.  Lane l owns d/32 consecutive output columns, so
// each gathered V row is read by the whole warp as one coalesced 128/256-byte
// (bf16) or 256/512-byte (fp32) transaction from L2.  Kept entries are
// processed 32 at a time: lane l loads index and logit l of the chunk,
// computes its weight exp(tau*(s - m)) once, and the warp broadcasts both.
// Accumulation is fp32; the result is divided by Z at the end.
#pragma once
#include "had_common.cuh"

namespace had {

template <typename T, int PER>
struct VRow;

template <>
struct VRow<__nv_bfloat16, 2> {
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&v)[2])
    {
        uint32_t u = __ldg(reinterpret_cast<const uint32_t *>(p));
        v[0] = bf16_lo(u); v[1] = bf16_hi(u);
    }
};
template <>
struct VRow<__nv_bfloat16, 4> {
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&v)[4])
    {
        uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    }
};
template <>
struct VRow<float, 2> {
    __device__ __forceinline__ static void load(const float *p, float (&v)[2])
    {
        float2 u = __ldg(reinterpret_cast<const float2 *>(p));
        v[0] = u.x; v[1] = u.y;
    }
};
template <>
struct VRow<float, 4> {
    __device__ __forceinline__ static void load(const float *p, float (&v)[4])
    {
        float4 u = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
sparse_softmax_av_kernel(const int32_t *__restrict__ idx, const int16_t *__restrict__ logits,
                         const T *__restrict__ V, int n, int N, float tau, long long rows,
                         float *__restrict__ out, float *__restrict__ p, int32_t *status)
{
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const long long row = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    if (row >= rows) return;
    const long long head = row / n;
    const int32_t *ir = idx + row * N;
    const int16_t *lr = logits + row * N;
    const T *vh = V + head * n * (long long)D;

    // an index of -1 marks an empty slot (rows of the causal form that see
    // fewer than N keys): it weighs nothing and takes no part in the max
    int m = -2147483647;
    for (int k = lane; k < N; k += 32)
        if (ir[k] != -1) m = max(m, (int)lr[k]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFullMask, m, o));

    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
    float z = 0.0f;
    for (int k0 = 0; k0 < N; k0 += 32) {
        const int k = k0 + lane;
        int j = 0;
        float w = 0.0f;
        if (k < N) {
            j = ir[k];
            if (j == -1) {
                w = 0.0f;
            } else if (j < 0 || j >= n) {
                flag(status, HAD_ERR_INVALID_ARG);
                j = 0;
                w = 0.0f;
            } else {
                w = expf(tau * (float)((int)lr[k] - m));
            }
        }
        z += w;
        const int cnt = min(32, N - k0);
        for (int t = 0; t < cnt; ++t) {
            const int jt = __shfl_sync(kFullMask, j, t);
            if (jt == -1) continue;   // empty slot; the same t on every lane
            const float wt = __shfl_sync(kFullMask, w, t);
            float v[PER];
            VRow<T, PER>::load(vh + (long long)jt * D + lane * PER, v);
#pragma unroll
            for (int e = 0; e < PER; ++e) acc[e] = fmaf(wt, v[e], acc[e]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFullMask, z, o);
    // z >= 1 whenever the row keeps a key (its largest logit weighs 1); a
    // row of empty slots only gets zeros
    const float inv = z > 0.0f ? 1.0f / z : 0.0f;
    float *orow = out + row * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) orow[e] = acc[e] * inv;
    if (p) {
        for (int k = lane; k < N; k += 32) {
            const int j = ir[k];
            const float w = (j < 0 || j >= n) ? 0.0f : expf(tau * (float)((int)lr[k] - m));
            p[row * N + k] = w * inv;
        }
    }
}

}  // namespace had
