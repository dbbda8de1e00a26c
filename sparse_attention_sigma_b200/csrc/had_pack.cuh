// had_pack.cuh -- standardize + sign + bit-pack (Eqs. 4-5 with the Eq. 12
// coefficients of "Hamming Attention Distillation", pith.science review,
// "What carries the argument").
//
// HBM-bound: every element is read once (16-byte vector loads) and 1 bit per
// element is written.  A thread turns 8 consecutive elements into one byte;
// four neighbouring lanes merge their bytes into a 32-bit word with two warp
// shuffles, so stores are whole words.  Word w of a row holds elements
// 32w..32w+31 with element 32w+k in bit k; bit = 1 means sign -1.
#pragma once
#include "had_common.cuh"

namespace had {

template <typename T>
struct Load8;

template <>
struct Load8<__nv_bfloat16> {
    __device__ __forceinline__ static void run(const __nv_bfloat16 *p, float (&v)[8])
    {
        uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
        v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
        v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
        v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
        v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
    }
};

template <>
struct Load8<float> {
    __device__ __forceinline__ static void run(const float *p, float (&v)[8])
    {
        float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

// groups = B*H*n*d/8 (a multiple of 4 because d is a multiple of 32).
template <typename T>
__global__ void __launch_bounds__(256)
pack_bits_kernel(const T *__restrict__ x, const float *__restrict__ sigma, int H,
                 int n, int d, long long groups, uint32_t *__restrict__ bits,
                 int32_t *status)
{
    const int lane = threadIdx.x & 31;
    const long long warp0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const int groups_per_row = d >> 3;
    for (long long base = warp0 * 32; base < groups; base += nwarps * 32) {
        const long long g = base + lane;
        uint32_t byte = 0;
        if (g < groups) {
            const long long row = g / groups_per_row;
            const int head = (int)((row / n) % H);
            const SignRule r = sign_rule(__ldg(sigma + head));
            if (r.bad) flag(status, HAD_ERR_BAD_SIGMA);
            float v[8];
            Load8<T>::run(x + g * 8, v);
#pragma unroll
            for (int k = 0; k < 8; ++k) byte |= negative_bit(v[k], r) << k;
        }
        uint32_t pair = byte | (__shfl_down_sync(kFullMask, byte, 1) << 8);
        uint32_t word = pair | (__shfl_down_sync(kFullMask, pair, 2) << 16);
        if ((lane & 3) == 0 && g < groups) bits[g >> 2] = word;
    }
}

}  // namespace had
