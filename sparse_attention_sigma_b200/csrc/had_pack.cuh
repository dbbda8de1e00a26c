// had_pack.cuh -- standardize + sign + bit-pack (Eqs. 4-5 with the Eq. 12
// coefficients of "Hamming Attention Distillation", pith.science review,
// "What carries the argument").
//
// HBM-bound: every element is read once (16-byte vector loads) and 1 bit per
// element is written, as whole 32-bit words.  Word w of a row holds elements
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

// One thread per output word: 32 consecutive elements of a row (16-byte
// vector loads) give the 32 bits of one uint32.  With a normal sigma an
// element at or below -sigma * 2^-100 is surely negative after the division
// and one at or above zero surely not, so the sign is a comparison; only a
// word holding an element strictly between (possible, never seen in
// practice) takes the exact IEEE division, for all 32 elements.
// words = B*H*n*d/32; word w covers elements 32w .. 32w+31 of the tensor.
template <typename T>
__global__ void __launch_bounds__(256)
pack_bits_kernel(const T *__restrict__ x, const float *__restrict__ sigma, int H, int n, int d,
                 long long words, uint32_t *__restrict__ bits, int32_t *status)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    const int words_per_row = d >> 5;
    int cached = -1;
    SignRule rule = sign_rule(1.0f);
    for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < words; w += stride) {
        const int head = (int)((w / words_per_row / n) % H);
        if (head != cached) {
            cached = head;
            rule = sign_rule(__ldg(sigma + head));
            if (rule.bad) flag(status, HAD_ERR_BAD_SIGMA);
        }
        float v[32];
#pragma unroll
        for (int c = 0; c < 4; ++c)
            Load8<T>::run(x + w * 32 + 8 * c, *reinterpret_cast<float(*)[8]>(v + 8 * c));
        uint32_t word = 0;
        bool unsure = !rule.fast;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            word |= (uint32_t)(v[i] <= -rule.thr) << i;
            unsure |= (v[i] < 0.0f) && (v[i] > -rule.thr);
        }
        if (unsure) {
            word = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) word |= negative_bit(v[i], rule) << i;
        }
        bits[w] = word;
    }
}

}  // namespace had
