// had_pack.cuh -- standardize + sign + bit-pack (Eqs. 4-5 with the Eq. 12
// coefficients of "Hamming Attention Distillation", pith.science review,
// "What carries the argument").
//
// HBM-bound: every element is read once (coalesced 16-byte vector loads) and
// 1 bit per element is written, as whole 32-bit words.  Word w of a row holds
// elements 32w..32w+31 with element 32w+k in bit k; bit = 1 means sign -1.
#pragma once
#include <type_traits>

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

// One (b, h) slab per blockIdx.y (striding over slabs beyond the grid), so
// sigma is read once per block and slab.  A warp streams 1024 consecutive
// elements per step in four 256-element chunks whose loads are in flight
// together: in a chunk lane L takes elements 8L..8L+7 (one 16-byte load for
// bf16, so the warp reads 512 contiguous bytes), forms their 8 bits, and the
// four lanes of a 32-element word join their bytes with two shuffles; every
// fourth lane stores the word.  With a normal
// sigma an element at or below -sigma * 2^-100 is surely negative after the
// division and one at or above zero surely not, so the sign is a
// comparison (for bf16 one on the raw bits, four values per few integer
// instructions: bf16_signs4); only a lane holding an element strictly
// between (possible, never seen in practice: -0, tiny values, -inf, NaN)
// takes the exact IEEE division, for its 8 elements.
// slab = n*d elements (a multiple of 32, so a word never straddles slabs).
template <typename T>
__global__ void __launch_bounds__(256)
pack_bits_kernel(const T *__restrict__ x, const float *__restrict__ sigma, int H, long long slab,
                 long long slabs, uint32_t *__restrict__ bits, int32_t *status)
{
    for (long long bh = blockIdx.y; bh < slabs; bh += gridDim.y) {
        const SignRule rule = sign_rule(__ldg(sigma + bh % H));
        const uint32_t kge = bf16_kge(rule);
        if (rule.bad && blockIdx.x == 0 && threadIdx.x == 0) flag(status, HAD_ERR_BAD_SIGMA);
        const T *xs = x + bh * slab;
        uint32_t *bs = bits + bh * (slab / 32);
        const int lane = threadIdx.x & 31;
        // four 256-element chunks per warp step, their loads in flight together
        const long long quads = (slab + 1023) / 1024;
        const long long step = (long long)gridDim.x * (blockDim.x / 32);
        const long long q0 = blockIdx.x * (long long)(blockDim.x / 32) + (threadIdx.x >> 5);
        for (long long q = q0; q < quads; q += step) {
            constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
            uint4 raw[4];                             // bf16: the 8 values' bits
            float v[4][8];                            // f32: the values
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const long long e0 = q * 1024 + k * 256 + 8 * lane;
                const bool in = e0 < slab;            // all 8 or none: slab is a multiple of 32
                if constexpr (kBf16) {
                    raw[k] = in ? __ldg(reinterpret_cast<const uint4 *>(xs + e0)) : make_uint4(0u, 0u, 0u, 0u);
                } else if (in) {
                    Load8<T>::run(xs + e0, v[k]);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[k][i] = 0.0f;
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const long long e0 = q * 1024 + k * 256 + 8 * lane;
                uint32_t byte = 0;
                bool unsure = !rule.fast;
                if constexpr (kBf16) {
                    uint32_t n0, u0, n1, u1;
                    bf16_signs4(raw[k].x, raw[k].y, kge, n0, u0);
                    bf16_signs4(raw[k].z, raw[k].w, kge, n1, u1);
                    byte = flags4(n0) | flags4(n1) << 4;
                    unsure |= (u0 | u1) != 0u;
                    if (unsure) {
                        v[k][0] = bf16_lo(raw[k].x); v[k][1] = bf16_hi(raw[k].x);
                        v[k][2] = bf16_lo(raw[k].y); v[k][3] = bf16_hi(raw[k].y);
                        v[k][4] = bf16_lo(raw[k].z); v[k][5] = bf16_hi(raw[k].z);
                        v[k][6] = bf16_lo(raw[k].w); v[k][7] = bf16_hi(raw[k].w);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        byte |= (uint32_t)(v[k][i] <= -rule.thr) << i;
                        unsure |= (v[k][i] < 0.0f) && (v[k][i] > -rule.thr);
                    }
                }
                if (unsure) {
                    byte = 0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) byte |= negative_bit(v[k][i], rule) << i;
                }
                uint32_t word = byte << (8 * (lane & 3));
                word |= __shfl_xor_sync(kFullMask, word, 1);
                word |= __shfl_xor_sync(kFullMask, word, 2);
                if (e0 < slab && (lane & 3) == 0) bs[e0 >> 5] = word;
            }
        }
    }
}

}  // namespace had
