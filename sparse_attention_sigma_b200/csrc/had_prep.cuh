// had_prep.cuh -- operand preparation for the tensor-core forward pass.
//
// The fused kernel feeds the 5th-generation tensor cores straight from
// shared memory, so the operands are written once, here, in the canonical
// no-swizzle K-major layout the MMA descriptors describe: 8-row x 16-byte
// "core matrices" of 128 contiguous bytes, core matrices adjacent along K
// 128 bytes apart, row groups (8 rows) (K bytes / 16) * 128 bytes apart.
// Tiles are stored contiguously so the kernel moves each with one bulk copy.
//
//   Qop1, Qop2 [BH][qtiles] tiles of 128 rows x d int8: the signs as +/-1
//                    and as +/-64 (0 padding; qtiles >= ceil(n/128), the
//                    extra tiles all padding)
//   Kop [BH][ceil(n/64)] tiles of 64 keys x d int8 (+4 / -4, 0 padding)
//   Qbits, Kbits [BH][n][d/32] the same signs bit-packed (1 = -1)
// With K as +/-4 the s32 accumulator holds 4 s against Qop1 (the counter
// shifts of the fused kernel's first pass are one integer add away) and
// 256 s against Qop2 (the byte offset of the logit's level in its per-row
// tables, again one integer add away).
//   Vop [BH][ceil(n/64)]  tiles of V^T: d rows x 64 keys fp16, scaled by
//                         2^-e_h so the head's largest |v| lies in
//                         [2^14, 2^15) (bf16 -> fp16 then loses no bits for
//                         any value within 2^39 of the head maximum)
//   vexp [BH] int          e_h, the power of two applied back to the output
// The signs are those of the standardize step (Eqs. 4-5, Eq. 12): -1 iff
// x / sigma_h < 0 in IEEE fp32.
#pragma once
#include <cuda_fp16.h>

#include "had_common.cuh"
#include "had_pack.cuh"

namespace had {
namespace prep {

constexpr int kQRows = 128;
constexpr int kKeys = 64;

// Byte offset of (row, kbyte) inside a tile whose rows are kbytes wide.
__device__ __forceinline__ uint32_t core_offset(uint32_t row, uint32_t kbyte, uint32_t kbytes)
{
    return ((row >> 3) * (kbytes >> 4) + (kbyte >> 4)) * 128u + (row & 7u) * 16u + (kbyte & 15u);
}

// One thread per 16 consecutive elements of a row -> 16 int8 signs.
// Works for Q (tile 128) and K (tile 64): `tile_rows` selects the tiling.
// The packed copy is written as 16-bit halves: chunk kc of a row is bits
// 16*(kc%2) .. 16*(kc%2)+15 of word kc/2.
// `op2` (may be null) receives a second copy with the codes pos2 / neg2.
template <typename T>
__global__ void __launch_bounds__(256)
sign_operand_kernel(const T *__restrict__ x, const float *__restrict__ sigma, int H, int n,
                    int d, int tile_rows, int tiles, long long chunks, uint32_t pos,
                    uint32_t neg, int8_t *__restrict__ op, uint32_t pos2, uint32_t neg2,
                    int8_t *__restrict__ op2, uint16_t *__restrict__ bits, int32_t *status)
{
    const int cpr = d >> 4;                                  // chunks per row
    const long long padded_rows = (long long)tiles * tile_rows;
    for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < chunks;
         c += (long long)gridDim.x * blockDim.x) {
        const long long prow = c / cpr;                      // padded row over all heads
        const int kc = (int)(c % cpr);
        const long long head = prow / padded_rows;
        const int r = (int)(prow % padded_rows);             // row within the head
        uint4 out = make_uint4(0, 0, 0, 0), out2 = make_uint4(0, 0, 0, 0);
        if (r < n) {
            const SignRule rule = sign_rule(__ldg(sigma + (head % H)));
            if (rule.bad) flag(status, HAD_ERR_BAD_SIGMA);
            const T *src = x + (head * n + r) * (long long)d + kc * 16;
            float v[16];
            float (&lo)[8] = *reinterpret_cast<float(*)[8]>(v);
            float (&hi)[8] = *reinterpret_cast<float(*)[8]>(v + 8);
            Load8<T>::run(src, lo);
            Load8<T>::run(src + 8, hi);
            uint32_t w[4], w2[4];
            uint32_t packed = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t word = 0, word2 = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const uint32_t nb = negative_bit(v[4 * q + b], rule);
                    word |= (nb ? neg : pos) << (8 * b);
                    word2 |= (nb ? neg2 : pos2) << (8 * b);
                    packed |= nb << (4 * q + b);
                }
                w[q] = word;
                w2[q] = word2;
            }
            out = make_uint4(w[0], w[1], w[2], w[3]);
            out2 = make_uint4(w2[0], w2[1], w2[2], w2[3]);
            bits[(head * n + r) * (long long)cpr + kc] = (uint16_t)packed;
        }
        const int t = r / tile_rows;
        const uint32_t rr = (uint32_t)(r % tile_rows);
        int8_t *tile = op + ((head * tiles + t) * (long long)tile_rows * d);
        *reinterpret_cast<uint4 *>(tile + core_offset(rr, kc * 16, d)) = out;
        if (op2) {
            int8_t *tile2 = op2 + ((head * tiles + t) * (long long)tile_rows * d);
            *reinterpret_cast<uint4 *>(tile2 + core_offset(rr, kc * 16, d)) = out2;
        }
    }
}

// Largest |v| of each head, as ordered float bits (non-negative floats
// compare like unsigned integers; NaN counts as infinity).  Each CTA reduces
// one contiguous chunk of one head and issues a single atomicMax.  vmax must
// be zeroed beforehand.
template <typename T>
__global__ void __launch_bounds__(256)
vmax_kernel(const T *__restrict__ v, long long groups_per_head, int chunks_per_head,
            unsigned int *__restrict__ vmax)
{
    __shared__ float wmax[8];
    const long long head = blockIdx.x / chunks_per_head;
    const int chunk = blockIdx.x % chunks_per_head;
    const long long per = (groups_per_head + chunks_per_head - 1) / chunks_per_head;
    const long long g_beg = head * groups_per_head + chunk * per;
    const long long g_end = head * groups_per_head + min(groups_per_head, (chunk + 1) * per);
    float m = 0.0f;
    for (long long g = g_beg + threadIdx.x; g < g_end; g += blockDim.x) {
        float e[8];
        Load8<T>::run(v + g * 8, e);
#pragma unroll
        for (int k = 0; k < 8; ++k) m = isnan(e[k]) ? __int_as_float(0x7f800000) : fmaxf(m, fabsf(e[k]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wmax[w]);
        atomicMax(vmax + head, __float_as_uint(m));
    }
}

// Power-of-two scale exponent of a head from its largest |v|.
__device__ __forceinline__ int vscale_exp(unsigned int bits)
{
    const float m = __uint_as_float(bits);
    if (!(m > 0.0f) || !isfinite(m)) return 0;
    int e;
    frexpf(m, &e);            // m = f * 2^e, f in [0.5, 1)  ->  m < 2^e
    return e - 15;            // m * 2^-(e-15) in [2^14, 2^15)
}

// One CTA per (head, 64-key tile): transpose the tile through shared memory
// and write V^T as fp16 core matrices.  Writes e_h for every head (by the
// CTA of tile 0).
template <typename T, int D>
__global__ void __launch_bounds__(256)
v_operand_kernel(const T *__restrict__ v, int n, const unsigned int *__restrict__ vmax,
                 __half *__restrict__ op, int *__restrict__ vexp)
{
    __shared__ float tile[kKeys][D + 1];
    const int tiles = (n + kKeys - 1) / kKeys;
    const long long head = blockIdx.x / tiles;
    const int t = blockIdx.x % tiles;
    const int e = vscale_exp(vmax[head]);
    const float scale = ldexpf(1.0f, -e);
    if (t == 0 && threadIdx.x == 0) vexp[head] = e;
    // load 64 keys x D values (coalesced, 8 elements per thread-iteration)
    constexpr int G = kKeys * D / 8;
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int key = g / (D / 8);
        const int c0 = (g % (D / 8)) * 8;
        const int j = t * kKeys + key;
        float e8[8];
        if (j < n) {
            Load8<T>::run(v + ((head * n + j) * (long long)D + c0), e8);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) e8[k] = 0.0f;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) tile[key][c0 + k] = e8[k] * scale;
    }
    __syncthreads();
    // write D rows x 64 keys: one thread per 16-byte chunk (8 keys of a dim)
    __half *dst = op + (head * tiles + t) * (long long)D * kKeys;
    constexpr int CH = D * (kKeys / 8);
    for (int c = threadIdx.x; c < CH; c += blockDim.x) {
        const int dim = c / (kKeys / 8);
        const int k0 = (c % (kKeys / 8)) * 8;
        __align__(16) __half h[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) h[k] = __float2half_rn(tile[k0 + k][dim]);
        const uint32_t off = core_offset(dim, k0 * 2, kKeys * 2);
        *reinterpret_cast<uint4 *>(reinterpret_cast<char *>(dst) + off) =
            *reinterpret_cast<const uint4 *>(h);
    }
}

}  // namespace prep
}  // namespace had
