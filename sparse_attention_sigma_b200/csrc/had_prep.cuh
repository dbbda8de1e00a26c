// had_prep.cuh -- operand preparation for the tensor-core forward pass.
//
// The fused kernel feeds the 5th-generation tensor cores straight from
// shared memory, so the operands are written once, here, in the canonical
// no-swizzle K-major layout the MMA descriptors describe: 8-row x 16-byte
// "core matrices" of 128 contiguous bytes, core matrices adjacent along K
// 128 bytes apart, row groups (8 rows) (K bytes / 16) * 128 bytes apart.
// Tiles are stored contiguously so the kernel moves each with one bulk copy.
//
//   Qop1, Qop2 [BH][qtiles] tiles of 128 rows x d int8: the signs negated,
//                    as -/+1, and as +/-64 (0 padding; qtiles >= ceil(n/128),
//                    the extra tiles all padding)
//   Kop [BH][kstride] tiles of 64 keys x d int8 (+4 / -4, 0 padding); kstride
//                    = ceil(n/64) rounded up to even, so that pairs of tiles
//                    (128 keys) always move as one whole copy
//   Qbits, Kbits [BH][n][d/32] the same signs bit-packed (1 = -1)
//   Kpart [BH][kstride][d] int8  per 64-key tile: sum over its keys of the
//                    +/-1 code of each dimension; Ksum [BH][d] int32 their
//                    sum over the head (the exact mean logit of a query row is
//                    q . Ksum / n)
// With K as +/-4 the s32 accumulator holds -4 s against Qop1 (so that a
// per-row bias added by the tensor core turns it into the counter shift of
// the fused kernel's first pass) and 256 s against Qop2 (the byte offset of
// the logit's level in its per-row tables, one integer add away).
//   Vop [BH][kstride]     tiles of V^T: d rows x 64 keys fp16, scaled by
//                         2^-e_h so the head's largest |v| lies in
//                         [2^14, 2^15) (bf16 -> fp16 then loses no bits for
//                         any value within 2^39 of the head maximum)
//   vexp [BH] int          e_h, the power of two applied back to the output
// The signs are those of the standardize step (Eqs. 4-5, Eq. 12): -1 iff
// x / sigma_h < 0 in IEEE fp32.
#pragma once
#include <cuda_fp16.h>
#include <type_traits>

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

// Signs of 16 consecutive elements as int8 codes (pos / neg) in four words,
// and as 16 packed bits (1 = negative).  With a normal sigma an element at
// or below -sigma * 2^-100 is surely negative after the division and one at
// or above zero surely not; only elements strictly between (never seen in
// practice, but possible) take the exact division, all 16 then together.
template <typename T>
__device__ __forceinline__ uint32_t sign16(const T *src, const SignRule &rule, uint32_t pos,
                                           uint32_t neg, uint32_t (&w)[4])
{
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        // on the raw bits: four values per bf16_signs4; a negative value's
        // byte flag, sign-replicated over its byte, selects the neg code
        if (rule.fast) {
            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(src));
            const uint4 b = __ldg(reinterpret_cast<const uint4 *>(src + 8));
            const uint32_t kge = bf16_kge(rule);
            uint32_t n[4], u[4];
            bf16_signs4(a.x, a.y, kge, n[0], u[0]);
            bf16_signs4(a.z, a.w, kge, n[1], u[1]);
            bf16_signs4(b.x, b.y, kge, n[2], u[2]);
            bf16_signs4(b.z, b.w, kge, n[3], u[3]);
            if (((u[0] | u[1]) | (u[2] | u[3])) == 0u) {
                const uint32_t pos4 = pos * 0x01010101u, flip4 = ((pos ^ neg) & 0xFFu) * 0x01010101u;
                uint32_t packed = 0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t m;
                    asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(m) : "r"(n[q]));   // 0xFF per negative byte
                    w[q] = pos4 ^ (m & flip4);
                    packed |= flags4(n[q]) << (4 * q);
                }
                return packed;
            }
        }
    }
    float v[16];
    Load8<T>::run(src, *reinterpret_cast<float(*)[8]>(v));
    Load8<T>::run(src + 8, *reinterpret_cast<float(*)[8]>(v + 8));
    uint32_t packed = 0;
    bool unsure = !rule.fast;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        packed |= (uint32_t)(v[i] <= -rule.thr) << i;
        unsure |= (v[i] < 0.0f) && (v[i] > -rule.thr);
    }
    if (unsure) {
        packed = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) packed |= negative_bit(v[i], rule) << i;
    }
    // byte b of word q is pos, or neg where bit 4q+b is set
    const uint32_t flip = (pos ^ neg) & 0xFFu;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t x = (packed >> (4 * q)) & 0xFu;
        const uint32_t spread = (x & 1u) | ((x & 2u) << 7) | ((x & 4u) << 14) | ((x & 8u) << 21);
        w[q] = (pos * 0x01010101u) ^ (spread * flip);
    }
    return packed;
}

// Rewrite of four code words from one code pair to another (a byte-wise map
// pos -> pos2, everything else -> neg2).
__device__ __forceinline__ uint4 recode(const uint32_t (&w)[4], uint32_t pos, uint32_t pos2,
                                        uint32_t neg2)
{
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
            word |= (((w[q] >> (8 * b)) & 0xFFu) == pos ? pos2 : neg2) << (8 * b);
        o[q] = word;
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// All operand preparation that needs only the inputs, in one launch.  Block
// b of the grid takes, in this order:
//   b <  BH*qtiles            one 128-row Q tile -> Qop1 (-/+1), Qop2 (+/-64, when
//                             qop2 is given: only the causal kernel reads it), Qbits
//   b <  BH*(qtiles+ktiles)   one 64-key K tile  -> Kop (+/-4), Kbits
//   otherwise                 one chunk of V     -> the chunk's largest |v|
// Rows past n are written as zero padding.  A thread handles 16 consecutive
// elements of a row; the packed bits are written as 16-bit halves (chunk kc
// of a row is bits 16*(kc%2) .. of word kc/2).  Block 0 also zeroes the miss
// counter of the fused kernel and the done counter of the fix-up kernel
// (which zeroes both again when it finishes, so the fused stage can run
// again on the same operands).
template <typename T, int D>
__global__ void __launch_bounds__(256)
operands_kernel(const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
                const float *__restrict__ sq, const float *__restrict__ sk, int H, int n,
                int bh, int qtiles, int ktiles, int vchunks, int8_t *__restrict__ qop,
                int8_t *__restrict__ qop2, int8_t *__restrict__ kop,
                uint16_t *__restrict__ qbits, uint16_t *__restrict__ kbits,
                int8_t *__restrict__ kpart, float *__restrict__ vpart,
                int *__restrict__ miss_count, int32_t *status)
{
    constexpr int CPR = D / 16;                                // 16-element chunks per row
    __shared__ uint16_t sbits[kKeys][CPR];                     // K tile signs, for column sums
    const int b = blockIdx.x;
    if (b == 0 && threadIdx.x < 2) miss_count[threadIdx.x] = 0;   // miss and fix-up done counters
    const int nq = bh * qtiles, nk = bh * ktiles;
    if (b < nq + nk) {
        const bool isq = b < nq;
        const int tiles = isq ? qtiles : ktiles;
        const int bb = isq ? b : b - nq;
        const int head = bb / tiles;
        const int t = bb - head * tiles;
        const int rows = isq ? kQRows : kKeys;
        const T *x = isq ? Q : K;
        const SignRule rule = sign_rule(__ldg((isq ? sq : sk) + head % H));
        if (rule.bad && threadIdx.x == 0) flag(status, HAD_ERR_BAD_SIGMA);
        int8_t *tile = (isq ? qop : kop) + (size_t)bb * rows * D;
        int8_t *tile2 = qop2 ? qop2 + (size_t)bb * rows * D : nullptr;
        uint16_t *bits = isq ? qbits : kbits;
        // Q as -1 / +1 for sign + / - (the pass-1 accumulator then holds -4 s),
        // K as +4 / -4
        const uint32_t pos = isq ? 0xFFu : 0x04u, neg = isq ? 0x01u : 0xFCu;
        for (int c = threadIdx.x; c < rows * CPR; c += blockDim.x) {
            const int r = c / CPR, kc = c % CPR;
            const int row = t * rows + r;
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            uint32_t packed = 0u;
            if (row < n) {
                const size_t e = ((size_t)head * n + row) * D + kc * 16;
                packed = sign16<T>(x + e, rule, pos, neg, w);
                bits[e / 16] = (uint16_t)packed;
            }
            if (!isq) sbits[r][kc] = (uint16_t)packed;
            const uint32_t off = core_offset(r, kc * 16, D);
            *reinterpret_cast<uint4 *>(tile + off) = make_uint4(w[0], w[1], w[2], w[3]);
            if (isq && qop2)
                *reinterpret_cast<uint4 *>(tile2 + off) =
                    row < n ? recode(w, 0xFFu, 0x40u, 0xC0u) : make_uint4(0u, 0u, 0u, 0u);
        }
        if (!isq) {
            // column sums of the tile's codes: valid keys minus twice the
            // negatives, each of the blockDim / D thread groups counting a
            // strided share of the rows
            static_assert(256 % D == 0, "thread groups of D columns");
            __shared__ int negp[256];
            __syncthreads();
            const int valid = max(0, min(kKeys, n - t * kKeys));
            const int a = threadIdx.x % D, grp = threadIdx.x / D, ngrp = blockDim.x / D;
            int neg_count = 0;
            for (int rr = grp; rr < valid; rr += ngrp) neg_count += (sbits[rr][a >> 4] >> (a & 15)) & 1;
            negp[threadIdx.x] = neg_count;
            __syncthreads();
            if (grp == 0) {
                for (int g2 = 1; g2 < ngrp; ++g2) neg_count += negp[g2 * D + a];
                kpart[(size_t)bb * D + a] = (int8_t)(valid - 2 * neg_count);
            }
        }
        return;
    }
    // largest |v| of one chunk of one head, as a float (NaN counts as inf)
    __shared__ float wmax[8];
    const int bb = b - nq - nk;
    const int head = bb / vchunks;
    const int chunk = bb - head * vchunks;
    const long long groups = (long long)n * D / 8;             // 8-element groups per head
    const long long per = (groups + vchunks - 1) / vchunks;
    const long long g0 = chunk * per, g1 = min(groups, g0 + per);
    const T *vh = V + (size_t)head * n * D;
    float m = 0.0f;
    for (long long g = g0 + threadIdx.x; g < g1; g += blockDim.x) {
        float e[8];
        Load8<T>::run(vh + g * 8, e);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            m = isnan(e[k]) ? __int_as_float(0x7f800000) : fmaxf(m, fabsf(e[k]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wmax[w]);
        vpart[bb] = m;
    }
}

// Power-of-two scale exponent of a head from its largest |v|.
__device__ __forceinline__ int vscale_exp(float m)
{
    if (!(m > 0.0f) || !isfinite(m)) return 0;
    int e;
    frexpf(m, &e);            // m = f * 2^e, f in [0.5, 1)  ->  m < 2^e
    return e - 15;            // m * 2^-(e-15) in [2^14, 2^15)
}

// The head's largest |v| from the chunk maxima of operands_kernel, then V^T
// as fp16 core matrices scaled by 2^-e_h (tiles past n are zeros).  A CTA
// takes 256 / D consecutive 64-key tiles of one head (ctiles per head);
// each thread one block of 8 keys x 8 dims: eight 16-byte rows of V in,
// transposed in registers, eight 16-byte core-matrix rows (8 keys of one
// dim) out.  The head's first CTA also writes e_h and reduces its key
// column sums to Ksum.
template <typename T, int D>
__global__ void __launch_bounds__(256)
v_operand_kernel(const T *__restrict__ v, int n, int tiles, int ctiles, const float *__restrict__ vpart,
                 int vchunks, __half *__restrict__ op, int *__restrict__ vexp,
                 const int8_t *__restrict__ kpart, int *__restrict__ ksum)
{
    static_assert(256 % D == 0, "thread groups of D columns / blocks");
    constexpr int TPC = 256 / D;                   // tiles per CTA (D threads per tile)
    __shared__ float head_max;
    const long long head = blockIdx.x / ctiles;
    const int ct = blockIdx.x % ctiles;
    if (threadIdx.x < 32) {
        float m = 0.0f;
        for (int c = threadIdx.x; c < vchunks; c += 32) m = fmaxf(m, vpart[head * vchunks + c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
        if (threadIdx.x == 0) head_max = m;
    }
    __syncthreads();
    const int e = vscale_exp(head_max);
    const float scale = ldexpf(1.0f, -e);
    if (ct == 0 && threadIdx.x == 0) vexp[head] = e;
    if (ct == 0) {
        // column sums over the head's key tiles: each of the blockDim / D
        // thread groups sums a strided share of the tiles (independent loads
        // in flight), then the groups' partial sums meet in shared memory
        __shared__ int kpsum[256];
        const int a = threadIdx.x % D, grp = threadIdx.x / D, ngrp = blockDim.x / D;
        int sum = 0;
#pragma unroll 4
        for (int k = grp; k < tiles; k += ngrp) sum += kpart[((size_t)head * tiles + k) * D + a];
        kpsum[threadIdx.x] = sum;
        __syncthreads();
        if (grp == 0) {
            for (int g2 = 1; g2 < ngrp; ++g2) sum += kpsum[g2 * D + a];
            ksum[head * D + a] = sum;
        }
    }
    const int t = ct * TPC + (int)threadIdx.x / D;  // this thread's tile
    if (t >= tiles) return;
    const int local = threadIdx.x % D;
    const int db = local % (D / 8), kb = local / (D / 8);   // dims 8 db.., keys 8 kb..
    // rows: keys 8 kb + r of the tile, dims 8 db .. 8 db + 7 (a warp's lanes
    // read D / 8 consecutive 16-byte pieces of each of 32 / (D / 8) rows)
    float x[8][8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int j = t * kKeys + kb * 8 + r;
        if (j < n) {
            Load8<T>::run(v + ((head * n + j) * (long long)D + db * 8), x[r]);
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) x[r][c] = 0.0f;
        }
    }
    char *dst = reinterpret_cast<char *>(op + (head * tiles + t) * (long long)D * kKeys);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t h2[4];
#pragma unroll
        for (int r = 0; r < 8; r += 2) {
            __half2 h = __halves2half2(__float2half_rn(x[r][c] * scale),
                                       __float2half_rn(x[r + 1][c] * scale));
            h2[r / 2] = *reinterpret_cast<uint32_t *>(&h);
        }
        const uint32_t off = core_offset(db * 8 + c, kb * 16, kKeys * 2);
        *reinterpret_cast<uint4 *>(dst + off) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
    }
}

}  // namespace prep
}  // namespace had
