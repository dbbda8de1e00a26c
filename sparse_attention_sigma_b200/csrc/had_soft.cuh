// had_soft.cuh -- forward pass on soft codes, for the tanh training stages
// ("Hamming Attention Distillation", pith.science review: the annealing
// schedule first trains with a scaled tanh, Eq. 13, whose scale c pushes
// it toward the sign; top-N mask, softmax and value product as in Eqs. 6-7).
//
// The codes t = tanh(c x / sigma) are fp32 and the logits s = tq . tk are
// continuous, so the d+1-level histogram of the binarized path does not
// apply.  Three kernels:
//   soft_codes_kernel   x -> t, elementwise (HBM-bound);
//   soft_logits_kernel  S = Tq Tk^T of a group of heads into a scratch
//                       matrix, fp32 FMA on the CUDA cores with a fixed
//                       summation order (k = 0 .. d-1), 128x128 tiles;
//   soft_select_kernel  one CTA per query row: a value histogram finds the
//                       slice of [-d, d] that holds the N-th largest logit,
//                       an exact radix select among that slice's keys finds
//                       the logit itself, then the kept keys are written in
//                       index order, ties at the threshold to the lower index.
// Softmax and the value product reuse sparse_softmax_av_kernel with fp32
// logits.
#pragma once
#include "had_common.cuh"
#include "had_pack.cuh"

namespace had {

// ----------------------------------------------------------------- codes

// groups = B*H*n*d/8; a thread turns 8 consecutive elements into 8 codes.
template <typename T>
__global__ void __launch_bounds__(256)
soft_codes_kernel(const T *__restrict__ x, const float *__restrict__ sigma, float c, int H,
                  int n, int d, long long groups, float *__restrict__ t, int32_t *status)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    const int groups_per_row = d >> 3;
    for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < groups; g += stride) {
        const long long row = g / groups_per_row;
        const float sg = __ldg(sigma + (int)((row / n) % H));
        if (!(sg > 0.0f) || !isfinite(sg)) flag(status, HAD_ERR_BAD_SIGMA);
        float v[8];
        Load8<T>::run(x + g * 8, v);
        float o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = tanhf(__fmul_rn(c, __fdiv_rn(v[k], sg)));
        float4 *dst = reinterpret_cast<float4 *>(t + g * 8);
        dst[0] = make_float4(o[0], o[1], o[2], o[3]);
        dst[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
}

// ---------------------------------------------------------------- logits

constexpr int kSoftTile = 128;
constexpr int kSoftPad = 4;     // row pitch 132 floats in shared memory

template <int D>
constexpr int soft_logits_smem_bytes()
{
    return 2 * D * (kSoftTile + kSoftPad) * 4;
}

// Grid (key tiles, query tiles, heads of this group).  S of head z of the
// group is [n, ld] with ld = n rounded up to a multiple of 4; columns n..ld-1
// hold logits of zero codes and are never read.  A thread owns an 8x8 block:
// rows 4ty..4ty+3 and 64+4ty..64+4ty+3, columns 4tx.. and 64+4tx.. of the
// tile, so its shared-memory reads are float4 (broadcast for the query side).
template <int D>
__global__ void __launch_bounds__(256)
soft_logits_kernel(const float *__restrict__ tq, const float *__restrict__ tk, int n,
                   long long ld, float *__restrict__ S)
{
    constexpr int P = kSoftTile + kSoftPad;
    extern __shared__ float sm[];
    float *As = sm;              // [D][P]: query codes, k-major
    float *Bs = sm + D * P;      // [D][P]: key codes, k-major
    const int tid = threadIdx.x;
    const long long head = blockIdx.z;
    const int i0 = blockIdx.y * kSoftTile;
    const int j0 = blockIdx.x * kSoftTile;
    const float *qh = tq + head * n * (long long)D;
    const float *kh = tk + head * n * (long long)D;

    // 16-byte loads along k, consecutive lanes on consecutive chunks of a row
    constexpr int CH = D / 4;                    // float4 chunks per row
    for (int e = tid; e < kSoftTile * CH; e += 256) {
        const int r = e / CH, kc = e % CH;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (i0 + r < n) a = __ldg(reinterpret_cast<const float4 *>(qh + (long long)(i0 + r) * D) + kc);
        if (j0 + r < n) b = __ldg(reinterpret_cast<const float4 *>(kh + (long long)(j0 + r) * D) + kc);
        As[(4 * kc + 0) * P + r] = a.x; As[(4 * kc + 1) * P + r] = a.y;
        As[(4 * kc + 2) * P + r] = a.z; As[(4 * kc + 3) * P + r] = a.w;
        Bs[(4 * kc + 0) * P + r] = b.x; Bs[(4 * kc + 1) * P + r] = b.y;
        Bs[(4 * kc + 2) * P + r] = b.z; Bs[(4 * kc + 3) * P + r] = b.w;
    }
    __syncthreads();

    const int ty = tid >> 4, tx = tid & 15;
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
        const float4 a0 = *reinterpret_cast<const float4 *>(As + k * P + 4 * ty);
        const float4 a1 = *reinterpret_cast<const float4 *>(As + k * P + 64 + 4 * ty);
        const float4 b0 = *reinterpret_cast<const float4 *>(Bs + k * P + 4 * tx);
        const float4 b1 = *reinterpret_cast<const float4 *>(Bs + k * P + 64 + 4 * tx);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
    }

    float *Sh = S + head * n * ld;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int i = i0 + (a < 4 ? 4 * ty + a : 64 + 4 * ty + (a - 4));
        if (i >= n) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = j0 + h * 64 + 4 * tx;           // a multiple of 4
            if (j < ld)
                *reinterpret_cast<float4 *>(Sh + (long long)i * ld + j) =
                    make_float4(acc[a][4 * h], acc[a][4 * h + 1], acc[a][4 * h + 2],
                                acc[a][4 * h + 3]);
        }
    }
}

// ---------------------------------------------------------------- select

constexpr int kSelThreads = 256;

// Unsigned key with the order of the float: larger float, larger key.
__device__ __forceinline__ uint32_t order_key(float f)
{
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

constexpr int kSelBins = 2048;

// Value bin of a logit: its place among kSelBins equal slices of [-d, d].
// (s + d) is rounded once and the scale is a power of two, so the bin never
// decreases as s grows; the clamp catches rounding at the ends.
template <int D>
__device__ __forceinline__ uint32_t value_bin(float s)
{
    constexpr float kScale = kSelBins / (2.0f * D);
    const int b = (int)floorf(__fmul_rn(__fadd_rn(s, (float)D), kScale));
    return (uint32_t)min(max(b, 0), kSelBins - 1);
}

// Bytes of dynamic shared memory: the row's keys and a list of candidates.
__host__ __device__ constexpr size_t soft_select_smem_bytes(int n)
{
    return ((size_t)n * 6 + 15) / 16 * 16;
}

// One CTA per row of S (row r of this group is flat output row out_row0 + r).
//   1. load the row as order-preserving keys, counting each logit into one
//      of 2048 value bins (one pass; the bins spread the atomic updates);
//   2. the bin that holds the N-th largest logit, by a scan from the top;
//   3. list the keys of that bin (few, except for strongly tied rows);
//   4. the exact N-th largest key among them: four 8-bit radix digits;
//   5. keep the keys above it and the first of its ties in index order,
//      each warp over a contiguous segment of the row.
template <int D>
__global__ void __launch_bounds__(kSelThreads)
soft_select_kernel(const float *__restrict__ S, long long ld, int n, int N, long long out_row0,
                   int32_t *__restrict__ idx, float *__restrict__ logits)
{
    extern __shared__ uint32_t dyn[];
    uint32_t *keys = dyn;                                     // [n]
    uint16_t *cand = reinterpret_cast<uint16_t *>(dyn + n);   // [n] (n <= 32768)
    __shared__ uint32_t hist[kSelBins];
    __shared__ uint32_t part[kSelThreads];
    __shared__ uint32_t s_sel, s_rank, s_ccount;
    __shared__ uint32_t wcnt[2][kSelThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = (1u << lane) - 1u;
    const long long r = blockIdx.x;
    const float *srow = S + r * ld;

    for (int b = tid; b < kSelBins; b += kSelThreads) hist[b] = 0;
    if (tid == 0) s_ccount = 0;
    __syncthreads();
#pragma unroll 4
    for (int j = tid; j < n; j += kSelThreads) {
        const float f = __fadd_rn(__ldg(srow + j), 0.0f);    // -0 becomes +0: equal values tie
        keys[j] = order_key(f);
        atomicAdd(&hist[value_bin<D>(f)], 1u);
    }
    __syncthreads();

    // 2. thread t sums the 8 bins kSelBins-1-8t downward; warp 0 scans the sums
    {
        uint32_t sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) sum += hist[kSelBins - 1 - 8 * tid - e];
        part[tid] = sum;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { c[e] = part[8 * lane + e]; tot += c[e]; }
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFullMask, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - tot, want = (uint32_t)N;
        if (excl < want && want <= incl) {
            uint32_t above = excl;
            for (int e = 0; e < 8; ++e) {
                if (above + c[e] >= want) {
                    const int p = 8 * lane + e;
                    for (int f = 0; f < 8; ++f) {
                        const int b = kSelBins - 1 - 8 * p - f;
                        const uint32_t h = hist[b];
                        if (above + h >= want) { s_sel = (uint32_t)b; s_rank = want - above; break; }
                        above += h;
                    }
                    break;
                }
                above += c[e];
            }
        }
    }
    __syncthreads();
    const uint32_t bstar = s_sel;
    uint32_t rank = s_rank;          // rank of the N-th largest inside bin bstar

    // 3. the keys of bin bstar, in any order; the two 256-bin buffers of the
    //    radix passes (part and the start of hist) are cleared meanwhile
    part[tid] = 0;
    hist[tid] = 0;
#pragma unroll 4
    for (int j0 = 0; j0 < n; j0 += kSelThreads) {
        const int j = j0 + tid;
        const bool is = j < n && value_bin<D>(key_value(keys[j])) == bstar;
        const unsigned bal = __ballot_sync(kFullMask, is);
        uint32_t base = 0;
        if (lane == 0 && bal) base = atomicAdd(&s_ccount, (uint32_t)__popc(bal));
        base = __shfl_sync(kFullMask, base, 0);
        if (is) cand[base + __popc(bal & lt)] = (uint16_t)j;
    }
    __syncthreads();
    const uint32_t cc = s_ccount;

    // 4. radix select among the candidates, most significant digit first;
    //    pass p counts into buffer p & 1 while warp 0 clears the other one
    uint32_t prefix = 0, mask = 0;
    for (int pos = 24, pass = 0; pos >= 0; pos -= 8, ++pass) {
        uint32_t *cnt = (pass & 1) ? hist : part;
        uint32_t *next = (pass & 1) ? part : hist;
        for (uint32_t i = tid; i < cc; i += kSelThreads) {
            const uint32_t k = keys[cand[i]];
            if ((k & mask) == prefix) atomicAdd(&cnt[(k >> pos) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l holds digits 255-8l down to 248-8l, largest first
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) { c[e] = cnt[255 - 8 * lane - e]; tot += c[e]; }
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(kFullMask, incl, o);
                if (lane >= o) incl += y;
            }
            const uint32_t excl = incl - tot;
            if (excl < rank && rank <= incl) {
                uint32_t above = excl;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (above + c[e] >= rank) {
                        s_sel = 255u - 8u * lane - e;
                        s_rank = rank - above;
                        break;
                    }
                    above += c[e];
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) next[8 * lane + e] = 0;
        }
        __syncthreads();
        prefix |= s_sel << pos;
        mask |= 0xffu << pos;
        rank = s_rank;
    }

    // 5. keys above prefix are kept; of those equal to it, the first rank
    //    ones in index order.  Warp w walks the contiguous segment
    //    [w seg, (w+1) seg): once to count, once (after one exchange of the
    //    counts) to write at its offsets.
    const uint32_t T = prefix, q = rank;
    const int seg = (n + kSelThreads - 1) / kSelThreads * 32;
    const int jb = warp * seg, je = min(n, jb + seg);
    uint32_t gt_n = 0, tie_n = 0;
    for (int j0 = jb; j0 < je; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t k = j < je ? keys[j] : 0u;
        gt_n += __popc(__ballot_sync(kFullMask, j < je && k > T));
        tie_n += __popc(__ballot_sync(kFullMask, j < je && k == T));
    }
    if (lane == 0) { wcnt[0][warp] = gt_n; wcnt[1][warp] = tie_n; }
    __syncthreads();
    uint32_t gt_before = 0, tie_before = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        gt_before += w < warp ? wcnt[0][w] : 0u;
        tie_before += w < warp ? wcnt[1][w] : 0u;
    }
    uint32_t ko = gt_before + min(tie_before, q);   // kept before this segment
    uint32_t tr = tie_before;                       // ties before this chunk
    int32_t *irow = idx + (out_row0 + r) * N;
    float *lrow = logits ? logits + (out_row0 + r) * N : nullptr;
    for (int j0 = jb; j0 < je && ko < (uint32_t)N; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t k = j < je ? keys[j] : 0u;
        const bool gt = j < je && k > T;
        const bool tie = j < je && k == T;
        const unsigned bt = __ballot_sync(kFullMask, tie);
        const bool keep = gt || (tie && tr + __popc(bt & lt) < q);
        const unsigned bk = __ballot_sync(kFullMask, keep);
        const uint32_t pos = ko + __popc(bk & lt);
        if (keep && pos < (uint32_t)N) {     // exactly N keys are kept; the bound is a guard
            irow[pos] = j;
            if (lrow) lrow[pos] = key_value(k);
        }
        tr += __popc(bt);
        ko += __popc(bk);
    }
}

}  // namespace had
