// had_mass.cuh -- top-N mass retention diagnostic: for each query row and
// threshold p, the smallest N whose N largest softmax weights (full softmax
// over all keys, temperature tau, binarized logits) hold at least a
// fraction p of the row's total.  It measures the premise the method rests
// on, that a small N keeps most of the attention mass ("Hamming Attention
// Distillation", pith.science review: the concrete test and the notes on
// the free parameter N).
//
// Only d + 1 logit levels exist, so a row's softmax is fixed by its
// histogram of Hamming distances: level l (logit s_l = d - 2 l) holds c_l
// keys of weight w_l = exp(tau (s_l - s_max)).  One thread owns one row; a
// CTA of 128 rows of one head streams the head's packed keys through shared
// memory (broadcast reads) and counts levels into hist[level][row].  Then,
// in fp64 and in order of decreasing logit: Z = sum c_l w_l, and for each p
// the crossing level l* where the running mass reaches p Z and the least
// number of its keys that gets there.
#pragma once
#include "had_common.cuh"
#include "had_topn.cuh"

namespace had {

constexpr int kMassMaxP = 8;

struct MassP {
    double p[kMassMaxP];
    int np;
};

template <int DW>
constexpr int mass_smem_bytes()
{
    return topn_smem_bytes<DW>();
}

template <int DW>
__global__ void __launch_bounds__(kTopnRows)
topn_mass_kernel(const uint32_t *__restrict__ qbits, const uint32_t *__restrict__ kbits, int n,
                 double tau, const MassP ps, int32_t *__restrict__ nmin)
{
    constexpr int D = DW * 32;
    constexpr int BINS = D + 1;
    extern __shared__ uint32_t smem[];
    uint32_t *hist = smem;                          // [BINS][kTopnRows]
    uint32_t *kch = smem + BINS * kTopnRows;        // [kTopnKeyChunk][DW]

    const int tid = threadIdx.x;
    const int tiles = (n + kTopnRows - 1) / kTopnRows;
    const long long head = blockIdx.x / tiles;
    const int row = (int)(blockIdx.x % tiles) * kTopnRows + tid;
    const bool active = row < n;

    uint32_t q[DW];
#pragma unroll
    for (int w = 0; w < DW; ++w) q[w] = active ? __ldg(qbits + (head * n + row) * DW + w) : 0u;
    for (int b = 0; b < BINS; ++b) hist[b * kTopnRows + tid] = 0;

    const uint32_t *kh = kbits + head * n * DW;
    for (int j0 = 0; j0 < n; j0 += kTopnKeyChunk) {
        const int cnt = min(kTopnKeyChunk, n - j0);
        __syncthreads();
        for (int t = tid; t < cnt * DW; t += kTopnRows) kch[t] = __ldg(kh + (long long)j0 * DW + t);
        __syncthreads();
        if (active) {
            for (int jj = 0; jj < cnt; ++jj) {
                int h = 0;
#pragma unroll
                for (int w = 0; w < DW; ++w) h += __popc(q[w] ^ kch[jj * DW + w]);
                hist[h * kTopnRows + tid] += 1;
            }
        }
    }
    if (!active) return;

    int hmin = 0;
    while (hmin < BINS - 1 && hist[hmin * kTopnRows + tid] == 0) ++hmin;
    // weight of level b relative to the best occupied level hmin
    auto weight = [&](int b) { return exp(tau * (double)(2 * (hmin - b))); };
    double Z = 0.0;
    for (int b = hmin; b < BINS; ++b) {
        const uint32_t c = hist[b * kTopnRows + tid];
        if (c) Z += (double)c * weight(b);
    }
    int32_t *dst = nmin + (head * n + row) * (long long)ps.np;
    for (int k = 0; k < ps.np; ++k) {
        const double target = ps.p[k] * Z;
        double cum = 0.0;
        long long kept = 0;
        int N = n;
        for (int b = hmin; b < BINS; ++b) {
            const uint32_t c = hist[b * kTopnRows + tid];
            if (!c) continue;
            const double w = weight(b);
            const double m = (double)c * w;
            if (cum + m >= target) {
                // least count of this level's keys that reaches the target
                long long kk = (long long)ceil((target - cum) / w);
                kk = kk < 1 ? 1 : (kk > (long long)c ? (long long)c : kk);
                while (kk > 1 && cum + (double)(kk - 1) * w >= target) --kk;
                while (kk < (long long)c && cum + (double)kk * w < target) ++kk;
                N = (int)(kept + kk);
                break;
            }
            cum += m;
            kept += c;
        }
        dst[k] = N;
    }
}

}  // namespace had
