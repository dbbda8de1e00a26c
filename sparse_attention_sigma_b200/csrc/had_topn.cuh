// had_topn.cuh -- Hamming logits + exact top-N selection, unfused (Eq. 5 and
// Eq. 6 of "Hamming Attention Distillation", pith.science review, "What
// carries the argument": QK^T by XNOR/popcount, then a mask keeping the
// largest logits of each row).
//
// One thread owns one query row.  A CTA of 128 rows of one head streams the
// head's packed keys through shared memory in chunks; every lane reads the
// same key word (a broadcast), so key traffic is one L2 read per CTA.
//   pass 1: Hamming distance h = popc(q ^ k) of every key, counted in a
//           per-row histogram of d+1 bins held in shared memory as
//           hist[bin][row] (each thread owns a column: conflict-free).
//   select: walk the bins from h = 0 up; the threshold t is the first bin
//           where the running count reaches N, and q = N - count(h < t) keys
//           of bin t are kept.
//   pass 2: recompute h; keep h < t, and h == t while fewer than q ties
//           were kept (ascending key index, so the lower index wins).
// Output per row: the N kept key indices in ascending order, and their
// logits s = d - 2h.
//
// Causal form (kCausal): query i of a head sees keys 0 .. i only and keeps
// N_i = min(N, i + 1) of them; slots N_i .. N-1 hold idx -1 and logit 0.  A
// CTA streams keys only up to its last row.
#pragma once
#include "had_common.cuh"

namespace had {

constexpr int kTopnRows = 128;
constexpr int kTopnKeyChunk = 512;

template <int DW>
constexpr int topn_smem_bytes()
{
    return ((DW * 32 + 1) * kTopnRows + kTopnKeyChunk * DW) * 4;
}

template <int DW, bool kCausal = false>
__global__ void __launch_bounds__(kTopnRows)
topn_simt_kernel(const uint32_t *__restrict__ qbits, const uint32_t *__restrict__ kbits,
                 int n, int N, int32_t *__restrict__ idx, int16_t *__restrict__ logits)
{
    constexpr int D = DW * 32;
    constexpr int BINS = D + 1;
    extern __shared__ uint32_t smem[];
    uint32_t *hist = smem;                          // [BINS][kTopnRows]
    uint32_t *kch = smem + BINS * kTopnRows;        // [kTopnKeyChunk][DW]

    const int tid = threadIdx.x;
    const int tiles = (n + kTopnRows - 1) / kTopnRows;
    const long long head = blockIdx.x / tiles;
    const int row0 = (int)(blockIdx.x % tiles) * kTopnRows;
    const int row = row0 + tid;
    const bool active = row < n;
    // keys this CTA streams, and the keys this row sees
    const int n_cta = kCausal ? min(n, row0 + kTopnRows) : n;
    const int n_row = kCausal ? row + 1 : n;
    const int N_row = min(N, n_row);

    uint32_t q[DW];
#pragma unroll
    for (int w = 0; w < DW; ++w) q[w] = active ? __ldg(qbits + (head * n + row) * DW + w) : 0u;
    for (int b = 0; b < BINS; ++b) hist[b * kTopnRows + tid] = 0;

    const uint32_t *kh = kbits + head * n * DW;
    for (int j0 = 0; j0 < n_cta; j0 += kTopnKeyChunk) {
        const int cnt = min(kTopnKeyChunk, n_cta - j0);
        __syncthreads();
        for (int t = tid; t < cnt * DW; t += kTopnRows) kch[t] = __ldg(kh + (long long)j0 * DW + t);
        __syncthreads();
        if (active) {
            const int lim = min(cnt, n_row - j0);
            for (int jj = 0; jj < lim; ++jj) {
                int h = 0;
#pragma unroll
                for (int w = 0; w < DW; ++w) h += __popc(q[w] ^ kch[jj * DW + w]);
                hist[h * kTopnRows + tid] += 1;
            }
        }
    }

    int t = BINS;
    uint32_t quota = 0;
    if (active) {
        uint32_t below = 0;
        for (int b = 0; b < BINS; ++b) {
            const uint32_t c = hist[b * kTopnRows + tid];
            if (below + c >= (uint32_t)N_row) { t = b; quota = (uint32_t)N_row - below; break; }
            below += c;
        }
    }

    const long long obase = (head * n + row) * (long long)N;
    int out = 0;
    uint32_t ties = 0;
    for (int j0 = 0; j0 < n_cta; j0 += kTopnKeyChunk) {
        const int cnt = min(kTopnKeyChunk, n_cta - j0);
        __syncthreads();
        for (int tt = tid; tt < cnt * DW; tt += kTopnRows) kch[tt] = __ldg(kh + (long long)j0 * DW + tt);
        __syncthreads();
        if (active) {
            const int lim = min(cnt, n_row - j0);
            for (int jj = 0; jj < lim; ++jj) {
                int h = 0;
#pragma unroll
                for (int w = 0; w < DW; ++w) h += __popc(q[w] ^ kch[jj * DW + w]);
                const bool tie = (h == t);
                const bool keep = (h < t) || (tie && ties < quota);
                ties += tie ? 1u : 0u;
                if (keep) {
                    idx[obase + out] = j0 + jj;
                    if (logits) logits[obase + out] = (int16_t)(D - 2 * h);
                    ++out;
                }
            }
        }
    }
    if (kCausal && active)
        for (int k = out; k < N; ++k) {
            idx[obase + k] = -1;
            if (logits) logits[obase + k] = 0;
        }
}

}  // namespace had
