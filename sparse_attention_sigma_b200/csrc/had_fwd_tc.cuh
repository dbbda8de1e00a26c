// had_fwd_tc.cuh -- the fused binarized top-N attention forward on the sm_100a
// tensor cores, in 128-key tiles ("Hamming Attention Distillation",
// pith.science review, "What carries the argument": sign-quantized Q/K,
// Hamming logits, top-N mask, softmax over the kept logits, value product;
// Eqs. 4-7).
//
// A CTA owns QT tiles of 128 query rows of one head (TMEM lane i = row i of a
// tile; one epilogue thread per row) and streams the head's keys twice, 128
// keys per step:
//   window  the row's threshold level (the Hamming distance of its N-th best
//           key) is estimated from the exact mean of its logits over all keys
//           (q . sum_j k_j, from per-head key column sums) and their spread
//           over the first key tile, as mean + z sd with z the standard normal
//           quantile at N/n.  Levels est-1 .. est+1 form the row's window.
//   pass 1  S = Q K^T (-/+1 x +/-4 int8: Q negated, the s32 accumulator holds
//           -4 s) plus, from the second key tile on, a third MMA step that
//           adds each row's bias (its window offset spread over 32 int8
//           columns, times a tile of ones), so that the accumulator is
//           directly the logit's shift in a thermometer of four 8-bit counters
//           of one register (level <= L0-1, L0, L0+1, L0+2).  One word of
//           counts per tile and row is kept in TMEM.  At the end the summed
//           counters give the exact threshold level t and the number q of
//           keys kept at it whenever t falls inside the window; rows where it
//           does not are listed and recomputed exactly by the fix-up kernel.
//           The tile words give the one tile where the row's tie quota runs
//           out.
//   regroup the CTA's rows are sorted by that tile (a counting sort in shared
//           memory) and the Q tiles are rewritten in that order, so that the
//           32 rows of a warp share few such tiles: they are the only tiles
//           that count ties key by key.
//   pass 2  S again, with Q as -64 times the signs and a bias step that adds
//           the offset of the thread's weight-table column, so that the
//           accumulator is directly the byte offset of the logit's weight:
//           exp2(c2 (s_l - ref)) for levels <= t, 0 beyond.  One shared load
//           per logit gives it; ties at level t are kept or zeroed through the
//           table, except in the quota tile, which keeps the first of them in
//           key order (the lower index wins).  P is packed to fp16 pairs over
//           the first half of its own S in TMEM and the tensor core
//           accumulates O += P V (fp16 x fp16 -> f32).
// The n x n logits never leave the SM.
//
// Warp roles: warp 0 bulk-copies the Q tiles once and streams K (twice) and
// V^T (pass 2) through shared-memory rings; warp 1 issues every MMA from one
// thread, in order, over a ring of three 128-column S slots shared by the
// query tiles (S tile k of the stream sits in slot k % 3; tile k + 3 is issued
// into it once the epilogue has released it in pass 1, or right after the
// P V that reads it in pass 2, since tcgen05 operations of one thread run in
// issue order); warps 2 .. 1 + 4 QT are the epilogue, four per query tile.
// Every wait is bounded by a caller-set limit: a CTA that hits it flags
// HAD_ERR_TIMEOUT, lets its copies and MMAs drain, frees its TMEM and returns.
#pragma once
#include <cuda_fp16.h>
#include <type_traits>

#include "had_common.cuh"
#include "had_tc.cuh"

namespace had {
namespace tcfwd {

constexpr int kRows = 128;      // query rows per tile (TMEM lanes)
constexpr int kKeys = 128;      // keys per S tile (TMEM columns of an S slot)
constexpr int kSub = 64;        // keys per operand tile in the workspace
constexpr int kSlots = 3;       // S slots in TMEM, shared by the CTA's query tiles

#ifndef HAD_TC_QT64
#define HAD_TC_QT64 2
#endif

template <int D>
struct Cfg {
    static constexpr int QT = D == 64 ? HAD_TC_QT64 : 1;   // query tiles per CTA
    static constexpr int EPI_WARPS = 4 * QT;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS);
    static constexpr int QBYTES = kRows * D;            // int8 Q tile
    static constexpr int KBYTES = kKeys * D;            // int8 K tile (two workspace tiles)
    static constexpr int VSUB = D * kSub * 2;           // fp16 V^T workspace tile
    static constexpr int VBYTES = 2 * VSUB;             // fp16 V^T of 128 keys
    static constexpr int KSTAGES = D == 64 ? 4 : 3;
    static constexpr int VSTAGES = D == 64 ? 3 : 2;
    static constexpr int BINS = D + 1;
    static constexpr int TAB_BYTES = BINS * kRows * 4;  // per query tile: [level][row] f32
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t O_COL = kSlots * kKeys;   // query tile g's O at O_COL + g D
    static constexpr int STASH_CAP = D;                 // tile words per row (in O's columns)
    static_assert(O_COL + QT * D <= TMEM_COLS, "TMEM budget");
    // shared memory layout (offsets from a 1024-aligned base)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QT * QBYTES;
    static constexpr int OFF_V = OFF_K + KSTAGES * KBYTES;
    static constexpr int OFF_TAB = OFF_V + VSTAGES * VBYTES;
    // pass-1 bias step: per query tile 128 rows x 32 int8 (one K=32 step),
    // and a 128-key x 32 tile of ones
    static constexpr int BIAS_BYTES = kRows * 32;
    static constexpr int ONES_BYTES = kKeys * 32;
    static constexpr int OFF_BIAS = OFF_TAB + QT * TAB_BYTES;
    static constexpr int OFF_ONES = OFF_BIAS + QT * BIAS_BYTES;
    // pass-2 bias step: per key 16 bytes of 127 then 16 bytes of 1, so that
    // a row's bias bytes (x0..x15, y0..y15) add 127 sum x + sum y
    static constexpr int OFF_ONES2 = OFF_ONES + ONES_BYTES;
    // between the passes the CTA's rows are regrouped by the key tile where
    // their tie quota runs out: per-row state at the new position, and the
    // bucket counts of the counting sort
    static constexpr int ROWS = QT * kRows;
    static constexpr int OFF_STATE = OFF_ONES2 + ONES_BYTES;
    static constexpr int OFF_SORT = OFF_STATE + ROWS * 32;
    static constexpr int SORT_BUCKETS = STASH_CAP + 2;
    static constexpr int OFF_BAR = OFF_SORT + ((SORT_BUCKETS * 4 + 15) / 16) * 16;
    static constexpr int NBARS = 1 + 2 * KSTAGES + 2 * VSTAGES + 3 * kSlots + 2 * QT + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + alignment slack
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    static constexpr uint32_t IDESC_QK = tc::idesc(2, 1, 1, kRows, kKeys);   // s32 <- s8 x s8
    static constexpr uint32_t IDESC_PV = tc::idesc(1, 0, 0, kRows, D);       // f32 <- f16 x f16
};

struct Params {
    const int8_t *qop;        // [BH][qtiles] 128 x D int8 tiles (-/+1: the negated signs)
    const int8_t *kop;        // [BH][kstride] 64 x D int8 tiles (+/-4); kstride even
    const __half *vop;        // [BH][kstride] D x 64 fp16 tiles (V^T, scaled)
    const int *vexp;          // [BH] power of two of the V scale
    const uint32_t *qbits;    // [BH][n][D/32] packed query signs (1 = -1)
    const int *ksum;          // [BH][D] sum over the head's keys of the +/-1 codes
    float *out;               // [BH][n][D]
    int32_t *dbg_idx;         // [BH][n][N] or null
    int16_t *dbg_logits;      // [BH][n][N] or null
    int32_t *status;
    int *miss_count;          // rows whose threshold fell outside the window
    int *miss_rows;           // their flat row ids (head * n + row)
    long long miss_cap;       // entries of miss_rows
    int n, N;
    int qtiles;               // query tiles per head in qop (a multiple of QT)
    int kstride;              // 64-key workspace tiles per head (even)
    int ctas_per_head;
    float c2;                 // tau * log2(e)
    float z;                  // standard normal quantile at N / n
    unsigned long long wait_ns;   // limit of every wait for another role
};

// Bounded wait: false if the deadline passed or another role aborted.  The
// deadline is checked after the first failed try and every 256 after it.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, uint64_t deadline,
                                         volatile int *abort_flag, int32_t *status)
{
    uint32_t spins = 0;
    while (!tc::mbar_try_wait(bar, parity)) {
        if ((spins++ & 255u) == 0) {
            if (*abort_flag) return false;
            if (tc::globaltimer_ns() > deadline) {
                *abort_flag = 1;
                flag(status, HAD_ERR_TIMEOUT);
                return false;
            }
        }
    }
    return true;
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Thermometer increment of the four 8-bit window counters for a logit whose
// first counter is 8 * amount bits up (amount <= 0: all four counters;
// >= 32: none): the high word of 0x01010101:0 shifted left by the amount,
// clamped at 32.
__device__ __forceinline__ uint32_t window_inc(int amount)
{
    return __funnelshift_lc(0u, 0x01010101u, (uint32_t)max(amount, 0));
}

// Barrier of the epilogue warps only (named barrier 1).
__device__ __forceinline__ void epi_sync(int nthreads)
{
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Per-row state handed from pass 1 to pass 2 at the row's new position.
struct RowState {
    int row;          // query index within the head
    int t;            // threshold level (-1: the fix-up kernel recomputes the row)
    int zero_at;      // key tile from which level t weighs nothing
    int jstar;        // key tile where the tie quota runs out (-1: none)
    int kstar;        // ties kept inside it
    int quota;        // ties kept in all (for the key-by-key mode)
    int pad[2];
};

// Make this thread's generic-proxy shared-memory writes visible to the
// tensor core (async proxy).
__device__ __forceinline__ void fence_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int D, bool kDbg>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1)
attention_tc_kernel(const Params p)
{
    using C = Cfg<D>;
    constexpr int QT = C::QT;
    // 1024-aligned base, as an offset from the shared array (so that the
    // compiler keeps shared-memory addressing for every access through it);
    // measured faster than the unaligned base for the weight lookups.
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *const q_full = bar;
    uint64_t *const k_full = bar + 1;
    uint64_t *const k_empty = k_full + C::KSTAGES;
    uint64_t *const v_full = k_empty + C::KSTAGES;
    uint64_t *const v_empty = v_full + C::VSTAGES;
    uint64_t *const s_full = v_empty + C::VSTAGES;     // [kSlots] S tile in the slot
    uint64_t *const s_free = s_full + kSlots;          // [kSlots] pass-1 slot read
    uint64_t *const p_full = s_free + kSlots;          // [kSlots] pass-2 P in the slot
    uint64_t *const q2_ready = p_full + kSlots;        // [QT] Q tile rewritten for pass 2
    uint64_t *const o_full = q2_ready + QT;            // [QT] last P V of the tile done
    uint64_t *const drain = o_full + QT;
    uint64_t *const bias_ready = drain + 1;            // bias rows and ones tile written
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long head = blockIdx.x / p.ctas_per_head;
    const int qtile0 = (blockIdx.x % p.ctas_per_head) * QT;
    const int T = (p.n + kKeys - 1) / kKeys;            // 128-key tiles
    const int J = T * QT;                               // S tiles per pass
    const uint64_t deadline = tc::globaltimer_ns() + p.wait_ns;
    constexpr uint64_t kDrainNs = 500000000ull;         // drains keep a long limit

    if (threadIdx.x == 0) {
        tc::mbar_init(q_full, 1);
        for (int s = 0; s < C::KSTAGES; ++s) {
            tc::mbar_init(k_full + s, 1);
            tc::mbar_init(k_empty + s, 1);
        }
        for (int s = 0; s < C::VSTAGES; ++s) {
            tc::mbar_init(v_full + s, 1);
            tc::mbar_init(v_empty + s, 1);
        }
        for (int s = 0; s < kSlots; ++s) {
            tc::mbar_init(s_full + s, 1);
            tc::mbar_init(s_free + s, 4);               // the four warps of the tile
            tc::mbar_init(p_full + s, 4);
        }
        for (int g = 0; g < QT; ++g) {
            tc::mbar_init(q2_ready + g, 4);
            tc::mbar_init(o_full + g, 1);
        }
        tc::mbar_init(drain, 1);
        tc::mbar_init(bias_ready, C::EPI_WARPS);
        int *buckets = reinterpret_cast<int *>(smem + C::OFF_SORT);
        for (int b = 0; b < C::SORT_BUCKETS; ++b) buckets[b] = 0;
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(tmem_holder, C::TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int8_t *qsrc = p.qop + (head * p.qtiles + qtile0) * (long long)C::QBYTES;
            const int8_t *ksrc = p.kop + head * (long long)p.kstride * (kSub * D);
            const uint8_t *vsrc = reinterpret_cast<const uint8_t *>(p.vop) +
                                  head * (long long)p.kstride * C::VSUB;
            tc::mbar_expect_tx(q_full, QT * C::QBYTES);
            tc::bulk_g2s(smem + C::OFF_Q, qsrc, QT * C::QBYTES, q_full);
            // K stream G = 0 .. 2T-1 (key tile G % T); V tile H follows K
            // stream entry T + H.
            int issued_k = 0, issued_v = 0;
            bool ok = true;
            for (int G = 0; G < 2 * T && ok; ++G) {
                const int ks = G % C::KSTAGES;
                ok = wait_bar(k_empty + ks, ((G / C::KSTAGES) & 1) ^ 1, deadline, abort_flag,
                              p.status);
                if (!ok) break;
                tc::mbar_expect_tx(k_full + ks, C::KBYTES);
                tc::bulk_g2s(smem + C::OFF_K + ks * C::KBYTES,
                             ksrc + (long long)(G % T) * C::KBYTES, C::KBYTES, k_full + ks);
                issued_k = G + 1;
                if (G >= T) {
                    const int H = G - T, vs = H % C::VSTAGES;
                    ok = wait_bar(v_empty + vs, ((H / C::VSTAGES) & 1) ^ 1, deadline, abort_flag,
                                  p.status);
                    if (!ok) break;
                    tc::mbar_expect_tx(v_full + vs, C::VBYTES);
                    tc::bulk_g2s(smem + C::OFF_V + vs * C::VBYTES,
                                 vsrc + (long long)H * C::VBYTES, C::VBYTES, v_full + vs);
                    issued_v = H + 1;
                }
            }
            if (!ok) {
                // let every copy already in flight land before the CTA exits
                const uint64_t dl = tc::globaltimer_ns() + kDrainNs;
                volatile int never = 0;
                wait_bar(q_full, 0, dl, &never, p.status);
                for (int G = max(0, issued_k - C::KSTAGES); G < issued_k; ++G)
                    wait_bar(k_full + G % C::KSTAGES, (G / C::KSTAGES) & 1, dl, &never, p.status);
                for (int H = max(0, issued_v - C::VSTAGES); H < issued_v; ++H)
                    wait_bar(v_full + H % C::VSTAGES, (H / C::VSTAGES) & 1, dl, &never, p.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // Descriptors are built once; a tile, stage or K step moves only
            // the start-address field (16-byte units).
            const uint64_t dq = tc::smem_desc(tc::smem_u32(smem + C::OFF_Q), 128, D * 8);
            const uint64_t dk = tc::smem_desc(tc::smem_u32(smem + C::OFF_K), 128, D * 8);
            const uint64_t dv = tc::smem_desc(tc::smem_u32(smem + C::OFF_V), 128, 8 * 128);
            // the bias step: K extent 32 bytes (two core matrices), rows 256 B apart
            const uint64_t dbias = tc::smem_desc(tc::smem_u32(smem + C::OFF_BIAS), 128, 256);
            const uint64_t dones = tc::smem_desc(tc::smem_u32(smem + C::OFF_ONES), 128, 256);
            const uint64_t dones2 = tc::smem_desc(tc::smem_u32(smem + C::OFF_ONES2), 128, 256);
            bool ok = wait_bar(q_full, 0, deadline, abort_flag, p.status);
            tc::fence_after_sync();
            // S tile kidx = S = Q_g K_u^T into slot kidx % 3; G is the K stream
            // entry that holds key tile u (the stage is waited for at g = 0 and
            // released after the last query tile's MMAs).
            // bias: 0 none, 1 the pass-1 window offset, 2 the pass-2 table offset.
            // synced: a barrier that epilogue threads arrive on was just waited
            // for, so their prior TMEM and shared-memory work must be ordered
            // before these MMAs (a fence); the copy barriers (async proxy, like
            // the MMA) and the in-order reuse of a slot after its P V need none.
            auto qk = [&](int kidx, int g, int G, int bias, bool synced) -> bool {
                const int ks = G % C::KSTAGES;
                if (g == 0 &&
                    !wait_bar(k_full + ks, (G / C::KSTAGES) & 1, deadline, abort_flag, p.status))
                    return false;
                if (synced) tc::fence_after_sync();
                const uint64_t dqa = dq + (uint64_t)((g * C::QBYTES) >> 4);
                const uint64_t dkb = dk + (uint64_t)((ks * C::KBYTES) >> 4);
                const uint32_t dcol = tmem + (kidx % kSlots) * kKeys;
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk)
                    tc::mma_i8_ss(dcol, dqa + (uint64_t)(kk * 16), dkb + (uint64_t)(kk * 16),
                                  C::IDESC_QK, kk > 0 ? 1u : 0u);
                if (bias)
                    tc::mma_i8_ss(dcol, dbias + (uint64_t)((g * C::BIAS_BYTES) >> 4),
                                  bias == 1 ? dones : dones2, C::IDESC_QK, 1u);
                tc::mma_commit(s_full + kidx % kSlots);
                if (g == QT - 1) tc::mma_commit(k_empty + ks);
                return true;
            };
            // pass 1: slot reuse waits for the epilogue to have read tile kidx - 3;
            // key tiles after the first add the rows' bias (written once the
            // first tile has placed each row's window)
            for (int kidx = 0; kidx < J && ok; ++kidx) {
                if (kidx >= kSlots &&
                    !wait_bar(s_free + kidx % kSlots, ((kidx - kSlots) / kSlots) & 1, deadline,
                              abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                if (kidx == QT && !wait_bar(bias_ready, 0, deadline, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                ok = qk(kidx, kidx % QT, kidx / QT, kidx >= QT ? 1 : 0,
                        kidx >= kSlots || kidx == QT);
            }
            // pass 2: tile j of the pass is stream tile J + j
            auto qk2 = [&](int j) -> bool {
                const int kidx = J + j, u = j / QT, g = j % QT;
                if (u == 0 && !wait_bar(q2_ready + g, 0, deadline, abort_flag, p.status))
                    return false;
                // the slot last held pass-1 tile kidx - 3 (if any): wait until read
                const bool after_pass1 = kidx >= kSlots && kidx - kSlots < J;
                if (after_pass1 &&
                    !wait_bar(s_free + kidx % kSlots, ((kidx - kSlots) / kSlots) & 1, deadline,
                              abort_flag, p.status))
                    return false;
                return qk(kidx, g, T + u, 2, u == 0 || after_pass1);
            };
            for (int j = 0; j < min(kSlots, J) && ok; ++j) ok = qk2(j);
            for (int j = 0; j < J && ok; ++j) {
                const int kidx = J + j, u = j / QT, g = j % QT;
                const int vs = u % C::VSTAGES;
                if (g == 0 &&
                    !wait_bar(v_full + vs, (u / C::VSTAGES) & 1, deadline, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                if (!wait_bar(p_full + kidx % kSlots, (j / kSlots) & 1, deadline, abort_flag,
                              p.status)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t pcol = tmem + (kidx % kSlots) * kKeys;   // P over S
                const uint32_t ocol = tmem + C::O_COL + g * D;
                const uint64_t dvs = dv + (uint64_t)((vs * C::VBYTES) >> 4);
#pragma unroll
                for (int c = 0; c < kKeys / 16; ++c) {
                    const uint32_t boff = (uint32_t)((c >> 2) * C::VSUB + (c & 3) * 256);
                    tc::mma_f16_ts(ocol, pcol + c * 8, dvs + (uint64_t)(boff >> 4), C::IDESC_PV,
                                   (u > 0 || c > 0) ? 1u : 0u);
                }
                if (g == QT - 1) tc::mma_commit(v_empty + vs);
                if (u == T - 1) tc::mma_commit(o_full + g);
                if (j + kSlots < J) ok = qk2(j + kSlots);
            }
            // drain: wait until every MMA this thread issued has completed
            tc::mma_commit(drain);
            volatile int never = 0;
            wait_bar(drain, 0, tc::globaltimer_ns() + kDrainNs, &never, p.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        using BT = std::integral_constant<bool, true>;
        using BF = std::integral_constant<bool, false>;
        constexpr int NT = C::EPI_WARPS * 32;
        const int g = (warp - 2) >> 2;                // query tile of this warp
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter ...
        const int r = quarter * 32 + lane;            // row (TMEM lane) within the tile
        const int f = g * kRows + r;                  // position among the CTA's rows
        const int row1 = (qtile0 + g) * kRows + r;    // pass-1 query index within the head
        const bool active1 = row1 < p.n;
        const int Nr = p.N;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t stash = lane_base + C::O_COL + g * D;
        const bool stash_ok = !kDbg && T <= C::STASH_CAP;
        const int T_full = p.n / kKeys;               // key tiles without padding keys
        bool ok = true;

        // exact mean of the row's logits over all keys: q . sum_j k_j / n
        int kdot = 0;
        {
            uint32_t qw[D / 32];
#pragma unroll
            for (int w = 0; w < D / 32; ++w)
                qw[w] = active1 ? __ldg(p.qbits + ((head * p.n) + row1) * (D / 32) + w) : 0u;
            const int *ks = p.ksum + head * D;
#pragma unroll
            for (int w = 0; w < D / 32; ++w) {
#pragma unroll 8
                for (int b = 0; b < 32; ++b) {
                    const int v = __ldg(ks + 32 * w + b);
                    kdot += ((qw[w] >> b) & 1u) ? -v : v;
                }
            }
        }

        uint32_t ra[32], rb[32];
        auto ld = [&](int kidx, int ch, uint32_t (&rr)[32]) {
            tc::tmem_ld32(lane_base + (kidx % kSlots) * kKeys + ch * 32, rr);
        };
        auto wait_s = [&](int kidx) -> bool {
            const bool w = __all_sync(kFullMask, wait_bar(s_full + kidx % kSlots,
                                                          (kidx / kSlots) & 1, deadline,
                                                          abort_flag, p.status));
            tc::fence_after_sync();
            return w;
        };
        auto release_s = [&](int kidx) {
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(s_free + kidx % kSlots);
        };
        auto chunk_valid = [&](int u, int ch) { return min(32, p.n - u * kKeys - ch * 32); };

        // ---------------------------------------------------------- window
        // Spread of the first key tile's logits (v = -4 s) -> estimated
        // threshold level est; counters cover levels L0 - 1 .. L0 + 2 with
        // L0 = est - 1, and a logit's counter shift is cshift + v: the bias
        // step adds cshift on the tensor core from the second key tile on.
        int cshift = 0, L0 = 0;
        if (ok) ok = wait_s(g);
        if (ok) {
            long long sv = 0, sv2 = 0;
            const int cnt = min(kKeys, p.n);
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
                ld(g, ch, ra);
                tc::tmem_wait_ld(ra);
                const int valid = chunk_valid(0, ch);
                int s1 = 0, s2 = 0;
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int v = c < valid ? (int)ra[c] : 0;
                    s1 += v;
                    s2 += v * v;
                }
                sv += s1;
                sv2 += s2;
            }
            const float inv = 1.0f / (float)cnt;
            const float m4 = (float)sv * inv;
            const float var4 = fmaxf((float)sv2 * inv - m4 * m4, 0.0f);
            const float mean_s = (float)kdot / (float)p.n;
            // level = (D - s) / 2: mean (D - mean_s) / 2, spread sd(s) / 2
            const float est_f = 0.5f * ((float)D - mean_s) + p.z * 0.125f * sqrtf(var4);
            const int est = min(D, max(0, __float2int_rn(est_f)));
            L0 = est - 1;
            cshift = 4 * D - 8 * L0 + 8;              // 8 (level - L0 + 1) = cshift + v
        }
        {
            // this row's bias: 32 int8 values summing to cshift (each within
            // one of cshift / 32), in the K-major layout of the bias step
            const int qb = cshift / 32, rem = cshift - 32 * qb;
            const int sgn = rem < 0 ? -1 : 1, nrem = rem < 0 ? -rem : rem;
            uint32_t wb[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t word = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int m = 4 * i + b;
                    word |= (uint32_t)(uint8_t)(int8_t)(qb + (m < nrem ? sgn : 0)) << (8 * b);
                }
                wb[i] = word;
            }
            uint8_t *bt = smem + C::OFF_BIAS + g * C::BIAS_BYTES;
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<uint4 *>(bt + ((r >> 3) * 2 + h) * 128 + (r & 7) * 16) =
                    make_uint4(wb[4 * h], wb[4 * h + 1], wb[4 * h + 2], wb[4 * h + 3]);
            // the constant tiles of the bias steps, shared by the query tiles:
            // all ones (pass 1); per key 16 x 127 then 16 x 1 (pass 2), which
            // in the K-major layout is core matrices of 127 then of 1
            for (int i = f; i < C::ONES_BYTES / 16; i += NT) {
                reinterpret_cast<uint4 *>(smem + C::OFF_ONES)[i] =
                    make_uint4(0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u);
                const uint32_t x = ((i >> 3) & 1) ? 0x01010101u : 0x7F7F7F7Fu;
                reinterpret_cast<uint4 *>(smem + C::OFF_ONES2)[i] = make_uint4(x, x, x, x);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bias_ready);
        }

        // ---------------------------------------------------------- pass 1
        uint32_t acc[4] = {0u, 0u, 0u, 0u};
        int tot[4] = {0, 0, 0, 0};                    // the four counters over all tiles
        // off = cshift for the first key tile (no bias step), 0 after it
        auto therm = [&](const uint32_t (&rr)[32], int valid, int off, auto masked) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
                if (!decltype(masked)::value || c < valid)
                    acc[c & 3] += window_inc(off + (int)rr[c]);
        };
        auto end_tile1 = [&](int u) {
            const uint32_t w = (acc[0] + acc[1]) + (acc[2] + acc[3]);   // fields <= 128
            acc[0] = acc[1] = acc[2] = acc[3] = 0u;
#pragma unroll
            for (int k = 0; k < 4; ++k) tot[k] += (int)((w >> (8 * k)) & 0xFFu);
            if (stash_ok) tc::tmem_st1(stash + u, w);
        };
        // one key tile; chunk 0 is in ra on entry, the next tile's chunk 0
        // on exit; first: no bias step (add cshift); masked: padding keys
        auto p1_tile = [&](int u, auto first, auto masked) {
            const int kidx = u * QT + g;
            const int off = decltype(first)::value ? cshift : 0;
            ld(kidx, 1, rb);
            therm(ra, chunk_valid(u, 0), off, masked);
            tc::tmem_wait_ld(rb);
            ld(kidx, 2, ra);
            therm(rb, chunk_valid(u, 1), off, masked);
            tc::tmem_wait_ld(ra);
            ld(kidx, 3, rb);
            therm(ra, chunk_valid(u, 2), off, masked);
            tc::tmem_wait_ld(rb);
            release_s(kidx);
            const bool more = u + 1 < T;
            if (more) {
                ok = wait_s(kidx + QT);
                if (ok) ld(kidx + QT, 0, ra);
            }
            therm(rb, chunk_valid(u, 3), off, masked);
            end_tile1(u);
            if (more && ok) tc::tmem_wait_ld(ra);
        };
        if (ok) {
            ld(g, 0, ra);
            tc::tmem_wait_ld(ra);
            p1_tile(0, BT{}, BT{});
        }
#pragma unroll 1
        for (int u = 1; u < T_full && ok; ++u) p1_tile(u, BF{}, BF{});
        if (ok && T > T_full && T_full >= 1) p1_tile(T - 1, BF{}, BT{});

        // threshold level t and the number q of keys kept at it
        const int f0 = tot[0], f1 = tot[1], f2 = tot[2], f3 = tot[3];
        int t = -1, quota = 0;
        bool miss = false;
        if (f0 < Nr && f3 >= Nr) {
            if (f1 >= Nr) { t = L0; quota = Nr - f0; }
            else if (f2 >= Nr) { t = L0 + 1; quota = Nr - f1; }
            else { t = L0 + 2; quota = Nr - f2; }
        } else {
            miss = true;
        }
        // Where the tie quota runs out: ties are kept in full before tile
        // jstar, kstar of them (the lowest indices) inside it, none after it;
        // from tile zero_at on the weight table maps level t to 0.
        int zero_at = T, jstar = -1, kstar = 0;
        if (stash_ok && ok) {
            tc::tmem_wait_st();
            const bool want = t >= 0 && !miss;
            const int ts = t - L0 + 1;                // 1..3: field of level t in a tile word
            bool found = !want;
            int cum = 0;
            for (int c0 = 0; c0 < T; c0 += 32) {
                uint32_t w[32];
                tc::tmem_ld32(stash + c0, w);
                tc::tmem_wait_ld(w);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int jj = c0 + i;
                    if (!found && jj < T) {
                        const int cnt = (int)((w[i] >> (8 * ts)) & 0xFFu) -
                                        (int)((w[i] >> (8 * ts - 8)) & 0xFFu);
                        if (cum + cnt >= quota) {
                            found = true;
                            zero_at = jj + 1;
                            if (quota - cum < cnt) { jstar = jj; kstar = quota - cum; }
                        }
                        cum += cnt;
                    }
                }
            }
            if (!found) miss = true;                  // counts disagree: recompute the row
        }
        if (miss && active1) {
            const int slot = atomicAdd(p.miss_count, 1);
            if (slot < p.miss_cap) p.miss_rows[slot] = (int)(head * p.n + row1);
        }
        // missed rows keep nothing here; the fix-up kernel rewrites them
        if (miss) { t = -1; quota = 0; zero_at = T; jstar = -1; }

        // ---------------------------------------------------------- regroup
        // Rows move to new positions sorted by jstar, so that the 32 rows of
        // a warp share few quota tiles (the only tiles that count ties key by
        // key).  Every pass-1 MMA has completed: each warp has seen its
        // tile's last pass-1 S before the first barrier.
        RowState *state = reinterpret_cast<RowState *>(smem + C::OFF_STATE);
        int *buckets = reinterpret_cast<int *>(smem + C::OFF_SORT);
        const int key = (stash_ok && active1 && jstar >= 0) ? jstar + 1 : 0;
        const int rank = atomicAdd(buckets + key, 1);
        uint4 qrow[D / 16];                           // this row's pass-1 Q bytes
        {
            const uint8_t *qt = smem + C::OFF_Q + g * C::QBYTES;
#pragma unroll
            for (int kc = 0; kc < D / 16; ++kc)
                qrow[kc] = *reinterpret_cast<const uint4 *>(
                    qt + ((r >> 3) * (D / 16) + kc) * 128 + (r & 7) * 16);
        }
        epi_sync(NT);
        if (f == 0) {                                 // exclusive prefix over the buckets
            int run = 0;
            for (int b = 0; b < C::SORT_BUCKETS; ++b) {
                const int c = buckets[b];
                buckets[b] = run;
                run += c;
            }
        }
        epi_sync(NT);
        const int fnew = buckets[key] + rank;
        {
            RowState st;
            st.row = row1;
            st.t = t;
            st.zero_at = zero_at;
            st.jstar = jstar;
            st.kstar = kstar;
            st.quota = quota;
            st.pad[0] = st.pad[1] = 0;
            state[fnew] = st;
            // the row's Q at its new position as -64 times the signs (64
            // times the negated signs): bytes 0xFF -> 0xC0, 0x01 -> 0x40
            const int gn = fnew / kRows, rn = fnew % kRows;
            uint8_t *qt = smem + C::OFF_Q + gn * C::QBYTES;
#pragma unroll
            for (int kc = 0; kc < D / 16; ++kc) {
                uint4 x = qrow[kc];
                x.x = (x.x << 6) & 0xC0C0C0C0u;
                x.y = (x.y << 6) & 0xC0C0C0C0u;
                x.z = (x.z << 6) & 0xC0C0C0C0u;
                x.w = (x.w << 6) & 0xC0C0C0C0u;
                *reinterpret_cast<uint4 *>(qt + ((rn >> 3) * (D / 16) + kc) * 128 +
                                           (rn & 7) * 16) = x;
            }
        }
        {
            // pass-2 bias of this thread's position: the byte offset of its
            // table column's level 0 plus 256 D, as 127 * X + Y with X spread
            // over the first 16 bias bytes and Y over the last 16
            const int hbv = g * C::TAB_BYTES + r * 4 + 256 * D;
            const int X = hbv / 127, Y = hbv - 127 * X;
            uint32_t wb[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int tot = i < 4 ? X : Y, base = tot / 16, extra = tot - 16 * base;
                uint32_t word = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int m = 4 * (i & 3) + b;
                    word |= (uint32_t)(base + (m < extra ? 1 : 0)) << (8 * b);
                }
                wb[i] = word;
            }
            uint8_t *bt = smem + C::OFF_BIAS + g * C::BIAS_BYTES;
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<uint4 *>(bt + ((r >> 3) * 2 + h) * 128 + (r & 7) * 16) =
                    make_uint4(wb[4 * h], wb[4 * h + 1], wb[4 * h + 2], wb[4 * h + 3]);
        }
        fence_async_smem();
        epi_sync(NT);                                 // every row of every tile rewritten
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(q2_ready + g);

        // this thread's pass-2 row: the one now at position f
        const RowState st = state[f];
        const int row = st.row;
        const bool active = row < p.n;
        t = st.t;
        zero_at = st.zero_at;
        jstar = st.jstar;
        kstar = st.kstar;
        // Weight table of the row, in this thread's own column (so the lanes
        // of a warp read distinct banks): level l holds exp2(c2 (s_l - ref))
        // for l <= t and 0 beyond.  ref is the threshold logit, raised where
        // needed so that no weight can exceed the fp16 range (s <= D).
        const int tab_off = g * C::TAB_BYTES + r * 4;
        float *tcol = reinterpret_cast<float *>(smem + C::OFF_TAB + tab_off);
        {
            const int headroom =
                p.c2 > 1.0e-6f ? (int)fminf(floorf(15.99f / p.c2), 1.0e6f) : 1000000;
            const int ref = max(D - 2 * max(t, 0), D - headroom);
            for (int bin = 0; bin < C::BINS; ++bin)
                tcol[bin * kRows] =
                    bin <= t ? ex2(p.c2 * (float)(D - 2 * bin - ref)) : 0.0f;
        }
        // The pass-2 accumulator holds a = hb - 256 s (the bias step adds
        // hb): level l = (D - s) / 2 sits l * 512 bytes past the column's
        // level 0, so a is the byte offset of the logit's weight in the tables.
        const uint8_t *tab = smem + C::OFF_TAB;
        const int hb = tab_off + 256 * D;
        auto weight = [&](uint32_t a) { return *reinterpret_cast<const float *>(tab + a); };

        const uint32_t vt = (uint32_t)(hb - 256 * (D - 2 * t));   // accumulator of the threshold
        int rem = st.quota;                           // ties still to keep (key-by-key mode)
        int kept = 0;
        float zacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const long long obase = ((head * p.n) + row) * (long long)p.N;
        constexpr int kAll = 1 << 30;

        // ---------------------------------------------------------- pass 2
        auto fast_chunk = [&](const uint32_t (&rr)[32], uint32_t (&pk)[16]) {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                const float w0 = weight(rr[c]);
                const float w1 = weight(rr[c + 1]);
                zacc[c & 2] += w0;
                zacc[(c & 2) + 1] += w1;
                __half2 h2 = __floats2half2_rn(w0, w1);
                pk[c >> 1] = *reinterpret_cast<uint32_t *>(&h2);
            }
        };
        // ties at the threshold are kept while rl > 0, in ascending key
        // order; keys past n weigh nothing
        auto slow_chunk = [&](int key0, const uint32_t (&rr)[32], uint32_t (&pk)[16], int &rl,
                              int valid) {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                float w2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const uint32_t a = rr[c + e];            // hb - 256 s
                    const bool in = (c + e) < valid;
                    float w = weight(a);                     // 0 below the threshold
                    const bool tie = (a == vt);
                    const bool drop = !in || (tie && rl <= 0);
                    rl -= tie ? 1 : 0;
                    w = drop ? 0.0f : w;
                    zacc[e + (c & 2)] += w;
                    w2[e] = w;
                    if (kDbg) {
                        // kept: above the threshold (a below vt) or a kept tie
                        if (active && !drop && ((int)a < (int)vt || tie) && kept < p.N) {
                            if (p.dbg_idx) p.dbg_idx[obase + kept] = key0 + c + e;
                            if (p.dbg_logits)
                                p.dbg_logits[obase + kept] = (int16_t)((hb - (int)a) / 256);
                            ++kept;
                        }
                    }
                }
                __half2 h2 = __floats2half2_rn(w2[0], w2[1]);
                pk[c >> 1] = *reinterpret_cast<uint32_t *>(&h2);
            }
        };
        auto chunk2 = [&](int u, int ch, bool slow, const uint32_t (&rr)[32], uint32_t (&pk)[16],
                          int &rl) {
            if (!slow) fast_chunk(rr, pk);
            else slow_chunk(u * kKeys + ch * 32, rr, pk, rl, chunk_valid(u, ch));
        };
        // one key tile; chunk 0 is in ra on entry, the next tile's in ra on exit
        auto p2_tile = [&](int u, bool masked) {
            const int kidx = J + u * QT + g;
            if (u == zero_at) tcol[t * kRows] = 0.0f;   // ties past the quota weigh nothing now
            const bool slow = masked || !stash_ok || __any_sync(kFullMask, u == jstar);
            int rl = !stash_ok ? rem : (u == jstar ? kstar : kAll);
            uint32_t pk[16];
            const uint32_t pcol = lane_base + (kidx % kSlots) * kKeys;   // P over S
            ld(kidx, 1, rb);
            chunk2(u, 0, slow, ra, pk, rl);
            tc::tmem_st16(pcol, pk);                  // S columns 0-15 are already read
            tc::tmem_wait_ld(rb);
            ld(kidx, 2, ra);
            chunk2(u, 1, slow, rb, pk, rl);
            tc::tmem_st16(pcol + 16, pk);
            tc::tmem_wait_ld(ra);
            ld(kidx, 3, rb);
            chunk2(u, 2, slow, ra, pk, rl);
            tc::tmem_st16(pcol + 32, pk);
            tc::tmem_wait_ld(rb);
            const bool more = u + 1 < T;
            if (more) {
                ok = wait_s(kidx + QT);
                if (ok) ld(kidx + QT, 0, ra);
            }
            chunk2(u, 3, slow, rb, pk, rl);
            if (!stash_ok) rem = rl;
            tc::tmem_st16(pcol + 48, pk);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (ok && lane == 0) tc::mbar_arrive(p_full + kidx % kSlots);
            if (more && ok) tc::tmem_wait_ld(ra);
        };
        if (ok) ok = wait_s(J + g);
        if (ok) {
            ld(J + g, 0, ra);
            tc::tmem_wait_ld(ra);
        }
#pragma unroll 1
        for (int u = 0; u < T_full && ok; ++u) p2_tile(u, false);
        if (ok && T > T_full) p2_tile(T - 1, true);
        float Z = (zacc[0] + zacc[1]) + (zacc[2] + zacc[3]);
        if (!(Z > 0.0f)) Z = 1.0f;                    // missed or inactive rows only

        // output: O / Z * 2^e_h
        if (ok)
            ok = __all_sync(kFullMask, wait_bar(o_full + g, 0, deadline, abort_flag, p.status));
        if (ok) {
            tc::fence_after_sync();
            const float scale = ldexpf(1.0f, p.vexp[head]) / Z;
            float *orow = p.out + ((head * p.n) + row) * (long long)D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                tc::tmem_ld32(lane_base + C::O_COL + g * D + c0, o);
                tc::tmem_wait_ld(o);
                if (active) {
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        float4 v = make_float4(__uint_as_float(o[c]) * scale,
                                               __uint_as_float(o[c + 1]) * scale,
                                               __uint_as_float(o[c + 2]) * scale,
                                               __uint_as_float(o[c + 3]) * scale);
                        *reinterpret_cast<float4 *>(orow + c0 + c) = v;
                    }
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace tcfwd
}  // namespace had
