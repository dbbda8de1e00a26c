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
//           -4 s).  Adding the row's window offset to it (one fused add-max
//           per logit) gives the logit's shift in a thermometer of four 8-bit
//           counters of one register (level <= L0-1, L0, L0+1, L0+2).  One
//           word of counts per tile and row is kept in shared memory.  At the
//           end the summed counters give the exact threshold level t and the
//           number q of keys kept at it whenever t falls inside the window;
//           rows where it does not are listed and recomputed exactly by the
//           fix-up kernel.  The tile words give the one tile where the row's
//           tie quota runs out.
//   pass 2  S again, with Q as -64 times the signs and a bias step that adds
//           the offset of the thread's weight-table column, so that the
//           accumulator is directly the byte offset of the logit's weight:
//           exp2(c2 (s_l - ref)) for levels <= t, 0 beyond.  One shared load
//           per logit gives it.  Ties at level t weigh w_t before the quota
//           tile and 0 from it on (the table entry is cleared there), so every
//           full tile takes the same path.  P is packed to fp16 pairs over
//           the first half of its own S in TMEM and the tensor core
//           accumulates O += P V (fp16 x fp16 -> f32).
//   quota   the kept ties of the quota tile (the first of them in key order:
//           the lower index wins), by one of three modes (kMode): found
//           between the passes by a scan of the head's packed key signs in
//           shared memory (Hamming distance = level) and set in P in pass 2;
//           masked in P from the S values in pass 2; or found after pass 2
//           from the key signs in global memory and added to O and Z by the
//           row's thread.
// The n x n logits never leave the SM.
//
// Warp roles: warp 0 bulk-copies the Q tiles once and streams K (twice) and
// V^T (pass 2) through shared-memory rings.  One thread of warp 1 issues the
// Q K^T MMAs and one thread of warp 2 + g the P V MMAs of query tile g (a
// thread that shares its scheduler with epilogue warps issues a tcgen05
// instruction only every ~100 cycles, so the streams go out in parallel).
// Pass 1 uses all four 128-column TMEM slots: key tile u's S tiles (one per
// query tile) go to stage u % (4 / QT), reused once every epilogue warp has
// read it; the row's tile words go to its weight-table column in shared
// memory.  Pass 2 uses three slots and O: S tile j (= u QT + g) goes to slot
// j % 3 once the P V of tile j - 3 has completed.  Warps 2 + QT .. 1 + 5 QT
// are the epilogue, four per query tile.
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
    static constexpr int EPI_WARP0 = 2 + QT;           // producer, Q K^T issuer, a P V issuer per query tile
    static constexpr int THREADS = 32 * (EPI_WARP0 + EPI_WARPS);
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
    // pass 1 uses all four 128-column slots (O's columns are free then):
    // stage st of key tile u (u % P1_STAGES) holds the QT S tiles of u
    static constexpr int P1_STAGES = 4 / QT;
    static constexpr int STASH_CAP = D;                 // tile words per row (its table column)
    static_assert(O_COL + QT * D <= TMEM_COLS, "TMEM budget");
    // shared memory layout (offsets from a 1024-aligned base)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QT * QBYTES;
    static constexpr int OFF_V = OFF_K + KSTAGES * KBYTES;
    static constexpr int OFF_TAB = OFF_V + VSTAGES * VBYTES;
    // pass-2 bias step: per query tile 128 rows x 32 int8 (one K=32 step),
    // and per key 16 bytes of 127 then 16 bytes of 1, so that a row's bias
    // bytes (x0..x15, y0..y15) add 127 sum x + sum y
    static constexpr int BIAS_BYTES = kRows * 32;
    static constexpr int ONES_BYTES = kKeys * 32;
    static constexpr int OFF_BIAS = OFF_TAB + QT * TAB_BYTES;
    static constexpr int OFF_ONES2 = OFF_BIAS + QT * BIAS_BYTES;
    static constexpr int OFF_BAR = OFF_ONES2 + ONES_BYTES;
    // the pass-2 bias (a shared address of the tables + 256 D, with up to 1 KB
    // of alignment and a small window base below it) is 127 X + Y with
    // X, Y <= 16 * 127
    static_assert(OFF_TAB + QT * TAB_BYTES + 256 * D + 4096 < 127 * (16 * 127 + 1),
                  "pass-2 bias range");
    static constexpr int NBARS = 1 + 2 * KSTAGES + 2 * VSTAGES + (2 + QT) * kSlots +
                                 2 * P1_STAGES + 3 * QT + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + alignment slack
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    // mode with the head's packed key signs in shared memory (n D / 8 bytes
    // widened to 16-byte boundaries, at most KB_CAP), after the rest of the
    // layout
    static constexpr int KB_CAP = D == 64 ? 32768 : 16384;
    static constexpr int OFF_KB = (OFF_MISC + 16 + 127) / 128 * 128;   // 16-byte aligned for the bulk copy
    static constexpr int OFF_KM = OFF_KB + KB_CAP;      // per row its 128-bit kept-tie mask
    static constexpr int SMEM_BYTES_KB = OFF_KM + QT * kRows * 16 + 1024;
    static_assert(SMEM_BYTES_KB <= 227 * 1024, "shared memory budget (key signs)");
    static constexpr uint32_t IDESC_QK = tc::idesc(2, 1, 1, kRows, kKeys);   // s32 <- s8 x s8
    static constexpr uint32_t IDESC_PV = tc::idesc(1, 0, 0, kRows, D);       // f32 <- f16 x f16
};

struct Params {
    const int8_t *qop;        // [BH][qtiles] 128 x D int8 tiles (-/+1: the negated signs)
    const int8_t *kop;        // [BH][kstride] 64 x D int8 tiles (+/-4); kstride even
    const __half *vop;        // [BH][kstride] D x 64 fp16 tiles (V^T, scaled)
    const int *vexp;          // [BH] power of two of the V scale
    const uint32_t *qbits;    // [BH][n][D/32] packed query signs (1 = -1)
    const uint32_t *kbits;    // [BH][n][D/32] packed key signs (1 = -1)
    const void *v;            // [BH][n][D] the values as given (bf16 or f32)
    int v_f32;                // 1: v is f32, 0: bf16
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
// abort flag and the deadline are checked every 32 failed tries (each try
// may suspend the thread for a while); reading the global timer on every
// failed try measurably slowed the issuing threads.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, uint64_t deadline,
                                         volatile int *abort_flag, int32_t *status)
{
    uint32_t spins = 0;
    while (!tc::mbar_try_wait(bar, parity)) {
        if ((++spins & 31u) == 0) {
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
// first counter is 8 * amount bits up, amount = v + shift (amount <= 0: all
// four counters; >= 32: none): the high word of 0x01010101:0 shifted left by
// the amount, clamped at 32 (the add and the clamp at 0 are one instruction).
__device__ __forceinline__ uint32_t window_inc(int v, int shift)
{
    return __funnelshift_lc(0u, 0x01010101u, (uint32_t)__viaddmax_s32(v, shift, 0));
}

// Make this thread's generic-proxy shared-memory writes visible to the
// tensor core (async proxy).
__device__ __forceinline__ void fence_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The quota tile's kept ties (its first kstar keys at level t), by kMode:
//   0: left out of pass 2 and gathered after it from global memory (a fixed
//      latency per CTA; the mode for any size);
//   1: every tie given its weight in pass 2, those past the quota masked out
//      by a per-chunk tie mask of the S values (cheaper with few key tiles);
//   2: found before pass 2 by a scan of the head's packed key signs, copied
//      to shared memory at the start, and set in P by pass 2 (heads whose
//      signs, widened to 16-byte boundaries, fit in KB_CAP bytes).
template <int D, bool kDbg, int kMode>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1)
attention_tc_kernel(const Params p)
{
    using C = Cfg<D>;
    constexpr bool kQ2 = kMode == 1;
    constexpr bool kKB = kMode == 2;
    static_assert(!(kDbg && kMode != 0), "the diagnostic outputs run in mode 0");
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
    uint64_t *const s_full = v_empty + C::VSTAGES;     // [kSlots] pass-2 S tile in the slot
    // [QT][kSlots] pass-2 P of query tile g in the slot: one barrier per
    // (tile, slot), so that the P V issuer of a tile, which skips the other
    // tile's S tiles, never waits on a phase more than one ahead
    uint64_t *const p_full = s_full + kSlots;
    uint64_t *const pv_done = p_full + QT * kSlots;    // [kSlots] the P V reading it done
    uint64_t *const q2_ready = pv_done + kSlots;       // [QT] Q tile rewritten for pass 2
    uint64_t *const o_full = q2_ready + QT;            // [QT] last P V of the tile done
    uint64_t *const drain = o_full + QT;               // [1 + QT] each issuer's MMAs done
    uint64_t *const s1_full = drain + 1 + QT;          // [P1_STAGES] pass-1 S tiles of a key tile
    uint64_t *const s1_free = s1_full + C::P1_STAGES;  // [P1_STAGES] ... read by every epilogue warp
    uint64_t *const kb_full = s1_free + C::P1_STAGES;  // the head's key signs (kMode 2)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long head = blockIdx.x / p.ctas_per_head;
    const int qtile0 = (blockIdx.x % p.ctas_per_head) * QT;
    const int T = (p.n + kKeys - 1) / kKeys;            // 128-key tiles
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
            tc::mbar_init(v_empty + s, QT);             // the P V issuer of every query tile
        }
        for (int s = 0; s < kSlots; ++s) {
            tc::mbar_init(s_full + s, 1);
            tc::mbar_init(pv_done + s, 1);
        }
        for (int s = 0; s < QT * kSlots; ++s) tc::mbar_init(p_full + s, 4);
        for (int g = 0; g < QT; ++g) {
            tc::mbar_init(q2_ready + g, 4);
            tc::mbar_init(o_full + g, 1);
        }
        for (int i = 0; i < 1 + QT; ++i) tc::mbar_init(drain + i, 1);
        for (int st = 0; st < C::P1_STAGES; ++st) {
            tc::mbar_init(s1_full + st, 1);
            tc::mbar_init(s1_free + st, C::EPI_WARPS);
        }
        tc::mbar_init(kb_full, 1);
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
            if (kKB) {
                // the head's packed key signs, for the quota-tile scan: from
                // the 16-byte boundary at or below their start, rounded up to
                // a whole 16 bytes (at most 30 bytes of the neighbouring heads
                // or of the workspace's padding come along)
                const long long b0 = head * p.n * (long long)(D / 8);
                const long long a0 = b0 & ~15ll, a1 = (b0 + p.n * (long long)(D / 8) + 15) & ~15ll;
                tc::mbar_expect_tx(kb_full, (uint32_t)(a1 - a0));
                tc::bulk_g2s(smem + C::OFF_KB, reinterpret_cast<const uint8_t *>(p.kbits) + a0,
                             (uint32_t)(a1 - a0), kb_full);
            }
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
            if (kKB) {
                // the key-sign copy lands before the CTA exits, whether or not
                // an epilogue warp got as far as waiting for it
                volatile int never = 0;
                wait_bar(kb_full, 0, tc::globaltimer_ns() + kDrainNs, &never, p.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ Q K^T issuer
        // The loop keeps every ring position and phase in counters and every
        // descriptor precomputed: this thread shares its scheduler with
        // epilogue warps, so each instruction between two MMAs costs.
        if (lane == 0) {
            uint64_t dq[QT], dbias[QT];
#pragma unroll
            for (int g = 0; g < QT; ++g) {
                dq[g] = tc::smem_desc(tc::smem_u32(smem + C::OFF_Q + g * C::QBYTES), 128, D * 8);
                // the bias step: K extent 32 bytes (two core matrices), rows 256 B apart
                dbias[g] = tc::smem_desc(tc::smem_u32(smem + C::OFF_BIAS + g * C::BIAS_BYTES),
                                         128, 256);
            }
            const uint64_t dk0 = tc::smem_desc(tc::smem_u32(smem + C::OFF_K), 128, D * 8);
            uint64_t dk = dk0;          // descriptor of the current K stage
            const uint64_t dones2 = tc::smem_desc(tc::smem_u32(smem + C::OFF_ONES2), 128, 256);
            bool ok = wait_bar(q_full, 0, deadline, abort_flag, p.status);
            tc::fence_after_sync();
            int ks = 0;                 // K stage of the current key tile
            uint32_t kph = 0;           // its fill phase
            // the D/32 (and, in pass 2, the bias) MMA steps of S = Q_g K^T into
            // the TMEM columns at dcol
            auto qk = [&](uint32_t dcol, int g, bool bias) {
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk)
                    tc::mma_i8_ss(dcol, dq[g] + (uint64_t)(kk * 16), dk + (uint64_t)(kk * 16),
                                  C::IDESC_QK, kk > 0 ? 1u : 0u);
                if (bias) tc::mma_i8_ss(dcol, dbias[g], dones2, C::IDESC_QK, 1u);
            };
            auto next_k = [&]() {
                tc::mma_commit(k_empty + ks);
                dk += (uint64_t)(C::KBYTES >> 4);
                if (++ks == C::KSTAGES) {
                    ks = 0;
                    kph ^= 1u;
                    dk = dk0;
                }
            };
            // Pass 1: key tile u's S tiles (all query tiles) go to stage
            // u % P1_STAGES, which is reused once every epilogue warp has read
            // it.  Every wait before the MMAs is on a barrier that other threads
            // arrive on, so a fence orders their prior TMEM and shared-memory
            // work first.
            for (int u = 0; u < T && ok; ++u) {
                const int st = u % C::P1_STAGES;
                if (u >= C::P1_STAGES)
                    ok = wait_bar(s1_free + st, ((u / C::P1_STAGES) - 1) & 1, deadline, abort_flag,
                                  p.status);
                ok = ok && wait_bar(k_full + ks, kph, deadline, abort_flag, p.status);
                if (!ok) break;
                tc::fence_after_sync();
#pragma unroll
                for (int g = 0; g < QT; ++g) qk(tmem + (st * QT + g) * kKeys, g, false);
                tc::mma_commit(s1_full + st);
                next_k();
            }
            // before the first pass-2 MMA: every query tile's rewritten Q and
            // bias rows, and the ones tile that all epilogue warps wrote; every
            // epilogue warp has then also read all of its pass-1 S tiles
            for (int g = 0; g < QT && ok; ++g)
                ok = wait_bar(q2_ready + g, 0, deadline, abort_flag, p.status);
            // Pass 2: tile j = u QT + g goes to slot j % 3, once the P V of
            // tile j - 3 (pv_done of the slot, its (j / 3 - 1)-th completion)
            // has read it.
            int sl = 0, jw = 0;         // j % 3 and j / 3
            for (int u = 0, j = 0; u < T && ok; ++u) {
                ok = wait_bar(k_full + ks, kph, deadline, abort_flag, p.status);
#pragma unroll
                for (int g = 0; g < QT; ++g, ++j) {
                    if (ok && j >= kSlots)
                        ok = wait_bar(pv_done + sl, (jw - 1) & 1, deadline, abort_flag, p.status);
                    if (ok) {
                        tc::fence_after_sync();
                        qk(tmem + sl * kKeys, g, true);
                        tc::mma_commit(s_full + sl);
                    }
                    if (++sl == kSlots) {
                        sl = 0;
                        ++jw;
                    }
                }
                if (!ok) break;
                next_k();
            }
            // drain: wait until every MMA this thread issued has completed
            tc::mma_commit(drain);
            volatile int never = 0;
            wait_bar(drain, 0, tc::globaltimer_ns() + kDrainNs, &never, p.status);
        }
    } else if (warp < C::EPI_WARP0) {
        // ------------------------------------------------------------ P V issuers
        // one per query tile: O_g += P V for the tile's pass-2 S tiles
        // (pass-2 tiles u QT + g), so that the two streams of eight MMAs
        // per key tile go out in parallel
        if (lane == 0) {
            const int g = warp - 2;
            const uint64_t dv0 = tc::smem_desc(tc::smem_u32(smem + C::OFF_V), 128, 8 * 128);
            uint64_t dv = dv0;          // descriptor of the current V stage
            const uint32_t ocol = tmem + C::O_COL + g * D;
            bool ok = true;
            int vs = 0;                 // V stage of the current key tile
            uint32_t vph = 0;           // its fill phase
            int j = g;                  // pass-2 tile index
            for (int u = 0; u < T && ok; ++u, j += QT) {
                const int sl = j % kSlots;
                // this tile's p_full of the slot completes the (u / 3)-th time
                // for key tile u (its S tiles visit the three slots in turn)
                ok = wait_bar(v_full + vs, vph, deadline, abort_flag, p.status) &&
                     wait_bar(p_full + g * kSlots + sl, (u / kSlots) & 1, deadline, abort_flag,
                              p.status);
                if (!ok) break;
                tc::fence_after_sync();
                const uint32_t pcol = tmem + sl * kKeys;           // P over S
#pragma unroll
                for (int c = 0; c < kKeys / 16; ++c) {
                    const uint32_t boff = (uint32_t)((c >> 2) * C::VSUB + (c & 3) * 256);
                    tc::mma_f16_ts(ocol, pcol + c * 8, dv + (uint64_t)(boff >> 4), C::IDESC_PV,
                                   (u > 0 || c > 0) ? 1u : 0u);
                }
                tc::mma_commit(pv_done + sl);
                tc::mma_commit(v_empty + vs);
                if (u == T - 1) tc::mma_commit(o_full + g);
                dv += (uint64_t)(C::VBYTES >> 4);
                if (++vs == C::VSTAGES) {
                    vs = 0;
                    vph ^= 1u;
                    dv = dv0;
                }
            }
            tc::mma_commit(drain + 1 + g);
            volatile int never = 0;
            wait_bar(drain + 1 + g, 0, tc::globaltimer_ns() + kDrainNs, &never, p.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        using BT = std::integral_constant<bool, true>;
        using BF = std::integral_constant<bool, false>;
        constexpr int NT = C::EPI_WARPS * 32;
        const int g = (warp - C::EPI_WARP0) >> 2;     // query tile of this warp
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter ...
        const int r = quarter * 32 + lane;            // row (TMEM lane) within the tile
        const int f = g * kRows + r;                  // position among the CTA's rows
        const int row1 = (qtile0 + g) * kRows + r;    // pass-1 query index within the head
        const bool active1 = row1 < p.n;
        const int Nr = p.N;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        // this thread's column of the weight table: in pass 1 it holds the
        // row's tile words (word u at u * kRows), later the weights
        const int tab_off = g * C::TAB_BYTES + r * 4;
        float *tcol = reinterpret_cast<float *>(smem + C::OFF_TAB + tab_off);
        uint32_t *stash = reinterpret_cast<uint32_t *>(tcol);
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
        // pass-2 S tile j (= u QT + g) sits in slot j % 3
        auto ld = [&](int j, int ch, uint32_t (&rr)[32]) {
            tc::tmem_ld32(lane_base + (j % kSlots) * kKeys + ch * 32, rr);
        };
        auto wait_s = [&](int j) -> bool {
            const bool w = __all_sync(kFullMask, wait_bar(s_full + j % kSlots, (j / kSlots) & 1,
                                                          deadline, abort_flag, p.status));
            tc::fence_after_sync();
            return w;
        };
        // pass-1 key tile u sits in stage u % P1_STAGES, slot stage * QT + g
        auto ld1 = [&](int u, int ch, uint32_t (&rr)[32]) {
            tc::tmem_ld32(lane_base + ((u % C::P1_STAGES) * QT + g) * kKeys + ch * 32, rr);
        };
        auto wait_s1 = [&](int u) -> bool {
            const bool w = __all_sync(kFullMask, wait_bar(s1_full + u % C::P1_STAGES,
                                                          (u / C::P1_STAGES) & 1, deadline,
                                                          abort_flag, p.status));
            tc::fence_after_sync();
            return w;
        };
        auto release_s1 = [&](int u) {
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(s1_free + u % C::P1_STAGES);
        };
        auto chunk_valid = [&](int u, int ch) { return min(32, p.n - u * kKeys - ch * 32); };

        // ---------------------------------------------------------- window
        // Spread of the first key tile's logits (v = -4 s) -> estimated
        // threshold level est; counters cover levels L0 - 1 .. L0 + 2 with
        // L0 = est - 1, and a logit's counter shift is cshift + v.
        int cshift = 0, L0 = 0;
        if (ok) ok = wait_s1(0);
        if (ok) {
            long long sv = 0, sv2 = 0;
            const int cnt = min(kKeys, p.n);
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
                ld1(0, ch, ra);
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
        // the constant tile of the pass-2 bias step, shared by the query
        // tiles: per key 16 x 127 then 16 x 1, which in the K-major layout is
        // core matrices of 127 then of 1 (made visible to the tensor core by
        // the fence before the pass-2 Q tiles are released)
        for (int i = f; i < C::ONES_BYTES / 16; i += NT) {
            const uint32_t x = ((i >> 3) & 1) ? 0x01010101u : 0x7F7F7F7Fu;
            reinterpret_cast<uint4 *>(smem + C::OFF_ONES2)[i] = make_uint4(x, x, x, x);
        }

        // ---------------------------------------------------------- pass 1
        uint32_t acc[4] = {0u, 0u, 0u, 0u};
        int tot[4] = {0, 0, 0, 0};                    // the four counters over all tiles
        auto therm = [&](const uint32_t (&rr)[32], int valid, auto masked) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
                if (!decltype(masked)::value || c < valid)
                    acc[c & 3] += window_inc((int)rr[c], cshift);
        };
        auto end_tile1 = [&](int u) {
            const uint32_t w = (acc[0] + acc[1]) + (acc[2] + acc[3]);   // fields <= 128
            acc[0] = acc[1] = acc[2] = acc[3] = 0u;
#pragma unroll
            for (int k = 0; k < 4; ++k) tot[k] += (int)((w >> (8 * k)) & 0xFFu);
            if (stash_ok) stash[u * kRows] = w;
        };
        // one key tile; chunk 0 is in ra on entry, the next tile's chunk 0
        // on exit; masked: padding keys
        auto p1_tile = [&](int u, auto masked) {
            ld1(u, 1, rb);
            therm(ra, chunk_valid(u, 0), masked);
            tc::tmem_wait_ld(rb);
            ld1(u, 2, ra);
            therm(rb, chunk_valid(u, 1), masked);
            tc::tmem_wait_ld(ra);
            ld1(u, 3, rb);
            therm(ra, chunk_valid(u, 2), masked);
            tc::tmem_wait_ld(rb);
            release_s1(u);
            const bool more = u + 1 < T;
            if (more) {
                ok = wait_s1(u + 1);
                if (ok) ld1(u + 1, 0, ra);
            }
            therm(rb, chunk_valid(u, 3), masked);
            end_tile1(u);
            if (more && ok) tc::tmem_wait_ld(ra);
        };
        if (ok) {
            ld1(0, 0, ra);
            tc::tmem_wait_ld(ra);
            p1_tile(0, BT{});
        }
#pragma unroll 1
        for (int u = 1; u < T_full && ok; ++u) p1_tile(u, BF{});
        if (ok && T > T_full && T_full >= 1) p1_tile(T - 1, BT{});

        // (kMode 2) the row's packed signs for the quota-tile scan, loaded
        // while the threshold and the pass-2 tables are set up
        uint32_t qw[D / 32];
#pragma unroll
        for (int w = 0; w < D / 32; ++w)
            qw[w] = kKB && active1 ? __ldg(p.qbits + ((head * p.n) + row1) * (D / 32) + w) : 0u;

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
        // jstar, kstar of them (the lowest indices) inside it, none after it.
        // From tile zero_at on the weight table maps level t to 0: the tile
        // after the last one with kept ties, or, when the quota tile's kept
        // ties are added after pass 2, the quota tile itself.
        int zero_at = T, jstar = -1, kstar = 0;
        if (stash_ok && ok) {
            const bool want = t >= 0 && !miss;
            const int ts = t - L0 + 1;                // 1..3: field of level t in a tile word
            bool found = !want;
            int cum = 0;
            for (int c0 = 0; c0 < T; c0 += 32) {
#pragma unroll 8
                for (int i = 0; i < 32; ++i) {
                    const int jj = c0 + i;
                    if (!found && jj < T) {
                        const uint32_t w = stash[jj * kRows];
                        const int cnt = (int)((w >> (8 * ts)) & 0xFFu) -
                                        (int)((w >> (8 * ts - 8)) & 0xFFu);
                        if (cum + cnt >= quota) {
                            found = true;
                            zero_at = jj + 1;
                            if (quota - cum < cnt) {
                                jstar = jj;
                                kstar = quota - cum;
                                if (!kQ2) zero_at = jj;
                            }
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

        // ---------------------------------------------------------- Q for pass 2
        // Every pass-1 MMA of this query tile has completed (this warp has
        // seen its last S), so the tile's Q rows can be rewritten in place as
        // -64 times the signs (64 times the negated signs): bytes 0xFF -> 0xC0,
        // 0x01 -> 0x40.
        {
            uint8_t *qt = smem + C::OFF_Q + g * C::QBYTES;
#pragma unroll
            for (int kc = 0; kc < D / 16; ++kc) {
                uint4 *q4 = reinterpret_cast<uint4 *>(qt + ((r >> 3) * (D / 16) + kc) * 128 +
                                                      (r & 7) * 16);
                uint4 x = *q4;
                x.x = (x.x << 6) & 0xC0C0C0C0u;
                x.y = (x.y << 6) & 0xC0C0C0C0u;
                x.z = (x.z << 6) & 0xC0C0C0C0u;
                x.w = (x.w << 6) & 0xC0C0C0C0u;
                *q4 = x;
            }
        }
        {
            // pass-2 bias of this row: the shared-memory address of its table
            // column's level 0 plus 256 D, as 127 * X + Y with X spread over
            // the first 16 bias bytes and Y over the last 16
            const int hbv = (int)tc::smem_u32(smem + C::OFF_TAB) + g * C::TAB_BYTES + r * 4 + 256 * D;
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
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(q2_ready + g);

        const int row = row1;
        const bool active = active1;
        // Weight table of the row, in this thread's own column (so the lanes
        // of a warp read distinct banks; its tile words are no longer needed):
        // level l holds exp2(c2 (s_l - ref)) for l <= t and 0 beyond.  ref is
        // the threshold logit, raised where needed so that no weight can
        // exceed the fp16 range (s <= D).
        const int headroom =
            p.c2 > 1.0e-6f ? (int)fminf(floorf(15.99f / p.c2), 1.0e6f) : 1000000;
        const int ref = max(D - 2 * max(t, 0), D - headroom);
        for (int bin = 0; bin < C::BINS; ++bin)
            tcol[bin * kRows] = bin <= t ? ex2(p.c2 * (float)(D - 2 * bin - ref)) : 0.0f;
        // The pass-2 accumulator holds a = hb - 256 s (the bias step adds
        // hb): level l = (D - s) / 2 sits l * 512 bytes past the column's
        // level 0, so a is the shared-memory address of the logit's weight.
        const int hb = (int)tc::smem_u32(smem + C::OFF_TAB) + tab_off + 256 * D;
        const uint32_t sbase = tc::smem_u32(smem_raw);
        auto weight = [&](uint32_t a) {
            return *reinterpret_cast<const float *>(smem_raw + (a - sbase));
        };

        const uint32_t vt = (uint32_t)(hb - 256 * (D - 2 * t));   // accumulator of the threshold
        const float wt_tab = t >= 0 ? tcol[t * kRows] : 0.0f;       // the table's weight of level t

        // (kMode 2) The kept ties of the quota tile, before pass 2: bit i of
        // word c is key 32 c + i of tile jstar.  The warp's rows go LPR at a
        // time with lane = key within a 32-key chunk (a chunk's sign words
        // are 32 consecutive entries of shared memory), all loads of a round
        // issued before any is used; lane L keeps the tie ballots of its own
        // row and then cuts them to the first kstar by itself.
        int zq = kstar;                                // ties of tile jstar that Z gains at the end
        uint32_t wt_x;                                 // (kMode 2) what P's changed ties become:
        {                                              // the tie weight as a pair of fp16, or 0
            __half2 h2 = __floats2half2_rn(wt_tab, wt_tab);
            wt_x = *reinterpret_cast<uint32_t *>(&h2);
        }
        if constexpr (kKB) {
            constexpr int DW = D / 32, LPR = D == 64 ? 4 : 2;
            const bool hq = ok && active && jstar >= 0 && kstar > 0;
            // (a CTA that has already aborted stays aborted)
            const bool kb_in = wait_bar(kb_full, 0, deadline, abort_flag, p.status);
            ok = __all_sync(kFullMask, ok && kb_in);
            // key j's sign words: (D / 32) words from byte (head n + j) D / 8 of
            // the packed signs, copied from the 16-byte boundary below the head
            const uint32_t *kbs = reinterpret_cast<const uint32_t *>(
                smem + C::OFF_KB + ((head * p.n * (long long)(D / 8)) & 15));
            uint32_t tw[4] = {0u, 0u, 0u, 0u};
            uint32_t todo = ok ? __ballot_sync(kFullMask, hq) : 0u;
            while (todo) {                            // warp-uniform
                int Ls[LPR], jl[LPR], tl[LPR];
                uint32_t ql[LPR][DW];
#pragma unroll
                for (int e = 0; e < LPR; ++e) {
                    Ls[e] = todo ? __ffs(todo) - 1 : -1;
                    todo &= todo - 1u;
                    const int Lc = max(Ls[e], 0);
                    jl[e] = max(__shfl_sync(kFullMask, jstar, Lc), 0);
                    tl[e] = Ls[e] >= 0 ? __shfl_sync(kFullMask, t, Lc) : -1;   // -1: no tie
#pragma unroll
                    for (int w = 0; w < DW; ++w) ql[e][w] = __shfl_sync(kFullMask, qw[w], Lc);
                }
                uint32_t kx[LPR][4][DW];
#pragma unroll
                for (int e = 0; e < LPR; ++e)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int key = min(jl[e] * kKeys + 32 * c + lane, p.n - 1);
                        if (DW == 2) {
                            const uint2 x = *reinterpret_cast<const uint2 *>(kbs + key * 2);
                            kx[e][c][0] = x.x;
                            kx[e][c][DW - 1] = x.y;
                        } else {
                            const uint4 x = *reinterpret_cast<const uint4 *>(kbs + key * 4);
                            kx[e][c][0] = x.x;
                            kx[e][c][1 % DW] = x.y;
                            kx[e][c][2 % DW] = x.z;
                            kx[e][c][3 % DW] = x.w;
                        }
                    }
#pragma unroll
                for (int e = 0; e < LPR; ++e)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        int ham = 0;
#pragma unroll
                        for (int w = 0; w < DW; ++w) ham += __popc(ql[e][w] ^ kx[e][c][w]);
                        const bool tie = ham == tl[e] && jl[e] * kKeys + 32 * c + lane < p.n;
                        const uint32_t b = __ballot_sync(kFullMask, tie);
                        tw[c] = lane == Ls[e] ? b : tw[c];
                    }
            }
            // this row's cut: its first kstar ties are kept, the rest dropped.
            // The smaller set is the one pass 2 changes in P: the kept ties,
            // set over the table's 0 (the table zeroes level t from tile
            // jstar on), or the dropped ties, cleared from the table's tie
            // weight (then level t keeps its weight through tile jstar).
            int need = hq ? kstar : 0, nkeep = 0, ndrop = 0;
            uint32_t kept[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int cnt = __popc(tw[c]);
                kept[c] = tw[c];
                if (need <= 0) {
                    kept[c] = 0u;
                } else if (cnt > need) {
                    kept[c] &= (1u << __fns(tw[c], 0, need + 1)) - 1u;
                    need = 0;
                } else {
                    need -= cnt;
                }
                nkeep += __popc(kept[c]);
                ndrop += cnt - __popc(kept[c]);
            }
            const bool drop_mode = hq && ndrop < nkeep;
            if (drop_mode) {
                zero_at = jstar + 1;
                zq = -ndrop;
            }
            // in shared memory through pass 2, read on the quota tile
            *reinterpret_cast<uint4 *>(smem + C::OFF_KM + f * 16) =
                drop_mode ? make_uint4(tw[0] & ~kept[0], tw[1] & ~kept[1], tw[2] & ~kept[2],
                                       tw[3] & ~kept[3])
                          : make_uint4(kept[0], kept[1], kept[2], kept[3]);
            if (drop_mode) wt_x = 0u;
        }
        float zdrop = 0.0f;                           // weights of ties dropped after the table
        int rem = quota;                              // ties still to keep (key-by-key mode)
        int kept = 0;
        float zacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};      // key-by-key chunks
        uint64_t zpair[2] = {0ull, 0ull};              // table chunks: pairs of f32 sums
        const long long obase = ((head * p.n) + row) * (long long)p.N;
        constexpr int kAll = 1 << 30;

        // ---------------------------------------------------------- pass 2
        auto fast_chunk = [&](const uint32_t (&rr)[32], uint32_t (&pk)[16]) {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                const float w0 = weight(rr[c]);
                const float w1 = weight(rr[c + 1]);
                // both weights into one pair of sums with one packed add
                asm("{\n\t.reg .b64 t;\n\tmov.b64 t, {%1, %2};\n\t"
                    "add.rn.f32x2 %0, %0, t;\n\t}"
                    : "+l"(zpair[(c >> 1) & 1])
                    : "f"(w0), "f"(w1));
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
        // Quota tile: rl ties of this chunk may still be kept (the lowest
        // indices); the table gave every tie its weight, so the ones past rl
        // are set to 0 in P and taken out of Z.  No per-key dependency: the
        // chunk's ties form a mask, the cut is the (rl+1)-th set bit.
        auto drop_ties = [&](const uint32_t (&rr)[32], uint32_t (&pk)[16], int &rl) {
            uint32_t m = 0;
#pragma unroll
            for (int c = 0; c < 32; ++c) m |= rr[c] == vt ? (1u << c) : 0u;
            const int cnt = __popc(m);
            uint32_t drop = 0;
            if (rl <= 0) drop = m;
            else if (rl < cnt) drop = m & ~((1u << __fns(m, 0, rl + 1)) - 1u);
            rl = max(rl - cnt, 0);
            if (__any_sync(kFullMask, drop != 0u)) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t b = (drop >> (2 * i)) & 3u;
                    pk[i] &= ~(((b & 1u) ? 0x0000FFFFu : 0u) | ((b & 2u) ? 0xFFFF0000u : 0u));
                }
                zdrop += wt_tab * (float)__popc(drop);
            }
        };
        // (kMode 2) the chunk's changed ties of the quota tile (mask m, bit i
        // = column i) become wt_x in P: the tie weight (kept ties, which the
        // table gave 0) or 0 (dropped ties, which it gave the tie weight).
        // Four mask bits are spread to the sign bits of four bytes (bit b to
        // bit 8 b + 7: the shifted copies of the multiply do not overlap), a
        // sign-replicating byte permute widens them to half-word masks, and
        // one three-input logic op selects.
        auto set_kept = [&](uint32_t m, uint32_t (&pk)[16]) {
            if (__any_sync(kFullMask, m != 0u)) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t sp = ((m >> (4 * i)) & 15u) * 0x10204080u;
                    uint32_t lo, hi;
                    asm("prmt.b32 %0, %1, 0, 0x9988;" : "=r"(lo) : "r"(sp));
                    asm("prmt.b32 %0, %1, 0, 0xBBAA;" : "=r"(hi) : "r"(sp));
                    pk[2 * i] = (pk[2 * i] & ~lo) | (wt_x & lo);
                    pk[2 * i + 1] = (pk[2 * i + 1] & ~hi) | (wt_x & hi);
                }
            }
        };
        // one key tile; chunk 0 is in ra on entry, the next tile's in ra on exit
        auto p2_tile = [&](int u, bool masked) {
            const int kidx = u * QT + g;               // pass-2 S tile index
            if (u == zero_at) tcol[t * kRows] = 0.0f;   // ties past the quota weigh nothing now
            // key by key only on the ragged last tile (keys past n) and in
            // the mode without tile words; ties there follow the table (and,
            // without tile words, the running quota)
            const bool slow = masked || !stash_ok;
            int rl = !stash_ok ? rem : (kQ2 && u == jstar ? kstar : kAll);
            // some row of the warp has its quota tile here (pass-2 mode):
            // every chunk also drops that row's ties past its quota
            const bool quota_tile =
                !slow && kQ2 && __any_sync(kFullMask, u == jstar);
            uint32_t pk[16];
            const uint32_t pcol = lane_base + (kidx % kSlots) * kKeys;   // P over S
            uint4 km = make_uint4(0u, 0u, 0u, 0u);    // (kMode 2) kept ties, quota tile only
            if (kKB && u == jstar) km = *reinterpret_cast<const uint4 *>(smem + C::OFF_KM + f * 16);
            ld(kidx, 1, rb);
            chunk2(u, 0, slow, ra, pk, rl);
            if (quota_tile) drop_ties(ra, pk, rl);
            if (kKB) set_kept(km.x, pk);
            tc::tmem_st16(pcol, pk);                  // S columns 0-15 are already read
            tc::tmem_wait_ld(rb);
            ld(kidx, 2, ra);
            chunk2(u, 1, slow, rb, pk, rl);
            if (quota_tile) drop_ties(rb, pk, rl);
            if (kKB) set_kept(km.y, pk);
            tc::tmem_st16(pcol + 16, pk);
            tc::tmem_wait_ld(ra);
            ld(kidx, 3, rb);
            chunk2(u, 2, slow, ra, pk, rl);
            if (quota_tile) drop_ties(ra, pk, rl);
            if (kKB) set_kept(km.z, pk);
            tc::tmem_st16(pcol + 32, pk);
            tc::tmem_wait_ld(rb);
            // The next tile's first chunk is loaded here only if its S is
            // already in, else after this P is released: releasing P never
            // waits for the next S (whose slot may wait on the P V of the
            // other query tile's last P).
            const bool more = u + 1 < T;
            const bool early = more && __all_sync(kFullMask, tc::mbar_test_wait(
                                                                 s_full + (kidx + QT) % kSlots,
                                                                 ((kidx + QT) / kSlots) & 1));
            if (early) {
                tc::fence_after_sync();
                ld(kidx + QT, 0, ra);
            }
            chunk2(u, 3, slow, rb, pk, rl);
            if (quota_tile) drop_ties(rb, pk, rl);
            if (kKB) set_kept(km.w, pk);
            if (!stash_ok) rem = rl;
            tc::tmem_st16(pcol + 48, pk);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(p_full + g * kSlots + kidx % kSlots);
            if (more && !early) {
                ok = wait_s(kidx + QT);
                if (ok) ld(kidx + QT, 0, ra);
            }
            if (more && ok) tc::tmem_wait_ld(ra);
        };
        if (ok) ok = wait_s(g);
        if (ok) {
            ld(g, 0, ra);
            tc::tmem_wait_ld(ra);
        }
#pragma unroll 1
        for (int u = 0; u < T_full && ok; ++u) p2_tile(u, false);
        if (ok && T > T_full) p2_tile(T - 1, true);
        float Z = (zacc[0] + zacc[1]) + (zacc[2] + zacc[3]);
#pragma unroll
        for (int i = 0; i < 2; ++i)
            Z += __uint_as_float((uint32_t)zpair[i]) + __uint_as_float((uint32_t)(zpair[i] >> 32));

        Z -= zdrop;                                   // ties the pass-2 quota masks dropped

        // ---------------------------------------------------------- quota tile
        // (mode for many key tiles) The kstar kept ties of tile jstar are its
        // first keys at level t in key order (level = Hamming distance of the
        // packed signs); they add w_t V_j to the output and w_t each to Z.
        // The 32 rows of a warp are served together so that every global load
        // is coalesced: the sign words of one row's quota tile (lane = key
        // within a 32-key word), then one value row per kept key (lane =
        // column pair).
        const bool has_quota = ok && jstar >= 0 && active && !kQ2;
        const float wq = has_quota ? ex2(p.c2 * (float)(D - 2 * t - ref)) : 0.0f;
        if (has_quota) Z += wq * (float)zq;
        if (!(Z > 0.0f)) Z = 1.0f;                    // missed or inactive rows only
        constexpr int DW = D / 32;                    // sign words per key
        uint32_t keep[4] = {0u, 0u, 0u, 0u};          // bit i of word c: key 32 c + i of tile jstar
        const uint32_t qlanes = kKB ? 0u : __ballot_sync(kFullMask, has_quota);   // kMode 2: set in P
        if (qlanes) {
            uint32_t qw[DW];
#pragma unroll
            for (int w = 0; w < DW; ++w)
                qw[w] = has_quota ? __ldg(p.qbits + ((head * p.n) + row) * DW + w) : 0u;
            const uint32_t *kbh = p.kbits + head * p.n * (long long)DW;
            constexpr int LPR = D == 64 ? 8 : 4;      // rows per round, their loads in flight together
            uint32_t todo = qlanes;
            while (todo) {                            // warp-uniform
                int Ls[LPR];
#pragma unroll
                for (int e = 0; e < LPR; ++e) {
                    Ls[e] = todo ? __ffs(todo) - 1 : -1;
                    todo &= todo - 1u;
                }
                uint32_t kw[LPR][4][DW];
#pragma unroll
                for (int e = 0; e < LPR; ++e) {
                    const int jl = __shfl_sync(kFullMask, jstar, max(Ls[e], 0));
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const long long key = min(jl * kKeys + 32 * k + lane, p.n - 1);
                        if (DW == 2) {
                            const uint2 x = __ldg(reinterpret_cast<const uint2 *>(kbh + key * DW));
                            kw[e][k][0] = x.x;
                            kw[e][k][DW - 1] = x.y;
                        } else {
                            const uint4 x = __ldg(reinterpret_cast<const uint4 *>(kbh + key * DW));
                            kw[e][k][0] = x.x;
                            kw[e][k][1 % DW] = x.y;
                            kw[e][k][2 % DW] = x.z;
                            kw[e][k][3 % DW] = x.w;
                        }
                    }
                }
#pragma unroll
                for (int e = 0; e < LPR; ++e) {
                    const int L = Ls[e];
                    if (L < 0) break;
                    const int jl = __shfl_sync(kFullMask, jstar, L);
                    const int tl = __shfl_sync(kFullMask, t, L);
                    uint32_t ql[DW];
#pragma unroll
                    for (int w = 0; w < DW; ++w) ql[w] = __shfl_sync(kFullMask, qw[w], L);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        int ham = 0;
#pragma unroll
                        for (int w = 0; w < DW; ++w) ham += __popc(ql[w] ^ kw[e][k][w]);
                        const bool tie = ham == tl && jl * kKeys + 32 * k + lane < p.n;
                        const uint32_t bits = __ballot_sync(kFullMask, tie);
                        if (lane == L) keep[k] = bits;
                    }
                }
            }
            // the first kstar of the ties
            int need = has_quota ? kstar : 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int cnt = __popc(keep[k]);
                if (need <= 0) {
                    keep[k] = 0u;
                } else if (cnt > need) {
                    const int cut = __fns(keep[k], 0, need + 1);   // position of tie need + 1
                    keep[k] &= (1u << cut) - 1u;
                    need = 0;
                } else {
                    need -= cnt;
                }
            }
        }

        // output: (O 2^e_h + w_t sum of the quota tile's kept V) / Z, in
        // halves of 64 columns.  Lane i loads columns 2i, 2i+1 of the half
        // from each kept value row and adds them to that row's sums, kept in
        // this warp's own bytes of the weight table (which pass 2 no longer
        // reads): row L, pair p sits in bin 2L + p / 16 at pair slot
        // (p ^ L) mod 16, so that both the writes and the reads spread over
        // the banks.
        const float scale = ok ? ldexpf(1.0f, p.vexp[head]) / Z : 0.0f;
        const float qscale = wq / Z;
        float *orow = p.out + ((head * p.n) + row) * (long long)D;
        uint8_t *vt_base = smem + C::OFF_TAB + g * C::TAB_BYTES + quarter * 128;
        auto vslot = [&](int L, int pr) -> float2 * {
            return reinterpret_cast<float2 *>(vt_base + (2 * L + pr / 16) * (kRows * 4) +
                                              ((pr ^ L) & 15) * 8);
        };
        // The warp's kept (row, key) pairs, numbered in lane order (lane L's
        // are off_L .. off_L + kstar_L - 1, in key order), are listed in this
        // warp's bytes of its query tile's Q (free once pass 2's Q K^T MMAs
        // are done) and gathered sixteen value rows at a time.
        const int nkeep = __popc(keep[0]) + __popc(keep[1]) + __popc(keep[2]) + __popc(keep[3]);
        int off = nkeep;
#pragma unroll
        for (int dd = 1; dd < 32; dd <<= 1) {
            const int y = __shfl_up_sync(kFullMask, off, dd);
            if (lane >= dd) off += y;
        }
        const int total = __shfl_sync(kFullMask, off, 31);
        off -= nkeep;
        constexpr int kListCap = 8 * D;               // 32 rows x D bytes of Q
        uint32_t *list = reinterpret_cast<uint32_t *>(smem + C::OFF_Q + g * C::QBYTES +
                                                      quarter * 32 * D);
#pragma unroll 1
        for (int h = 0; h < D / 64 && ok; ++h) {
            float vq[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) vq[c] = 0.0f;
            if (total > 0) {
#pragma unroll
                for (int L = 0; L < 32; ++L) *vslot(L, lane) = make_float2(0.0f, 0.0f);
                const long long col = 64 * h + 2 * lane;
                for (int w0 = 0; w0 < total; w0 += kListCap) {
                    const int w1 = min(total, w0 + kListCap);
                    // this lane's pairs in the window, in key order
                    __syncwarp();
                    int idx = off;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        for (uint32_t m = keep[k]; m != 0u && idx < w1; m &= m - 1u, ++idx)
                            if (idx >= w0)
                                list[idx - w0] = ((uint32_t)lane << 24) |
                                                 (uint32_t)(jstar * kKeys + 32 * k + __ffs(m) - 1);
                    }
                    __syncwarp();
                    // KV value rows per step, all loads issued before any is used
                    // (the entries past the list load row 0 and add nothing)
                    constexpr int KV = 32;
                    auto add = [&](const uint32_t (&ent)[KV], const float2 (&x)[KV], int b0) {
#pragma unroll
                        for (int e = 0; e < KV; ++e)
                            if (b0 + e < w1) {
                                float2 *sl = vslot((int)(ent[e] >> 24), lane);
                                float2 y = *sl;
                                y.x += x[e].x;
                                y.y += x[e].y;
                                *sl = y;
                            }
                    };
                    for (int b0 = w0; b0 < w1; b0 += KV) {
                        uint32_t ent[KV];
                        float2 x[KV];
#pragma unroll
                        for (int e = 0; e < KV; ++e)
                            ent[e] = b0 + e < w1 ? list[b0 + e - w0] : 0u;
                        if (p.v_f32) {
                            const float *vb = static_cast<const float *>(p.v) + col;
#pragma unroll
                            for (int e = 0; e < KV; ++e)
                                x[e] = __ldg(reinterpret_cast<const float2 *>(
                                    vb + ((head * p.n) + (ent[e] & 0xFFFFFFu)) * (long long)D));
                        } else {
                            const uint16_t *vb = static_cast<const uint16_t *>(p.v) + col;
                            uint32_t b2[KV];
#pragma unroll
                            for (int e = 0; e < KV; ++e)
                                b2[e] = __ldg(reinterpret_cast<const uint32_t *>(
                                    vb + ((head * p.n) + (ent[e] & 0xFFFFFFu)) * (long long)D));
#pragma unroll
                            for (int e = 0; e < KV; ++e)
                                x[e] = make_float2(__uint_as_float(b2[e] << 16),
                                                   __uint_as_float(b2[e] & 0xFFFF0000u));
                        }
                        add(ent, x, b0);
                    }
                }
                __syncwarp();
#pragma unroll
                for (int pr = 0; pr < 32; ++pr) {
                    const float2 v2 = *vslot(lane, pr);
                    vq[2 * pr] = v2.x;
                    vq[2 * pr + 1] = v2.y;
                }
                __syncwarp();
            }
            if (h == 0) {
                ok = __all_sync(kFullMask,
                                wait_bar(o_full + g, 0, deadline, abort_flag, p.status));
                if (!ok) break;
                tc::fence_after_sync();
            }
#pragma unroll
            for (int c1 = 0; c1 < 64; c1 += 32) {
                const int c0 = 64 * h + c1;
                uint32_t o[32];
                tc::tmem_ld32(lane_base + C::O_COL + g * D + c0, o);
                tc::tmem_wait_ld(o);
                if (active) {
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        float4 v = make_float4(
                            fmaf(__uint_as_float(o[c]), scale, vq[c1 + c] * qscale),
                            fmaf(__uint_as_float(o[c + 1]), scale, vq[c1 + c + 1] * qscale),
                            fmaf(__uint_as_float(o[c + 2]), scale, vq[c1 + c + 2] * qscale),
                            fmaf(__uint_as_float(o[c + 3]), scale, vq[c1 + c + 3] * qscale));
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
