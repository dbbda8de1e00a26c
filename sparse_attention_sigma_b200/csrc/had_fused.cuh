// had_fused.cuh -- the fused binarized top-N attention forward on the sm_100a
// tensor cores ("Hamming Attention Distillation", pith.science review, "What
// carries the argument": sign-quantized Q/K, Hamming logits, top-N mask,
// softmax over the kept logits, value product; Eqs. 4-7).
//
// A CTA owns QT tiles of 128 query rows of one head (TMEM lane i = row i of
// a tile) and streams the head's keys in tiles of 64, twice:
//   pass 1  S = Q K^T on the tensor core (+/-4 x -/+1 int8 operands, Q
//           negated, so the s32 accumulator holds -4 s); each epilogue
//           thread reads its row.
//           The first key tiles are counted exactly into a per-row histogram
//           of the d+1 logit levels (shared memory); it places a window of
//           three levels around the row's threshold, and the remaining tiles
//           only update four 8-bit cumulative counters packed in one
//           register (one shifted add per logit).  That yields the exact
//           threshold level t and the number q of keys kept at it whenever t
//           falls inside the window; rows where it does not are listed and
//           recomputed exactly by fixup_rows_kernel.  Each tile's counter
//           word is also kept in TMEM, so the row knows in which tile its
//           tie quota runs out.
//   pass 2  S again (Q now +/-64: the accumulator holds 256 s, a byte
//           offset into the row's weight table); the thread turns its row
//           into P = exp(tau (s - ref)) for logits above the threshold and
//           for the first q logits at it (ascending key index: the lower
//           index wins the tie), 0 elsewhere, sums them into Z, packs P to
//           fp16 pairs in TMEM, and the tensor core accumulates O += P V
//           (fp16 operands, f32 accumulate).  Only the sampled tiles and the
//           tile where some row's quota runs out count ties key by key; in
//           every other tile one table load gives a key's weight.
// The n x n logits never leave the SM.
//
// Warp roles: warp 0 bulk-copies Q once and K (twice) / V (once) tiles into
// shared-memory rings; warp 1 issues every MMA from one thread; warps
// 2 .. 2+4*QT-1 are the epilogue, one query row per thread, four warps per
// query tile.  The QT tiles share every K and V tile.  Each query tile has
// three S buffers in TMEM, so the QK^T of a tile is issued about one and a
// half tiles before the epilogue reads it; in pass 2 the tile's P is written
// over the first half of its own S, and the P V that reads it frees the
// buffer for the next QK^T in the MMA thread's (in-order) stream.  Every
// wait is bounded by a deadline: a CTA that hits it flags HAD_ERR_TIMEOUT,
// lets its copies and MMAs drain, frees its TMEM and returns.
#pragma once
#include <cuda_fp16.h>
#include <type_traits>

#include "had_common.cuh"
#include "had_prep.cuh"
#include "had_tc.cuh"

namespace had {
namespace fused {

constexpr int kRows = 128;
constexpr int kKeys = 64;
constexpr uint64_t kWaitNs = 2000000000ull;         // 2 s: far beyond any real wait
constexpr int kMagic = 0x4B400000;                  // bits of 1.5 * 2^23

template <int D>
struct Cfg {
    static constexpr int QT = D == 64 ? 2 : 1;            // query tiles per CTA
    // warp 0 producer, warp 1 MMA issuer of query tile 0, warps 2 .. 1+4*QT
    // epilogue, warp 2+4*QT MMA issuer of query tile 1 (QT = 2)
    static constexpr int THREADS = 32 * (2 + 4 * QT + (QT - 1));
    static constexpr int QBYTES = kRows * D;              // int8 Q tile
    static constexpr int KBYTES = kKeys * D;              // int8 K tile
    static constexpr int VBYTES = D * kKeys * 2;          // fp16 V^T tile
    // K and V move in groups of consecutive tiles, 16 KB per bulk copy: a
    // cp.async.bulk costs an SM about the same time whatever its size up to
    // 16 KB, so few large copies keep the operand stream off the critical
    // path.  Rings of KGROUPS / VGROUPS groups; one commit frees a group.
    static constexpr int GK = 16384 / KBYTES;             // K tiles per copy
    static constexpr int GV = 16384 / VBYTES;             // V tiles per copy
    static constexpr int KGROUPS = 3;
    static constexpr int VGROUPS = 3;
    static constexpr int KSTAGES = KGROUPS * GK;          // K tile slots
    static constexpr int VSTAGES = VGROUPS * GV;          // V tile slots
    static constexpr int SBUF = 3;                        // S buffers per query tile
    static constexpr int BINS = D + 1;
    static constexpr int HIST_BYTES = BINS * kRows * 4;   // per query tile
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t GROUP_COLS = 256;           // TMEM columns per query tile
    // S of key tile u in buffer u % SBUF (s32, 64 columns); in pass 2 the
    // tile's P (fp16 pairs, 32 columns) overwrites the first half of its S.
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t O_COL = SBUF * 64;          // f32, D columns
    // pass 1 only: one word of window counts per key tile, in the O columns
    // (unused until the first P V)
    static constexpr uint32_t STASH_COL = O_COL;
    static constexpr int STASH_CAP = D;
    static_assert(QT * GROUP_COLS <= TMEM_COLS || QT == 1, "TMEM budget");
    static_assert(O_COL + D <= (QT == 1 ? TMEM_COLS : GROUP_COLS), "TMEM budget");
    // shared memory layout (offsets from a 1024-aligned base)
    static constexpr int OFF_Q = 0;                       // Q as +/-1 (pass 1)
    static constexpr int OFF_Q2 = OFF_Q + QT * QBYTES;     // Q as +/-64 (pass 2)
    static constexpr int OFF_K = OFF_Q2 + QT * QBYTES;
    static constexpr int OFF_V = OFF_K + KSTAGES * KBYTES;
    static constexpr int OFF_HIST = OFF_V + VSTAGES * VBYTES;
    static constexpr int OFF_BAR = OFF_HIST + QT * HIST_BYTES;
    static constexpr int NBARS = 1 + 2 * KGROUPS + 2 * VGROUPS + QT * (3 * SBUF + 2);
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + alignment slack
    static constexpr uint32_t IDESC_QK = tc::idesc(2, 1, 1, kRows, kKeys);   // s32 <- s8 x s8
    static constexpr uint32_t IDESC_PV = tc::idesc(1, 0, 0, kRows, D);       // f32 <- f16 x f16
};

struct Params {
    const int8_t *qop;        // [BH][qtiles] 128 x D int8 tiles (-/+1: the negated signs)
    const int8_t *qop2;       // [BH][qtiles] 128 x D int8 tiles (+/-64)
    const int8_t *kop;        // [BH][ktiles] 64 x D int8 tiles (+/-4)
    const __half *vop;        // [BH][ktiles] D x 64 fp16 tiles (V^T, scaled)
    const int *vexp;          // [BH] power of two of the V scale
    float *out;               // [BH][n][D]
    int32_t *dbg_idx;         // [BH][n][N] or null
    int16_t *dbg_logits;      // [BH][n][N] or null
    int32_t *status;
    int *miss_count;          // rows whose threshold fell outside the window
    int *miss_rows;           // their flat row ids (head * n + row)
    long long miss_cap;       // entries of miss_rows (every row of the grid)
    int sample_tiles;         // key tiles counted exactly before the window
    int n, N;
    int qtiles;               // query tiles per head in qop (a multiple of QT)
    int ktiles;               // 64-key tiles holding keys (ceil(n / 64))
    int kstride;              // 64-key tiles per head in kop / vop (ktiles rounded up)
    int ctas_per_head;
    float c2;                 // tau * log2(e)
};

struct Bars {
    uint64_t *q_full;
    uint64_t *k_full, *k_empty;     // [KGROUPS]
    uint64_t *v_full, *v_empty;     // [VGROUPS]
    // per query tile g (each has its own MMA issuer):
    // s_full[SBUF] s_empty[SBUF] p_full[SBUF] o_full drain
    uint64_t *grp;
    __device__ uint64_t *s_full(int g, int b) const { return grp + 11 * g + b; }
    __device__ uint64_t *s_empty(int g, int b) const { return grp + 11 * g + 3 + b; }
    __device__ uint64_t *p_full(int g, int b) const { return grp + 11 * g + 6 + b; }
    __device__ uint64_t *o_full(int g) const { return grp + 11 * g + 9; }
    __device__ uint64_t *drain(int g) const { return grp + 11 * g + 10; }
};

// Bounded wait: false if the deadline passed or another role aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, uint64_t deadline,
                                         volatile int *abort_flag, int32_t *status)
{
    uint32_t spins = 0;
    while (!tc::mbar_try_wait(bar, parity)) {
        if ((++spins & 255u) == 0) {
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

__device__ __forceinline__ void red_add1(uint32_t saddr)
{
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(saddr), "r"(1u) : "memory");
}

__device__ __forceinline__ float lds_f32(uint32_t saddr)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(saddr) : "memory");
    return v;
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Weight of an accumulator value v (a multiple of the logit):
// exp2(k1 * (v - ref)) evaluated as exp2(k1 * float(1.5*2^23 + v) + k0) with
// k0 = -k1 * (ref + 1.5*2^23); the int -> float step is exact and costs one
// integer add.
__device__ __forceinline__ float weight_of(int v, float k1, float k0)
{
    return ex2(fmaf(__int_as_float(v + kMagic), k1, k0));
}

// Increment of the four cumulative 8-bit window counters for a logit whose
// counter index is amount / 8 (amount <= 0: every counter; >= 32: none).
// shl.b32 clamps shift amounts above 32, which gives the "none" case.
__device__ __forceinline__ uint32_t window_inc(int amount)
{
    uint32_t r;
    asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(0x01010101u), "r"((uint32_t)max(amount, 0)));
    return r;
}

template <int D, bool kDbg, bool kCausal = false>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1)
attention_fwd_kernel(const Params p)
{
    using C = Cfg<D>;
    constexpr int QT = C::QT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    Bars b;
    b.q_full = bar;
    b.k_full = bar + 1;
    b.k_empty = b.k_full + C::KGROUPS;
    b.v_full = b.k_empty + C::KGROUPS;
    b.v_empty = b.v_full + C::VGROUPS;
    b.grp = b.v_empty + C::VGROUPS;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long head = blockIdx.x / p.ctas_per_head;
    // Causal: the CTAs of a head run from its last query tiles (the most
    // keys) to its first, and each streams keys only up to its last row.
    // Every role derives T from blockIdx alone, so all agree on it.
    const int cta_in_head = blockIdx.x % p.ctas_per_head;
    const int qtile0 = (kCausal ? p.ctas_per_head - 1 - cta_in_head : cta_in_head) * QT;
    const int T = kCausal ? min(p.ktiles, ((qtile0 + QT) * kRows + kKeys - 1) / kKeys)
                          : p.ktiles;
    const uint64_t deadline = tc::globaltimer_ns() + kWaitNs;

    if (threadIdx.x == 0) {
        tc::mbar_init(b.q_full, 1);
        for (int s = 0; s < C::KGROUPS; ++s) {
            tc::mbar_init(b.k_full + s, 1);
            tc::mbar_init(b.k_empty + s, QT);             // one commit per MMA issuer
        }
        for (int s = 0; s < C::VGROUPS; ++s) {
            tc::mbar_init(b.v_full + s, 1);
            tc::mbar_init(b.v_empty + s, QT);
        }
        for (int g = 0; g < QT; ++g) {
            for (int s = 0; s < C::SBUF; ++s) {
                tc::mbar_init(b.s_full(g, s), 1);
                tc::mbar_init(b.s_empty(g, s), 4);      // one arrive per epilogue warp
                tc::mbar_init(b.p_full(g, s), 4);
            }
            tc::mbar_init(b.o_full(g), 1);
            tc::mbar_init(b.drain(g), 1);
        }
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
            const int8_t *ksrc = p.kop + head * (long long)p.kstride * C::KBYTES;
            const uint8_t *vsrc = reinterpret_cast<const uint8_t *>(p.vop) +
                                  head * (long long)p.kstride * C::VBYTES;
            const int8_t *qsrc2 = p.qop2 + (head * p.qtiles + qtile0) * (long long)C::QBYTES;
            tc::mbar_expect_tx(b.q_full, 2 * QT * C::QBYTES);
            tc::bulk_g2s(smem + C::OFF_Q, qsrc, QT * C::QBYTES, b.q_full);
            tc::bulk_g2s(smem + C::OFF_Q2, qsrc2, QT * C::QBYTES, b.q_full);
            // Group G of the K stream holds key tiles GK*q .. of pass G / nkg
            // (q = G % nkg); V group H holds key tiles GV*H .. (pass 2 only).
            const int nkg = (T + C::GK - 1) / C::GK;
            int issued_k = 0, issued_v = 0;
            bool ok = true;
            auto load_v = [&](int H) -> bool {
                const int vs = H % C::VGROUPS;
                if (!wait_bar(b.v_empty + vs, ((H / C::VGROUPS) & 1) ^ 1, deadline, abort_flag,
                              p.status))
                    return false;
                const int cnt = min(C::GV, T - H * C::GV);
                tc::mbar_expect_tx(b.v_full + vs, cnt * C::VBYTES);
                tc::bulk_g2s(smem + C::OFF_V + vs * C::GV * C::VBYTES,
                             vsrc + (long long)H * C::GV * C::VBYTES, cnt * C::VBYTES,
                             b.v_full + vs);
                issued_v = H + 1;
                return true;
            };
            for (int G = 0; G < 2 * nkg && ok; ++G) {
                const int pass = G / nkg, q = G % nkg;
                const int ks = G % C::KGROUPS;
                ok = wait_bar(b.k_empty + ks, ((G / C::KGROUPS) & 1) ^ 1, deadline, abort_flag,
                              p.status);
                if (!ok) break;
                const int cnt = min(C::GK, T - q * C::GK);
                tc::mbar_expect_tx(b.k_full + ks, cnt * C::KBYTES);
                tc::bulk_g2s(smem + C::OFF_K + ks * C::GK * C::KBYTES,
                             ksrc + (long long)q * C::GK * C::KBYTES, cnt * C::KBYTES,
                             b.k_full + ks);
                issued_k = G + 1;
                // pass 2: the V groups of these key tiles follow their K group
                if (pass == 1) {
                    const int hend = (q * C::GK + cnt + C::GV - 1) / C::GV;
                    for (int H = issued_v; H < hend && ok; ++H) ok = load_v(H);
                }
            }
            if (!ok) {
                // let every copy already in flight land before the CTA exits
                const uint64_t drain_deadline = tc::globaltimer_ns() + kWaitNs / 4;
                volatile int never = 0;
                wait_bar(b.q_full, 0, drain_deadline, &never, p.status);
                for (int G = (issued_k > C::KGROUPS ? issued_k - C::KGROUPS : 0); G < issued_k; ++G)
                    wait_bar(b.k_full + G % C::KGROUPS, (G / C::KGROUPS) & 1, drain_deadline,
                             &never, p.status);
                for (int H = (issued_v > C::VGROUPS ? issued_v - C::VGROUPS : 0); H < issued_v; ++H)
                    wait_bar(b.v_full + H % C::VGROUPS, (H / C::VGROUPS) & 1, drain_deadline,
                             &never, p.status);
            }
        }
    } else if (warp == 1 || warp == 2 + 4 * QT) {
        // ------------------------------------------------------------ MMA issuers
        // One thread per query tile g issues that tile's MMAs; the two
        // issuers share only the K and V rings (each commits once per group).
        if (lane == 0) {
            const int g = warp == 1 ? 0 : 1;
            // Descriptors are computed once; a tile or K step moves only the
            // start-address field (bits 0-13, in 16-byte units).
            const uint64_t dq1 =
                tc::smem_desc(tc::smem_u32(smem + C::OFF_Q + g * C::QBYTES), 128, D * 8);
            const uint64_t dq2 =
                tc::smem_desc(tc::smem_u32(smem + C::OFF_Q2 + g * C::QBYTES), 128, D * 8);
            const uint64_t dk = tc::smem_desc(tc::smem_u32(smem + C::OFF_K), 128, D * 8);
            const uint64_t dv = tc::smem_desc(tc::smem_u32(smem + C::OFF_V), 128, 8 * 128);
            const uint32_t gcol = g * C::GROUP_COLS;
            bool ok = wait_bar(b.q_full, 0, deadline, abort_flag, p.status);
            tc::fence_after_sync();
            const int nkg = (T + C::GK - 1) / C::GK;
            // O += P V for pass-2 key tile j; P sits in the S buffer of tile
            // T + j.  The V group's barrier is waited for at its first tile.
            auto pv = [&](int j) -> bool {
                const int H = j / C::GV;
                const int vg = H % C::VGROUPS;
                const int vs = vg * C::GV + j % C::GV;        // tile slot in the V ring
                if ((j % C::GV == 0 &&
                     !wait_bar(b.v_full + vg, (H / C::VGROUPS) & 1, deadline, abort_flag,
                               p.status)) ||
                    !wait_bar(b.p_full(g, j % C::SBUF), (j / C::SBUF) & 1, deadline, abort_flag,
                              p.status))
                    return false;
                tc::fence_after_sync();
                const uint64_t dvs = dv + (uint64_t)((vs * C::VBYTES) >> 4);
                const uint32_t pcol = C::S_COL + ((T + j) % C::SBUF) * 64;
#pragma unroll
                for (int kk = 0; kk < kKeys / 16; ++kk)
                    tc::mma_f16_ts(tmem + gcol + C::O_COL, tmem + gcol + pcol + kk * 8,
                                   dvs + (uint64_t)(kk * 16), C::IDESC_PV,
                                   (j > 0 || kk > 0) ? 1u : 0u);
                if (j % C::GV == C::GV - 1 || j == T - 1) tc::mma_commit(b.v_empty + vg);
                return true;
            };
            // S = Q K^T for key tile u of the stream (pass 1: u < T).  Its
            // buffer u % SBUF last held tile u - SBUF: a pass-1 tile is given
            // back by the epilogue (s_empty); a pass-2 tile is free once the
            // P V that read its P is issued, which happens earlier in this
            // thread's (in-order) stream.  The K group's barrier is waited
            // for at its first tile.
            auto qk = [&](int u) -> bool {
                const int jt = u < T ? u : u - T;             // key tile
                const int G = (u < T ? 0 : nkg) + jt / C::GK;  // its K group
                const int kg = G % C::KGROUPS;
                const int ks = kg * C::GK + jt % C::GK;         // tile slot in the K ring
                const int sb = u % C::SBUF;
                const int prev = u - C::SBUF;
                if (jt % C::GK == 0 &&
                    !wait_bar(b.k_full + kg, (G / C::KGROUPS) & 1, deadline, abort_flag, p.status))
                    return false;
                if (prev >= 0 && prev < T &&
                    !wait_bar(b.s_empty(g, sb), (prev / C::SBUF) & 1, deadline, abort_flag,
                              p.status))
                    return false;
                tc::fence_after_sync();
                const uint64_t dks = dk + (uint64_t)((ks * C::KBYTES) >> 4);
                const uint64_t dqp = u < T ? dq1 : dq2;
                const uint32_t scol = gcol + C::S_COL + sb * 64;
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk)
                    tc::mma_i8_ss(tmem + scol, dqp + (uint64_t)(kk * 16), dks + (uint64_t)(kk * 16),
                                  C::IDESC_QK, kk > 0 ? 1u : 0u);
                tc::mma_commit(b.s_full(g, sb));
                if (jt % C::GK == C::GK - 1 || jt == T - 1) tc::mma_commit(b.k_empty + kg);
                return true;
            };
            // Pass 1, then the first SBUF tiles of pass 2; after that each
            // P V frees the buffer for the QK^T SBUF tiles ahead.
            for (int u = 0; u < T && ok; ++u) ok = qk(u);
            for (int u = T; u < T + min(T, C::SBUF) && ok; ++u) ok = qk(u);
            for (int j = 0; j < T && ok; ++j) {
                ok = pv(j);
                if (ok && j + C::SBUF < T) ok = qk(T + j + C::SBUF);
            }
            if (ok) tc::mma_commit(b.o_full(g));
            // drain: wait until every MMA this thread issued has completed
            tc::mma_commit(b.drain(g));
            volatile int never = 0;
            wait_bar(b.drain(g), 0, tc::globaltimer_ns() + kWaitNs / 4, &never, p.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int g = (warp - 2) >> 2;                // query tile of this warp
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter ...
        const int r = quarter * 32 + lane;            // row within the tile
        const int row = (qtile0 + g) * kRows + r;     // query index within the head
        const bool active = row < p.n;
        // keys this row sees and keeps: all n and N, or (causal) keys 0..row
        // and min(N, row + 1)
        const int vis = kCausal ? min(p.n, row + 1) : p.n;
        const int Nr = min(p.N, vis);
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + g * C::GROUP_COLS;
        uint32_t *hist = reinterpret_cast<uint32_t *>(smem + C::OFF_HIST + g * C::HIST_BYTES);
        uint32_t *hcol = hist + r;                    // hist[bin][r] at hcol[bin * kRows]
        for (int bin = 0; bin < C::BINS; ++bin) hcol[bin * kRows] = 0;
        // The pass-1 accumulator holds v = -4 s.  The level of a logit is its
        // Hamming distance (D - s)/2; its histogram bin sits (D - s) * 256
        // bytes = 256 D + 64 v past this row's bin 0, and its counter shift
        // is cshift + v.
        const uint32_t hbase = tc::smem_u32(hcol) + 256u * D;
        const int A = min(T, p.sample_tiles);         // tiles counted exactly
        // Pass 1 keeps one word of window counts per key tile in the TMEM
        // columns that P and O only use in pass 2; from it each row learns
        // the one tile where its tie quota runs out, and every other tile of
        // pass 2 needs no per-key tie bookkeeping.
        const bool stash_ok = !kDbg && T - A <= C::STASH_CAP;
        const int fast_from = stash_ok ? A : T;
        bool ok = true;
        using BT = std::integral_constant<bool, true>;
        using BF = std::integral_constant<bool, false>;

        // Each S tile is read in two halves of 32 columns; the load of the
        // next half is in flight while the current one is processed.
        uint32_t sa[32], sb[32];
        auto ld_half = [&](int u, int h, uint32_t (&rr)[32]) {
            tc::tmem_ld32(lane_base + C::S_COL + (u % C::SBUF) * 64 + h * 32, rr);
        };
        auto wait_s = [&](int u) -> bool {
            const bool w = __all_sync(kFullMask, wait_bar(b.s_full(g, u % C::SBUF),
                                                          (u / C::SBUF) & 1, deadline, abort_flag,
                                                          p.status));
            tc::fence_after_sync();
            return w;
        };
        auto release_s = [&](int u) {
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(b.s_empty(g, u % C::SBUF));
        };
        auto half_valid = [&](int j, int h) { return min(32, vis - j * kKeys - h * 32); };

        // pass 1a: exact histogram of the first A key tiles
        auto hist_half = [&](const uint32_t (&rr)[32], auto full, int valid) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
                if (decltype(full)::value || c < valid) red_add1(hbase + (rr[c] << 6));
        };
        // pass 1b: four cumulative 8-bit window counters in one register;
        // four independent counter registers keep the adds off one chain
        uint32_t acc[4] = {0u, 0u, 0u, 0u};
        uint32_t run = 0u;                            // sum of up to three tile words
        int tot0 = 0, tot1 = 0, tot2 = 0, tot3 = 0;
        int cshift = 0, L0 = 0, hmin = C::BINS - 1;
        auto flush = [&]() {
            tot0 += (int)(run & 0xFFu);
            tot1 += (int)((run >> 8) & 0xFFu);
            tot2 += (int)((run >> 16) & 0xFFu);
            tot3 += (int)(run >> 24);
            run = 0u;
        };
        auto window_half = [&](const uint32_t (&rr)[32], auto full, int valid) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
                if (decltype(full)::value || c < valid)
                    acc[c & 3] += window_inc(cshift + (int)rr[c]);
        };
        // Window from the sample: est = the level of the sample's
        // (N * sampled / n)-th best key.  Levels L0 = est - 1 .. est + 1 are
        // resolved exactly; the rest of the row updates four cumulative
        // counters f_k = #{level <= L0 - 1 + k}, k = 0..3.
        auto place_window = [&]() {
            const int sampled = min(vis, A * kKeys);
            const int ns = max(1, (int)(((long long)Nr * sampled + vis / 2) / vis));
            int cum = 0, est = C::BINS - 1;
            bool seen = false, found = false;
            for (int bin = 0; bin < C::BINS; ++bin) {
                const int c = (int)hcol[bin * kRows];
                if (!seen && c) { hmin = bin; seen = true; }
                cum += c;
                if (!found && cum >= ns) { est = bin; found = true; }
            }
            L0 = est - 1;
            cshift = 4 * D - 8 * L0 + 8;              // 8 * (level - L0 + 1) = cshift + v
        };
        auto pass1_half = [&](int j, int h, const uint32_t (&rr)[32]) {
            const int valid = half_valid(j, h);
            if (j < A) {
                if (valid >= 32) hist_half(rr, BT{}, 32);
                else hist_half(rr, BF{}, valid);
            } else {
                if (valid >= 32) window_half(rr, BT{}, 32);
                else window_half(rr, BF{}, valid);
            }
            // causal: valid differs from lane to lane, so the lanes meet
            // again before the next warp-wide TMEM access
            if constexpr (kCausal) __syncwarp();
        };
        auto pass1_end_tile = [&](int j) {
            if (j == A - 1) place_window();
            if (j >= A) {
                const uint32_t w = (acc[0] + acc[1]) + (acc[2] + acc[3]);   // fields <= 64
                acc[0] = acc[1] = acc[2] = acc[3] = 0u;
                run += w;
                if ((j - A) % 3 == 2) flush();        // fields stay below 3 * 64 < 256
                if (stash_ok) tc::tmem_st1(lane_base + C::STASH_COL + (j - A), w);
            }
        };
        ok = wait_s(0);
        if (ok) {
            ld_half(0, 0, sa);
            tc::tmem_wait_ld(sa);
        }
        for (int j = 0; j < T && ok; ++j) {
            ld_half(j, 1, sb);
            pass1_half(j, 0, sa);
            tc::tmem_wait_ld(sb);
            release_s(j);
            const bool more = j + 1 < T;
            if (more) {
                ok = wait_s(j + 1);
                if (ok) ld_half(j + 1, 0, sa);
            }
            pass1_half(j, 1, sb);
            pass1_end_tile(j);
            if (more && ok) tc::tmem_wait_ld(sa);
        }
        flush();

        // threshold level t and the number q of keys kept at it
        int t = -1, quota = 0;
        bool miss = false;
        if (A >= T) {
            int below = 0;
            for (int bin = 0; bin < C::BINS; ++bin) {
                const int c = (int)hcol[bin * kRows];
                if (below + c >= Nr) { t = bin; quota = Nr - below; break; }
                below += c;
            }
        } else {
            int f0 = tot0, f1 = tot1, f2 = tot2, f3 = tot3;
            for (int bin = 0; bin < C::BINS; ++bin) {
                const int c = (int)hcol[bin * kRows];
                if (bin <= L0 - 1) f0 += c;
                if (bin <= L0) f1 += c;
                if (bin <= L0 + 1) f2 += c;
                if (bin <= L0 + 2) f3 += c;
            }
            if (f0 < Nr && f3 >= Nr) {
                if (f1 >= Nr) { t = L0; quota = Nr - f0; }
                else if (f2 >= Nr) { t = L0 + 1; quota = Nr - f1; }
                else { t = L0 + 2; quota = Nr - f2; }
            } else {
                miss = true;
            }
        }
        // Where the tie quota runs out.  The sampled tiles hold the first
        // hist[t] keys at level t; past them, tile words give each tile's
        // count at t.  Ties are kept in full before tile jstar, kstar of them
        // (the lowest indices) inside it, and none after it: from tile
        // zero_at on the weight table maps level t to 0.
        int zero_at = T, jstar = -1, kstar = 0;
        __syncwarp();                                 // lanes left the threshold loops apart
        if (stash_ok && ok && A < T) {
            tc::tmem_wait_st();
            const bool want = t >= 0 && !miss;
            const int ts = t - L0 + 1;                // 1..3: field of level t in a tile word
            const int rem0 = want ? quota - (int)hcol[t * kRows] : 0;
            bool found = !want || rem0 <= 0;
            if (want && rem0 <= 0) zero_at = A;
            int cum = 0;
            for (int c0 = 0; c0 < T - A; c0 += 32) {
                uint32_t w[32];
                tc::tmem_ld32(lane_base + C::STASH_COL + c0, w);
                tc::tmem_wait_ld(w);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int jj = c0 + i;
                    if (!found && jj < T - A) {
                        const int cnt = (int)((w[i] >> (8 * ts)) & 0xFFu) -
                                        (int)((w[i] >> (8 * ts - 8)) & 0xFFu);
                        if (cum + cnt >= rem0) {
                            found = true;
                            zero_at = A + jj + 1;
                            if (rem0 - cum < cnt) { jstar = A + jj; kstar = rem0 - cum; }
                        }
                        cum += cnt;
                    }
                }
            }
            if (!found) miss = true;                  // counts disagree: recompute the row
        }
        if (miss && active) {
            const int slot = atomicAdd(p.miss_count, 1);
            if (slot < p.miss_cap) p.miss_rows[slot] = (int)(head * p.n + row);
        }
        // missed rows keep nothing here; the fix-up kernel rewrites them
        if (miss) { t = -1; quota = 0; zero_at = T; jstar = -1; }
        // Softmax reference: the sample's best logit, raised if needed so that
        // no weight can exceed the fp16 range (s <= D).  The histogram column
        // becomes the row's weight table: level l holds exp2(c2 (s_l - ref))
        // for l <= t and 0 beyond the threshold, so pass 2 reads a logit's
        // weight with one shared load at the same address its histogram bin
        // had.
        {
            const int headroom = p.c2 > 1.0e-6f ? (int)fminf(floorf(15.99f / p.c2), 1.0e6f) : 1000000;
            const int ref = max(D - 2 * hmin, D - headroom);
            for (int bin = 0; bin < C::BINS; ++bin)
                hcol[bin * kRows] =
                    bin <= t ? __float_as_uint(ex2(p.c2 * (float)(D - 2 * bin - ref))) : 0u;
        }
        const uint32_t vt = 256u * (uint32_t)(D - 2 * t);   // accumulator value of the threshold
        int rem = quota;                              // ties still to keep (slow tiles before fast_from)
        int kept = 0;
        float zacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const long long obase = ((head * p.n) + row) * (long long)p.N;
        constexpr int kAll = 1 << 30;

        // pass 2: P = kept weights (fp16) -> TMEM; the MMA warp does O += P V
        // Fast half: the table alone decides (0 beyond the threshold).
        auto fast_half = [&](const uint32_t (&rr)[32], uint32_t (&pk)[16]) {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                const float w0 = lds_f32(hbase - rr[c]);
                const float w1 = lds_f32(hbase - rr[c + 1]);
                zacc[c & 2] += w0;
                zacc[(c & 2) + 1] += w1;
                __half2 h2 = __floats2half2_rn(w0, w1);
                pk[c >> 1] = *reinterpret_cast<uint32_t *>(&h2);
            }
        };
        // Slow half: ties at the threshold are kept while rl > 0, in
        // ascending key order; keys past n weigh nothing.
        auto slow_half = [&](int key0, const uint32_t (&rr)[32], uint32_t (&pk)[16], int &rl,
                             auto full, int valid) {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                float w2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const uint32_t v = rr[c + e];            // 256 s
                    const bool in = decltype(full)::value || (c + e) < valid;
                    float w = lds_f32(hbase - v);            // 0 below the threshold
                    const bool tie = (v == vt);
                    const bool drop = !in || (tie && rl <= 0);
                    rl -= tie ? 1 : 0;
                    w = drop ? 0.0f : w;
                    zacc[e + (c & 2)] += w;
                    w2[e] = w;
                    if (kDbg) {
                        if (active && !drop && ((int)v > (int)vt || tie)) {
                            if (p.dbg_idx) p.dbg_idx[obase + kept] = key0 + c + e;
                            if (p.dbg_logits) p.dbg_logits[obase + kept] = (int16_t)((int)v / 256);
                            ++kept;
                        }
                    }
                }
                __half2 h2 = __floats2half2_rn(w2[0], w2[1]);
                pk[c >> 1] = *reinterpret_cast<uint32_t *>(&h2);
            }
        };
        auto pass2_half = [&](int j, int h, bool slow, const uint32_t (&rr)[32],
                              uint32_t (&pk)[16], int &rl) {
            if (!slow) {
                fast_half(rr, pk);
            } else {
                const int valid = half_valid(j, h);
                if (valid >= 32) slow_half(j * kKeys + h * 32, rr, pk, rl, BT{}, 32);
                else slow_half(j * kKeys + h * 32, rr, pk, rl, BF{}, valid);
            }
            if constexpr (kCausal) __syncwarp();      // slow differs from lane to lane
        };
        if (ok) ok = wait_s(T);
        if (ok) {
            ld_half(T, 0, sa);
            tc::tmem_wait_ld(sa);
        }
        for (int j = 0; j < T && ok; ++j) {
            const int u = T + j;
            if (j == zero_at) hcol[t * kRows] = 0u;  // ties past the quota weigh nothing now
            bool slow;
            if constexpr (kCausal) {
                // half_valid depends on the lane's row: the vote must not sit
                // behind a short-circuit that some lanes take
                const bool hit = __any_sync(kFullMask, j == jstar);
                slow = j < fast_from || half_valid(j, 1) < 32 || hit;
            } else {
                slow = j < fast_from || half_valid(j, 1) < 32 || __any_sync(kFullMask, j == jstar);
            }
            int rl = j < fast_from ? rem : (j == jstar ? kstar : kAll);
            uint32_t pk[16];
            const uint32_t pcol = lane_base + C::S_COL + (u % C::SBUF) * 64;   // P over S
            ld_half(u, 1, sb);
            pass2_half(j, 0, slow, sa, pk, rl);
            tc::tmem_st16(pcol, pk);                  // S columns 0-15 are already read
            tc::tmem_wait_ld(sb);
            const bool more = j + 1 < T;
            if (more) {
                ok = wait_s(u + 1);
                if (ok) ld_half(u + 1, 0, sa);
            }
            pass2_half(j, 1, slow, sb, pk, rl);
            if (j < fast_from) rem = rl;
            tc::tmem_st16(pcol + 16, pk);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (ok && lane == 0) tc::mbar_arrive(b.p_full(g, j % C::SBUF));
            if (more && ok) tc::tmem_wait_ld(sa);
        }
        float Z = (zacc[0] + zacc[1]) + (zacc[2] + zacc[3]);
        if (!(Z > 0.0f)) Z = 1.0f;                    // missed or inactive rows only
        // causal rows that see fewer than N keys: the unused slots are empty
        if (kDbg && kCausal && active && !miss)
            for (int k = kept; k < p.N; ++k) {
                if (p.dbg_idx) p.dbg_idx[obase + k] = -1;
                if (p.dbg_logits) p.dbg_logits[obase + k] = 0;
            }

        // output: O / Z * 2^e_h
        if (ok) ok = __all_sync(kFullMask, wait_bar(b.o_full(g), 0, deadline, abort_flag, p.status));
        if (ok) {
            tc::fence_after_sync();
            const float scale = ldexpf(1.0f, p.vexp[head]) / Z;
            float *orow = p.out + ((head * p.n) + row) * (long long)D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                tc::tmem_ld32(lane_base + C::O_COL + c0, o);
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

// Exact recomputation of the rows the fused kernel listed.  One CTA of
// eight warps per row, over the keys in segments of kFixSeg:
//   1. the Hamming distance of every key to the row (packed bits, loads of
//      several keys in flight per thread) into a shared byte array, and
//      their histogram -> threshold level t and quota q;
//   2. per segment, each warp takes one contiguous range of it; per-warp
//      counts of ties and of keys above the threshold, prefix-summed across
//      warps (and carried across segments), give every warp its share of
//      the quota (ties go to the lower key index) and its output positions;
//   3. the warp lists its kept keys with their weights exp(tau (s - m)) in
//      shared memory and gathers their V rows eight at a time (lane l owns
//      D/32 columns, so each row is one coalesced read), accumulating fp32;
//      the partial sums meet in shared memory.
// For n <= kFixSeg the distances of step 1 are kept for step 2; longer rows
// recompute each segment's distances.  The last CTA to finish copies the
// miss count to miss_count[2] (the diagnostic's copy) and zeroes the miss
// counter and its own done counter for the next fused pass.
constexpr int kFixSeg = 16384;
constexpr int kFixList = 256;                     // kept keys a warp lists per round

// A whole warp reads one V row, d/32 consecutive elements a lane.
template <typename T, int PER>
struct VRow;

template <>
struct VRow<__nv_bfloat16, 2> {
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&v)[2])
    {
        uint32_t u = __ldg(reinterpret_cast<const uint32_t *>(p));
        v[0] = bf16_lo(u); v[1] = bf16_hi(u);
    }
};
template <>
struct VRow<__nv_bfloat16, 4> {
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&v)[4])
    {
        uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    }
};
template <>
struct VRow<float, 2> {
    __device__ __forceinline__ static void load(const float *p, float (&v)[2])
    {
        float2 u = __ldg(reinterpret_cast<const float2 *>(p));
        v[0] = u.x; v[1] = u.y;
    }
};
template <>
struct VRow<float, 4> {
    __device__ __forceinline__ static void load(const float *p, float (&v)[4])
    {
        float4 u = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
};

template <typename T, int D, bool kCausal = false>
__global__ void __launch_bounds__(256)
fixup_rows_kernel(const uint32_t *__restrict__ qbits, const uint32_t *__restrict__ kbits,
                  const T *__restrict__ V, int n, int N, float tau,
                  int *__restrict__ miss_count, int *__restrict__ done_count,
                  const int *__restrict__ miss_rows,
                  float *__restrict__ out, int32_t *dbg_idx, int16_t *dbg_logits)
{
    constexpr int DW = D / 32, BINS = D + 1, PER = D / 32, NW = 8;
    __shared__ uint8_t dist[kFixSeg];
    __shared__ int hist[BINS];
    __shared__ int wties[NW], wabove[NW];
    __shared__ int lidx[NW][kFixList];
    __shared__ float lw[NW][kFixList];
    __shared__ float opart[NW][D];
    __shared__ float zpart[NW];
    __shared__ int sh_t, sh_quota, sh_hmin;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned below_me = (1u << lane) - 1u;
    const int count = *miss_count;
    for (int m = blockIdx.x; m < count; m += gridDim.x) {
        const int r = miss_rows[m];
        const long long head = r / n;
        // keys the row sees and keeps (causal: keys 0 .. its position)
        const int nv = kCausal ? (int)(r - head * n) + 1 : n;
        const int Nr = min(N, nv);
        uint32_t q[DW];
#pragma unroll
        for (int w = 0; w < DW; ++w) q[w] = qbits[(long long)r * DW + w];
        const uint32_t *kh = kbits + head * n * DW;
        // distances of keys [s0, s1) into dist[j - s0], four keys in flight per thread
        auto fill = [&](int s0, int s1) {
            for (int j0 = s0 + threadIdx.x; j0 < s1; j0 += 4 * blockDim.x) {
                uint32_t kw[4][DW];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = j0 + u * blockDim.x;
#pragma unroll
                    for (int w = 0; w < DW; ++w)
                        kw[u][w] = j < s1 ? __ldg(kh + (long long)j * DW + w) : 0u;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = j0 + u * blockDim.x;
                    int h = 0;
#pragma unroll
                    for (int w = 0; w < DW; ++w) h += __popc(q[w] ^ kw[u][w]);
                    if (j < s1) dist[j - s0] = (uint8_t)h;
                }
            }
        };
        for (int b = threadIdx.x; b < BINS; b += blockDim.x) hist[b] = 0;
        __syncthreads();
        for (int s0 = 0; s0 < nv; s0 += kFixSeg) {
            const int s1 = min(nv, s0 + kFixSeg);
            fill(s0, s1);
            __syncthreads();
            for (int j = threadIdx.x; j < s1 - s0; j += blockDim.x) atomicAdd(&hist[dist[j]], 1);
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            int t = BINS - 1, quota = 0, hmin = BINS - 1, below = 0;
            bool found = false, seen = false;
            for (int b = 0; b < BINS; ++b) {
                const int c = hist[b];
                if (!seen && c) { hmin = b; seen = true; }
                if (!found) {
                    if (below + c >= Nr) { t = b; quota = Nr - below; found = true; }
                    else below += c;
                }
            }
            sh_t = t; sh_quota = quota; sh_hmin = hmin;
        }
        __syncthreads();
        const int t = sh_t, quota = sh_quota, smax = D - 2 * sh_hmin;
        int ties_all = 0, kept_all = 0;           // over earlier segments (block-uniform)
        float acc[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
        float z = 0.0f;
        const T *vh = V + head * n * (long long)D;
        for (int s0 = 0; s0 < nv; s0 += kFixSeg) {
            const int s1 = min(nv, s0 + kFixSeg);
            if (nv > kFixSeg) {
                __syncthreads();
                fill(s0, s1);
                __syncthreads();
            }
            // this warp's range of the segment: a multiple of 32 keys
            const int len = s1 - s0;
            const int span = ((len + NW - 1) / NW + 31) / 32 * 32;
            const int jb = min(len, warp * span), je = min(len, jb + span);
            int nt = 0, na = 0;
            for (int j = jb + lane; j < je; j += 32) {
                const int h = dist[j];
                nt += (h == t);
                na += (h < t);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                nt += __shfl_xor_sync(kFullMask, nt, o);
                na += __shfl_xor_sync(kFullMask, na, o);
            }
            if (lane == 0) { wties[warp] = nt; wabove[warp] = na; }
            __syncthreads();
            int ties_before = ties_all, kept_before = kept_all;
            {
                int tb = ties_all, ka = kept_all;
                for (int w = 0; w < NW; ++w) {
                    const int take = wabove[w] + min(max(quota - tb, 0), wties[w]);
                    if (w == warp) { ties_before = tb; kept_before = ka; }
                    tb += wties[w];
                    ka += take;
                }
                ties_all = tb;
                kept_all = ka;
            }
            for (int base = jb; base < je; base += kFixList) {
                const int lim = min(je, base + kFixList);
                int cnt = 0;
                for (int j0 = base; j0 < lim; j0 += 32) {
                    const int j = j0 + lane;
                    const int h = j < lim ? dist[j] : BINS;
                    const bool tie = (h == t);
                    const unsigned tmask = __ballot_sync(kFullMask, tie);
                    const int rank = ties_before + __popc(tmask & below_me);
                    const bool keep = (h < t) || (tie && rank < quota);
                    ties_before += __popc(tmask);
                    const unsigned kmask = __ballot_sync(kFullMask, keep);
                    if (keep) {
                        const int sv = D - 2 * h;
                        const int slot = cnt + __popc(kmask & below_me);
                        lidx[warp][slot] = s0 + j;
                        lw[warp][slot] = expf(tau * (float)(sv - smax));
                        if (dbg_idx || dbg_logits) {
                            const long long pos = (long long)r * N + kept_before + slot;
                            if (dbg_idx) dbg_idx[pos] = s0 + j;
                            if (dbg_logits) dbg_logits[pos] = (int16_t)sv;
                        }
                    }
                    cnt += __popc(kmask);
                }
                kept_before += cnt;
                __syncwarp();
                // gather the listed V rows, GU loads in flight per lane (at d
                // 128, 16 rows cost more in occupancy than they save in latency)
                constexpr int GU = D == 64 ? 16 : 8;
                for (int i0 = 0; i0 < cnt; i0 += GU) {
                    float v[GU][PER];
                    float ww[GU];
#pragma unroll
                    for (int u = 0; u < GU; ++u) {
                        const bool has = i0 + u < cnt;
                        const int jj = has ? lidx[warp][i0 + u] : 0;
                        ww[u] = has ? lw[warp][i0 + u] : 0.0f;
                        VRow<T, PER>::load(vh + (long long)jj * D + lane * PER, v[u]);
                    }
#pragma unroll
                    for (int u = 0; u < GU; ++u) {
#pragma unroll
                        for (int e = 0; e < PER; ++e) acc[e] = fmaf(ww[u], v[u][e], acc[e]);
                        z += ww[u];
                    }
                }
                __syncwarp();
            }
            __syncthreads();
        }
#pragma unroll
        for (int e = 0; e < PER; ++e) opart[warp][lane * PER + e] = acc[e];
        if (lane == 0) zpart[warp] = z;
        __syncthreads();
        float zt = 0.0f;
#pragma unroll
        for (int w = 0; w < NW; ++w) zt += zpart[w];
        for (int c = threadIdx.x; c < D; c += blockDim.x) {
            float o = 0.0f;
#pragma unroll
            for (int w = 0; w < NW; ++w) o += opart[w][c];
            out[(long long)r * D + c] = o / zt;
        }
        if (kCausal)           // slots past the row's N_i keys are empty
            for (int k = Nr + threadIdx.x; k < N; k += blockDim.x) {
                const long long pos = (long long)r * N + k;
                if (dbg_idx) dbg_idx[pos] = -1;
                if (dbg_logits) dbg_logits[pos] = 0;
            }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(done_count, 1) == (int)gridDim.x - 1) {
            miss_count[2] = *miss_count;          // kept for had_attention_window_misses
            *miss_count = 0;
            *done_count = 0;
            __threadfence();
        }
    }
}

}  // namespace fused
}  // namespace had
