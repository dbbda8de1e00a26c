// had_common.cuh -- small device helpers shared by the HAD kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "had.h"

namespace had {

constexpr unsigned kFullMask = 0xffffffffu;

// OR a device-detected condition into the caller's status word (if any).
__device__ __forceinline__ void flag(int32_t *status, int code)
{
    if (status) atomicOr(status, 1 << code);
}

__device__ __forceinline__ float bf16_lo(uint32_t two) { return __uint_as_float(two << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t two) { return __uint_as_float(two & 0xffff0000u); }

// Per-head constants of the standardize-and-sign step.  sigma must be a
// positive finite number; for a normal sigma the quotient x / sigma can only
// round to zero when |x| is below sigma * 2^-100, so larger negative x take
// the sign without dividing and only tiny ones pay for the IEEE division.
struct SignRule {
    float sigma;
    float thr;
    bool fast;
    bool bad;
};

__device__ __forceinline__ SignRule sign_rule(float sigma)
{
    SignRule r;
    r.sigma = sigma;
    r.bad = !(sigma > 0.0f) || !isfinite(sigma);
    r.fast = !r.bad && sigma >= 1.17549435e-38f;          // normal, positive
    // sigma * 2^-100, kept at or above the smallest subnormal: a sigma below
    // 2^-50 would round it to 0, and x <= -0 would then hold for x = +-0,
    // whose quotient is not negative (with thr >= 2^-149 and sigma < 2^-49
    // any x <= -thr still has |x / sigma| > 2^-100)
    r.thr = fmaxf(sigma * 7.88860905e-31f, 1.40129846e-45f);
    return r;
}

// 1 iff x / sigma (IEEE fp32, round to nearest, subnormals kept) is < 0.
__device__ __forceinline__ uint32_t negative_bit(float x, const SignRule &r)
{
    if (r.fast) {
        if (!(x < 0.0f)) return 0u;
        if (x <= -r.thr) return 1u;
    }
    return __fdiv_rn(x, r.sigma) < 0.0f ? 1u : 0u;
}

// Sign test of four bf16 values on their raw bits, under a normal sigma
// (SignRule::fast).  The values are the low then the high halves of words a
// and b (memory order); byte i of each result is 0x80 or 0 for value i:
//   neg: surely negative after the division: sign set and exponent field
//        e >= 2 e7 (e < 255), so |x| >= 2^(2 e7 - 127) > sigma 2^-100 and
//        x / sigma < -2^-100;
//   uns: the exact division must decide: sign set and a smaller exponent
//        (-0 and tiny values), or e = 255 (-inf, NaN).
// Non-negative values (sign clear, +NaN included) are in neither.  kge =
// (0x80 - e7) per byte, from bf16_kge: adding it to a byte's top 7 exponent
// bits sets the byte's bit 7 iff they are >= e7 (no carry leaves a byte).
__device__ __forceinline__ uint32_t bf16_kge(const SignRule &r)
{
    const uint32_t e_thr = (__float_as_uint(r.thr) >> 23) & 0xFFu;   // thr < 2^(e_thr - 126)
    const uint32_t e7 = (e_thr + 2u) >> 1;                           // 2 e7 >= e_thr + 1; 1 .. 128
    return (0x80u - e7) * 0x01010101u;
}

__device__ __forceinline__ void bf16_signs4(uint32_t a, uint32_t b, uint32_t kge, uint32_t &neg,
                                            uint32_t &uns)
{
    const uint32_t hi = __byte_perm(a, b, 0x7531);     // the four high bytes: sign, e[7:1]
    const uint32_t t7 = hi & 0x7F7F7F7Fu;
    const uint32_t ge = t7 + kge;                       // bit 7: e[7:1] >= e7
    const uint32_t sp = t7 + 0x01010101u;               // bit 7: e[7:1] = 127 (inf, NaN)
    neg = hi & ge & ~sp & 0x80808080u;
    uns = hi & (~ge | sp) & 0x80808080u;
}

// The four bit-7 flags of a byte-lane word as bits 0..3 (the shifted copies
// of the multiply land on distinct bits, so no carries).
__device__ __forceinline__ uint32_t flags4(uint32_t x) { return (x * 0x00204081u) >> 28; }

}  // namespace had
