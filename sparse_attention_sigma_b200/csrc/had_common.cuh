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
    r.thr = sigma * 7.88860905e-31f;                       // sigma * 2^-100
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

}  // namespace had
