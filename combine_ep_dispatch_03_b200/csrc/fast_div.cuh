// fast_div.cuh -- x / s rounded to nearest even, for the FP8 cast's many
// quotients by one block scale s, without a full division per element.
//
// Markstein's method (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with
// y = RN(1/s), q0 = RN(x * y) and the exact remainder r = x - s * q0 (one
// fused multiply-add), RN(q0 + r * y) is RN(x / s) when no step leaves the
// normal range. fast_group_ok keeps every step there for a group of elements:
// the block's amax in [2^-60, 2^120] (so s and y are normal), and the group's
// smallest nonzero |x| at least 2^-100 with RN(|x| * y) at least 2^-100 (so r
// is exact and the quotient normal). Zeros take the sign of x, as a division
// gives them. tests/fast_div_exhaustive.cu checks div_by_scale_fast against
// __fdiv_rn on every pair of finite bf16 x and positive finite bf16 amax that
// these conditions admit.
#pragma once

namespace epb {

// RN(x / s) given y = RN(1 / s), inside the range fast_group_ok admits
__device__ __forceinline__ float div_by_scale_fast(float x, float s, float y) {
    const float q0 = __fmul_rn(x, y);
    return copysignf(__fmaf_rn(__fmaf_rn(-s, q0, x), y, q0), x);
}

// amax: the block's largest |x| (s = RN(amax / 448)); minnz: the group's
// smallest nonzero |x| (+inf if it has none)
__device__ __forceinline__ bool fast_group_ok(float amax, float minnz, float y) {
    return amax >= 0x1p-60f && amax <= 0x1p+120f && minnz >= 0x1p-100f && __fmul_rn(minnz, y) >= 0x1p-100f;
}

} // namespace epb
