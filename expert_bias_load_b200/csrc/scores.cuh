// scores.cuh -- the logits-mode routing score with one defined rounding.
//
// s = (float)(1 / (1 + exp(-(double)x))): the sigmoid evaluated in fp64 and
// rounded once to fp32.  Logits mode fixes this rounding so that any
// implementation of the formula agrees with the kernels value for value (up
// to a last-ulp difference between two fp64 exp implementations).
#pragma once

namespace ebl {

__device__ __forceinline__ float sigmoid_rounded_once(float x) {
    const double e = exp(-(double)x);
    return __double2float_rn(__drcp_rn(__dadd_rn(1.0, e)));  // correctly rounded 1/y, the same as 1.0/y
}

}  // namespace ebl
