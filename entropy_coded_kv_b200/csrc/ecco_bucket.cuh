// The encoder's threshold bucket map (see ecco_encode.cu, quantise_bucket),
// shared with the table builder that fills the per-pattern bucket counts.
#pragma once

#include <cstdint>

namespace ecco {

// Bucket of v in a pattern's threshold map: n = round(255 * sat(a v + b)),
// by two fused multiply-adds (the second one adds 1.5 * 2^23, so the integer
// lands in the low mantissa bits).  Every step is monotone (a > 0), so n never
// decreases as v grows: a threshold in a higher bucket than v is above v, one
// in a lower bucket is below it.  The table builder and the encoder both call
// this, so the buckets of v and of the thresholds come from the same
// operations.
__device__ __forceinline__ uint32_t threshold_bucket(float v, float a, float b)
{
    const float s = __saturatef(__fmaf_rn(v, a, b));
    return __float_as_uint(__fmaf_rn(s, 255.0f, 12582912.0f)) & 0xffu;
}

}  // namespace ecco
