// dec_bins.cuh -- the absolute indexer-score bins of the decode selection
// (decode_select.cu bins every score into them; decode_variants.cu reads the
// counts back): bin b = floor(s * kappa), kappa = kDecKappa bins per unit.
#pragma once

#include "rtp_host.h"

namespace rtp {

// Absolute score bin floor(s * kappa), rounding toward -inf.  kappa * s is
// clamped to +-2^21 (far outside the histogram's range); adding 1.5 * 2^23 with
// rounding toward -inf leaves floor(x) in the low mantissa bits, exactly, for
// |x| < 2^22.  sbin_m returns that sum: the bin is bin_f / bin_i of it.
__device__ __forceinline__ float sbin_m(float s) {
  const float x = fminf(fmaxf(__fmul_rn(s, kDecKappa), -2097152.0f), 2097152.0f);
  return __fadd_rd(x, 12582912.0f);
}
__device__ __forceinline__ float bin_f(float m) { return __fsub_rn(m, 12582912.0f); }
__device__ __forceinline__ int bin_i(float m) { return __float_as_int(m) - 0x4B400000; }
__device__ __forceinline__ int sbin(float s) { return bin_i(sbin_m(s)); }

}  // namespace rtp
