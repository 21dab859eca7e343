// Device self-check of the hardware conversions the kernels rely on.
//
// The quantiser encodes with the sm_100a conversion instructions (E2M1
// round-to-nearest, E2M1 stochastic rounding with a 32-bit random operand, E4M3
// round-to-nearest).  This kernel compares each with its definition written out
// in common.cuh, so a library user can confirm on their own GPU that the bytes
// the kernels produce follow the stated rounding rules:
//   counts[0]  E2M1 RNE mismatches over every 2^32 float pattern (NaN skipped)
//   counts[1]  E4M3 mismatches over every non-negative finite float
//   counts[2]  E2M1 SR mismatches over n_sr pseudo-random (value, word) pairs
#pragma once

#include "common.cuh"

namespace nvfp4 {

__global__ void __launch_bounds__(256) check_conversions_kernel(unsigned long long* counts, uint64_t n_sr) {
  const uint64_t tid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  unsigned long long bad_rn = 0, bad_e4 = 0, bad_sr = 0;
  for (uint64_t i = tid; i < (1ull << 32); i += stride) {
    const uint32_t bits = (uint32_t)i;
    const float x = __uint_as_float(bits);
    if (isnan(x)) continue;
    const float y[8] = {x, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if ((e2m1x8_rn(y) & 0xFu) != e2m1_rne(x)) ++bad_rn;
    if (!(bits >> 31) && isfinite(x) && e4m3_encode_hw(x) != e4m3_encode(x)) ++bad_e4;
  }
  for (uint64_t i = tid; i < n_sr; i += stride) {
    const uint4 r = philox4x32_10(make_uint4((uint32_t)i, (uint32_t)(i >> 32), 0x5EEDu, 0u), 0x9E3779B9u, 7u);
    const uint4 e = philox4x32_10(make_uint4((uint32_t)i, (uint32_t)(i >> 32), 0xE4Du, 1u), 0x9E3779B9u, 7u);
    float v[4];
    const uint32_t raw[4] = {r.x, r.y, r.z, e.x};
    const uint32_t ex[4] = {e.y, e.z, e.w, e.y >> 8};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // exponents spread from far below E2M1's range to above it, random mantissa and sign
      const uint32_t expo = 100u + (ex[k] & 31u);
      uint32_t b = (raw[k] & 0x807FFFFFu) | (expo << 23);
      if ((ex[k] & 0x3E0u) == 0) b = raw[k] & 0xFF7FFFFFu;   // occasionally any finite pattern
      v[k] = __uint_as_float(b);
    }
    const uint32_t w = r.w ^ e.w;
    const uint32_t hw = e2m1x4_rs(v[0], v[1], v[2], v[3], w);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (((hw >> (4 * k)) & 0xFu) != e2m1_sr16(v[k], group_noise(w, k))) ++bad_sr;
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) {
    bad_rn += __shfl_xor_sync(0xFFFFFFFFu, bad_rn, s);
    bad_e4 += __shfl_xor_sync(0xFFFFFFFFu, bad_e4, s);
    bad_sr += __shfl_xor_sync(0xFFFFFFFFu, bad_sr, s);
  }
  if ((threadIdx.x & 31) == 0) {
    if (bad_rn) atomicAdd(counts + 0, bad_rn);
    if (bad_e4) atomicAdd(counts + 1, bad_e4);
    if (bad_sr) atomicAdd(counts + 2, bad_sr);
  }
}

}  // namespace nvfp4
