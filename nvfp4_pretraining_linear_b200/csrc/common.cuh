// Device helpers shared by the NVFP4 kernels: format conversions written from
// the E2M1 / E4M3 definitions, the Philox4x32-10 generator (Salmon et al.,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11), the 16-point
// Hadamard butterfly, the tensor-core scale-tile addressing, and bounded
// mbarrier waits.
//
// Every floating-point step of the quantiser is one IEEE round-to-nearest
// operation (__fdiv_rn / __fmul_rn / __fadd_rn): no contraction into FMA, no
// flush-to-zero, so the encoded bytes do not depend on compiler choices.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

// ----------------------------------------------------------------- errors

// Bits of the device error word (one per device, module scope).
constexpr unsigned kErrTimeout = 1u;
__device__ unsigned int g_error_word;

// A bounded wait gives up after this long (ns of %globaltimer) and reports
// kErrTimeout instead of hanging the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------- BF16

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// float -> BF16 bits, round to nearest even (finite inputs).
__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
  uint32_t b = __float_as_uint(f);
  return (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;
}

// ----------------------------------------------------------------- E4M3 scales

// Non-negative float -> E4M3 byte, round to nearest even, saturating at 448.
// E4M3: bias 7, 3 mantissa bits; normals (1 + m/8) * 2^(e-7), subnormals m * 2^-9.
__device__ __forceinline__ uint32_t e4m3_encode(float v) {
  if (!(v < 448.0f)) return 0x7Eu;                 // saturate (also +inf)
  if (v < 0.015625f) {                             // below 2^-6: subnormal grid 2^-9
    return (uint32_t)__float2int_rn(__fmul_rn(v, 512.0f));   // 0..8, exact scaling
  }
  const uint32_t bits = __float_as_uint(v);
  const int e = (int)((bits >> 23) & 0xFFu) - 127;  // -6 .. 8
  const uint32_t mant = bits & 0x7FFFFFu;
  const uint32_t keep = mant >> 20;                 // top 3 mantissa bits
  const uint32_t rest = mant & 0xFFFFFu;
  uint32_t q = 8u + keep;
  if (rest > 0x80000u || (rest == 0x80000u && (keep & 1u))) q += 1u;   // ties to even
  return (uint32_t)((e + 6) * 8) + q;              // q == 16 carries into the next binade
}

__device__ __forceinline__ float e4m3_decode(uint32_t b) {
  const uint32_t e = b >> 3, m = b & 7u;
  if (e == 0) return __fmul_rn((float)m, 0.001953125f);        // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));      // (1 + m/8) * 2^(e-7)
}

// ----------------------------------------------------------------- E2M1 elements

// float -> 4-bit E2M1 code (sign << 3 | index), nearest magnitude of
// {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the even index, saturating at 6, sign kept.
__device__ __forceinline__ uint32_t e2m1_rne(float y) {
  const float a = fabsf(y);
  const uint32_t idx = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) +
                       (uint32_t)(a >= 1.75f) + (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) +
                       (uint32_t)(a > 5.0f);
  return idx | ((__float_as_uint(y) >> 31) << 3);
}

// Stochastic rounding between the two neighbouring magnitudes lo <= |y| < hi
// with a 16-bit random integer n: up iff floor(f * 2^16) + n >= 2^16, f =
// (|y| - lo) / (hi - lo); |y| >= 6 gives 6; sign kept.
__device__ __forceinline__ uint32_t e2m1_sr16(float y, uint32_t n) {
  const float a = fabsf(y);
  const uint32_t sign = (__float_as_uint(y) >> 31) << 3;
  if (a >= 6.0f) return 7u | sign;
  const uint32_t lo = (uint32_t)(a >= 0.5f) + (uint32_t)(a >= 1.0f) + (uint32_t)(a >= 1.5f) +
                      (uint32_t)(a >= 2.0f) + (uint32_t)(a >= 3.0f) + (uint32_t)(a >= 4.0f);
  const float lo_v = lo < 4u ? __fmul_rn((float)lo, 0.5f) : (float)lo - 2.0f;   // 0,.5,1,1.5 | 2,3,4
  const float inv_step = lo < 4u ? 2.0f : (lo < 6u ? 1.0f : 0.5f);
  const float frac = __fmul_rn(__fsub_rn(a, lo_v), inv_step);                  // exact, in [0, 1)
  const uint32_t fixed = (uint32_t)__float2int_rd(__fmul_rn(frac, 65536.0f));  // exact scaling, floor
  return (lo + (fixed + n >= 65536u ? 1u : 0u)) | sign;
}

// 16-bit reversal and the random integers of the four elements of a group.
__device__ __forceinline__ uint32_t bitrev16(uint32_t x) { return __brev(x) >> 16; }

__device__ __forceinline__ uint32_t group_noise(uint32_t w, int e) {
  const uint32_t n0 = (((w >> 16) & 0xFFu) << 8) | (w & 0xFFu);
  const uint32_t n2 = (((w >> 24) & 0xFFu) << 8) | ((w >> 8) & 0xFFu);
  return e == 0 ? n0 : (e == 1 ? bitrev16(n0) : (e == 2 ? n2 : bitrev16(n2)));
}

// ----------------------------------------------------------------- hardware conversions
//
// The sm_100a conversions below are used by the kernels; each was checked on
// every input it can receive against the definitions above (e2m1_rne: all 2^32
// float patterns; e4m3_encode: all non-negative floats).

// Eight floats -> eight E2M1 codes (RNE, saturating), element j in nibble j.
__device__ __forceinline__ uint32_t e2m1x8_rn(const float* y) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  return out;
}

// Four floats -> four E2M1 codes with stochastic rounding (element j in nibble
// j).  The 32-bit word w supplies each element's 16-bit random integer:
// e0: w[23:16]:w[7:0], e1: its 16-bit reversal, e2: w[31:24]:w[15:8], e3: its
// reversal; an element rounds up iff floor(f * 2^16) + n >= 2^16.
__device__ __forceinline__ uint32_t e2m1x4_rs(float y0, float y1, float y2, float y3, uint32_t w) {
  uint16_t out;
  asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%1, %2, %3, %4}, %5;"
      : "=h"(out)
      : "f"(y3), "f"(y2), "f"(y1), "f"(y0), "r"(w));
  return out;
}

// Non-negative float -> E4M3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_encode_hw(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(v), "f"(0.0f));
  return out & 0xFFu;
}

// ----------------------------------------------------------------- Philox4x32-10

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    // one 32 x 32 -> 64-bit product gives both halves of each multiplication
    const uint64_t p0 = (uint64_t)0xD2511F53u * c.x;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c.z;
    c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ k1, (uint32_t)p0);
  }
  return c;
}

// The same generator with its round keys precomputed (rk[r] = k0 + r * 0x9E3779B9,
// rk[10 + r] = k1 + r * 0xBB67AE85, modulo 2^32): when rk lives in a kernel's
// parameter space, a round is two wide multiplies and two three-input XORs.
__device__ __forceinline__ uint4 philox4x32_10_rk(uint4 c, const uint32_t* rk) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c.x;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c.z;
    c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ rk[r], (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ rk[10 + r],
                   (uint32_t)p0);
  }
  return c;
}


// ----------------------------------------------------------------- packed FP32 pairs
//
// sm_100 executes two FP32 additions or multiplications as one instruction on a
// 64-bit register pair (add/sub/mul.rn.f32x2); each lane is the IEEE
// round-to-nearest operation of its scalar counterpart, so results are unchanged.

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t p, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// ----------------------------------------------------------------- Hadamard

// Butterfly stage h over N values held in registers: (v[i], v[i+h]) <- (v[i]+v[i+h], v[i]-v[i+h]).
template <int N>
__device__ __forceinline__ void wht_stage(float* v, int h) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    if (!(i & h)) {
      const float a = v[i], b = v[i + h];
      v[i] = __fadd_rn(a, b);
      v[i + h] = __fsub_rn(a, b);
    }
  }
}

// ----------------------------------------------------------------- scales

// Per-tensor decode scale S = amax / (6 * 448); 1 for an all-zero tensor.
__device__ __forceinline__ float tensor_scale_from_amax(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

struct BlockScale {
  float r;        // encode multiplier 1 / (s * S), 0 for a dead block
  uint32_t sbyte; // E4M3 block scale
};

// Block scale s = E4M3((b / 6) / S), d = s * S, r = 1 / d.  A block whose scale
// or decode factor is zero, or whose multiplier overflows, encodes all-zero codes.
__device__ __forceinline__ BlockScale block_scale(float bmax, float S) {
  BlockScale out;
  const float s_f = __fdiv_rn(__fdiv_rn(bmax, 6.0f), S);
  out.sbyte = e4m3_encode_hw(s_f);
  const float d = __fmul_rn(e4m3_decode(out.sbyte), S);
  const float r = __fdiv_rn(1.0f, d);
  const bool dead = (out.sbyte == 0u) || (d == 0.0f) || !isfinite(r);
  out.r = dead ? 0.0f : r;
  return out;
}

// The encode multiplier of an E4M3 scale byte under tensor scale S, with the
// dead-block rule of block_scale (0 when s == 0, s * S == 0 or 1 / (s * S) is not
// finite).  A kernel tabulates it for all 128 non-negative bytes once per S.
__device__ __forceinline__ float scale_multiplier(uint32_t sbyte, float S) {
  const float d = __fmul_rn(e4m3_decode(sbyte), S);
  const float r = __fdiv_rn(1.0f, d);
  return (sbyte == 0u || d == 0.0f || !isfinite(r)) ? 0.0f : r;
}

// block_scale with the multiplier looked up in such a table (bit-identical).
__device__ __forceinline__ BlockScale block_scale_tab(float bmax, float S, const float* rtab) {
  BlockScale out;
  out.sbyte = e4m3_encode_hw(__fdiv_rn(__fdiv_rn(bmax, 6.0f), S));
  out.r = rtab[out.sbyte & 0x7Fu];
  return out;
}

// Per-tensor factor of block_scale_fast: K = fl(1 / fl(6 S)), or 0 where the fast
// path's error bound is not established (S below 2^-100, or K not finite).
__device__ __forceinline__ float fast_scale_factor(float S) {
  if (!(S >= 0x1p-100f)) return 0.0f;
  const float k = __fdiv_rn(1.0f, __fmul_rn(6.0f, S));
  return isfinite(k) ? k : 0.0f;
}

// block_scale_tab with one multiply where that provably gives the same byte.
// s_a = fl(b K) carries three roundings of at most 2^-24 relative each, s = fl(fl(b / 6)
// / S) two (b / 6 normal, below), so they are within 5 ulps of s_a of each other.  E4M3
// rounding changes only at the midpoints between its values; for s_a in E4M3's normal
// range (>= 2^-6), a midpoint is where the 20 FP32 mantissa bits below E4M3's 3 are
// exactly 0x80000.  If those bits of s_a are more than 16 away from it, s rounds to the
// byte s_a rounds to (values above 448 saturate either way).  Otherwise -- and for s_a
// below 2^-6 or not a number -- the two divisions are done.  s_a >= 2^-6 also implies
// K != 0 (K = 0 gives s_a = 0 or NaN) and, as K = 0 unless S >= 2^-100,
// b >= 2^-6 * 6 S * (1 - 2^-22) > 2^-104, which keeps b / 6 normal.
__device__ __forceinline__ BlockScale block_scale_fast(float bmax, float S, float K, const float* rtab) {
  const float sa = __fmul_rn(bmax, K);
  const int dm = (int)(__float_as_uint(sa) & 0xFFFFFu) - 0x80000;
  float s = sa;
  if (!(sa >= 0x1p-6f && (uint32_t)(dm + 16) > 32u))   // |dm| > 16
    s = __fdiv_rn(__fdiv_rn(bmax, 6.0f), S);
  BlockScale out;
  out.sbyte = e4m3_encode_hw(s);
  out.r = rtab[out.sbyte & 0x7Fu];
  return out;
}

// Byte offset of block scale (row r, block j) in the tensor-core scale layout:
// tiles of 128 rows x 4 blocks, tile-major along the blocks.
__device__ __forceinline__ int64_t mma_scale_offset(int64_t r, int64_t j, int64_t kgroups) {
  return (((r >> 7) * kgroups + (j >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (j & 3);
}

// ----------------------------------------------------------------- PTX wrappers

// Programmatic dependent launch: a kernel launched as a programmatic dependent of
// the one before it in the stream may start once every CTA of that one has called
// griddep_launch_dependents (or exited); griddep_wait then blocks until that kernel
// has completed and its memory operations are visible.  In a normal launch the wait
// returns at once.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// One lane of the (fully active) warp, chosen by elect.sync (the same lane every time
// the whole warp calls it).  Single-thread operations -- tcgen05 MMAs, copies and
// commits, TMA copies, barrier arming -- are issued under it with operands the whole
// warp computed, so that they stay warp-uniform; issuing them under lane == 0 with
// operands computed inside the branch measured 5-8 % slower in the GEMM.
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(e));
  return e != 0;
}

// Wait until the phase with the given parity of mbarrier `bar` has completed.
// Gives up after kWaitLimitNs, or as soon as *abort is set by another role of
// the CTA: records kErrTimeout, raises *abort and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        atomicOr(&g_error_word, kErrTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

}  // namespace nvfp4
