// Element-wise kernels of the NVFP4 Newton-Schulz iteration (nvfp4_newton_schulz).
//
// The iteration is the optimizer passage of "Full-Stack FP4: Preentrenamiento
// Estable de LLM" (Newton-Schulz run natively in NVFP4 for Muon), taken as the
// coefficient-free cubic iteration for the orthogonal polar factor (Bjorck and
// Bowie, SIAM J. Numer. Anal. 8, 1971) in residual form:
//   X_0 = G / ||G||_F,   R = I - X X^T,   X <- X + R X / 2,
// both products NVFP4 GEMMs (gemm.cuh) on operands from the quantiser
// (quantize.cuh).  What is left for this file is HBM-bound element-wise work:
// the sum of squares of G, the normalisation, and the identity that the first
// product accumulates into.  Matrices are BF16, row-major, rows 16-byte aligned,
// columns a multiple of 8; every kernel walks whole rows with one block per row
// (grid-stride over rows) and 16-byte vectors per thread.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace nvfp4 {
namespace ns {

constexpr int kThreads = 256;

// acc += sum of g[r][c]^2 over the matrix, in FP64 (each square of a BF16 value
// is exact in FP64).  acc must be zeroed before the launch.
__global__ void __launch_bounds__(kThreads) sumsq_kernel(const uint16_t* __restrict__ g, int64_t rows, int64_t cols,
                                                         int64_t ld, double* __restrict__ acc) {
  __shared__ double part[kThreads / 32];
  const int64_t vecs = cols / 8;
  double s = 0.0;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(g + r * ld);
    for (int64_t v = threadIdx.x; v < vecs; v += blockDim.x) {
      const uint4 w = row[v];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double a = (double)bf16_lo(ws[e]);
        const double b = (double)bf16_hi(ws[e]);
        s = __dadd_rn(s, __dmul_rn(a, a));
        s = __dadd_rn(s, __dmul_rn(b, b));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s = __dadd_rn(s, __shfl_down_sync(0xffffffffu, s, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) part[warp] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) t = __dadd_rn(t, part[i]);
    if (t != 0.0) atomicAdd(acc, t);
  }
}

// x = BF16(fl32(g / n)) with n = FP32(sqrt(acc)), the Frobenius norm; n == 0 gives
// x = 0.  norm_out (optional) receives n.  g and x may be the same matrix (each
// element is read and written by the same thread).
__global__ void __launch_bounds__(kThreads) normalize_kernel(const uint16_t* g, int64_t ldg, uint16_t* x, int64_t ldx,
                                                             int64_t rows, int64_t cols,
                                                             const double* __restrict__ acc, float* norm_out) {
  const float nrm = __double2float_rn(__dsqrt_rn(*acc));
  if (norm_out && blockIdx.x == 0 && threadIdx.x == 0) *norm_out = nrm;
  const int64_t vecs = cols / 8;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(g + r * ldg);
    uint4* dst = reinterpret_cast<uint4*>(x + r * ldx);
    for (int64_t v = threadIdx.x; v < vecs; v += blockDim.x) {
      const uint4 w = src[v];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      uint32_t out[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = nrm == 0.0f ? 0.0f : __fdiv_rn(bf16_lo(ws[e]), nrm);
        const float b = nrm == 0.0f ? 0.0f : __fdiv_rn(bf16_hi(ws[e]), nrm);
        out[e] = f32_to_bf16_bits(a) | (f32_to_bf16_bits(b) << 16);
      }
      dst[v] = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

// r = I (BF16 [m x m], row stride ld): the matrix the product -X X^T adds into.
__global__ void __launch_bounds__(kThreads) identity_kernel(uint16_t* __restrict__ r, int64_t m, int64_t ld) {
  const int64_t vecs = m / 8;
  for (int64_t row = blockIdx.x; row < m; row += gridDim.x) {
    uint4* dst = reinterpret_cast<uint4*>(r + row * ld);
    for (int64_t v = threadIdx.x; v < vecs; v += blockDim.x) {
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      const int64_t d = row - 8 * v;                      // the diagonal's place in this vector
      if (d >= 0 && d < 8) w[d >> 1] = (d & 1) ? 0x3F800000u : 0x00003F80u;   // BF16 1.0, even index low
      dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

}  // namespace ns
}  // namespace nvfp4
