// NVFP4 quantiser kernels: the amax pass, the fused quantise pass and the
// dequantiser.
//
// What they compute follows the format and recipe passages of "Preentrenamiento
// de 4 bits con NVFP4 en un hibrido Mamba-Transformer de 12B": 16-element blocks
// with an E4M3 scale each and an FP32 scale per tensor; 16x16 two-dimensional
// blocks for weights; a 16x16 random Hadamard transform on the weight-gradient
// operands; stochastic rounding for gradients only.
//
// Work decomposition (both passes).  A warp owns a slab of 16 rows x 256
// columns; lane l holds the 16 x 8 sub-block at columns 8l..8l+7, loaded as
// sixteen 16-byte vectors (each row of the slab is one 512-byte coalesced
// segment).  The slab contains, per lane, half of 16 row blocks (the other half
// is the neighbouring lane: one shuffle joins them) and 8 whole column blocks,
// so the row and the col (transposed) layouts are both produced from one read
// of the input.  A CTA of 8 warps stacks 8 slabs vertically (128 rows), so that
// each column's col-layout codes for the CTA are one 64-byte run.
#pragma once

#include "common.cuh"

namespace nvfp4 {

constexpr int kQuantWarps = 8;
constexpr int kQuantThreads = kQuantWarps * 32;
constexpr int kSlabRows = 16;
constexpr int kSlabCols = 256;

struct QuantLayout {
  uint8_t* codes;       // nullptr when the layout is not emitted
  uint8_t* scales;
  float* tensor_scale;
  int64_t kgroups;      // 4-block groups per row (tensor-core scale layout)
  int32_t mma_layout;   // scales in the tensor-core layout (else row-major)
};

struct QuantParams {
  const uint16_t* x;    // BF16 bits
  int64_t rows, cols, ld;
  QuantLayout row, col;
  const float* amax;    // 3 floats: raw, transformed col layout, transformed row layout
  float* amax_out;      // nullptr or 3 floats
  uint32_t key0, key1;  // Philox key (seed)
  uint32_t offset;      // Philox counter word 3
  uint32_t signs;       // RHT sign mask
};

__device__ __forceinline__ int64_t scale_index(const QuantLayout& L, int64_t r, int64_t j, int64_t nblk) {
  return L.mma_layout ? mma_scale_offset(r, j, L.kgroups) : r * nblk + j;
}

// Load the 16 x 8 sub-block of lane `lane` (zero rows past `nrows`, zero lanes past `cols`).
__device__ __forceinline__ void load_slab(const uint16_t* __restrict__ x, int64_t ld, int64_t r0, int64_t c0,
                                          int nrows, bool active, uint4 (&raw)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    raw[i] = make_uint4(0u, 0u, 0u, 0u);
    if (active && i < nrows) raw[i] = __ldg(reinterpret_cast<const uint4*>(x + (r0 + i) * ld + c0));
  }
}

__device__ __forceinline__ void unpack8(const uint4& w, float* v) {
  v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x);
  v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
  v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z);
  v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}

__device__ __forceinline__ float column_value(const uint4& w, int j) {
  const uint32_t word = j < 2 ? w.x : (j < 4 ? w.y : (j < 6 ? w.z : w.w));
  return (j & 1) ? bf16_hi(word) : bf16_lo(word);
}

// Row-block transform: this lane holds elements e = 8*(lane&1) + j of a 16-group
// spread over a lane pair.  Stages h = 1, 2, 4 are local, stage 8 crosses the
// pair, then the 1/4 normalisation -- the same operation order as rht16().
__device__ __forceinline__ void rht16_pair(float* v, uint32_t signs, int lane) {
  const uint32_t half = (uint32_t)(lane & 1) * 8u;
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = flip_sign(v[j], (signs >> (half + j)) & 1u);
  wht_stage<8>(v, 1);
  wht_stage<8>(v, 2);
  wht_stage<8>(v, 4);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float other = __shfl_xor_sync(0xFFFFFFFFu, v[j], 1);
    v[j] = (lane & 1) ? __fsub_rn(other, v[j]) : __fadd_rn(v[j], other);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(v[j], 0.25f);
}

__device__ __forceinline__ float absmax8(const float* v) {
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
  return m;
}

__device__ __forceinline__ unsigned float_as_ordered(float f) { return __float_as_uint(f); }

// ------------------------------------------------------------------ amax pass
//
// out[0] = max |x|; out[1] = max over the col layout's transformed blocks;
// out[2] = max over the row layout's transformed blocks.  Non-negative floats
// order like their bit patterns, so atomicMax on the bits is a float max.
template <bool RHT_COL, bool RHT_ROW>
__global__ void __launch_bounds__(kQuantThreads) amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                             int64_t cols, int64_t ld, uint32_t signs,
                                                             unsigned* __restrict__ out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row_groups = (rows + kSlabRows - 1) / kSlabRows;
  const int64_t chunks = (cols + kSlabCols - 1) / kSlabCols;
  const int64_t items = row_groups * chunks;
  float m_raw = 0.0f, m_col = 0.0f, m_row = 0.0f;
  for (int64_t it = (int64_t)blockIdx.x * kQuantWarps + warp; it < items; it += (int64_t)gridDim.x * kQuantWarps) {
    const int64_t rg = it / chunks, ch = it - rg * chunks;
    const int64_t r0 = rg * kSlabRows, c0 = ch * kSlabCols + lane * 8;
    const bool active = c0 < cols;
    const int nrows = (int)(rows - r0 < kSlabRows ? rows - r0 : kSlabRows);
    uint4 raw[16];
    load_slab(x, ld, r0, c0, nrows, active, raw);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float v[8];
      unpack8(raw[i], v);
      m_raw = fmaxf(m_raw, absmax8(v));
      if (RHT_ROW) {
        rht16_pair(v, signs, lane);
        m_row = fmaxf(m_row, absmax8(v));
      }
    }
    if (RHT_COL) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = column_value(raw[i], j);
        rht16(v, signs);
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
        m_col = fmaxf(m_col, m);
      }
    }
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) {
    m_raw = fmaxf(m_raw, __shfl_xor_sync(0xFFFFFFFFu, m_raw, s));
    if (RHT_COL) m_col = fmaxf(m_col, __shfl_xor_sync(0xFFFFFFFFu, m_col, s));
    if (RHT_ROW) m_row = fmaxf(m_row, __shfl_xor_sync(0xFFFFFFFFu, m_row, s));
  }
  __shared__ float red[3][kQuantWarps];
  if (lane == 0) {
    red[0][warp] = m_raw;
    red[1][warp] = m_col;
    red[2][warp] = m_row;
  }
  __syncthreads();
  if (threadIdx.x < 3) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < kQuantWarps; ++w) m = fmaxf(m, red[threadIdx.x][w]);
    if (threadIdx.x == 0 || (threadIdx.x == 1 && RHT_COL) || (threadIdx.x == 2 && RHT_ROW))
      atomicMax(out + threadIdx.x, float_as_ordered(m));
  }
}

// ------------------------------------------------------------------ quantise pass

template <bool SR>
__device__ __forceinline__ uint32_t encode8(const float* v, float r, uint4 w0, uint4 w1) {
  uint32_t packed = 0;
  const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float y = __fmul_rn(v[j], r);
    const uint32_t c = SR ? e2m1_sr(y, words[j]) : e2m1_rne(y);
    packed |= c << (4 * j);
  }
  return packed;
}

template <bool EMIT_ROW, bool EMIT_COL, bool SR, bool RHT_ROW, bool RHT_COL, bool TWO_D>
__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(QuantParams p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float amax_raw = p.amax[0];
  const float amax_col = RHT_COL ? p.amax[1] : amax_raw;
  const float amax_row = RHT_ROW ? p.amax[2] : amax_raw;
  const float S_row = tensor_scale_from_amax(amax_row);
  const float S_col = tensor_scale_from_amax(amax_col);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (EMIT_ROW) *p.row.tensor_scale = S_row;
    if (EMIT_COL) *p.col.tensor_scale = S_col;
    if (p.amax_out) {
      p.amax_out[0] = amax_raw;
      p.amax_out[1] = RHT_COL ? amax_col : 0.0f;
      p.amax_out[2] = RHT_ROW ? amax_row : 0.0f;
    }
  }
  const int64_t rows = p.rows, cols = p.cols;
  const int64_t row_groups = (rows + kSlabRows - 1) / kSlabRows;
  const int64_t chunks = (cols + kSlabCols - 1) / kSlabCols;
  const int64_t row_tiles = (row_groups + kQuantWarps - 1) / kQuantWarps;
  const int64_t tiles = row_tiles * chunks;
  const int64_t nblk_row = cols / 16, nblk_col = rows / 16;

  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
    const int64_t rt = t / chunks, ch = t - rt * chunks;
    const int64_t rg = rt * kQuantWarps + warp;
    if (rg >= row_groups) continue;                       // whole warp
    const int64_t r0 = rg * kSlabRows, c0 = ch * kSlabCols + lane * 8;
    const bool active = c0 < cols;
    const int nrows = (int)(rows - r0 < kSlabRows ? rows - r0 : kSlabRows);
    uint4 raw[16];
    load_slab(p.x, p.ld, r0, c0, nrows, active, raw);

    float tile_max = 0.0f;
    if (TWO_D) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float v[8];
        unpack8(raw[i], v);
        tile_max = fmaxf(tile_max, absmax8(v));
      }
      tile_max = fmaxf(tile_max, __shfl_xor_sync(0xFFFFFFFFu, tile_max, 1));
    }

    if (EMIT_ROW) {
      BlockScale tbs;
      if (TWO_D) tbs = block_scale(tile_max, S_row);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i >= nrows) break;                            // warp-uniform
        const int64_t r = r0 + i;
        float v[8];
        unpack8(raw[i], v);
        if (RHT_ROW) rht16_pair(v, p.signs, lane);
        BlockScale bs;
        if (TWO_D) {
          bs = tbs;
        } else {
          float m = absmax8(v);
          m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
          bs = block_scale(m, S_row);
        }
        uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
        if (SR) {
          const uint64_t ctr = (uint64_t)(r * cols + c0) >> 2;
          w0 = philox_block(ctr, 0u, p.offset, p.key0, p.key1);
          w1 = philox_block(ctr + 1, 0u, p.offset, p.key0, p.key1);
        }
        uint32_t packed = encode8<SR>(v, bs.r, w0, w1);
        if (bs.r == 0.0f) packed = 0u;                    // dead block: all-zero codes
        if (active) {
          *reinterpret_cast<uint32_t*>(p.row.codes + r * (cols / 2) + c0 / 2) = packed;
          if (!(lane & 1)) p.row.scales[scale_index(p.row, r, c0 / 16, nblk_row)] = (uint8_t)bs.sbyte;
        }
      }
    }

    if (EMIT_COL) {
      BlockScale tbs;
      if (TWO_D) tbs = block_scale(tile_max, S_col);
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = column_value(raw[i], j);
        if (RHT_COL) rht16(v, p.signs);
        BlockScale bs;
        if (TWO_D) {
          bs = tbs;
        } else {
          float m = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
          bs = block_scale(m, S_col);
        }
        const int64_t c = c0 + j;
        uint4 w[4] = {};
        if (SR) {
          const uint64_t ctr = (uint64_t)(c * rows + r0) >> 2;
#pragma unroll
          for (int q = 0; q < 4; ++q) w[q] = philox_block(ctr + q, 1u, p.offset, p.key0, p.key1);
        }
        uint32_t lo = encode8<SR>(v, bs.r, w[0], w[1]);
        uint32_t hi = encode8<SR>(v + 8, bs.r, w[2], w[3]);
        if (bs.r == 0.0f) lo = hi = 0u;
        if (active) {
          *reinterpret_cast<uint2*>(p.col.codes + c * (rows / 2) + r0 / 2) = make_uint2(lo, hi);
          p.col.scales[scale_index(p.col, c, r0 / 16, nblk_col)] = (uint8_t)bs.sbyte;
        }
      }
    }
  }
}

// ------------------------------------------------------------------ dequantiser

__device__ __forceinline__ float e2m1_value(uint32_t code) {
  const uint32_t idx = code & 7u;
  const float mag = idx < 4u ? __fmul_rn((float)idx, 0.5f) : (idx < 7u ? (float)idx - 2.0f : 6.0f);
  return (code & 8u) ? -mag : mag;
}

// One thread per 16-element block: out = (code * s) * S.
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t* __restrict__ codes,
                                                         const uint8_t* __restrict__ scales,
                                                         const float* __restrict__ tensor_scale, int64_t rows,
                                                         int64_t cols, int32_t mma_layout, int64_t kgroups,
                                                         void* out, int64_t ldo, int32_t out_f32) {
  const int64_t nblk = cols / 16;
  const int64_t total = rows * nblk;
  const float S = *tensor_scale;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < total; b += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = b / nblk, j = b - r * nblk;
    const uint2 c8 = *reinterpret_cast<const uint2*>(codes + r * (cols / 2) + j * 8);
    const uint32_t sb = scales[mma_layout ? mma_scale_offset(r, j, kgroups) : r * nblk + j];
    const float s = e4m3_decode(sb);
    float v[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const uint32_t code = ((t < 8 ? c8.x : c8.y) >> (4 * (t & 7))) & 0xFu;
      v[t] = __fmul_rn(__fmul_rn(e2m1_value(code), s), S);
    }
    if (out_f32) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + r * ldo + j * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
      uint32_t w[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) w[q] = f32_to_bf16_bits(v[2 * q]) | (f32_to_bf16_bits(v[2 * q + 1]) << 16);
      uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + r * ldo + j * 16);
      o[0] = make_uint4(w[0], w[1], w[2], w[3]);
      o[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
}

}  // namespace nvfp4
