// Kernels of the LoRA-SVD linear (nvfp4_lora_*): the weight is split as
// W = W_res + L R so that NVFP4 quantisation noise falls on the residual, and the
// rank-r part runs in BF16 ("Full-Stack FP4: Preentrenamiento Estable de LLM",
// linear-projection passage: a light LoRA-SVD decomposition that lowers the
// quantisation error of direct 4-bit quantisation).
//
//   lora_residual_kernel   W_res = BF16(fl32(W - s)), s = sum_j L[n][j] R[j][k]
//                          accumulated in FP32 in increasing j (each product of two
//                          BF16 values is exact in FP32, so a fused multiply-add
//                          rounds exactly as the separate product and sum would).
//   lowrank_project_kernel U = BF16(A B^T), A [M x K] BF16, B [r x K] (or given as
//                          [K x r]); HBM-bound on A.
//   lowrank_expand_kernel  Y = BF16(fl32(Y + U C^T)), U [M x r], C [N x r] (or given
//                          as [r x N]); HBM-bound on the read-modify-write of Y,
//                          persistent, with a ring of Y tiles in flight.
//
// The two products are dense contractions with a short side (r <= 64), so they run
// on the warp-level BF16 tensor-core MMA (m16n8k16, FP32 accumulation) from shared
// memory; the tiles are small and the work is bound by streaming A or Y, not by the
// MMA rate.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace nvfp4 {
namespace lowrank {

constexpr int kMaxRank = 64;
constexpr int kResidualThreads = 256;
constexpr int kResRows = 4;            // rows of W per residual thread
constexpr int kProjRows = 64;          // rows of A per CTA (4 warps x 16)
constexpr int kProjThreads = 128;
constexpr int kProjKc = 64;            // K per pipeline stage
constexpr int kProjStages = 4;
constexpr int kPad = 72;               // shared row stride in BF16 elements (144 B, conflict-free)
constexpr int kProjSmemBytes = kProjStages * (kProjRows + kMaxRank) * kPad * 2;
constexpr int kExpTile = 128;          // Y tile 128 x 128
constexpr int kExpThreads = 256;

// One warp-level BF16 MMA: d += a(16x16, row) * b(16x8, col), FP32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_pending() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ------------------------------------------------------------------ residual

// A thread computes 8 consecutive columns k of kResRows consecutive rows n, so each
// 16-byte load of R serves kResRows rows (row groups grid-stride over blockIdx.y).
// The products are exact barring FP32 underflow (BF16 factors below about 1e-19).
__global__ void __launch_bounds__(kResidualThreads) lora_residual_kernel(
    const uint16_t* __restrict__ w, int64_t ldw, const uint16_t* __restrict__ l, int64_t ldl,
    const uint16_t* __restrict__ r, int64_t ldr, uint16_t* __restrict__ out, int64_t ldo, int64_t N, int64_t K,
    int rank) {
  const int64_t k0 = ((int64_t)blockIdx.x * kResidualThreads + threadIdx.x) * 8;
  if (k0 >= K) return;
  for (int64_t n0 = (int64_t)blockIdx.y * kResRows; n0 < N; n0 += (int64_t)gridDim.y * kResRows) {
    float s[kResRows][8];
#pragma unroll
    for (int i = 0; i < kResRows; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) s[i][e] = 0.f;
    for (int j = 0; j < rank; ++j) {
      const uint4 rv = *reinterpret_cast<const uint4*>(r + (int64_t)j * ldr + k0);
      const float rf[8] = {bf16_lo(rv.x), bf16_hi(rv.x), bf16_lo(rv.y), bf16_hi(rv.y),
                           bf16_lo(rv.z), bf16_hi(rv.z), bf16_lo(rv.w), bf16_hi(rv.w)};
#pragma unroll
      for (int i = 0; i < kResRows; ++i) {
        const int64_t n = min(n0 + i, N - 1);           // rows past N compute row N-1 and are not stored
        const float lj = __uint_as_float((uint32_t)l[n * ldl + j] << 16);
#pragma unroll
        for (int e = 0; e < 8; ++e) s[i][e] = __fmaf_rn(lj, rf[e], s[i][e]);
      }
    }
#pragma unroll
    for (int i = 0; i < kResRows; ++i) {
      const int64_t n = n0 + i;
      if (n >= N) break;
      const uint4 wv = *reinterpret_cast<const uint4*>(w + n * ldw + k0);
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        o[e] = f32_to_bf16_bits(__fsub_rn(bf16_lo(ww[e]), s[i][2 * e])) |
               (f32_to_bf16_bits(__fsub_rn(bf16_hi(ww[e]), s[i][2 * e + 1])) << 16);
      *reinterpret_cast<uint4*>(out + n * ldo + k0) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// ------------------------------------------------------------------ U = BF16(A B^T)

// Two floats rounded to BF16 (nearest even, the hardware conversion) and packed, lo in
// the low half.
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t out;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(hi), "f"(lo));
  return out;
}

// Two BF16 values from shared memory packed as one MMA operand register, the first in
// the low half (the operand element with the lower K index).
__device__ __forceinline__ uint32_t pack_bf16_pair(const uint16_t* lo, const uint16_t* hi) {
  return (uint32_t)*lo | ((uint32_t)*hi << 16);
}

// RT = rank / 8 (n8 tiles).  CTA: 64 rows of A; warp w owns rows 16w..16w+15 and all
// rank columns.  K streams through a kProjStages-deep cp.async ring of 64-column
// chunks (dynamic shared memory, kProjSmemBytes), so about 24 KB of A is in flight per
// CTA.  B is staged as given: [r x K] rows (BT false) give each MMA operand register
// as one 32-bit load; [K x r] rows (BT true, e.g. L in dgrad) are staged unchanged and
// each register is packed from two 16-bit loads.
//
// With scale_a and scale_b given, the sums are divided by g = fl32(*scale_a * *scale_b)
// before the rounding: U' = BF16(fl32(fl32(sum) * fl32(1 / g))) -- the projection that
// joins an NVFP4 GEMM's accumulator, which that GEMM multiplies by g.
template <int RT, bool BT>
__global__ void __launch_bounds__(kProjThreads) lowrank_project_kernel(const uint16_t* __restrict__ a, int64_t lda,
                                                                       const uint16_t* __restrict__ b, int64_t ldb,
                                                                       int64_t K, uint16_t* __restrict__ u,
                                                                       int64_t ldu, const float* scale_a,
                                                                       const float* scale_b) {
  constexpr int R = RT * 8, RSn = R + 8;          // RSn: row stride of a staged [K x r] chunk
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint16_t (*As)[kProjRows][kPad] = reinterpret_cast<uint16_t (*)[kProjRows][kPad]>(smem_raw);
  uint16_t (*Bs)[kMaxRank][kPad] =
      reinterpret_cast<uint16_t (*)[kMaxRank][kPad]>(smem_raw + kProjStages * kProjRows * kPad * 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int64_t m0 = (int64_t)blockIdx.x * kProjRows;
  const int chunks = (int)(K / kProjKc);

  auto load = [&](int c, int buf) {
    const int64_t k0 = (int64_t)c * kProjKc;
#pragma unroll
    for (int i = 0; i < (kProjRows * 8) / kProjThreads; ++i) {
      const int idx = tid + i * kProjThreads, row = idx >> 3, ch = idx & 7;
      cp_async16(&As[buf][row][ch * 8], a + (m0 + row) * lda + k0 + ch * 8);
    }
    if constexpr (!BT) {
      for (int idx = tid; idx < R * 8; idx += kProjThreads) {
        const int j = idx >> 3, ch = idx & 7;
        cp_async16(&Bs[buf][j][ch * 8], b + (int64_t)j * ldb + k0 + ch * 8);
      }
    } else {
      uint16_t* bn = &Bs[buf][0][0];                 // [kProjKc][RSn] within the same stage buffer
      for (int idx = tid; idx < kProjKc * RT; idx += kProjThreads) {
        const int kr = idx / RT, jc = idx - kr * RT;
        cp_async16(bn + kr * RSn + jc * 8, b + (k0 + kr) * ldb + jc * 8);
      }
    }
  };

  float acc[RT][4];
#pragma unroll
  for (int nt = 0; nt < RT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

  // prologue: chunks 0 .. S-2, one commit group each (empty past the end)
#pragma unroll
  for (int c = 0; c < kProjStages - 1; ++c) {
    if (c < chunks) load(c, c);
    cp_async_commit();
  }
  for (int c = 0; c < chunks; ++c) {
    cp_async_wait_pending<kProjStages - 2>();         // chunk c has landed (this thread's copies)
    __syncthreads();                                  // ... everyone's; chunk c-1's buffer is free
    const int nc = c + kProjStages - 1;
    if (nc < chunks) load(nc, nc % kProjStages);
    cp_async_commit();
    const int buf = c % kProjStages;
    const int r0 = warp * 16 + g;
#pragma unroll
    for (int kk = 0; kk < kProjKc / 16; ++kk) {
      const int kc = kk * 16 + 2 * t;
      uint32_t af[4];
      af[0] = *reinterpret_cast<const uint32_t*>(&As[buf][r0][kc]);
      af[1] = *reinterpret_cast<const uint32_t*>(&As[buf][r0 + 8][kc]);
      af[2] = *reinterpret_cast<const uint32_t*>(&As[buf][r0][kc + 8]);
      af[3] = *reinterpret_cast<const uint32_t*>(&As[buf][r0 + 8][kc + 8]);
#pragma unroll
      for (int nt = 0; nt < RT; ++nt) {
        uint32_t bfr[2];
        if constexpr (!BT) {
          bfr[0] = *reinterpret_cast<const uint32_t*>(&Bs[buf][nt * 8 + g][kc]);
          bfr[1] = *reinterpret_cast<const uint32_t*>(&Bs[buf][nt * 8 + g][kc + 8]);
        } else {
          const uint16_t* bn = &Bs[buf][0][0] + nt * 8 + g;
          bfr[0] = pack_bf16_pair(bn + kc * RSn, bn + (kc + 1) * RSn);
          bfr[1] = pack_bf16_pair(bn + (kc + 8) * RSn, bn + (kc + 9) * RSn);
        }
        mma_bf16_16816(acc[nt], af, bfr);
      }
    }
  }
  cp_async_wait_pending<0>();
  const int64_t row = m0 + warp * 16 + g;
  if (scale_a) {
    const float inv = __fdiv_rn(1.0f, __fmul_rn(*scale_a, *scale_b));
#pragma unroll
    for (int nt = 0; nt < RT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = __fmul_rn(acc[nt][e], inv);
  }
#pragma unroll
  for (int nt = 0; nt < RT; ++nt) {
    const int col = nt * 8 + 2 * t;
    *reinterpret_cast<uint32_t*>(u + row * ldu + col) = pack_bf16x2_rn(acc[nt][0], acc[nt][1]);
    *reinterpret_cast<uint32_t*>(u + (row + 8) * ldu + col) = pack_bf16x2_rn(acc[nt][2], acc[nt][3]);
  }
}

// ------------------------------------------------------------------ Y = BF16(Y + U C^T)

// Ring depth of the expansion and its shared-memory bytes per stage: the staged Y tile
// (128 x 136 BF16), the U tile and the C tile (128 x (r + 8) BF16 each; a C given as
// [r x N] takes r x 136 of that space).
template <int KS>
__host__ __device__ constexpr int exp_stages() { return KS <= 2 ? 4 : 3; }
constexpr int kYStride = kExpTile + 8;
template <int KS>
__host__ __device__ constexpr int exp_stage_bytes() { return kExpTile * kYStride * 2 + 2 * kExpTile * (KS * 16 + 8) * 2; }
template <int KS>
__host__ __device__ constexpr int exp_smem_bytes() { return exp_stages<KS>() * exp_stage_bytes<KS>(); }

// KS = rank / 16 (k16 steps).  Persistent: CTA b takes the 128 x 128 tiles b, b + G,
// ... of Y (G = gridDim.x, N tiles fastest) through a ring of exp_stages() stages, so
// the Y tiles of the next stages stream in (cp.async) while one is computed.  Per
// tile: warp w multiplies rows 32(w/2).. by columns 64(w%2).. (r/16 MMAs of m16n8k16
// per 16 x 8 block), adds its FP32 results into the staged BF16 Y in place (each
// element belongs to one lane), and the CTA writes the tile back in 16-byte chunks.
// C is staged as given: [N x r] rows (CT false) or [r x N] rows (CT true, e.g. R^T in
// dgrad), whose MMA operand registers are packed from two 16-bit loads.
template <int KS, bool CT>
__global__ void __launch_bounds__(kExpThreads) lowrank_expand_kernel(uint16_t* __restrict__ y, int64_t ldy,
                                                                     const uint16_t* __restrict__ u, int64_t ldu,
                                                                     const uint16_t* __restrict__ c, int64_t ldc,
                                                                     int32_t tiles_n, int32_t tiles) {
  constexpr int R = KS * 16, RS = R + 8, S = exp_stages<KS>();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int wm = (warp >> 1) * 32, wn = (warp & 1) * 64;
  auto Ys = [&](int st) { return reinterpret_cast<uint16_t (*)[kYStride]>(smem_raw + st * exp_stage_bytes<KS>()); };
  auto Us = [&](int st) {
    return reinterpret_cast<uint16_t (*)[RS]>(smem_raw + st * exp_stage_bytes<KS>() + kExpTile * kYStride * 2);
  };
  auto Cs = [&](int st) {
    return reinterpret_cast<uint16_t (*)[RS]>(smem_raw + st * exp_stage_bytes<KS>() + kExpTile * kYStride * 2 +
                                              kExpTile * RS * 2);
  };

  auto load = [&](int tile, int st) {
    const int64_t m0 = (int64_t)(tile / tiles_n) * kExpTile, n0 = (int64_t)(tile % tiles_n) * kExpTile;
    uint16_t (*ys)[kYStride] = Ys(st);
    uint16_t (*us)[RS] = Us(st);
    uint16_t (*cs)[RS] = Cs(st);
#pragma unroll
    for (int i = 0; i < (kExpTile * kExpTile / 8) / kExpThreads; ++i) {
      const int idx = tid + i * kExpThreads, row = idx >> 4, ch = idx & 15;
      cp_async16(&ys[row][ch * 8], y + (m0 + row) * ldy + n0 + ch * 8);
    }
    for (int idx = tid; idx < kExpTile * (R / 8); idx += kExpThreads) {
      const int row = idx / (R / 8), ch = idx - row * (R / 8);
      cp_async16(&us[row][ch * 8], u + (m0 + row) * ldu + ch * 8);
    }
    if constexpr (!CT) {
      for (int idx = tid; idx < kExpTile * (R / 8); idx += kExpThreads) {
        const int row = idx / (R / 8), ch = idx - row * (R / 8);
        cp_async16(&cs[row][ch * 8], c + (n0 + row) * ldc + ch * 8);
      }
    } else {
      uint16_t* cn = &cs[0][0];                      // [R][kYStride] within the same stage buffer
      for (int idx = tid; idx < R * (kExpTile / 8); idx += kExpThreads) {
        const int j = idx / (kExpTile / 8), ch = idx - j * (kExpTile / 8);
        cp_async16(cn + j * kYStride + ch * 8, c + (int64_t)j * ldc + n0 + ch * 8);
      }
    }
  };

  const int first = blockIdx.x, step = gridDim.x;
#pragma unroll
  for (int k = 0; k < S - 1; ++k) {
    const int tile = first + k * step;
    if (tile < tiles) load(tile, k);
    cp_async_commit();
  }
  for (int k = 0;; ++k) {
    const int tile = first + k * step;
    if (tile >= tiles) break;
    const int st = k % S;
    cp_async_wait_pending<S - 2>();                   // tile k has landed (this thread's copies)
    __syncthreads();                                  // ... everyone's; the stage of tile k-1 is free
    const int ahead = first + (k + S - 1) * step;
    if (ahead < tiles) load(ahead, (k + S - 1) % S);
    cp_async_commit();

    uint16_t (*ys)[kYStride] = Ys(st);
    uint16_t (*us)[RS] = Us(st);
    uint16_t (*cs)[RS] = Cs(st);
    float acc[2][8][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
#pragma unroll 1
    for (int ks = 0; ks < KS; ++ks) {
      const int kc = ks * 16 + 2 * t;
      uint32_t af[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int r0 = wm + mt * 16 + g;
        af[mt][0] = *reinterpret_cast<const uint32_t*>(&us[r0][kc]);
        af[mt][1] = *reinterpret_cast<const uint32_t*>(&us[r0 + 8][kc]);
        af[mt][2] = *reinterpret_cast<const uint32_t*>(&us[r0][kc + 8]);
        af[mt][3] = *reinterpret_cast<const uint32_t*>(&us[r0 + 8][kc + 8]);
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        uint32_t bfr[2];
        if constexpr (!CT) {
          bfr[0] = *reinterpret_cast<const uint32_t*>(&cs[wn + nt * 8 + g][kc]);
          bfr[1] = *reinterpret_cast<const uint32_t*>(&cs[wn + nt * 8 + g][kc + 8]);
        } else {
          const uint16_t* cn = &cs[0][0] + wn + nt * 8 + g;
          bfr[0] = pack_bf16_pair(cn + kc * kYStride, cn + (kc + 1) * kYStride);
          bfr[1] = pack_bf16_pair(cn + (kc + 8) * kYStride, cn + (kc + 9) * kYStride);
        }
        mma_bf16_16816(acc[0][nt], af[0], bfr);
        mma_bf16_16816(acc[1][nt], af[1], bfr);
      }
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t* p = reinterpret_cast<uint32_t*>(&ys[wm + mt * 16 + g + 8 * h][wn + nt * 8 + 2 * t]);
          const uint32_t old = *p;
          *p = pack_bf16x2_rn(__fadd_rn(bf16_lo(old), acc[mt][nt][2 * h]),
                              __fadd_rn(bf16_hi(old), acc[mt][nt][2 * h + 1]));
        }
    __syncthreads();
    const int64_t m0 = (int64_t)(tile / tiles_n) * kExpTile, n0 = (int64_t)(tile % tiles_n) * kExpTile;
#pragma unroll
    for (int i = 0; i < (kExpTile * kExpTile / 8) / kExpThreads; ++i) {
      const int idx = tid + i * kExpThreads, row = idx >> 4, ch = idx & 15;
      __stcs(reinterpret_cast<uint4*>(y + (m0 + row) * ldy + n0 + ch * 8),
             *reinterpret_cast<const uint4*>(&ys[row][ch * 8]));
    }
  }
  cp_async_wait_pending<0>();
}

}  // namespace lowrank
}  // namespace nvfp4
