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
//                          [K x r]); HBM-bound on A: persistent, one CTA per SM,
//                          each CTA a balanced run of 16-row units, A and B
//                          streamed by TMA through a deep ring.
//   lowrank_expand_kernel  Y = BF16(fl32(Y + U C^T)), U [M x r], C [N x r] (or given
//                          as [r x N]); HBM-bound on the read-modify-write of Y,
//                          persistent, with a ring of Y tiles in flight.
//
// The two products are dense contractions with a short side (r <= 64), so they run
// on the warp-level BF16 tensor-core MMA (m16n8k16, FP32 accumulation) from shared
// memory; the work is bound by streaming A or Y, not by the MMA rate, and the 16-row
// granularity of the warp-level MMA lets the projection split M evenly over the SMs.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace nvfp4 {
namespace lowrank {

constexpr int kMaxRank = 64;
constexpr int kResidualThreads = 256;
constexpr int kResRows = 4;            // rows of W per residual thread
constexpr int kProjUnit = 16;          // rows of A per work unit (one m16 MMA row block)
constexpr int kProjUnits = 8;          // units a CTA holds at once, one consumer warp each
constexpr int kProjThreads = 32 * (1 + kProjUnits);   // TMA producer warp + consumer warps
constexpr int kProjKc = 64;            // K per TMA box (128 bytes of BF16: one swizzle row)
constexpr int kProjBoxBytes = kProjUnit * 128;                        // 2 KB: one A box
constexpr int kProjBBytes = 64 * 128;                                 // B box, at most 64 rows x 128 B
constexpr int kProjBoxSets = 8;        // ring capacity in sets of (kProjUnits A boxes + one B box)
constexpr int kProjSetBytes = kProjUnits * kProjBoxBytes + kProjBBytes;   // 24 KB
constexpr int kProjBarOffset = kProjBoxSets * kProjSetBytes;          // 192 KB of ring
constexpr int kProjSmemBytes = kProjBarOffset + 256 + 1024;           // ring, barriers, alignment slack
// Boxes along K per unit and stage (H; each row is then read 128 * H contiguous bytes
// per stage) and ring depth kProjBoxSets / H.  Measured at the 12B shapes: H = 4 (two
// stages) for B given as [K x r] (the dgrad projection dY L, 671 MB of A), H = 2 (four
// stages) for B as [r x K] (X R^T, 168 MB).
template <bool BT>
__host__ __device__ constexpr int proj_halves() { return BT ? 4 : 2; }
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

// Four 8x8 BF16 matrices from shared memory (lane l gives the address of row l % 8 of
// matrix l / 8); .trans delivers each transposed.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Shared address of 16-byte chunk `chunk` of row `row` in a box written by TMA with the
// 128-byte swizzle (rows of 128 bytes, 1024-byte aligned box): the chunk index is
// XORed with row % 8.
__device__ __forceinline__ uint32_t sw128_addr(uint32_t box, int row, int chunk) {
  return box + (uint32_t)(row * 128) + (uint32_t)(((chunk ^ row) & 7) << 4);
}

__device__ __forceinline__ void proj_tma_load(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// RT = rank / 8 (n8 tiles).  A persistent CTA owns the 16-row units [u0, u1) of A, an
// even split of the M / 16 units over the grid, and takes them kProjUnits at a time:
// warp 1 + j computes unit j of the group for all r columns while warp 0 streams the
// group's K range through a ring of 64H-column chunks (H = proj_halves: per chunk H
// 16 x 64 TMA boxes per unit, adjacent along K so that each row is read 128H bytes at
// a time, and H boxes of B; 128-byte swizzle).  K need not be a multiple of 64H: the
// boxes of a last partial chunk lie past K and TMA fills them with zeros.  Operand registers come
// from ldmatrix: A and B given as [r x K] row-major, B given as [K x r] (BT, e.g. L in
// dgrad) transposed on the way.  B boxes are 64 columns wide; with BT the columns past
// r are zero-filled by TMA and never read.
//
// With scale_a and scale_b given, the sums are divided by g = fl32(*scale_a * *scale_b)
// before the rounding: U' = BF16(fl32(fl32(sum) * fl32(1 / g))) -- the projection that
// joins an NVFP4 GEMM's accumulator, which that GEMM multiplies by g.
template <int RT, bool BT>
__global__ void __launch_bounds__(kProjThreads, 1)
    lowrank_project_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                           int64_t units, int32_t chunks, uint16_t* __restrict__ u, int64_t ldu,
                           const float* scale_a, const float* scale_b) {
  constexpr int R = RT * 8;
  constexpr uint32_t kBBoxBytes = BT ? (uint32_t)kProjBBytes : (uint32_t)(R * 128);
  constexpr int kProjHalves = proj_halves<BT>();
  constexpr int kProjStages = kProjBoxSets / kProjHalves;
  constexpr int kProjStageBytes = kProjHalves * kProjSetBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t base = smem_u32(smem);
  const uint32_t bar_base = base + kProjBarOffset;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kProjBarOffset + 16 * kProjStages);
  auto full_bar = [&](int st) { return bar_base + 8u * st; };
  auto empty_bar = [&](int st) { return bar_base + 8u * (kProjStages + st); };
  auto a_box = [&](int st, int h, int j) {
    return base + (uint32_t)(st * kProjStageBytes + (h * kProjUnits + j) * kProjBoxBytes);
  };
  auto b_box = [&](int st, int h) {
    return base + (uint32_t)(st * kProjStageBytes + kProjHalves * kProjUnits * kProjBoxBytes + h * kProjBBytes);
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kProjStages; ++st) {
      mbar_init(full_bar(st), 1);
      mbar_init(empty_bar(st), kProjUnits);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  const int64_t u0 = (int64_t)blockIdx.x * units / gridDim.x;
  const int64_t u1 = (int64_t)(blockIdx.x + 1) * units / gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop; one elected lane arms the barrier and issues the copies.
    {
      int st = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool issued[kProjStages] = {};
      uint32_t issued_phase[kProjStages] = {};
      for (int64_t g0 = u0; g0 < u1 && ok; g0 += kProjUnits) {
        const int nu = (int)(u1 - g0 < kProjUnits ? u1 - g0 : kProjUnits);
        for (int c = 0; c < chunks; ++c) {
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(empty_bar(st), phase ^ 1u, abort_flag))) {
            ok = false;
            break;
          }
          if (elect_one()) {
            mbar_arrive_expect_tx(full_bar(st),
                                  (uint32_t)kProjHalves * ((uint32_t)(nu * kProjBoxBytes) + kBBoxBytes));
            for (int j = 0; j < nu; ++j)
              for (int h = 0; h < kProjHalves; ++h)
                proj_tma_load(a_box(st, h, j), &amap, (c * kProjHalves + h) * kProjKc,
                              (int32_t)((g0 + j) * kProjUnit), full_bar(st));
            for (int h = 0; h < kProjHalves; ++h) {
              if (BT)
                proj_tma_load(b_box(st, h), &bmap, 0, (c * kProjHalves + h) * kProjKc, full_bar(st));
              else
                proj_tma_load(b_box(st, h), &bmap, (c * kProjHalves + h) * kProjKc, 0, full_bar(st));
            }
          }
          __syncwarp();
          issued[st] = true;
          issued_phase[st] = phase;
          if (++st == kProjStages) {
            st = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // wind down: let every load already issued land before the CTA exits
        for (int k = 0; k < kProjStages; ++k) {
          if (!issued[k]) continue;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(full_bar(k), issued_phase[k]) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumer warps
  const int j = warp - 1;                        // unit of the group
  const int g = lane >> 2, t = lane & 3;
  float inv = 1.0f;
  if (scale_a) inv = __fdiv_rn(1.0f, __fmul_rn(*scale_a, *scale_b));
  // ldmatrix lane roles: A (16 x 16 per k-step): row lane % 16, k half lane / 16;
  // B [r x K]: row 8 * (lane / 16) + lane % 8 of an n8 pair, k half (lane / 8) % 2;
  // B [K x r] (transposed): k row lane % 16, n tile of the pair lane / 16.
  const int a_row = lane & 15, a_half = lane >> 4;
  const int b_row = (lane & 7) + ((lane >> 4) << 3), b_half = (lane >> 3) & 1;
  int st = 0;
  uint32_t phase = 0;
  bool ok = true;
  for (int64_t g0 = u0; g0 < u1 && ok; g0 += kProjUnits) {
    const int nu = (int)(u1 - g0 < kProjUnits ? u1 - g0 : kProjUnits);
    const bool active = j < nu;
    float acc[RT][4];
#pragma unroll
    for (int nt = 0; nt < RT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    for (int c = 0; c < chunks; ++c) {
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(full_bar(st), phase, abort_flag));
      if (!ok) break;
      if (active) {
#pragma unroll
        for (int k16 = 0; k16 < kProjHalves * kProjKc / 16; ++k16) {
          const int kk = k16 % (kProjKc / 16);
          const uint32_t abox = a_box(st, k16 / (kProjKc / 16), j), bbox = b_box(st, k16 / (kProjKc / 16));
          uint32_t af[4];
          ldsm_x4(sw128_addr(abox, a_row, 2 * kk + a_half), af);
#pragma unroll
          for (int np = 0; np < RT / 2; ++np) {
            uint32_t bf[4];                      // b0, b1 of n tile 2np, then of 2np + 1
            if constexpr (!BT) {
              ldsm_x4(sw128_addr(bbox, 16 * np + b_row, 2 * kk + b_half), bf);
            } else {
              const int krow = 16 * kk + (lane & 15);
              uint32_t tr[4];
              ldsm_x4_trans(sw128_addr(bbox, krow, 2 * np + (lane >> 4)), tr);
              bf[0] = tr[0], bf[1] = tr[1], bf[2] = tr[2], bf[3] = tr[3];
            }
            mma_bf16_16816(acc[2 * np], af, bf);
            mma_bf16_16816(acc[2 * np + 1], af, bf + 2);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(st));
      if (++st == kProjStages) {
        st = 0;
        phase ^= 1u;
      }
    }
    if (!ok || !active) continue;
    const int64_t row = (g0 + j) * kProjUnit + g;
    if (scale_a) {
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
