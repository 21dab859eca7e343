// Block-scaled NVFP4 GEMM for sm_100a: C = alpha * S_A * S_B * A . B^T.
//
// The performance passage of "Preentrenamiento de 4 bits con NVFP4 en un hibrido
// Mamba-Transformer de 12B" rests on the FP4 tensor-core GEMM; "Full-Stack FP4"
// notes how fast error accumulates in low-precision products, so the
// accumulator is FP32 in tensor memory and the global scales are applied once,
// in the epilogue.
//
// Two kernels.  gemm_kernel_pair (further below) serves M >= 256, and M = 128 while
// its tiles fit one wave of pairs: CTA pairs (cta_group::2) on 256 x 256 output
// tiles, block scales stored into tensor memory by writer warps, two MMA-issuing
// warps, output through TMA stores.  gemm_kernel serves the other 128-row problems
// and devices that cannot co-schedule a pair.  In both, a role warp runs its loop as
// a whole warp and issues single-thread operations (TMA copies, barrier arming,
// MMAs, commits) from one elected lane with warp-uniform operands.
//
// Structure (one CTA per SM, persistent over output tiles of 128 x 256):
//   warp 0      TMA producer: per K-stage of 256 elements, one tiled TMA load of
//               A (128 rows x 128 bytes) and of B (256 x 128 bytes), 128-byte
//               swizzled, plus bulk copies of the matching block-scale tiles
//               (already in the tensor-core order, 512 bytes per 128 rows x 64 K).
//   warp 1      MMA issuer (one elected lane): copies each stage's scales into tensor
//               memory (tcgen05.cp) and issues four tcgen05.mma kind::mxf4nvf4
//               block16 (M=128, N=256, K=64) into an FP32 accumulator in tensor
//               memory; tcgen05.commit frees the stage and, after the last one,
//               hands the accumulator to the epilogue.
//   warps 2..9  epilogue: tcgen05.ld of their 32-lane quarter of the
//               accumulator, scale by alpha*S_A*S_B, round to BF16 (or keep FP32),
//               store; then release the accumulator.
// All waits are bounded (see mbar_wait): a stuck pipeline records an error
// and the CTA winds down instead of hanging.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace nvfp4 {
namespace gemm {

constexpr int BM = 128;                 // rows of A per tile (MMA M)
constexpr int BN = 256;                 // rows of B per tile (MMA N)
constexpr int BK = 256;                 // K elements per pipeline stage
constexpr int BK_BYTES = BK / 2;        // 128: one 128-byte swizzle row
constexpr int MMA_K = 64;               // K per tcgen05.mma (kind::mxf4nvf4)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK_BYTES;                        // 16 KiB
constexpr int B_BYTES = BN * BK_BYTES;                        // 32 KiB
constexpr int SF_ATOM = 512;                                  // 128 rows x 4 scales
constexpr int SFA_BYTES = (BM / 128) * (BK / MMA_K) * SF_ATOM;  // 2 KiB
constexpr int SFB_BYTES = (BN / 128) * (BK / MMA_K) * SF_ATOM;  // 4 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COL = 0;              // 256 FP32 columns
constexpr int SFA_COL = 256;            // 4 columns per MMA k-step -> 16
constexpr int SFB_COL = 256 + 16;       // 8 columns per MMA k-step -> 32
constexpr int EPI_WARP0 = 2;
constexpr int NUM_EPI_WARPS = 8;                  // two per tensor-memory lane quarter
constexpr int NUM_THREADS = 32 * (EPI_WARP0 + NUM_EPI_WARPS);
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;

struct Params {
  int32_t M, N, K;
  int32_t num_m, num_n, num_k_stages, tail_atoms;   // tail_atoms: MMA k-steps in the last stage
  int32_t group_m;
  const uint8_t* sfa;       // tensor-core scale layout of A
  const uint8_t* sfb;
  int64_t sf_kgroups;       // 64-element K groups per 128-row scale block of B (= K / 64)
  int64_t sf_kgroups_a;     // the same for A
  const float* scale_a;
  const float* scale_b;
  float alpha;
  void* C;
  int64_t ldc;
  int32_t out_f32;
  int32_t accumulate;
  unsigned* amax_acc;       // nullptr, or 2 words receiving max|C| and max|RHT16 col(C)| (float bits)
  uint32_t rht_signs;       // sign mask of that transform
  int64_t skip_stage;       // fault injection (pair kernel): CTA pair 0 never loads its K-stage
                            // number skip_stage (counted over all its tiles); -1: off
  int32_t lr_ksteps;        // pair kernel: BF16 MMAs (K = 16 each) of the low-rank stage that ends
                            // every tile, accumulating U V^T into the same accumulator; 0: none
};

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1), UE4M3
// scales, K-major operands, M = 128, N = n, dense K = 64.
__host__ __device__ constexpr uint32_t make_idesc(int n) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | (uint32_t)(BM >> 4) << 24;
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Descriptor of one 512-byte scale tile as tcgen05.cp 32x128b source: 32 rows
// of 16 bytes, no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_copy_scales(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate, uint32_t sfa_tmem, uint32_t sfb_tmem) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 32 lanes x 32 columns of 32-bit accumulator: lane i of the warp gets row i.
// Asynchronous: the registers are valid after tc_wait_loads().
__device__ __forceinline__ void tc_load_32cols(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tc_wait_loads() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }


// Scale 32 accumulator columns by g and store them (BF16 or FP32, optionally
// adding the existing values) at crow (row-major C, 16-byte aligned).
__device__ __forceinline__ void store_32cols(const Params& p, const uint32_t* r, float g, void* crow_v) {
  if (p.out_f32) {
    float* crow = static_cast<float*>(crow_v);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 v = make_float4(__fmul_rn(__uint_as_float(r[4 * q]), g), __fmul_rn(__uint_as_float(r[4 * q + 1]), g),
                             __fmul_rn(__uint_as_float(r[4 * q + 2]), g), __fmul_rn(__uint_as_float(r[4 * q + 3]), g));
      if (p.accumulate) {
        const float4 o = reinterpret_cast<const float4*>(crow)[q];
        v.x = __fadd_rn(v.x, o.x);
        v.y = __fadd_rn(v.y, o.y);
        v.z = __fadd_rn(v.z, o.z);
        v.w = __fadd_rn(v.w, o.w);
      }
      reinterpret_cast<float4*>(crow)[q] = v;
    }
  } else {
    uint16_t* crow = static_cast<uint16_t*>(crow_v);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t w[4];
      uint4 old = make_uint4(0u, 0u, 0u, 0u);
      if (p.accumulate) old = reinterpret_cast<const uint4*>(crow)[q];
      const uint32_t oldw[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v0 = __fmul_rn(__uint_as_float(r[8 * q + 2 * e]), g);
        float v1 = __fmul_rn(__uint_as_float(r[8 * q + 2 * e + 1]), g);
        if (p.accumulate) {
          v0 = __fadd_rn(v0, bf16_lo(oldw[e]));
          v1 = __fadd_rn(v1, bf16_hi(oldw[e]));
        }
        w[e] = f32_to_bf16_bits(v0) | (f32_to_bf16_bits(v1) << 16);
      }
      reinterpret_cast<uint4*>(crow)[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// Wait with a time limit only (teardown after an abort).
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_error_word, kErrTimeout);
      return;
    }
  }
}

struct TileCoord {
  int32_t m_blk, n_blk;
};

// Grouped rasterisation: runs of group_m row-blocks sweep all column blocks, so
// the CTAs in flight share their A and B tiles through L2.
__device__ __forceinline__ TileCoord tile_coord(const Params& p, int32_t t) {
  const int32_t per_group = p.group_m * p.num_n;
  const int32_t g = t / per_group, w = t - g * per_group;
  const int32_t m_first = g * p.group_m;
  const int32_t gm = min(p.group_m, p.num_m - m_first);
  TileCoord c;
  c.m_blk = m_first + w % gm;
  c.n_blk = w / gm;
  return c;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t smem_base = smem_u32(smem);
  uint8_t* bar_area = smem + STAGES * STAGE_BYTES;
  const uint32_t bar_base = smem_u32(bar_area);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  const uint32_t acc_full = bar_base + 8u * (2 * STAGES);
  const uint32_t acc_empty = bar_base + 8u * (2 * STAGES + 1);
  const uint32_t mma_done = bar_base + 8u * (2 * STAGES + 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_area + 8 * (2 * STAGES + 3));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 8 * (2 * STAGES + 3) + 4);

  auto a_smem = [&](int s) { return smem_base + (uint32_t)(s * STAGE_BYTES); };
  auto b_smem = [&](int s) { return smem_base + (uint32_t)(s * STAGE_BYTES + A_BYTES); };
  auto sfa_smem = [&](int s) { return smem_base + (uint32_t)(s * STAGE_BYTES + A_BYTES + B_BYTES); };
  auto sfb_smem = [&](int s) { return smem_base + (uint32_t)(s * STAGE_BYTES + A_BYTES + B_BYTES + SFA_BYTES); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, NUM_EPI_WARPS);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int32_t num_tiles = p.num_m * p.num_n;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop; one elected lane arms the barrier and issues the copies.
    {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_phase[STAGES];
      bool issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_phase[s] = 0;
      bool ok = true;
      for (int32_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_coord(p, t);
        const int nb_valid = min(2, (p.N - tc.n_blk * BN) / 128);
        for (int ks = 0; ks < p.num_k_stages; ++ks) {
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag))) {
            ok = false;
            break;
          }
          const int atoms = (ks == p.num_k_stages - 1) ? p.tail_atoms : BK / MMA_K;
          const uint32_t sf_bytes = (uint32_t)atoms * SF_ATOM;
          const int64_t kg = (int64_t)ks * (BK / MMA_K);
          if (elect_one()) {
            mbar_arrive_expect_tx(full_bar(stage), (uint32_t)(A_BYTES + B_BYTES) + sf_bytes * (1u + nb_valid));
            tma_load_2d(a_smem(stage), &tma_a, ks * BK_BYTES, tc.m_blk * BM, full_bar(stage));
            tma_load_2d(b_smem(stage), &tma_b, ks * BK_BYTES, tc.n_blk * BN, full_bar(stage));
            bulk_load(sfa_smem(stage), p.sfa + ((int64_t)tc.m_blk * p.sf_kgroups + kg) * SF_ATOM, sf_bytes,
                      full_bar(stage));
            for (int nb = 0; nb < nb_valid; ++nb)
              bulk_load(sfb_smem(stage) + nb * (BK / MMA_K) * SF_ATOM,
                        p.sfb + ((int64_t)(tc.n_blk * 2 + nb) * p.sf_kgroups + kg) * SF_ATOM, sf_bytes,
                        full_bar(stage));
          }
          __syncwarp();
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // wind down: let every load already issued land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) mbar_wait_drain(full_bar(s), issued_phase[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and computes the operands (warp-uniform); one
    // elected lane issues the scale copies, the MMAs and the commits.
    {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int32_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_coord(p, t);
        const int nb_valid = min(2, (p.N - tc.n_blk * BN) / 128);
        const uint32_t idesc = make_idesc(nb_valid * 128);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int ks = 0; ks < p.num_k_stages; ++ks) {
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(full_bar(stage), phase, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int atoms = (ks == p.num_k_stages - 1) ? p.tail_atoms : BK / MMA_K;
          const uint64_t a_desc0 = sw128_desc(a_smem(stage)), b_desc0 = sw128_desc(b_smem(stage));
          if (elect_one()) {
            for (int kk = 0; kk < atoms; ++kk) {
              tc_copy_scales(tmem + SFA_COL + 4 * kk, sf_desc(sfa_smem(stage) + kk * SF_ATOM));
              for (int nb = 0; nb < nb_valid; ++nb)
                tc_copy_scales(tmem + SFB_COL + 8 * kk + 4 * nb,
                               sf_desc(sfb_smem(stage) + (nb * (BK / MMA_K) + kk) * SF_ATOM));
              tc_mma(tmem + ACC_COL, a_desc0 + (uint64_t)(kk * (MMA_K / 2 / 16)),
                     b_desc0 + (uint64_t)(kk * (MMA_K / 2 / 16)), idesc, (ks | kk) != 0 ? 1u : 0u,
                     tmem + SFA_COL + 4 * kk, tmem + SFB_COL + 8 * kk);
            }
            tc_commit(empty_bar(stage));
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (elect_one()) tc_commit(acc_full);
        __syncwarp();
        acc_phase ^= 1u;
      }
      // every MMA issued by the elected lanes has finished once mma_done flips
      if (elect_one()) tc_commit(mma_done);
      __syncwarp();
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp w reads tensor-memory lanes 32*(w%4).. (its hardware lane quarter)
    // and one half of the 256 accumulator columns.  It copies its whole share to
    // registers, hands the accumulator back to the MMA warp at once, and then
    // scales, converts and stores while the next tile's main loop runs.
    const int ew = warp - EPI_WARP0;               // 0..7
    const int quarter = warp & 3;
    const int half = ew >> 2;                      // accumulator columns 128*half ..
    const int row_in_tile = quarter * 32 + lane;
    const float g = __fmul_rn(__fmul_rn(*p.scale_a, *p.scale_b), p.alpha);
    uint32_t acc_phase = 0;
    for (int32_t t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const TileCoord tc = tile_coord(p, t);
      const int n_cols = min(BN, p.N - tc.n_blk * BN);
      const bool mine = n_cols > half * 128;
      // every lane polls; the warp proceeds (converged) only if all saw the phase complete
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, acc_phase, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t r[128];
      if (mine) {
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + ACC_COL + half * 128;
#pragma unroll
        for (int k = 0; k < 4; ++k) tc_load_32cols(taddr + 32 * k, r + 32 * k);
        tc_wait_loads();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1u;
      if (mine) {
        const int64_t m = (int64_t)tc.m_blk * BM + row_in_tile;
        const int64_t n0 = (int64_t)tc.n_blk * BN + half * 128;
        const size_t esz = p.out_f32 ? 4 : 2;
        uint8_t* crow = static_cast<uint8_t*>(p.C) + (size_t)(m * p.ldc + n0) * esz;
#pragma unroll
        for (int k = 0; k < 4; ++k) store_32cols(p, r + 32 * k, g, crow + (size_t)32 * k * esz);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}


// =====================================================================================
// CTA-pair variant (cta_group::2): one 256 x 256 output tile per pair of SMs.
//
// CTA r of the pair (r = 0 leads) loads A rows 128r.. of the tile, B rows 128r..
// (its half of N), the block scales of its A rows and the scales of all 256 B
// rows; the leader alone issues tcgen05.mma with cta_group::2 (M = 256, N = 256,
// K = 64), which reads each CTA's shared memory at the same offsets and
// accumulates rows 128r.. of the tile in CTA r's tensor memory.  Each CTA streams
// 38 KB per K-stage (the single-CTA kernel streams 54 KB for half the work), so a
// 5-stage ring covers more memory latency.  All loads are TMA tile loads without
// multicast; the pair's operand loads complete on the leader's stage barrier, each
// CTA's scale loads on its own; the leader's commits arrive on both CTAs' barriers.
//
// Block scales reach tensor memory through tcgen05.st from four scale-writer warps
// per CTA (one per 32-lane quarter), not through tcgen05.cp from the MMA thread:
// measured with copies and MMAs issued from a lane == 0 branch, copies between the
// MMAs stretched each M256N256K64 MMA from 128 to about 275 cycles on random
// operands, while stores from other warps left the MMA stream at 128.  Each operand stage has its own scale slot in tensor memory (48
// columns: 16 of A scales, 32 of B scales), freed with the stage.  The layout
// written is the one a 32x128b.warpx4 copy of the 512-byte scale tile gives:
// every quarter holds the same 32 lanes x 4 columns per tile.  The scales stream
// through a shared-memory ring of their own, deeper than the operand ring and fed
// by a second producer warp, so that a stage's scales are in shared memory before
// its tensor-memory slot frees.  The writers' hand-over to the MMA issuers is a
// relaxed cluster-scope arrival: ordering tensor-memory accesses takes only the
// tcgen05 fences around it, and a release arrival costs over a thousand cycles.
// =====================================================================================

constexpr int P_STAGES = 5;                                         // operand ring
constexpr int P_SF_STAGES = 4;                                      // scale ring (shared memory)
constexpr int P_SF_SLOTS = 5;                                       // scale slots in tensor memory
constexpr int P_A_BYTES = 128 * BK_BYTES;                           // 16 KiB, own A rows
constexpr int P_B_BYTES = 128 * BK_BYTES;                           // 16 KiB, own half of B
constexpr int P_SFA_BYTES = (BK / MMA_K) * SF_ATOM;                 // 2 KiB
constexpr int P_SFB_BYTES = 2 * (BK / MMA_K) * SF_ATOM;             // 4 KiB, all 256 B rows
constexpr int P_AB_BYTES = P_A_BYTES + P_B_BYTES;                   // operand bytes per CTA and stage
constexpr int P_SF_BYTES = P_SFA_BYTES + P_SFB_BYTES;               // scale bytes per CTA and stage
constexpr int P_SF_OFFSET = P_STAGES * P_AB_BYTES;                  // scale ring after the operands
constexpr int P_EPI_BOX_COLS = 64;                                  // BF16 output box: 64 columns x 32 rows
constexpr int P_EPI_BOX_BYTES = 32 * P_EPI_BOX_COLS * 2;            // 4 KiB, one per epilogue warp
constexpr int P_EPI_OFFSET = P_SF_OFFSET + P_SF_STAGES * P_SF_BYTES;
constexpr int P_BAR_OFFSET = P_EPI_OFFSET + NUM_EPI_WARPS * P_EPI_BOX_BYTES;
constexpr int P_NUM_BARS = 3 * P_STAGES + 2 * P_SF_STAGES + 4;
constexpr int P_BAR_BYTES = 512;
constexpr int P_SMEM_BYTES = P_BAR_OFFSET + P_BAR_BYTES + 1024;
constexpr int P_BM = 256;                                           // tile rows per pair
constexpr int P_ISSUER2 = EPI_WARP0 + NUM_EPI_WARPS;                // warp 10: second MMA issuer
constexpr int P_WRITER0 = P_ISSUER2 + 1;                            // warps 11..14: scale writers
constexpr int P_NUM_WRITERS = 4;
constexpr int P_SF_PRODUCER = P_WRITER0 + P_NUM_WRITERS;            // warp 15: scale loads
constexpr int P_NUM_THREADS = 32 * (P_SF_PRODUCER + 1);             // 512
constexpr int P_SF_COL0 = 256;                                      // scale slot s at 256 + 48 s
constexpr int P_SF_SLOT_COLS = 48;                                  // 16 A-scale + 32 B-scale columns
constexpr int P_PREFETCH = 4;                                       // next-tile stages warmed in L2
static_assert(P_SF_COL0 + P_SF_SLOTS * P_SF_SLOT_COLS <= TMEM_COLS, "scale slots exceed tensor memory");
static_assert(P_SF_SLOTS <= P_STAGES, "a scale slot must free no later than the operand stage it serves");
static_assert(8 * P_NUM_BARS + 8 <= P_BAR_BYTES, "barrier area too small");
static_assert(P_SMEM_BYTES <= 232448, "shared memory above the sm_100 limit");
static_assert(P_SF_BYTES % 128 == 0 && P_AB_BYTES % 1024 == 0, "ring alignment");

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t saddr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
  return out;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrival that only hands over tensor-memory accesses: the arriving warp has waited
// for its tcgen05.ld / tcgen05.st (wait::ld / wait::st) and issued
// tcgen05.fence::before_thread_sync; the waiter issues tcgen05.fence::after_thread_sync
// before its next tcgen05 operation.  No generic-memory release is needed, and the
// cluster-scope release costs over a thousand cycles per arrival.
__device__ __forceinline__ void mbar_arrive_cluster_tc(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA tile load whose completion is signalled on `bar`, which may be the peer CTA's barrier.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                                 uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Warm L2 with a tile that a later TMA load will read (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
               : "memory");
}

// TMA store of a tile from shared memory (bulk async group of the issuing thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int32_t x, int32_t y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(x),
               "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the shared memory of every committed store has been read (it may be reused).
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until every committed store has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Maxima of a staged 32 x 64 BF16 output box (rows 128 bytes, 128-byte swizzle) that
// the next quantiser of C needs, folded into mraw / mrht: max |x|, and max |w| over
// the 16-point Walsh-Hadamard transforms w (before their 1/4) of each 16-row group
// of each column, signs applied first -- the col layout's transform, blocks along M.
// Lane t takes columns 2t and 2t+1 (one word per row); the butterflies run on the
// column pair as packed FP32, in the transform's own order (stages 1, 2, 4, 8).
__device__ __forceinline__ void box_amax(const uint8_t* stg, int lane, uint32_t signs, float& mraw, float& mrht) {
  const uint32_t chunk = (uint32_t)lane >> 2, wsub = ((uint32_t)lane & 3u) * 4u;
#pragma unroll
  for (int grp = 0; grp < 2; ++grp) {
    uint64_t pr[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = 16 * grp + i;
      uint32_t w = *reinterpret_cast<const uint32_t*>(stg + r * 128 + ((chunk ^ (uint32_t)(r & 7)) << 4) + wsub);
      mraw = fmaxf(mraw, fmaxf(fabsf(bf16_lo(w)), fabsf(bf16_hi(w))));
      w ^= ((signs >> i) & 1u) * 0x80008000u;
      pr[i] = f2_pack(bf16_lo(w), bf16_hi(w));
    }
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (!(i & h)) {
          const uint64_t a = pr[i], b = pr[i + h];
          pr[i] = f2_add(a, b);
          pr[i + h] = f2_sub(a, b);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float lo, hi;
      f2_unpack(pr[i], lo, hi);
      mrht = fmaxf(mrht, fmaxf(fabsf(lo), fabsf(hi)));
    }
  }
}

// Two FP32 values scaled by g, rounded to BF16 (nearest even) and packed, lo in the low half.
__device__ __forceinline__ uint32_t scale_pack_bf16x2(uint32_t lo, uint32_t hi, float g) {
  uint32_t out;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
      : "=r"(out)
      : "f"(__fmul_rn(__uint_as_float(hi), g)), "f"(__fmul_rn(__uint_as_float(lo), g)));
  return out;
}

// Two FP32 values rounded to BF16 (nearest even) and packed, a in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  uint32_t out;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(b), "f"(a));
  return out;
}

__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate, uint32_t sfa_tmem, uint32_t sfb_tmem) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor of the pair MMA: M = 256, N = 256.
__host__ __device__ constexpr uint32_t make_idesc_pair() {
  return (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

// Instruction descriptor of the low-rank stage's MMA, kind::f16: BF16 A and B (format 1),
// FP32 accumulator (format 1), K-major, M = 256, N = 256, K = 16.
__host__ __device__ constexpr uint32_t make_idesc_pair_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_pair_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, 1, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc)
      : "memory");
}

__device__ __forceinline__ TileCoord pair_tile_coord(const Params& p, int32_t t) {
  // p.num_m counts 256-row tiles here
  return tile_coord(p, t);
}

// Output modes of the pair kernel's epilogue (one instantiation each).
enum EpiMode : int { EPI_BF16 = 0, EPI_BF16_ACC = 1, EPI_F32 = 2, EPI_F32_ACC = 3 };

// Tensor maps of one GEMM problem of the pair kernel.
struct PairMaps {
  CUtensorMap a, b, sfa, sfb, c;
};

// The problems one pair-kernel launch works through: MAXP = 1 for a single GEMM, more for
// a grouped launch (one persistent grid over several GEMMs of the same output mode, e.g.
// a layer's weight gradients).  Their output tiles form one queue: problem i owns the
// global tile indices tile_end[i - 1] .. tile_end[i] - 1.  u and v are the low-rank
// factors of a single GEMM's low-rank stage (unused otherwise).
template <int MAXP>
struct PairGroup {
  PairMaps maps[MAXP];
  CUtensorMap u, v;
  Params p[MAXP];
  int32_t tile_end[MAXP];
  int32_t count;
};
constexpr int kMaxGroup = 8;

struct TileRef {
  int pi;       // problem
  int32_t lt;   // tile within the problem
};

template <int MAXP>
__device__ __forceinline__ TileRef locate(const PairGroup<MAXP>& g, int32_t t) {
  int pi = 0;
  if constexpr (MAXP > 1) {
    while (pi + 1 < g.count && t >= g.tile_end[pi]) ++pi;
  }
  return TileRef{pi, t - (pi ? g.tile_end[pi - 1] : 0)};
}

// Stages of a tile: the NVFP4 K-stages, then (LR) the low-rank stage.
template <bool LR>
__device__ __forceinline__ int stages_of(const Params& p) {
  return LR ? p.num_k_stages + 1 : p.num_k_stages;
}

// EPI: output mode; MAXP: problems per launch; LR: a low-rank stage ends every tile (a
// separate instantiation, so that the plain GEMM carries none of its branches).
template <int EPI, int MAXP, bool LR>
__global__ void __launch_bounds__(P_NUM_THREADS, 1)
    gemm_kernel_pair(const __grid_constant__ PairGroup<MAXP> grp) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t smem_base = smem_u32(smem);
  uint8_t* bar_area = smem + P_BAR_OFFSET;
  const uint32_t bar_base = smem_u32(bar_area);
  // operand ring: full (leader; both CTAs' loads complete on it), empty (MMA commits, both CTAs)
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (P_STAGES + s); };
  auto sf_ready_bar = [&](int s) { return bar_base + 8u * (2 * P_STAGES + s); };   // scales in TMEM (leader)
  // scale ring (each CTA its own): landed in shared memory / written to TMEM by the four writers
  auto sf_full_bar = [&](int j) { return bar_base + 8u * (3 * P_STAGES + j); };
  auto sf_empty_bar = [&](int j) { return bar_base + 8u * (3 * P_STAGES + P_SF_STAGES + j); };
  const uint32_t acc_full = bar_base + 8u * (P_NUM_BARS - 4);
  const uint32_t acc_empty = bar_base + 8u * (P_NUM_BARS - 3);
  const uint32_t mma_done = bar_base + 8u * (P_NUM_BARS - 2);
  const uint32_t mma_done2 = bar_base + 8u * (P_NUM_BARS - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_area + 8 * P_NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 8 * P_NUM_BARS + 4);

  auto a_smem = [&](int s) { return smem_base + (uint32_t)(s * P_AB_BYTES); };
  auto b_smem = [&](int s) { return smem_base + (uint32_t)(s * P_AB_BYTES + P_A_BYTES); };
  auto sfa_smem = [&](int j) { return smem_base + (uint32_t)(P_SF_OFFSET + j * P_SF_BYTES); };
  auto sfb_smem = [&](int j) { return smem_base + (uint32_t)(P_SF_OFFSET + j * P_SF_BYTES + P_SFA_BYTES); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();           // 0 = leader
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(sf_ready_bar(s), 2 * P_NUM_WRITERS);
    }
    for (int j = 0; j < P_SF_STAGES; ++j) {
      mbar_init(sf_full_bar(j), 1);
      mbar_init(sf_empty_bar(j), P_NUM_WRITERS);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * NUM_EPI_WARPS);
    mbar_init(mma_done, 1);
    mbar_init(mma_done2, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();                                     // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The launch may be a programmatic dependent of the kernel before it in the stream:
  // nothing above touches global memory, and every role below starts after that
  // kernel has completed.  A dependent of this kernel may start as its CTAs leave.
  griddep_launch_dependents();
  griddep_wait();

  const int32_t num_tiles = grp.tile_end[grp.count - 1];
  const int32_t pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const uint32_t leader_full0 = map_to_cta(full_bar(0), 0);
  const uint32_t leader_acc_empty = map_to_cta(acc_empty, 0);

  if (warp == 0) {
    // ------------------------------------------------------------ operand producer (both CTAs)
    {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // During the last P_PREFETCH stages of a tile, the first stages of the pair's next
      // tile are prefetched into L2: every pair starts its next tile at about the same
      // time, and without this those first loads all miss L2 at once.
      int64_t q = 0;                                    // stage sequence number over this pair's tiles
      for (int32_t t = pair; t < num_tiles && ok; t += num_pairs) {
        const TileRef tr = locate(grp, t);
        const Params& p = grp.p[tr.pi];
        const PairMaps& M = grp.maps[tr.pi];
        const int tile_stages = stages_of<LR>(p);
        const int pf_n = min(P_PREFETCH, p.num_k_stages);
        const TileCoord tc = pair_tile_coord(p, tr.lt);
        const bool has_next = t + num_pairs < num_tiles;
        const TileRef nr = locate(grp, has_next ? t + num_pairs : t);
        const Params& pn = grp.p[nr.pi];
        const PairMaps& Mn = grp.maps[nr.pi];
        const TileCoord nc = pair_tile_coord(pn, nr.lt);
        for (int ks = 0; ks < tile_stages; ++ks, ++q) {
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag))) {
            ok = false;
            break;
          }
          if (pair == 0 && q == grp.p[0].skip_stage) {
            // fault injection: neither CTA loads this stage and the leader never arms its
            // barrier, so the MMA issuers' bounded wait on it expires (kErrTimeout) and
            // every role winds down; nothing is in flight for this stage
            if (++stage == P_STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          const uint32_t fb = leader_full0 + 8u * stage;
          const int32_t kx = ks * BK_BYTES;
          const int pf = ks - (p.num_k_stages - pf_n);
          if (elect_one()) {
            if (leader) mbar_arrive_expect_tx(full_bar(stage), 2u * P_AB_BYTES);
            if (LR && ks == p.num_k_stages) {
              // low-rank stage: 128 rows x 64 BF16 of U (this CTA's A rows) and of V (its half
              // of the B rows), zero-filled past the rank
              tma_load_2d_pair(a_smem(stage), &grp.u, 0, tc.m_blk * P_BM + (int32_t)rank * 128, fb);
              tma_load_2d_pair(b_smem(stage), &grp.v, 0, tc.n_blk * BN + (int32_t)rank * 128, fb);
            } else {
              tma_load_2d_pair(a_smem(stage), &M.a, kx, tc.m_blk * P_BM + (int32_t)rank * 128, fb);
              tma_load_2d_pair(b_smem(stage), &M.b, kx, tc.n_blk * BN + (int32_t)rank * 128, fb);
            }
            if (has_next && pf >= 0 && (!LR || pf < pf_n) && (MAXP == 1 || pf < pn.num_k_stages)) {
              tma_prefetch_2d(&Mn.a, pf * BK_BYTES, nc.m_blk * P_BM + (int32_t)rank * 128);
              tma_prefetch_2d(&Mn.b, pf * BK_BYTES, nc.n_blk * BN + (int32_t)rank * 128);
            }
          }
          __syncwarp();
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1 || warp == P_ISSUER2) {
    // ------------------------------------------------------------ MMA issuers (leader only)
    // Two warps take the K-stages in turn (stage sequence q over all tiles of this
    // pair: warp 1 issues even q, warp 10 odd q).  An issuer waits for its stage's
    // data while the other warp's MMAs keep the tensor pipe busy -- a thread that
    // polls an mbarrier stalls its own MMA issue, so one issuer alone cannot keep
    // the pipe full.  Named barriers hand the turn over (1: warp 1 -> warp 10,
    // 2: warp 10 -> warp 1), which keeps the MMAs in stage order; the tensor fences
    // around them order the tensor-memory accesses across the two issuers.  After
    // a failed wait an issuer keeps taking part in the hand-over (so the other
    // issuer is never left waiting at a named barrier) but issues nothing.
    if (leader) {
      const int me = warp == 1 ? 0 : 1;
      const uint32_t idesc = make_idesc_pair();
      bool ok = true;
      int64_t q = 0;                                    // stage sequence number
      int stage = 0, slot = 0;                          // operand stage, scale slot (q % P_SF_SLOTS)
      uint32_t phase = 0, acc_phase = 0;
      int64_t total = 0;                                // stages over all tiles of this pair
      if constexpr (MAXP == 1) {
        total = (int64_t)((num_tiles - pair + num_pairs - 1) / num_pairs) * stages_of<LR>(grp.p[0]);
      } else {
        for (int32_t t = pair; t < num_tiles; t += num_pairs) total += stages_of<LR>(grp.p[locate(grp, t).pi]);
      }
      for (int32_t t = pair; t < num_tiles; t += num_pairs) {
        const Params& p = grp.p[locate(grp, t).pi];
        const int tile_stages = stages_of<LR>(p);
        for (int ks = 0; ks < tile_stages; ++ks, ++q) {
          if ((q & 1) == me) {
            if (ok && ks == 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag));
            if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(full_bar(stage), phase, abort_flag));
            if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(sf_ready_bar(stage), phase, abort_flag));
            if (q > 0) asm volatile("bar.sync %0, 64;" ::"r"(me == 0 ? 2 : 1) : "memory");
            tc_fence_after();
            // Operands of this stage's MMAs, computed by every lane so that they stay
            // warp-uniform; one lane chosen by elect.sync issues.  (Computing them under a
            // lane == 0 branch instead cost 5 % of the GEMM's throughput.)
            const uint64_t a_desc0 = sw128_desc(a_smem(stage)), b_desc0 = sw128_desc(b_smem(stage));
            const uint32_t sfa0 = tmem + P_SF_COL0 + P_SF_SLOT_COLS * slot;
            const int atoms_u = (ks == p.num_k_stages - 1) ? p.tail_atoms : BK / MMA_K;
            if (ok && elect_one()) {
              if (LR && ks == p.num_k_stages) {
                // low-rank stage: U V^T (BF16, K = 16 per MMA) into the same accumulator
                for (int kk = 0; kk < p.lr_ksteps; ++kk)
                  tc_mma_pair_bf16(tmem + ACC_COL, sw128_desc(a_smem(stage) + kk * 32),
                                   sw128_desc(b_smem(stage) + kk * 32), make_idesc_pair_bf16());
              } else {
                for (int kk = 0; kk < atoms_u; ++kk)
                  tc_mma_pair(tmem + ACC_COL, a_desc0 + (uint64_t)(kk * (MMA_K / 2 / 16)),
                              b_desc0 + (uint64_t)(kk * (MMA_K / 2 / 16)), idesc, (ks | kk) != 0 ? 1u : 0u,
                              sfa0 + 4 * kk, sfa0 + 16 + 8 * kk);
              }
              tc_commit_pair(empty_bar(stage));
              if (ks == tile_stages - 1) tc_commit_pair(acc_full);
            }
            tc_fence_before();
            __syncwarp();
            if (q + 1 < total) asm volatile("bar.arrive %0, 64;" ::"r"(me == 0 ? 1 : 2) : "memory");
          }
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          if (++slot == P_SF_SLOTS) slot = 0;
        }
        acc_phase ^= 1u;
      }
      // every MMA this warp issued has finished once mma_done flips (one barrier per
      // issuer; the commit comes from the lane that issued them)
      const uint32_t done = me == 0 ? mma_done : mma_done2;
      if (elect_one())
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(done)
                     : "memory");
      __syncwarp();
      mbar_wait_drain(done, 0);
    }
  } else if (warp == P_SF_PRODUCER) {
    // ------------------------------------------------------------ scale producer (both CTAs)
    // Each CTA loads the scales of its own A rows and of all 256 B rows of the tile,
    // up to P_SF_STAGES stages ahead; a slot is reused once the four writers of this
    // CTA have stored it to tensor memory.
    {
      int j = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int32_t t = pair; t < num_tiles && ok; t += num_pairs) {
        const TileRef tr = locate(grp, t);
        const Params& p = grp.p[tr.pi];
        const PairMaps& M = grp.maps[tr.pi];
        const int tile_stages = stages_of<LR>(p);
        const int pf_n = min(P_PREFETCH, p.num_k_stages);
        const TileCoord tc = pair_tile_coord(p, tr.lt);
        const bool has_next = t + num_pairs < num_tiles;
        const TileRef nr = locate(grp, has_next ? t + num_pairs : t);
        const Params& pn = grp.p[nr.pi];
        const PairMaps& Mn = grp.maps[nr.pi];
        const TileCoord nc = pair_tile_coord(pn, nr.lt);
        for (int ks = 0; ks < tile_stages; ++ks) {
          const int pf = ks - (p.num_k_stages - pf_n);
          if (has_next && pf >= 0 && (!LR || pf < pf_n) && (MAXP == 1 || pf < pn.num_k_stages) && elect_one()) {
            // the next tile's scales
            const int32_t pk = pf * (BK / MMA_K);
            tma_prefetch_2d(&Mn.sfa, 0, (int32_t)((nc.m_blk * 2 + (int32_t)rank) * pn.sf_kgroups_a) + pk);
            tma_prefetch_2d(&Mn.sfb, 0, (int32_t)((nc.n_blk * 2) * pn.sf_kgroups) + pk);
            tma_prefetch_2d(&Mn.sfb, 0, (int32_t)((nc.n_blk * 2 + 1) * pn.sf_kgroups) + pk);
          }
          __syncwarp();
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(sf_empty_bar(j), phase ^ 1u, abort_flag))) {
            ok = false;
            break;
          }
          const uint32_t sb = sf_full_bar(j);
          if (LR && ks == p.num_k_stages) {
            // the low-rank stage has no block scales: complete the slot's phase without
            // loading, so the writers' and issuers' stage counts stay in step
            if (elect_one()) mbar_arrive(sb);
            __syncwarp();
            if (++j == P_SF_STAGES) {
              j = 0;
              phase ^= 1u;
            }
            continue;
          }
          const int32_t katom = ks * (BK / MMA_K);
          if (elect_one()) {
            mbar_arrive_expect_tx(sb, (uint32_t)P_SF_BYTES);
            tma_load_2d(sfa_smem(j), &M.sfa, 0, (int32_t)((tc.m_blk * 2 + (int32_t)rank) * p.sf_kgroups_a) + katom,
                        sb);
            tma_load_2d(sfb_smem(j), &M.sfb, 0, (int32_t)((tc.n_blk * 2) * p.sf_kgroups) + katom, sb);
            tma_load_2d(sfb_smem(j) + (BK / MMA_K) * SF_ATOM, &M.sfb, 0,
                        (int32_t)((tc.n_blk * 2 + 1) * p.sf_kgroups) + katom, sb);
          }
          __syncwarp();
          if (++j == P_SF_STAGES) {
            j = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp >= P_WRITER0) {
    // ------------------------------------------------------------ scale writers (both CTAs)
    // Warp w writes lane quarter w % 4 of each stage's scale slot: lane i takes row i
    // of every 512-byte scale tile of the stage (16 bytes = 4 columns per tile) and
    // stores them with tcgen05.st; then it tells the leader's MMA issuers and frees
    // the shared-memory slot (the stores have consumed the loaded registers, so the
    // loads are complete).  Stage q uses tensor-memory slot q % P_SF_SLOTS, free once
    // the MMAs of stage q - P_SF_SLOTS have completed: the commit that frees operand
    // stage (q - P_SF_SLOTS) % P_STAGES, phase (q - P_SF_SLOTS) / P_STAGES.  That
    // barrier cannot be a phase behind (the MMAs of stage q - 1 - P_SF_SLOTS, older,
    // are complete: this warp waited for them) nor a phase ahead (stage q + 1 needs
    // this warp's scales), so its parity names the phase.
    const int quarter = warp & 3;
    const uint32_t tq = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t leader_ready0 = map_to_cta(sf_ready_bar(0), 0);
    const uint32_t own_empty0 = map_to_cta(sf_empty_bar(0), rank);
    int stage = 0, j = 0, slot = 0, lag_stage = 0;
    uint32_t sf_phase = 0, lag_phase = 0;
    int64_t q = 0;
    bool ok = true;
    for (int32_t t = pair; t < num_tiles && ok; t += num_pairs) {
      const int tile_stages = stages_of<LR>(grp.p[locate(grp, t).pi]);
      for (int ks = 0; ks < tile_stages; ++ks, ++q) {
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(sf_full_bar(j), sf_phase, abort_flag));
        if (!ok) break;
        const uint8_t* sa = smem + P_SF_OFFSET + j * P_SF_BYTES + lane * 16;
        uint32_t v[48];
#pragma unroll
        for (int kk = 0; kk < BK / MMA_K; ++kk) {
          const uint4 xa = *reinterpret_cast<const uint4*>(sa + kk * SF_ATOM);
          const uint4 x0 = *reinterpret_cast<const uint4*>(sa + P_SFA_BYTES + kk * SF_ATOM);
          const uint4 x1 = *reinterpret_cast<const uint4*>(sa + P_SFA_BYTES + ((BK / MMA_K) + kk) * SF_ATOM);
          v[4 * kk] = xa.x, v[4 * kk + 1] = xa.y, v[4 * kk + 2] = xa.z, v[4 * kk + 3] = xa.w;
          v[16 + 8 * kk] = x0.x, v[17 + 8 * kk] = x0.y, v[18 + 8 * kk] = x0.z, v[19 + 8 * kk] = x0.w;
          v[20 + 8 * kk] = x1.x, v[21 + 8 * kk] = x1.y, v[22 + 8 * kk] = x1.z, v[23 + 8 * kk] = x1.w;
        }
        if (q >= P_SF_SLOTS) {
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(empty_bar(lag_stage), lag_phase, abort_flag));
          if (!ok) break;
          if (++lag_stage == P_STAGES) {
            lag_stage = 0;
            lag_phase ^= 1u;
          }
        }
        tc_fence_after();
        const uint32_t taddr = tq + P_SF_COL0 + P_SF_SLOT_COLS * slot;
        asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
                     "%15,%16};" ::"r"(taddr),
                     "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
                     "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
                     : "memory");
        asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
                     "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr + 16),
                     "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]),
                     "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]),
                     "r"(v[30]), "r"(v[31]), "r"(v[32]), "r"(v[33]), "r"(v[34]), "r"(v[35]), "r"(v[36]),
                     "r"(v[37]), "r"(v[38]), "r"(v[39]), "r"(v[40]), "r"(v[41]), "r"(v[42]), "r"(v[43]),
                     "r"(v[44]), "r"(v[45]), "r"(v[46]), "r"(v[47])
                     : "memory");
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cluster_tc(leader_ready0 + 8u * stage);
          mbar_arrive_cluster_tc(own_empty0 + 8u * j);
        }
        if (++stage == P_STAGES) stage = 0;
        if (++slot == P_SF_SLOTS) slot = 0;
        if (++j == P_SF_STAGES) {
          j = 0;
          sf_phase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Output paths, by output type:
    //   BF16            scale and round while reading the accumulator (64 registers for
    //                   the warp's 128 columns), release it, then two 32 x 64 TMA stores;
    //   BF16 + C        the warp's 128 old values of C are loaded into registers before
    //                   the accumulator is ready (while the main loop runs), added while
    //                   reading it (BF16(fl32(fl32(acc * g) + C))), then as BF16;
    //   FP32            four 32 x 32 boxes, each staged and stored as soon as read; the
    //                   accumulator is released after the last read;
    //   FP32 + C        32 columns at a time, direct loads and stores.
    // Staging uses the warp's own 4 KB of shared memory, rows of 128 bytes with the
    // 128-byte swizzle (lane r puts 16-byte chunk c of its row at chunk c ^ (r % 8),
    // which keeps each quarter-warp on distinct banks); whole-line bulk stores instead
    // of per-row 16-byte stores keep the output burst at every tile change off the
    // operand loads.
    const int ew = warp - EPI_WARP0;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    const int row_in_tile = (int)rank * 128 + quarter * 32 + lane;
    constexpr bool bf16_out = EPI == EPI_BF16 || EPI == EPI_BF16_ACC;
    constexpr bool accumulate = EPI == EPI_BF16_ACC || EPI == EPI_F32_ACC;
    uint8_t* stg = smem + P_EPI_OFFSET + ew * P_EPI_BOX_BYTES;
    uint32_t acc_phase = 0;
    auto scale_of = [](const Params& q) { return __fmul_rn(__fmul_rn(*q.scale_a, *q.scale_b), q.alpha); };
    const float g1 = MAXP == 1 ? scale_of(grp.p[0]) : 0.0f;   // one problem: read once
    for (int32_t t = pair; t < num_tiles; t += num_pairs) {
      const TileRef tr = locate(grp, t);
      const Params& p = grp.p[tr.pi];
      const CUtensorMap* tma_c = &grp.maps[tr.pi].c;
      const float g = MAXP == 1 ? g1 : scale_of(p);
      const TileCoord tc = pair_tile_coord(p, tr.lt);
      const int n_cols = min(BN, p.N - tc.n_blk * BN);
      const int64_t m = (int64_t)tc.m_blk * P_BM + row_in_tile;
      const bool mine = n_cols > half * 128;          // N % 128 == 0: a half is whole or absent
      const int64_t n0 = (int64_t)tc.n_blk * BN + half * 128;
      const int32_t m0 = tc.m_blk * P_BM + (int32_t)rank * 128 + quarter * 32;
      const bool rows_in = m0 < p.M;                  // M % 128 == 0: the warp's 32 rows are all in or all out
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + ACC_COL + half * 128;
      uint32_t pk[64];                                // BF16 pairs: old C, then the result
      if constexpr (EPI == EPI_BF16_ACC) {
        if (mine && rows_in) {
          const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.C) + m * p.ldc + n0);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const uint4 v = src[q];
            pk[4 * q] = v.x, pk[4 * q + 1] = v.y, pk[4 * q + 2] = v.z, pk[4 * q + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 64; ++q) pk[q] = 0u;
        }
      }
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, acc_phase, abort_flag));
      if (!ok) break;
      tc_fence_after();
      if constexpr (bf16_out) {
        if (mine) {
          if constexpr (accumulate) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint32_t r[32];
              tc_load_32cols(taddr + 32 * k, r);
              tc_wait_loads();
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const uint32_t o = pk[16 * k + j];
                const float v0 = __fadd_rn(__fmul_rn(__uint_as_float(r[2 * j]), g), bf16_lo(o));
                const float v1 = __fadd_rn(__fmul_rn(__uint_as_float(r[2 * j + 1]), g), bf16_hi(o));
                pk[16 * k + j] = pack_bf16x2(v0, v1);
              }
            }
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint32_t r[32];
              tc_load_32cols(taddr + 32 * k, r);
              tc_wait_loads();
#pragma unroll
              for (int j = 0; j < 16; ++j) pk[16 * k + j] = scale_pack_bf16x2(r[2 * j], r[2 * j + 1], g);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_tc(leader_acc_empty);
        float mraw = 0.0f, mrht = 0.0f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if (!mine || !rows_in) continue;                                 // box outside C
          if (lane == 0) bulk_wait_read();                                 // staging buffer free again
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_uint4(pk[32 * hh + 4 * c], pk[32 * hh + 4 * c + 1], pk[32 * hh + 4 * c + 2],
                           pk[32 * hh + 4 * c + 3]);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(tma_c, (int32_t)n0 + hh * P_EPI_BOX_COLS, m0, smem_u32(stg));
            bulk_commit();
          }
          if (EPI == EPI_BF16 && p.amax_acc) box_amax(stg, lane, p.rht_signs, mraw, mrht);
        }
        if (EPI == EPI_BF16 && p.amax_acc) {
          // boxes past the end of C hold zeros (their operand rows were zero-filled), so
          // the maxima need no masking; 0.25 * max |w| = max |w / 4| (scaling by 1/4 is
          // monotonic in round-to-nearest)
          mrht = __fmul_rn(mrht, 0.25f);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            mraw = fmaxf(mraw, __shfl_xor_sync(0xFFFFFFFFu, mraw, o));
            mrht = fmaxf(mrht, __shfl_xor_sync(0xFFFFFFFFu, mrht, o));
          }
          if (lane == 0) {
            atomicMax(p.amax_acc, __float_as_uint(mraw));          // non-negative floats order as their bits
            atomicMax(p.amax_acc + 1, __float_as_uint(mrht));
          }
        }
      } else if constexpr (!accumulate) {
        // FP32: 32 columns (one 128-byte box row per lane) at a time
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          uint32_t r[32];
          if (mine) {
            tc_load_32cols(taddr + 32 * k, r);
            tc_wait_loads();
          }
          if (k == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_tc(leader_acc_empty);
          }
          if (!mine || !rows_in) continue;
          if (lane == 0) bulk_wait_read();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_float4(__fmul_rn(__uint_as_float(r[4 * c]), g), __fmul_rn(__uint_as_float(r[4 * c + 1]), g),
                            __fmul_rn(__uint_as_float(r[4 * c + 2]), g), __fmul_rn(__uint_as_float(r[4 * c + 3]), g));
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(tma_c, (int32_t)n0 + 32 * k, m0, smem_u32(stg));
            bulk_commit();
          }
        }
      } else {
        // FP32 accumulation into C: 32 columns at a time, released at the end.
        uint8_t* crow = static_cast<uint8_t*>(p.C) + (size_t)(m * p.ldc + n0) * 4;
        if (mine) {
#pragma unroll 1
          for (int k = 0; k < 4; ++k) {
            uint32_t r[32];
            tc_load_32cols(taddr + 32 * k, r);
            tc_wait_loads();
            if (rows_in) store_32cols(p, r, g, crow + (size_t)32 * k * 4);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_tc(leader_acc_empty);
      }
      acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();                   // this warp's output stores have landed
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                                     // the leader's MMAs are done with both CTAs
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}
}  // namespace gemm
}  // namespace nvfp4
