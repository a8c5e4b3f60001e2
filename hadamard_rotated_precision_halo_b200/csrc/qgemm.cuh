// qgemm.cuh -- low-precision GEMM on 8-bit codes with a dequantising epilogue.
//
//     C[i, j] = (sum_k A[i, k] B[j, k]) * s_a[i] * s_b[j]
//
// INT8 codes multiply on the 5th-generation tensor cores with exact int32
// accumulation (tcgen05.mma kind::i8), E4M3 codes with fp32 accumulation
// (kind::f8f6f4).  "All large matrix multiplications ... in lower precision"
// with INT8 or FP8: HALO paper page, abstract and "key design".
//
// Structure (one CTA per SM, persistent over output tiles of 128 x 256):
//   warp 0      TMA producer: 128-byte-swizzled A / B tiles (K block of 128
//               codes) into a 4-stage shared-memory ring.
//   warp 1      tensor-memory allocator and MMA issuer (one thread): four
//               128x256x32 MMAs per K block into a tensor-memory accumulator.
//   warps 2-5   epilogue: tensor memory -> registers, int32 -> fp32, times
//               s_a[row] * s_b[col], store fp32 or bf16.
// Two 256-column accumulators in tensor memory let the epilogue of one tile
// overlap the main loop of the next.  Operands may be K-major (contraction
// dimension contiguous) or MN-major; the shared-memory descriptors describe
// either, so dimension-0-rotated codes are consumed without a transpose.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace halo {

enum : unsigned int {
  kSiteGemmProducer = 0x301,
  kSiteGemmMma = 0x302,
  kSiteGemmMmaAcc = 0x303,
  kSiteGemmEpilogue = 0x304,
  kSiteGemmDrain = 0x305,
};

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 128;  // codes (bytes) per K block
constexpr int kGemmStages = 4;
constexpr int kGemmABytes = kGemmBM * kGemmBK;  // 16 KB
constexpr int kGemmBBytes = kGemmBN * kGemmBK;  // 32 KB
constexpr int kGemmThreads = 192;
constexpr uint32_t kGemmTmemCols = 512;  // two 256-column fp32/int32 accumulators
constexpr int kGemmGroupM = 16;           // tile raster: groups of 16 M tiles
constexpr int kSnakeMinKBlocks = 128;     // K >= 16384: odd passes walk K backwards
// Dynamic shared memory: stages + 1 KB alignment slack + barriers.
constexpr size_t kGemmSmemBytes = kGemmStages * (kGemmABytes + kGemmBBytes) + 1024 + 256;

struct GemmParams {
  int m, n, k;
  int tiles_m, tiles_n, num_tiles;
  int a_mn, b_mn;  // operand storage: 0 = K-major, 1 = MN-major
  int group_m;     // tile raster of the pair kernel (M tiles per group)
  uint32_t idesc;  // tcgen05 instruction descriptor
  const float* sa;
  const float* sb;
  void* c;
  int64_t ldc;
  int out_bf16;
};

// Tile raster: groups of `group_m` M tiles; inside a group the M tiles of one
// N column come one after another, so that consecutive tiles (computed at the
// same time by neighbouring CTAs) share B panels and the group's A panels.
__device__ __forceinline__ void gemm_tile_coords(int tile, int tiles_m, int tiles_n, int group_m, int& tm, int& tn) {
  const int per_group = group_m * tiles_n;
  const int group = tile / per_group;
  const int first_m = group * group_m;
  const int gm = min(tiles_m - first_m, group_m);
  const int in_group = tile - group * per_group;
  tm = first_m + in_group % gm;
  tn = in_group / gm;
}

__device__ __forceinline__ void gemm_tile_coords(int tile, int tiles_m, int tiles_n, int& tm, int& tn) {
  gemm_tile_coords(tile, tiles_m, tiles_n, kGemmGroupM, tm, tn);
}

template <int QT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGemmStages * kGemmABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kGemmStages * kGemmBBytes);
  uint64_t* empty = full + kGemmStages;
  uint64_t* tfull = empty + kGemmStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);  // one arrival per epilogue warp
    }
    fence_mbar_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kGemmTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kblocks = (p.k + kGemmBK - 1) / kGemmBK;
  griddep_wait();  // codes and scales written, output read, by the previous kernels
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t ld_issued = 0, ld_par = 0;  // loads issued per stage, for the drain below
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        int tm, tn;
        gemm_tile_coords(tile, p.tiles_m, p.tiles_n, tm, tn);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, kSiteGemmProducer)) { ok = false; break; }
          note_load(ld_issued, ld_par, stage, phase);
          mbar_arrive_expect_tx(&full[stage], kGemmABytes + kGemmBBytes);
          uint8_t* a_dst = sA + stage * kGemmABytes;
          uint8_t* b_dst = sB + stage * kGemmBBytes;
          if (p.a_mn)
            tma_load_2d(a_dst, &tm_a, &full[stage], tm * kGemmBM, kb * kGemmBK);
          else
            tma_load_2d(a_dst, &tm_a, &full[stage], kb * kGemmBK, tm * kGemmBM);
          if (p.b_mn) {
            tma_load_2d(b_dst, &tm_b, &full[stage], tn * kGemmBN, kb * kGemmBK);
            tma_load_2d(b_dst + kGemmBBytes / 2, &tm_b, &full[stage], tn * kGemmBN + 128, kb * kGemmBK);
          } else {
            tma_load_2d(b_dst, &tm_b, &full[stage], kb * kGemmBK, tn * kGemmBN);
          }
          if (++stage == kGemmStages) { stage = 0; phase ^= 1u; }
        }
      }
      drain_loads(full, kGemmStages, ld_issued, ld_par, kSiteGemmDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int lt = 0;
      // Per-K-step descriptor advance: 32 codes along K.  K-major tiles step 32
      // bytes inside the swizzled 128-byte row; MN-major tiles step 32 rows.
      const uint32_t a_step = p.a_mn ? 32u * 128u : 32u;
      const uint32_t b_step = p.b_mn ? 32u * 128u : 32u;
      const uint32_t a_lbo = p.a_mn ? static_cast<uint32_t>(kGemmBK * 128) : 16u;
      const uint32_t b_lbo = p.b_mn ? static_cast<uint32_t>(kGemmBK * 128) : 16u;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++lt) {
        const uint32_t acc = lt & 1;
        const uint32_t acc_phase = (lt >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, kSiteGemmMmaAcc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256u;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, kSiteGemmMma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * kGemmABytes);
          const uint32_t b_base = smem_u32(sB + stage * kGemmBBytes);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 32; ++kk) {
            const uint64_t adesc = smem_desc_sw128(a_base + kk * a_step, a_lbo, 1024u);
            const uint64_t bdesc = smem_desc_sw128(b_base + kk * b_step, b_lbo, 1024u);
            const uint32_t accumulate = (kb > 0 || kk > 0) ? 1u : 0u;
            if (QT == 0)
              mma_i8(d_tmem, adesc, bdesc, p.idesc, accumulate);
            else
              mma_f8(d_tmem, adesc, bdesc, p.idesc, accumulate);
          }
          mma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == kGemmStages) { stage = 0; phase ^= 1u; }
        }
        mma_commit(&tfull[acc]);  // accumulator complete
      }
    }
    __syncwarp();
  } else {
    // Epilogue: warp w reads tensor-memory lanes 32*(w%4) .. +31 = tile rows.
    const int quad = warp & 3;
    int lt = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++lt) {
      int tm, tn;
      gemm_tile_coords(tile, p.tiles_m, p.tiles_n, tm, tn);
      const uint32_t acc = lt & 1;
      const uint32_t acc_phase = (lt >> 1) & 1;
      const bool ok = mbar_wait(&tfull[acc], acc_phase, kSiteGemmEpilogue);
      if (bar_or(1, 128, !ok)) break;
      tc_fence_after();
      const int row = tm * kGemmBM + quad * 32 + lane;
      const bool row_ok = row < p.m;
      const float sa = row_ok ? p.sa[row] : 0.f;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * 256u;
#pragma unroll 1
      for (int ch = 0; ch < kGemmBN / 32; ++ch) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(t_row + ch * 32, r);
        tmem_ld_wait();
        const int col0 = tn * kGemmBN + ch * 32;
        if (row_ok && col0 < p.n) {
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float a = (QT == 0) ? __int2float_rn(static_cast<int>(r[j])) : __uint_as_float(r[j]);
          const int col = col0 + j;
          const float sb = col < p.n ? __ldg(p.sb + col) : 0.f;
          y[j] = (a * sa) * sb;
        }
        const bool full_chunk = col0 + 32 <= p.n;
        if (p.out_bf16) {
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.c) + static_cast<int64_t>(row) * p.ldc + col0;
          if (full_chunk) {
            uint4* o4 = reinterpret_cast<uint4*>(out);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(y[8 * q + 2 * e], y[8 * q + 2 * e + 1]);
                w[e] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              o4[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.n) out[j] = __float2bfloat16_rn(y[j]);
          }
        } else {
          float* out = static_cast<float*>(p.c) + static_cast<int64_t>(row) * p.ldc + col0;
          if (full_chunk) {
            float4* o4 = reinterpret_cast<float4*>(out);
#pragma unroll
            for (int q = 0; q < 8; ++q) o4[q] = make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.n) out[j] = y[j];
          }
        }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kGemmTmemCols);
  }
}


// ------------------------------------------------------------------------------------------
// qgemm_pair_kernel: the same GEMM with 256 x 256 output tiles computed by a
// pair of CTAs (a 2-CTA cluster on two SMs) with tcgen05.mma.cta_group::2.
// Each CTA holds half of the A tile (128 rows) and half of the B tile (128
// of the 256 N indices) in its own shared memory, so per K block an SM loads
// 32 KB instead of 48 KB for the same tensor work.  The even CTA issues the
// MMAs; both CTAs' TMA loads complete on the even CTA's stage barrier; the
// MMA commits arrive on both CTAs' barriers; each CTA drains its own 128 rows
// of the accumulator from its tensor memory and releases it on the even CTA's
// barrier.  Loads are plain (no multicast).
// ------------------------------------------------------------------------------------------
constexpr int kPairStages = 6;
constexpr int kPairABytes = 128 * kGemmBK;  // 16 KB: 128 rows of A
constexpr int kPairBBytes = 128 * kGemmBK;  // 16 KB: 128 N indices of B
// Output staging of the epilogue: per epilogue warp two buffers of 32 rows x
// 128 bytes (32 fp32 or 64 bf16 columns), 128-byte swizzled.
constexpr int kPairOutBytes = 32 * 128;
// Dynamic shared memory: stages, output staging, 1 KB alignment slack, barriers.
constexpr size_t kPairSmemBytes = kPairStages * (kPairABytes + kPairBBytes) + 4 * 2 * kPairOutBytes + 1024 + 256;

enum : unsigned int {
  kSitePairProducer = 0x311,
  kSitePairMma = 0x312,
  kSitePairMmaAcc = 0x313,
  kSitePairEpilogue = 0x314,
  kSitePairDrain = 0x315,
};

// Epilogue: each epilogue warp converts 32 rows x 128 bytes of its accumulator
// quarter at a time into a swizzled shared-memory buffer (two per warp,
// alternating) and one lane writes it with a bulk tensor store (this GPU's own
// memory; the copy clips rows and columns past the matrix), so the stores
// leave as whole lines and overlap the next chunk.  OB = 1: bf16 out, else fp32.
template <int QT, int OB>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qgemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_c, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPairStages * kPairABytes;
  uint8_t* sOut = sB + kPairStages * kPairBBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + 4 * 2 * kPairOutBytes);
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);  // four epilogue warps in each CTA of the pair
    }
    fence_mbar_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kGemmTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_arrive();  // both CTAs' barriers and tensor memory are ready
  cluster_wait();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kblocks = (p.k + kGemmBK - 1) / kGemmBK;
  griddep_wait();  // codes and scales written, output read, by the previous kernels
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t ld_issued = 0, ld_par = 0;  // loads issued per stage, for the drain below
      int lt = 0;
      for (int tile = pair; tile < p.num_tiles && ok; tile += npairs, ++lt) {
        int tm, tn;
        gemm_tile_coords(tile, p.tiles_m, p.tiles_n, p.group_m, tm, tn);
        const int a_row = tm * 256 + static_cast<int>(rank) * 128;
        const int b_row = tn * 256 + static_cast<int>(rank) * 128;
        // Every pair takes its lt-th tile at about the same time, so the tiles
        // of one pass over the grid share A panels with the pass before.  When
        // those panels are too long to stay in L2 (K >= 16384), odd passes walk
        // K backwards: their first K blocks are the ones the previous pass read
        // last, still in L2.  (The MMA loop accumulates in arrival order; INT8
        // sums are exact in any order.)  Shorter K keeps one direction: there
        // the reversal measured a few percent more DRAM reads.
        const bool reverse = (lt & 1) != 0 && kblocks >= kSnakeMinKBlocks;
        for (int kb = 0; kb < kblocks; ++kb) {
          const int kpos = reverse ? kblocks - 1 - kb : kb;
          if (!mbar_wait(&empty[stage], phase ^ 1u, kSitePairProducer)) { ok = false; break; }
          note_load(ld_issued, ld_par, stage, phase);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * (kPairABytes + kPairBBytes));
          const uint32_t bar = map_to_rank(&full[stage], 0);
          uint8_t* a_dst = sA + stage * kPairABytes;
          uint8_t* b_dst = sB + stage * kPairBBytes;
          if (p.a_mn)
            tma_load_2d_pair(a_dst, &tm_a, bar, a_row, kpos * kGemmBK);
          else
            tma_load_2d_pair(a_dst, &tm_a, bar, kpos * kGemmBK, a_row);
          if (p.b_mn)
            tma_load_2d_pair(b_dst, &tm_b, bar, b_row, kpos * kGemmBK);
          else
            tma_load_2d_pair(b_dst, &tm_b, bar, kpos * kGemmBK, b_row);
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
      }
      // Both CTAs' loads complete bytes on the leader's barriers: the leader
      // drains them; the other CTA stays until the final cluster barrier.
      if (leader) drain_loads(full, kPairStages, ld_issued, ld_par, kSitePairDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int lt = 0;
      const uint32_t a_step = p.a_mn ? 32u * 128u : 32u;
      const uint32_t b_step = p.b_mn ? 32u * 128u : 32u;
      const uint32_t lbo = p.a_mn || p.b_mn ? static_cast<uint32_t>(kGemmBK * 128) : 16u;
      for (int tile = pair; tile < p.num_tiles && ok; tile += npairs, ++lt) {
        const uint32_t acc = lt & 1;
        const uint32_t acc_phase = (lt >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, kSitePairMmaAcc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256u;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, kSitePairMma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * kPairABytes);
          const uint32_t b_base = smem_u32(sB + stage * kPairBBytes);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 32; ++kk) {
            const uint64_t adesc = smem_desc_sw128(a_base + kk * a_step, p.a_mn ? lbo : 16u, 1024u);
            const uint64_t bdesc = smem_desc_sw128(b_base + kk * b_step, p.b_mn ? lbo : 16u, 1024u);
            const uint32_t accumulate = (kb > 0 || kk > 0) ? 1u : 0u;
            if (QT == 0)
              mma_i8_pair(d_tmem, adesc, bdesc, p.idesc, accumulate);
            else
              mma_f8_pair(d_tmem, adesc, bdesc, p.idesc, accumulate);
          }
          mma_commit_pair_mc(&empty[stage], 0x3);  // both CTAs' stage is free once these MMAs have read it
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
        mma_commit_pair_mc(&tfull[acc], 0x3);  // both halves of the accumulator complete
      }
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const uint32_t tempty_leader0 = map_to_rank(&tempty[0], 0);
    const uint32_t tempty_leader1 = map_to_rank(&tempty[1], 0);
    constexpr int kChunkCols = OB ? 64 : 32;  // columns per 128-byte row chunk
    uint8_t* outbuf = sOut + quad * (2 * kPairOutBytes);
    const uint32_t swz = static_cast<uint32_t>(lane & 7);
    int nbuf = 0;
    int lt = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs, ++lt) {
      int tm, tn;
      gemm_tile_coords(tile, p.tiles_m, p.tiles_n, p.group_m, tm, tn);
      const uint32_t acc = lt & 1;
      const uint32_t acc_phase = (lt >> 1) & 1;
      const bool ok = mbar_wait(&tfull[acc], acc_phase, kSitePairEpilogue);
      if (bar_or(1, 128, !ok)) break;
      tc_fence_after();
      const int row0 = tm * 256 + static_cast<int>(rank) * 128 + quad * 32;  // this warp's 32 rows
      const int row = row0 + lane;
      const float sa = row < p.m ? p.sa[row] : 0.f;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * 256u;
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += kChunkCols) {
        const int col0 = tn * 256 + c0;
        uint32_t w[32];  // this row's 128 bytes of the chunk
#pragma unroll
        for (int hh = 0; hh < (OB ? 2 : 1); ++hh) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + c0 + 32 * hh, r);
          tmem_ld_wait();
          reg_fence32(r);
          float y[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float a = (QT == 0) ? __int2float_rn(static_cast<int>(r[j])) : __uint_as_float(r[j]);
            const int col = col0 + 32 * hh + j;
            const float sb = col < p.n ? __ldg(p.sb + col) : 0.f;
            y[j] = (a * sa) * sb;
          }
          if (OB) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(y[2 * e], y[2 * e + 1]);
              w[16 * hh + e] = *reinterpret_cast<const uint32_t*>(&b2);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(y[j]);
          }
        }
        uint8_t* buf = outbuf + (nbuf & 1) * kPairOutBytes;
        if (lane == 0) bulk_wait_read<1>();  // the store that last read this buffer is done with it
        __syncwarp();
        // Row `lane` at byte lane * 128; its 16-byte unit j at position j ^ (lane % 8)
        // (the 128-byte swizzle the tensor map describes): conflict-free 16-byte stores.
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(buf + lane * 128 + ((static_cast<uint32_t>(j) ^ swz) << 4)) =
              make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < p.m && col0 < p.n) {
          tma_store_2d(&tm_c, buf, col0, row0);
          bulk_commit();
        }
        ++nbuf;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
    if (lane == 0) bulk_wait<0>();  // every output store has completed
  }

  tc_fence_before();
  __syncthreads();
  cluster_arrive();  // neither CTA leaves while the other may still address its memory
  cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kGemmTmemCols);
  }
}

}  // namespace halo
