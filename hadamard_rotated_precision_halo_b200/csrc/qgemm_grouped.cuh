// qgemm_grouped.cuh -- low-precision GEMM on codes with group-wise scales along
// the contraction dimension:
//
//     C[i, j] = sum_G s_a[i, G] * s_b[j, G] * sum_{k in group G} A[i, k] B[j, k]
//
// Groups of `group` (64 or 128) consecutive K positions, each with its own
// scale per operand row (QWHA page sec. 3.1, group_quantize; sec. 3.2: group
// size 64).  A group's partial product cannot be scaled inside the tensor
// core, so each group is accumulated on its own and promoted:
//
//   warp 0      TMA producer: a 128 x 128 A tile and a 256 x 128 B tile (as
//               two 128-wide boxes) per K block of 128 codes, 128-byte
//               swizzle, into a 4-stage ring.
//   warp 1      tensor-memory allocator and MMA issuer: for every group, the
//               group's K steps (group / 32 MMAs of 128x256x32) into one of
//               two 256-column partial accumulators in tensor memory, then a
//               commit that marks that partial full.
//   warps 2-9   promotion: eight warps, two per tensor-memory lane quarter;
//               each thread owns 128 columns of one tile row and keeps their
//               fp32 running sums in registers.  Per group it reads its slice
//               of the partial (tcgen05.ld, 4 columns at a time: small loads
//               leave the registers to the sums), converts it (INT8: exact
//               int32 -> fp32, |partial| <= 127^2 * 128 < 2^24), multiplies
//               by s_a[i, G] * s_b[j, G] and adds, and frees the partial once
//               its last slice is in registers.  The s_a and s_b of 8 groups
//               are staged in shared memory at a time by asynchronous copies
//               issued one chunk ahead, so the promotion warps meet at a
//               barrier once per 8 groups and never wait on a global load.
// Each group's hand-over (the MMA thread's waits, fences and commits, the
// promotion warps' wait and release) costs about the same whatever the tile
// width, so the 256-column tile does twice the tensor work per hand-over of a
// 128-column one; the price is two partials instead of four (the MMAs run one
// group ahead of the promotion).
// After the last group the running sums are stored as fp32 or bf16.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "qgemm.cuh"

namespace halo {

enum : unsigned int {
  kSiteGgProducer = 0x321,
  kSiteGgMma = 0x322,
  kSiteGgPartial = 0x323,
  kSiteGgPromote = 0x324,
  kSiteGgDrain = 0x325,
};

constexpr int kGgBM = 128;
constexpr int kGgBN = 256;
constexpr int kGgBK = 128;
constexpr int kGgStages = 4;
constexpr int kGgABytes = kGgBM * kGgBK;  // 16 KB
constexpr int kGgBBytes = kGgBN * kGgBK;  // 32 KB: two 128-row (K-major) or 128-column (MN-major) boxes
constexpr int kGgBHalf = kGgBBytes / 2;
constexpr int kGgPartials = 2;            // 256-column partial accumulators
constexpr uint32_t kGgTmemCols = 512;
constexpr int kGgPromWarps = 8;                      // a multiple of 4 (lane quarters)
constexpr int kGgThreads = 64 + 32 * kGgPromWarps;  // producer, MMA, promotion
constexpr int kGgPromThreads = 32 * kGgPromWarps;
constexpr int kGgColsPerThread = kGgBN * 4 / kGgPromWarps;  // columns of a tile row per promotion thread
constexpr int kGgChunk = 8;  // groups whose scales are staged together
constexpr int kGgLdCols = 4;  // columns per tensor-memory load (registers: 128 sums + 4)
// Dynamic shared memory: stages + 1 KB alignment slack + scale staging (2
// buffers x kGgChunk groups x (256 s_b + 128 s_a) floats) + barriers.
constexpr size_t kGgSmemBytes =
    kGgStages * (kGgABytes + kGgBBytes) + 1024 + 2 * kGgChunk * (kGgBN + kGgBM) * 4 + 256;

struct GroupedGemmParams {
  int m, n, k, group;
  int tiles_m, tiles_n, num_tiles;
  int a_mn, b_mn;  // operand storage: 0 = K-major, 1 = MN-major
  uint32_t idesc;
  // Scale of (row i, group G): sa[i * sa_row + G * sa_grp] (likewise sb).
  const float* sa;
  int64_t sa_row, sa_grp;
  const float* sb;
  int64_t sb_row, sb_grp;
  void* c;
  int64_t ldc;
  int out_bf16;
};

template <int QT>
__global__ void __launch_bounds__(kGgThreads, 1)
    qgemm_grouped_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                         GroupedGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGgStages * kGgABytes;
  float* sbuf = reinterpret_cast<float*>(sB + kGgStages * kGgBBytes);  // s_b [2][kGgChunk][256], s_a [2][kGgChunk][128]
  uint64_t* full = reinterpret_cast<uint64_t*>(sbuf + 2 * kGgChunk * (kGgBN + kGgBM));
  uint64_t* empty = full + kGgStages;
  uint64_t* pfull = empty + kGgStages;
  uint64_t* pempty = pfull + kGgPartials;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pempty + kGgPartials);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGgStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kGgPartials; ++b) {
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], kGgPromWarps);  // one arrival per promotion warp
    }
    fence_mbar_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kGgTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kblocks = p.k / kGgBK;            // K is a multiple of 128
  const int gpb = kGgBK / p.group;            // groups per K block: 1 or 2
  const int steps_per_group = p.group / 32;   // MMAs (K = 32 each) per group
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
          if (!mbar_wait(&empty[stage], phase ^ 1u, kSiteGgProducer)) { ok = false; break; }
          note_load(ld_issued, ld_par, stage, phase);
          mbar_arrive_expect_tx(&full[stage], kGgABytes + kGgBBytes);
          uint8_t* a_dst = sA + stage * kGgABytes;
          uint8_t* b_dst = sB + stage * kGgBBytes;
          if (p.a_mn)
            tma_load_2d(a_dst, &tm_a, &full[stage], tm * kGgBM, kb * kGgBK);
          else
            tma_load_2d(a_dst, &tm_a, &full[stage], kb * kGgBK, tm * kGgBM);
          // B in two 128-wide boxes (a box row holds at most 128 swizzled
          // bytes); a box past the matrix reads as zeros.
          if (p.b_mn) {
            tma_load_2d(b_dst, &tm_b, &full[stage], tn * kGgBN, kb * kGgBK);
            tma_load_2d(b_dst + kGgBHalf, &tm_b, &full[stage], tn * kGgBN + 128, kb * kGgBK);
          } else {
            tma_load_2d(b_dst, &tm_b, &full[stage], kb * kGgBK, tn * kGgBN);
            tma_load_2d(b_dst + kGgBHalf, &tm_b, &full[stage], kb * kGgBK, tn * kGgBN + 128);
          }
          if (++stage == kGgStages) { stage = 0; phase ^= 1u; }
        }
      }
      drain_loads(full, kGgStages, ld_issued, ld_par, kSiteGgDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t gi = 0;  // groups issued so far (all tiles)
      const uint32_t a_step = p.a_mn ? 32u * 128u : 32u;
      const uint32_t b_step = p.b_mn ? 32u * 128u : 32u;
      const uint32_t a_lbo = p.a_mn ? static_cast<uint32_t>(kGgBK * 128) : 16u;
      const uint32_t b_lbo = p.b_mn ? static_cast<uint32_t>(kGgBK * 128) : 16u;
      const uint64_t as4 = a_step >> 4, bs4 = b_step >> 4;  // one K step in descriptor units
      const uint32_t idesc = p.idesc;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < kblocks && ok; ++kb) {
          if (!mbar_wait(&full[stage], phase, kSiteGgMma)) { ok = false; break; }
          tc_fence_after();
          // Descriptors of the stage's first K step.  A K step adds its byte
          // offset / 16 to the start-address field (shared-memory offsets stay
          // below 256 KB, so the 14-bit field never carries).  The issue loop
          // is short: one thread issues every MMA, and its per-group cost
          // paces the kernel.
          const uint64_t adesc0 = smem_desc_sw128(smem_u32(sA + stage * kGgABytes), a_lbo, 1024u);
          const uint64_t bdesc0 = smem_desc_sw128(smem_u32(sB + stage * kGgBBytes), b_lbo, 1024u);
          for (int gs = 0; gs < gpb; ++gs, ++gi) {
            const uint32_t pb = gi % kGgPartials;
            if (!mbar_wait(&pempty[pb], ((gi / kGgPartials) & 1u) ^ 1u, kSiteGgPartial)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + pb * static_cast<uint32_t>(kGgBN);
            const uint64_t ad = adesc0 + ((gs * steps_per_group * a_step) >> 4);
            const uint64_t bd = bdesc0 + ((gs * steps_per_group * b_step) >> 4);
            // group 64: two MMAs of K = 32; group 128: four
            if (QT == 0) {
              mma_i8(d_tmem, ad, bd, idesc, 0u);
              mma_i8(d_tmem, ad + as4, bd + bs4, idesc, 1u);
              if (steps_per_group == 4) {
                mma_i8(d_tmem, ad + 2 * as4, bd + 2 * bs4, idesc, 1u);
                mma_i8(d_tmem, ad + 3 * as4, bd + 3 * bs4, idesc, 1u);
              }
            } else {
              mma_f8(d_tmem, ad, bd, idesc, 0u);
              mma_f8(d_tmem, ad + as4, bd + bs4, idesc, 1u);
              if (steps_per_group == 4) {
                mma_f8(d_tmem, ad + 2 * as4, bd + 2 * bs4, idesc, 1u);
                mma_f8(d_tmem, ad + 3 * as4, bd + 3 * bs4, idesc, 1u);
              }
            }
            mma_commit(&pfull[pb]);  // this group's partial is complete
          }
          mma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == kGgStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else {
    // Promotion.  A warp may only read tensor-memory lanes 32*(warp%4) .. +31:
    // that quarter gives the tile rows, (warp - 2) / 4 the 128-column half.
    const int quad = warp & 3;
    const int slice = (warp - 2) >> 2;  // this thread's kGgColsPerThread columns: 0 or 1
    const int row_in_tile = quad * 32 + lane;
    const int ngroups = p.k / p.group;
    // Scale staging: for a chunk of kGgChunk groups, each of the 256 promotion
    // threads copies one column's s_b per group into shared memory, and the
    // 128 threads of warps 2-5 (lane quarters 2, 3, 0, 1: the tile's 128 rows)
    // one row's s_a.  The copies of the next chunk are issued as soon as a
    // chunk starts and land while it is promoted.
    const bool sb_stager = (warp - 2) < kGgBN / 32;  // warps 2-9: one column each
    const bool sa_stager = (warp - 2) < 4;           // warps 2-5: one row each
    const bool stager = sb_stager;
    const int scol_in_tile = (warp - 2) * 32 + lane;  // valid for s_b stagers: 0..255
    float* const sb_bufs = sbuf;                               // [2][kGgChunk][256]
    float* const sa_bufs = sbuf + 2 * kGgChunk * kGgBN;        // [2][kGgChunk][128]
    auto stage_chunk = [&](int tile, int g0, uint32_t buf) {
      int tm, tn;
      gemm_tile_coords(tile, p.tiles_m, p.tiles_n, tm, tn);
      const int gn = min(kGgChunk, ngroups - g0);
      const int scol = tn * kGgBN + scol_in_tile;
      const int srow = tm * kGgBM + row_in_tile;
      const bool cok = scol < p.n, rok = srow < p.m;
      const float* sbp = p.sb + static_cast<int64_t>(cok ? scol : 0) * p.sb_row + static_cast<int64_t>(g0) * p.sb_grp;
      const float* sap = p.sa + static_cast<int64_t>(rok ? srow : 0) * p.sa_row + static_cast<int64_t>(g0) * p.sa_grp;
      float* db = sb_bufs + buf * (kGgChunk * kGgBN) + scol_in_tile;
      float* da = sa_bufs + buf * (kGgChunk * kGgBM) + row_in_tile;
      for (int gg = 0; gg < gn; ++gg)
        cp_async_4(db + gg * kGgBN, sbp + static_cast<int64_t>(gg) * p.sb_grp, cok ? 4u : 0u);
      if (sa_stager)
        for (int gg = 0; gg < gn; ++gg)
          cp_async_4(da + gg * kGgBM, sap + static_cast<int64_t>(gg) * p.sa_grp, rok ? 4u : 0u);
      cp_async_commit();
    };
    uint32_t gi = 0;
    uint32_t ci = 0;  // chunks started so far (all tiles): picks the staging buffer
    bool dead = false;
    if (stager && static_cast<int>(blockIdx.x) < p.num_tiles) stage_chunk(blockIdx.x, 0, 0);
    for (int tile = blockIdx.x; tile < p.num_tiles && !dead; tile += gridDim.x) {
      int tm, tn;
      gemm_tile_coords(tile, p.tiles_m, p.tiles_n, tm, tn);
      const int row = tm * kGgBM + row_in_tile;
      const bool row_ok = row < p.m;
      float run[kGgColsPerThread];
#pragma unroll
      for (int j = 0; j < kGgColsPerThread; ++j) run[j] = 0.f;
      const uint32_t t_cols = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + slice * kGgColsPerThread;
#pragma unroll 1
      for (int g0 = 0; g0 < ngroups; g0 += kGgChunk, ++ci) {
        const uint32_t buf = ci & 1u;
        if (stager) cp_async_wait_all();  // this chunk's copies, issued one chunk ago
        // All promotion threads: publishes the chunk's scales, and every thread
        // has finished the previous chunk, whose buffer is refilled next; a
        // wait that ran out in the previous chunk stops all.
        if (bar_or(1, kGgPromThreads, dead)) { dead = true; break; }
        if (stager) {
          int nt = tile, ng0 = g0 + kGgChunk;
          if (ng0 >= ngroups) { nt = tile + gridDim.x; ng0 = 0; }
          if (nt < p.num_tiles) stage_chunk(nt, ng0, buf ^ 1u);
        }
        const float* sb_chunk = sb_bufs + buf * (kGgChunk * kGgBN);
        const float* sa_chunk = sa_bufs + buf * (kGgChunk * kGgBM);
        const int gn = min(kGgChunk, ngroups - g0);
#pragma unroll 1
        for (int gg = 0; gg < gn; ++gg, ++gi) {
          const float sa = sa_chunk[gg * kGgBM + row_in_tile];
          const uint32_t pb = gi % kGgPartials;
          if (!dead && !mbar_wait(&pfull[pb], (gi / kGgPartials) & 1u, kSiteGgPromote)) dead = true;
          dead = __any_sync(0xffffffffu, dead);
          if (dead) continue;  // still reach the next chunk barrier
          tc_fence_after();
          const float* sb_buf = sb_chunk + gg * kGgBN;
#pragma unroll
          for (int ch = 0; ch < kGgColsPerThread / kGgLdCols; ++ch) {
          uint32_t r[kGgLdCols];
          tmem_ld_32x32b_x4(t_cols + pb * static_cast<uint32_t>(kGgBN) + ch * kGgLdCols, r);
          tmem_ld_wait();
          reg_fence4(r);  // no use of r is scheduled above the wait
          if (ch == kGgColsPerThread / kGgLdCols - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[pb]);  // the partial is in registers: free it early
          }
          const float4* sbv4 = reinterpret_cast<const float4*>(sb_buf + slice * kGgColsPerThread + ch * kGgLdCols);
#pragma unroll
          for (int q = 0; q < kGgLdCols / 4; ++q) {
            const float4 sbq = sbv4[q];
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              const int j = 4 * q + e;
              const int jr = ch * kGgLdCols + j;  // index into run[]
              float2 a;
              if (QT == 0)
                a = make_float2(__int2float_rn(static_cast<int>(r[j])), __int2float_rn(static_cast<int>(r[j + 1])));
              else
                a = make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1]));
              const float2 w = __fmul2_rn(make_float2(sa, sa), e == 0 ? make_float2(sbq.x, sbq.y)
                                                                        : make_float2(sbq.z, sbq.w));
              const float2 acc = __ffma2_rn(a, w, make_float2(run[jr], run[jr + 1]));
              run[jr] = acc.x;
              run[jr + 1] = acc.y;
            }
          }
          }
        }
      }
      if (bar_or(1, kGgPromThreads, dead)) dead = true;  // agree before the stores
      if (dead) break;
      // Store this thread's columns of the tile row, 32 at a time.
#pragma unroll
      for (int ch = 0; ch < kGgColsPerThread / 32; ++ch) {
      const int col0 = tn * kGgBN + slice * kGgColsPerThread + ch * 32;
      const float* run32 = run + ch * 32;
      if (row_ok && col0 < p.n) {
        if (p.out_bf16) {
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.c) + static_cast<int64_t>(row) * p.ldc + col0;
          if (col0 + 32 <= p.n) {
            uint4* o4 = reinterpret_cast<uint4*>(out);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(run32[8 * q + 2 * e], run32[8 * q + 2 * e + 1]);
                w[e] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              o4[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.n) out[j] = __float2bfloat16_rn(run32[j]);
          }
        } else {
          float* out = static_cast<float*>(p.c) + static_cast<int64_t>(row) * p.ldc + col0;
          if (col0 + 32 <= p.n) {
            float4* o4 = reinterpret_cast<float4*>(out);
#pragma unroll
            for (int q = 0; q < 8; ++q) o4[q] = make_float4(run32[4 * q], run32[4 * q + 1], run32[4 * q + 2], run32[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.n) out[j] = run32[j];
          }
        }
      }
      }
    }
  }

  if (warp >= 2) cp_async_wait_all();  // no scale copy lands after the CTA exits
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kGgTmemCols);
  }
}

}  // namespace halo
