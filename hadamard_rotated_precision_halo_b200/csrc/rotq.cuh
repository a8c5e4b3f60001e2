// rotq.cuh -- fused block Walsh-Hadamard rotation + absmax + symmetric quantisation.
//
// Kernels, by rotation axis of a bf16 matrix X[rows, cols]:
//
//   rotq_rows_kernel        rotate along the contiguous dimension (blocks of
//                           128 or 256 consecutive elements of a row), one
//                           scale per row (or per group of 64 / 128 elements).
//   rotq_rows_pair_kernel   the same for rows of 193..256 whole 128-element
//                           blocks, each row split over a two-CTA cluster.
//   rotq_cols_1pass_kernel  rotate along dimension 0 (blocks of 128
//   rotq_cols_kernel        consecutive rows of a column), one scale per
//                           column: a single pass for up to 8192 rows, two
//                           passes above.
//   rotq_cols_grouped_kernel  dimension 0 with one scale per group of 64 / 128
//                           rows of a column.
// A rotated length that is not a multiple of the block is zero-padded.
//
// All compute, for every group g (a row, a column or a part of one),
//     u      = H_blk x            (unnormalised Sylvester transform, fp32)
//     amax_g = max |u|            (over the whole group)
//     s_g    = amax_g / (qmax sqrt(blk))        -> scale of the normalised value
//     q      = round_half_even(u * qmax / amax_g)   (INT8; |q| <= 127 by construction)
//            | e4m3_rn_satfinite(u * qmax / amax_g) (E4M3)
// which equals quantising the normalised rotation H_blk x / sqrt(blk) with
// scale s_g: the 1/sqrt(blk) factor cancels in the codes and only enters s_g.
// Walsh-Hadamard transform and quantiser: QWHA page sec. 2.1-2.2; INT8 / FP8:
// HALO paper page, "key design"; block-local rotation: HALO blog page sec. 5.
//
// Memory path (HBM-bound): one TMA read of the bf16 input, one TMA write of the
// 1-byte codes, one fp32 scale per group.  Every FWHT butterfly runs in
// registers (packed f32x2 adds), no data crosses threads except the top stage
// of a 256-block (one shuffle per element).
#pragma once

#include <cuda_fp8.h>

#include "ptx.cuh"

namespace halo {

enum : unsigned int {
  kSiteRotqRowsLoad = 0x101,
  kSiteRotqRowsDrain = 0x102,
  kSiteRotqColsLoad = 0x201,
  kSiteRotqColsDrain = 0x208,
};

// Per-thread slot sizes in shared memory for rotq_rows: 128 bf16 (256 B) plus
// 16 B of padding, and 128 code bytes plus 16 B of padding.  The padding makes
// the per-thread 16-byte accesses of a quarter warp hit eight distinct bank
// groups.
constexpr int kRowsInSlot = 272;   // bytes (136 bf16)
constexpr int kRowsOutSlot = 144;  // bytes

__device__ __forceinline__ float2 f2_add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.f, -1.f), a);
}

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// In-register unnormalised Walsh-Hadamard transform of 128 values held as 64
// float2 pairs (v[i] = elements 2i, 2i+1), natural Sylvester order.
__device__ __forceinline__ void fwht128_pairs(float2 (&v)[64]) {
  // h = 1: butterflies inside each pair.
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float a = v[i].x, b = v[i].y;
    v[i] = make_float2(a + b, a - b);
  }
  // h = 2 .. 64: pair i with pair i + h/2.
#pragma unroll
  for (int hp = 1; hp < 64; hp *= 2) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      if ((i & hp) == 0) {
        const float2 a = v[i], b = v[i + hp];
        v[i] = f2_add(a, b);
        v[i + hp] = f2_sub(a, b);
      }
    }
  }
}

// max |v| over 128 values as a balanced tree (depth 7 instead of a 128-long
// dependency chain; fmaxf chains are not reassociated by the compiler).
__device__ __forceinline__ float absmax128(const float2 (&v)[64]) {
  float m[32];
#pragma unroll
  for (int i = 0; i < 32; ++i)
    m[i] = fmaxf(fmaxf(fabsf(v[2 * i].x), fabsf(v[2 * i].y)), fmaxf(fabsf(v[2 * i + 1].x), fabsf(v[2 * i + 1].y)));
#pragma unroll
  for (int w = 16; w >= 1; w /= 2) {
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  }
  return m[0];
}

// max |v| over elements 0..63 (x) and 64..127 (y) of 128 values held as 64
// float2 pairs, as two trees.
__device__ __forceinline__ float2 absmax128_halves(const float2 (&v)[64]) {
  float m[32];
#pragma unroll
  for (int i = 0; i < 32; ++i)
    m[i] = fmaxf(fmaxf(fabsf(v[2 * i].x), fabsf(v[2 * i].y)), fmaxf(fabsf(v[2 * i + 1].x), fabsf(v[2 * i + 1].y)));
#pragma unroll
  for (int w = 8; w >= 1; w /= 2) {
#pragma unroll
    for (int i = 0; i < w; ++i) {
      m[i] = fmaxf(m[i], m[i + w]);
      m[16 + i] = fmaxf(m[16 + i], m[16 + i + w]);
    }
  }
  return make_float2(m[0], m[16]);
}

// Column-wise max |v| of 64 float2 (x and y are two columns), as trees.
__device__ __forceinline__ float2 absmax64_cols(const float2 (&v)[64]) {
  float mx[32], my[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    mx[i] = fmaxf(fabsf(v[2 * i].x), fabsf(v[2 * i + 1].x));
    my[i] = fmaxf(fabsf(v[2 * i].y), fabsf(v[2 * i + 1].y));
  }
#pragma unroll
  for (int w = 16; w >= 1; w /= 2) {
#pragma unroll
    for (int i = 0; i < w; ++i) {
      mx[i] = fmaxf(mx[i], mx[i + w]);
      my[i] = fmaxf(my[i], my[i + w]);
    }
  }
  return make_float2(mx[0], my[0]);
}

// Round-half-even of t (|t| <= 2^22) to an int8 code in the low byte of the
// returned word: adding 1.5 * 2^23 puts the rounded integer into the low
// mantissa bits (round-to-nearest-even of the fused multiply-add).
__device__ __forceinline__ uint32_t q_int8_bits(float u, float r) {
  return __float_as_uint(__fmaf_rn(u, r, 12582912.0f));
}

__device__ __forceinline__ uint32_t pack4_int8(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  const uint32_t lo = __byte_perm(b0, b1, 0x0040);
  const uint32_t hi = __byte_perm(b2, b3, 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

__device__ __forceinline__ uint32_t e4m3x2_bits(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// Optional inputs of the rotate+quantise variants (used when a kernel is
// instantiated with EXT = 1):
//   signs  +-1 per position along the rotated dimension (random-sign
//          rotation H (D x)); only the sign bit is used.  nullptr: none.
//   rand   16 random bits per element, layout [rows, cols] with row stride
//          ld_rand: stochastic rounding with u = rand / 65536.  nullptr:
//          round to nearest even.
struct RotqExtras {
  const int8_t* signs;
  const uint16_t* rand;
  int64_t ld_rand;
};

// bf16x2 sign-flip mask from two sign bytes of a 4-byte group (pair 0: bytes
// 0, 1; pair 1: bytes 2, 3): bit 15 and bit 31 take the bytes' sign bits.
__device__ __forceinline__ uint32_t sign_mask_pair(uint32_t s4, int pair) {
  return __byte_perm(s4, 0u, pair ? 0x3424 : 0x1404) & 0x80008000u;
}

// bf16x2 sign-flip mask for both halves from sign byte `b` (0..3) of s4.
__device__ __forceinline__ uint32_t sign_mask_row(uint32_t s4, int b) {
  const uint32_t sel = (static_cast<uint32_t>(b) << 12) | (4u << 8) | (static_cast<uint32_t>(b) << 4) | 4u;
  return __byte_perm(s4, 0u, sel) & 0x80008000u;
}

// Stochastic rounding onto the INT8 grid: the upper neighbour of t when
// uu < t - floor(t); clamped to +-127; the code in the low byte.
__device__ __forceinline__ uint32_t q_int8_sr(float t, float uu) {
  const float lo = floorf(t);
  float q = (uu < t - lo) ? lo + 1.f : lo;
  q = fminf(fmaxf(q, -127.f), 127.f);
  return static_cast<uint32_t>(__float2int_rn(q)) & 0xFFu;
}

// Stochastic rounding onto the E4M3 grid: the signed grid value to encode.
// Grid spacing 2^-9 below 2^-6, else 2^(floor(log2|t|) - 3); |t| >= 448 gives 448.
__device__ __forceinline__ float e4m3_sr_value(float t, float uu) {
  const float a = fabsf(t);
  float mag;
  if (a >= 448.f) {
    mag = 448.f;
  } else {
    const float quantum =
        a < 0.015625f ? 0.001953125f : __uint_as_float(((__float_as_uint(a) >> 23) - 3u) << 23);
    const float lo = floorf(__fdiv_rn(a, quantum)) * quantum;  // exact: quantum is a power of two
    mag = (uu < __fdiv_rn(a - lo, quantum)) ? lo + quantum : lo;
  }
  return copysignf(mag, t);
}

__device__ __forceinline__ float rand_unit(uint32_t bits16) { return static_cast<float>(bits16) * (1.f / 65536.f); }

// ------------------------------------------------------------------------------------------
// rotq_rows: one thread owns one 128-element chunk of one row.  A row is
// handled by a "row group" of G = ceil(nb / 32) warps (one warp when the row
// has 4096 elements); a CTA holds 4 / G groups (or one group of G > 4 warps),
// and every group streams its own rows independently with its own 2-stage TMA
// ring, so warps do not wait on each other beyond their own row.  A row
// arrives by one 3-D TMA load of the view [rows][nb][128] with a 136-element
// box along the innermost dimension: the 8 elements past each chunk fall
// outside the tensor, read as zeros and give the padded per-thread slot for
// free.  Codes leave the same way (144-byte box; the out-of-range tail is not
// written).  Row absmax: redux.sync within a warp, shared memory across the
// group's warps.
// ------------------------------------------------------------------------------------------
struct RotqRowsParams {
  float* scales;
  int64_t rows;
  int nb;        // 128-element chunks per padded row (cols rounded up to the block, / 128)
  int nbt;       // whole 128-element chunks of the input row (loaded by the 3-D TMA view)
  int tail;      // elements of the input's last, partial chunk (0: none; loaded by a 2-D TMA box)
  int gw;        // warps per row group
  int groups;    // row groups per CTA
  float qmax;
  float scale_mult;  // 1 / (qmax * sqrt(blk))
  RotqExtras ex;     // EXT = 1 only
  float* scales2;    // QT = 2 only: the E4M3 scales (`scales` holds the INT8 ones)
  float scale_mult2; // QT = 2 only: 1 / (448 * sqrt(blk))
  int group;         // GR = 1 only: elements per scale group (64 or 128), scales [rows][nb * 128 / group]
  int out_tiles;     // code tiles per row group: 0 (codes written into the consumed input stage), 1, or 2 (QT = 2)
};

// QT = 2: both code sets from one read of the input -- INT8 codes with their
// scales through tm_q / scales, E4M3 codes with theirs through tm_q2 / scales2.
constexpr int kQtDual = 2;

// Shared-memory bytes of one row group: 2 input stages (the per-thread slots,
// then, when padding, 256 bytes for a partial last chunk) and `ntiles` code
// tiles (none when the codes go into the consumed input stage; two for the
// dual output).
__host__ __device__ inline uint32_t rows_group_slots_bytes(int gw) { return static_cast<uint32_t>(gw) * 32 * kRowsInSlot; }
__host__ __device__ inline uint32_t rows_group_in_bytes(int gw, int pad) { return rows_group_slots_bytes(gw) + (pad ? 256 : 0); }
__host__ __device__ inline uint32_t rows_group_out_bytes(int gw) { return static_cast<uint32_t>(gw) * 32 * kRowsOutSlot; }
__host__ __device__ inline uint32_t rows_group_smem(int gw, int ntiles, int pad) {
  return 2 * rows_group_in_bytes(gw, pad) + ntiles * rows_group_out_bytes(gw);
}

__device__ __forceinline__ void group_sync(int gw, int grp) {
  if (gw == 1)
    __syncwarp();
  else
    named_bar_sync(1 + grp, gw * 32);
}

// PAD = 1: the row length is not a multiple of the block (zero padding); the
// instantiation for whole blocks (PAD = 0) carries none of that logic.
// GR = 1: group-wise scales, one per p.group (64 or 128) consecutive elements
// of a row instead of one per row (QT 0 / 1, EXT 0 only).
// p.out_tiles = 0 (one output, chosen by the launcher when it fits more CTAs
// on an SM): a row's codes are written into the input stage the row was read
// from, and that stage is refilled with the next row once their store has read
// them, so only one row is in flight ahead; with <= 168 registers (the bound
// below) three 4-warp CTAs of 8192-wide rows fit on an SM.  Otherwise the codes
// go to tiles of their own and two rows are in flight ahead.
template <int BLK, int QT, int EXT, int PAD, int GR = 0>
__global__ void __launch_bounds__(BLK == 128 && EXT == 0 && QT != kQtDual ? 384 : 256)
    rotq_rows_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xt,
                     const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q2,
                     RotqRowsParams p) {
  const bool in_stage = QT != kQtDual && p.out_tiles == 0;  // codes written into the consumed input stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t full_bar[8][2];
  __shared__ uint32_t s_wmax[2][8];  // per-warp row maxima, by row parity

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int gw = p.gw;
  const int grp = warp / gw;
  const int wig = warp - grp * gw;          // warp index inside the group
  const int chunk = wig * 32 + lane;        // this thread's 128-element chunk of the row
  const bool is_active = chunk < p.nb;
  // Chunks past the input (zero padding up to the block) hold zeros.
  const bool is_zero = PAD && (chunk > p.nbt || (chunk == p.nbt && p.tail == 0));
  const bool leader = (wig == 0 && lane == 0);
  // One row: the 3-D box of whole chunks, plus the partial chunk's 2-D box.
  const uint32_t in_bytes = PAD ? static_cast<uint32_t>(p.nbt) * kRowsInSlot + (p.tail ? 256u : 0u)
                               : static_cast<uint32_t>(p.nb) * kRowsInSlot;
  uint8_t* g_in = smem + grp * rows_group_smem(gw, p.out_tiles, PAD);
  uint8_t* g_out = g_in + 2 * rows_group_in_bytes(gw, PAD);  // code tile (unused when in_stage)
  uint8_t* g_out2 = g_out + rows_group_out_bytes(gw);        // QT = 2 only

  if (leader) {
    mbar_init(&full_bar[grp][0], 1);
    mbar_init(&full_bar[grp][1], 1);
    fence_mbar_init();
    prefetch_tmap(&tm_x);
    if (PAD && p.tail) prefetch_tmap(&tm_xt);
    prefetch_tmap(&tm_q);
    if (QT == kQtDual) prefetch_tmap(&tm_q2);
  }
  __syncthreads();
  griddep_wait();  // inputs written and codes read by the previous kernel
  griddep_launch_dependents();

  const int64_t first = static_cast<int64_t>(blockIdx.x) * p.groups + grp;
  const int64_t step = static_cast<int64_t>(gridDim.x) * p.groups;
  const int64_t nmine = first < p.rows ? (p.rows - first + step - 1) / step : 0;

  uint32_t ld_issued = 0, ld_par = 0;  // loads issued per stage, for the drain at the end
  auto issue = [&](int64_t it) {
    const int st = static_cast<int>(it & 1);
    const int32_t row = static_cast<int32_t>(first + it * step);
    uint8_t* dst = g_in + st * rows_group_in_bytes(gw, PAD);
    note_load(ld_issued, ld_par, st, static_cast<uint32_t>(it >> 1));
    mbar_arrive_expect_tx(&full_bar[grp][st], in_bytes);
    if (!PAD || p.nbt > 0) tma_load_3d(dst, &tm_x, &full_bar[grp][st], 0, 0, row);
    // Partial last chunk: elements past the row's end are out of the 2-D
    // tensor and arrive as zeros (the zero padding).
    if (PAD && p.tail) tma_load_2d(dst + rows_group_slots_bytes(gw), &tm_xt, &full_bar[grp][st], p.nbt * 128, row);
  };
  if (leader) {
    if (nmine > 0) issue(0);
    if (nmine > 1) issue(1);
  }

  bool dead = false;  // a load wait ran out: stop waiting and loading, keep every barrier
  for (int64_t it = 0; it < nmine; ++it) {
    const int st = static_cast<int>(it & 1);
    const int par = static_cast<int>(it & 1);
    const int64_t row = first + it * step;
    if (EXT && p.ex.rand != nullptr && is_active) {
      // This chunk's random bits (two 128-byte lines) into L2 while the row
      // is rotated: the code loop below reads them.
      const uint16_t* rl = p.ex.rand + row * p.ex.ld_rand + static_cast<int64_t>(chunk) * 128;
      prefetch_l2(rl);
      prefetch_l2(rl + 64);
    }
    if (!dead) {
      const bool ok = mbar_wait(&full_bar[grp][st], static_cast<uint32_t>((it >> 1) & 1), kSiteRotqRowsLoad);
      dead = !ok;
    }
    float2 v[64];
    if (is_active && !is_zero && !dead) {
      const uint8_t* stage = g_in + st * rows_group_in_bytes(gw, PAD);
      const uint4* src = reinterpret_cast<const uint4*>(!PAD || chunk < p.nbt ? stage + chunk * kRowsInSlot
                                                                              : stage + rows_group_slots_bytes(gw));
      const uint4* sgn = reinterpret_cast<const uint4*>(p.ex.signs + static_cast<int64_t>(chunk) * 128);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        uint4 raw = src[k];
        if (EXT && p.ex.signs != nullptr) {
          // elements 8k .. 8k+7: sign bytes 8k .. 8k+7 = half of sign vector k/2
          const uint4 sv = __ldg(sgn + k / 2);
          const uint32_t s01 = (k & 1) ? sv.z : sv.x;
          const uint32_t s23 = (k & 1) ? sv.w : sv.y;
          raw.x ^= sign_mask_pair(s01, 0);
          raw.y ^= sign_mask_pair(s01, 1);
          raw.z ^= sign_mask_pair(s23, 0);
          raw.w ^= sign_mask_pair(s23, 1);
        }
        v[4 * k + 0] = bf16x2_to_f2(raw.x);
        v[4 * k + 1] = bf16x2_to_f2(raw.y);
        v[4 * k + 2] = bf16x2_to_f2(raw.z);
        v[4 * k + 3] = bf16x2_to_f2(raw.w);
      }
      fwht128_pairs(v);
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = make_float2(0.f, 0.f);
    }
    group_sync(gw, grp);  // stage `st` fully read
    if (leader) {
      if (in_stage) {
        // The other stage holds the previous row's codes: once their store
        // has read them, it takes the next row.
        if (!dead && it >= 1 && it + 1 < nmine) {
          bulk_wait_read<0>();
          issue(it + 1);
        }
      } else {
        if (!dead && it + 2 < nmine) issue(it + 2);
        bulk_wait_read<0>();  // the previous row's store has read the code tiles
      }
    }
    uint8_t* out = in_stage ? g_in + st * rows_group_in_bytes(gw, PAD) : g_out;
    if (BLK == 256) {
      // Top stage of the 256-point transform: chunk pairs (2j, 2j+1) sit on
      // adjacent lanes.  Lower half keeps a + b, upper half a - b.
      const bool upper = (chunk & 1) != 0;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        float2 o;
        o.x = __shfl_xor_sync(0xffffffffu, v[i].x, 1);
        o.y = __shfl_xor_sync(0xffffffffu, v[i].y, 1);
        v[i] = upper ? f2_sub(o, v[i]) : f2_add(v[i], o);
      }
    }
    if (GR) {
      // Group-wise scales: every group lies inside one thread's 128-element
      // chunk, so no reduction crosses threads.
      const float2 hm = absmax128_halves(v);
      const bool g64 = p.group == 64;
      const float a0 = g64 ? hm.x : fmaxf(hm.x, hm.y);
      const float a1 = g64 ? hm.y : a0;
      const float r0 = a0 > 0.f ? __fdiv_rn(p.qmax, a0) : 0.f;
      const float r1 = a1 > 0.f ? __fdiv_rn(p.qmax, a1) : 0.f;
      if (!in_stage) group_sync(gw, grp);  // orders the leader's store wait before the code writes
      if (is_active) {
        const int gpc = g64 ? 2 : 1;  // scale groups per 128-element chunk
        float* srow = p.scales + row * static_cast<int64_t>(p.nb) * gpc + chunk * gpc;
        srow[0] = a0 * p.scale_mult;
        if (g64) srow[1] = a1 * p.scale_mult;
        uint4* dst = reinterpret_cast<uint4*>(out + chunk * kRowsOutSlot);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float r = k < 4 ? r0 : r1;  // elements 16k .. 16k + 15
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 a = v[8 * k + 2 * j];
            const float2 b = v[8 * k + 2 * j + 1];
            if (QT == 0)
              w[j] = pack4_int8(q_int8_bits(a.x, r), q_int8_bits(a.y, r), q_int8_bits(b.x, r), q_int8_bits(b.y, r));
            else
              w[j] = e4m3x2_bits(a.x * r, a.y * r) | (e4m3x2_bits(b.x * r, b.y * r) << 16);
          }
          dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    } else {
    const float amax = absmax128(v);
    uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if (gw > 1) {
      if (lane == 0) s_wmax[par][warp] = wmax;
      group_sync(gw, grp);  // (code tiles: also orders the leader's store wait before the code writes)
      for (int w = 0; w < gw; ++w) wmax = max(wmax, s_wmax[par][grp * gw + w]);
    } else {
      __syncwarp();
    }
    const float row_amax = __uint_as_float(wmax);
    const float r = row_amax > 0.f ? __fdiv_rn(p.qmax, row_amax) : 0.f;
    if (chunk == 0) p.scales[row] = row_amax * p.scale_mult;
    if (QT == kQtDual) {
      const float r2 = row_amax > 0.f ? __fdiv_rn(448.0f, row_amax) : 0.f;
      if (chunk == 0) p.scales2[row] = row_amax * p.scale_mult2;
      if (is_active) {
        uint4* dst = reinterpret_cast<uint4*>(g_out + chunk * kRowsOutSlot);
        uint4* dst2 = reinterpret_cast<uint4*>(g_out2 + chunk * kRowsOutSlot);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint32_t w[4], w2[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 a = v[8 * k + 2 * j];
            const float2 b = v[8 * k + 2 * j + 1];
            w[j] = pack4_int8(q_int8_bits(a.x, r), q_int8_bits(a.y, r), q_int8_bits(b.x, r), q_int8_bits(b.y, r));
            w2[j] = e4m3x2_bits(a.x * r2, a.y * r2) | (e4m3x2_bits(b.x * r2, b.y * r2) << 16);
          }
          dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
          dst2[k] = make_uint4(w2[0], w2[1], w2[2], w2[3]);
        }
      }
    } else if (is_active) {
      uint4* dst = reinterpret_cast<uint4*>(out + chunk * kRowsOutSlot);
      if (EXT && p.ex.rand != nullptr) {
        // Stochastic rounding: the chunk's 128 random values in two batches of
        // 8 vectors, loaded before the code stores so that the loads overlap.
        const uint4* rnd =
            reinterpret_cast<const uint4*>(p.ex.rand + row * p.ex.ld_rand + static_cast<int64_t>(chunk) * 128);
#pragma unroll
        for (int kb = 0; kb < 8; kb += 4) {
          uint4 rv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) rv[i] = __ldg(rnd + 2 * kb + i);
#pragma unroll
          for (int k = kb; k < kb + 4; ++k) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // elements 16k + 4j .. +3: random halves 4(j%2) .. +3 of vector 2k + j/2
              const float2 a = v[8 * k + 2 * j];
              const float2 b = v[8 * k + 2 * j + 1];
              const uint4 rq = rv[2 * (k - kb) + j / 2];
              const uint32_t r01 = (j & 1) ? rq.z : rq.x;
              const uint32_t r23 = (j & 1) ? rq.w : rq.y;
              const float u0 = rand_unit(r01 & 0xFFFFu), u1 = rand_unit(r01 >> 16);
              const float u2 = rand_unit(r23 & 0xFFFFu), u3 = rand_unit(r23 >> 16);
              if (QT == 0) {
                w[j] = pack4_int8(q_int8_sr(a.x * r, u0), q_int8_sr(a.y * r, u1), q_int8_sr(b.x * r, u2),
                                  q_int8_sr(b.y * r, u3));
              } else {
                w[j] = e4m3x2_bits(e4m3_sr_value(a.x * r, u0), e4m3_sr_value(a.y * r, u1)) |
                       (e4m3x2_bits(e4m3_sr_value(b.x * r, u2), e4m3_sr_value(b.y * r, u3)) << 16);
              }
            }
            dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 a = v[8 * k + 2 * j];
          const float2 b = v[8 * k + 2 * j + 1];
          if (QT == 0) {
            w[j] = pack4_int8(q_int8_bits(a.x, r), q_int8_bits(a.y, r), q_int8_bits(b.x, r),
                              q_int8_bits(b.y, r));
          } else {
            w[j] = e4m3x2_bits(a.x * r, a.y * r) | (e4m3x2_bits(b.x * r, b.y * r) << 16);
          }
        }
        dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      }
    }
    }  // GR
    fence_proxy_async_smem();
    group_sync(gw, grp);
    if (leader) {
      tma_store_3d(&tm_q, out, 0, 0, static_cast<int32_t>(row));
      if (QT == kQtDual) tma_store_3d(&tm_q2, g_out2, 0, 0, static_cast<int32_t>(row));
      bulk_commit();  // one group for both stores: the wait above covers both tiles
    }
  }
  if (leader) {
    drain_loads(full_bar[grp], 2, ld_issued, ld_par, kSiteRotqRowsDrain);
    bulk_wait<0>();
  }
}

// ------------------------------------------------------------------------------------------
// rotq_rows_pair: rows of 193..256 whole 128-element chunks (e.g. 28672
// elements), each split over a cluster of two CTAs of 4 warps: rank r owns
// chunks [r h, r h + h), h = nb / 2 <= 128, one thread per chunk.  One CTA per
// row would need 7-8 warps and two ~61 KB input stages, i.e. one CTA (7-8
// warps) per SM; the halves fit three CTAs (12 warps) per SM.  Each CTA's
// half-row maximum goes to the partner's slot with one 16-byte st.async that
// completes bytes on the partner's mbarrier; two slot buffers alternate over
// rows (the partner writes row k+2's slot only after it has this CTA's row k+1
// maximum, which is sent after this CTA has read row k's slot).  Codes are
// written into the consumed input stage, which is refilled with the next row
// once their store has read them.
// ------------------------------------------------------------------------------------------
struct RotqRowsPairParams {
  float* scales;
  int64_t rows;
  int h;             // chunks per CTA (nb / 2)
  float qmax;
  float scale_mult;  // 1 / (qmax * sqrt(128))
};

enum : unsigned int { kSiteRotqPairLoad = 0x105, kSiteRotqPairReduce = 0x106, kSiteRotqPairDrain = 0x107 };

constexpr uint32_t kRowsPairStageBytes = 128 * kRowsInSlot;  // one stage: up to 128 chunk slots

template <int QT>
__global__ void __launch_bounds__(128, 3)
    rotq_rows_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_q,
                          RotqRowsPairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t full_bar[2];                 // input stage loaded
  __shared__ uint64_t red_bar[2];                  // partner's maximum received, per row parity
  __shared__ uint32_t s_wmax[2][4];                // per-warp maxima, per row parity
  __shared__ __align__(16) uint32_t s_slot[2][4];  // the partner's half-row maximum (element 0)

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t crank = cluster_ctarank();
  const uint32_t peer = crank ^ 1u;
  const int chunk = threadIdx.x;  // this thread's chunk within the CTA's half row
  const bool is_active = chunk < p.h;

  if (threadIdx.x == 0) {
    mbar_init(&full_bar[0], 1);
    mbar_init(&full_bar[1], 1);
    mbar_init(&red_bar[0], 1);
    mbar_init(&red_bar[1], 1);
    fence_mbar_init();
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_q);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&red_bar[0], 16);  // armed for rows 0 and 1
    mbar_arrive_expect_tx(&red_bar[1], 16);
  }
  cluster_arrive();  // the partner is running and initialised before the first remote store
  cluster_wait();
  griddep_wait();
  griddep_launch_dependents();

  const int64_t cid = blockIdx.x / 2;  // this cluster: rows cid, cid + ncl, ...
  const int64_t ncl = gridDim.x / 2;
  const int64_t nmine = cid < p.rows ? (p.rows - cid + ncl - 1) / ncl : 0;

  uint32_t ld_issued = 0, ld_par = 0;  // loads issued per stage, for the drain at the end
  auto issue = [&](int64_t it) {
    const int st = static_cast<int>(it & 1);
    note_load(ld_issued, ld_par, st, static_cast<uint32_t>(it >> 1));
    mbar_arrive_expect_tx(&full_bar[st], static_cast<uint32_t>(p.h) * kRowsInSlot);
    tma_load_3d(smem + st * kRowsPairStageBytes, &tm_x, &full_bar[st], 0, static_cast<int32_t>(crank) * p.h,
                static_cast<int32_t>(cid + it * ncl));
  };
  if (threadIdx.x == 0) {
    if (nmine > 0) issue(0);
    if (nmine > 1) issue(1);
  }

  bool dead = false;  // a wait ran out: stop waiting and loading, keep every barrier and send every maximum
  for (int64_t it = 0; it < nmine; ++it) {
    const int st = static_cast<int>(it & 1);
    const uint32_t ph = static_cast<uint32_t>((it >> 1) & 1);
    const int64_t row = cid + it * ncl;
    uint8_t* stage = smem + st * kRowsPairStageBytes;
    if (!dead) dead = !mbar_wait(&full_bar[st], ph, kSiteRotqPairLoad);
    float2 v[64];
    if (is_active && !dead) {
      const uint4* src = reinterpret_cast<const uint4*>(stage + chunk * kRowsInSlot);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const uint4 raw = src[k];
        v[4 * k + 0] = bf16x2_to_f2(raw.x);
        v[4 * k + 1] = bf16x2_to_f2(raw.y);
        v[4 * k + 2] = bf16x2_to_f2(raw.z);
        v[4 * k + 3] = bf16x2_to_f2(raw.w);
      }
      fwht128_pairs(v);
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = make_float2(0.f, 0.f);
    }
    __syncthreads();  // stage `st` fully read
    if (threadIdx.x == 0 && !dead && it >= 1 && it + 1 < nmine) {
      // The other stage holds the previous row's codes: once their store has
      // read them, it takes the next row.
      bulk_wait_read<0>();
      issue(it + 1);
    }
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(absmax128(v)));
    if (lane == 0) s_wmax[st][warp] = wmax;
    __syncthreads();
    const uint32_t cmax = max(max(s_wmax[st][0], s_wmax[st][1]), max(s_wmax[st][2], s_wmax[st][3]));
    if (threadIdx.x == 0)
      st_async_v4(map_to_rank(&s_slot[st][0], peer), make_uint4(cmax, 0u, 0u, 0u), map_to_rank(&red_bar[st], peer));
    if (!dead) dead = !mbar_wait_cluster(&red_bar[st], ph, kSiteRotqPairReduce);
    const uint32_t pmax = s_slot[st][0];
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&red_bar[st], 16);  // re-armed for row it + 2
    const float row_amax = __uint_as_float(max(cmax, pmax));
    const float r = row_amax > 0.f ? __fdiv_rn(p.qmax, row_amax) : 0.f;
    if (crank == 0 && threadIdx.x == 0) p.scales[row] = row_amax * p.scale_mult;
    if (is_active) {
      uint4* dst = reinterpret_cast<uint4*>(stage + chunk * kRowsOutSlot);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 a = v[8 * k + 2 * j];
          const float2 b = v[8 * k + 2 * j + 1];
          if (QT == 0)
            w[j] = pack4_int8(q_int8_bits(a.x, r), q_int8_bits(a.y, r), q_int8_bits(b.x, r), q_int8_bits(b.y, r));
          else
            w[j] = e4m3x2_bits(a.x * r, a.y * r) | (e4m3x2_bits(b.x * r, b.y * r) << 16);
        }
        dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tma_store_3d(&tm_q, stage, 0, static_cast<int32_t>(crank) * p.h, static_cast<int32_t>(row));
      bulk_commit();
    }
  }
  if (threadIdx.x == 0) {
    drain_loads(full_bar, 2, ld_issued, ld_par, kSiteRotqPairDrain);
    bulk_wait<0>();
  }
  __syncthreads();
  cluster_arrive();  // no CTA leaves while its partner could still store into its shared memory
  cluster_wait();
}

constexpr int kColsStrip = 32;
constexpr int kColsInBytes = 128 * kColsStrip * 2;  // one 128 x 32 bf16 block
constexpr int kColsStages = 2;

// Lane (pcol, h) of a warp owns columns (2 pcol, 2 pcol + 1) and the 64 rows
// 2i + h of a 128-row block held in shared memory as [128][32] bf16.  Reading
// both rows of every pair forms the bottom butterfly stage on the way in
// (h = 0 keeps the sum, h = 1 the difference); the other six stages run on
// the lane's own rows.
// `row_signs` (EXT only): the +-1 signs of the block's 128 rows, or nullptr.
template <int EXT = 0>
__device__ __forceinline__ void cols_load_fwht(const uint32_t* blkw, int pcol, int h, float2 (&v)[64],
                                               const int8_t* row_signs = nullptr) {
  const float sg = h ? -1.f : 1.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    uint32_t wa = blkw[(2 * i) * 16 + pcol];
    uint32_t wb = blkw[(2 * i + 1) * 16 + pcol];
    if (EXT && row_signs != nullptr) {
      const uint32_t s4 = __ldg(reinterpret_cast<const uint32_t*>(row_signs) + i / 2);  // rows 4(i/2) .. +3
      wa ^= sign_mask_row(s4, 2 * (i & 1));
      wb ^= sign_mask_row(s4, 2 * (i & 1) + 1);
    }
    const float2 a = bf16x2_to_f2(wa);
    const float2 b = bf16x2_to_f2(wb);
    v[i] = __ffma2_rn(b, make_float2(sg, sg), a);
  }
}

__device__ __forceinline__ void cols_fwht_rest(float2 (&v)[64]) {
#pragma unroll
  for (int hp = 1; hp < 64; hp *= 2) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      if ((i & hp) == 0) {
        const float2 a = v[i], b = v[i + hp];
        v[i] = f2_add(a, b);
        v[i + hp] = f2_sub(a, b);
      }
    }
  }
}

// Codes of 16 of the lane's rows (v16[i] is row 2 (i0 + i) + h, two columns)
// into a [128][32]-byte tile.  `rnd` (EXT only): random bits of this lane's
// two columns in the block's first row (stride ld_rand between rows), or
// nullptr for round to nearest.
template <int QT, int EXT = 0>
__device__ __forceinline__ void cols_write_codes16(uint8_t* tile, const float2* v16, int i0, float r0, float r1,
                                                   int pcol, int h, const uint16_t* rnd, int64_t ld_rand) {
  uint16_t* outw = reinterpret_cast<uint16_t*>(tile);
  if (EXT && rnd != nullptr) {
    // The 16 rows' random bits are loaded before the code stores so that the
    // loads overlap instead of waiting one by one behind each store.
    uint32_t rb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      rb[i] = __ldg(reinterpret_cast<const uint32_t*>(rnd + (2 * (i0 + i) + h) * ld_rand));
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float u0 = rand_unit(rb[i] & 0xFFFFu), u1 = rand_unit(rb[i] >> 16);
      const float2 x = v16[i];
      uint32_t code;
      if (QT == 0)
        code = __byte_perm(q_int8_sr(x.x * r0, u0), q_int8_sr(x.y * r1, u1), 0x0040) & 0xFFFFu;
      else
        code = e4m3x2_bits(e4m3_sr_value(x.x * r0, u0), e4m3_sr_value(x.y * r1, u1));
      outw[(2 * (i0 + i) + h) * 16 + pcol] = static_cast<uint16_t>(code);
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    uint32_t code;
    if (QT == 0) {
      // Both columns in one packed FMA (same rounding as q_int8_bits).
      const float2 t = __ffma2_rn(v16[i], make_float2(r0, r1), make_float2(12582912.0f, 12582912.0f));
      code = __byte_perm(__float_as_uint(t.x), __float_as_uint(t.y), 0x0040);  // low 16 bits stored
    } else {
      code = e4m3x2_bits(v16[i].x * r0, v16[i].y * r1);
    }
    outw[(2 * (i0 + i) + h) * 16 + pcol] = static_cast<uint16_t>(code);
  }
}

// Stochastic rounding along dimension 0: the random bits of one 128-row block
// of a 32-column strip (128 lines of 64 bytes, 4 per lane) into L2 ahead of
// cols_write_codes, whose loads would otherwise wait on memory.
__device__ __forceinline__ void prefetch_block_rand(const uint16_t* rand, int64_t ld_rand, int64_t row0, int c0,
                                                    int64_t cols, int lane) {
  if (rand == nullptr || c0 >= cols) return;
#pragma unroll
  for (int j = 0; j < 4; ++j) prefetch_l2(rand + (row0 + 4 * lane + j) * ld_rand + c0);
}

// Codes of all of the lane's 64 rows x 2 columns.
template <int QT, int EXT = 0>
__device__ __forceinline__ void cols_write_codes(uint8_t* tile, const float2 (&v)[64], float r0, float r1, int pcol,
                                                 int h, const uint16_t* rnd = nullptr, int64_t ld_rand = 0) {
#pragma unroll
  for (int i0 = 0; i0 < 64; i0 += 16) cols_write_codes16<QT, EXT>(tile, v + i0, i0, r0, r1, pcol, h, rnd, ld_rand);
}

struct RotqColsParams {
  float* scales;
  int64_t cols;
  int nblocks;     // rows / 128
  int warps;       // warps per CTA
  float qmax;
  float scale_mult;  // 1 / (qmax * sqrt(128))
  RotqExtras ex;     // EXT = 1 only
};

template <int QT, int EXT>
__global__ void __launch_bounds__(128, EXT ? 2 : 3)
    rotq_cols_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_q,
                     RotqColsParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t bars[4][kColsStages];
  __shared__ uint32_t s_part[kColsStrip];
  __shared__ float s_colmax[kColsStrip];

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int pcol = lane & 15;  // column pair within the strip
  const int h = lane >> 4;     // row parity
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const int c0 = blockIdx.y * kColsStrip;

  uint8_t* s_in = smem + warp * (kColsStages * kColsInBytes);

  if (threadIdx.x < kColsStrip) s_part[threadIdx.x] = 0u;
  if (lane == 0) {
    for (int s = 0; s < kColsStages; ++s) mbar_init(&bars[warp][s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();  // not resident all at once: no early launch of dependents

  // This warp's blocks: b_i = crank + csize * (warp + warps * i).
  const int first = static_cast<int>(crank) + static_cast<int>(csize) * warp;
  const int step = static_cast<int>(csize) * p.warps;
  const int nmine = first < p.nblocks ? (p.nblocks - first + step - 1) / step : 0;
  // Pass 1 then pass 2 over the same blocks, pass 2 in reverse order: the
  // blocks read last in pass 1 are the likeliest still to be in L2.
  const int nseq = 2 * nmine;

  uint32_t ld_issued = 0, ld_par = 0;  // loads issued per stage, for the drain at the end
  auto issue = [&](int j) {
    const int b = first + step * (j < nmine ? j : 2 * nmine - 1 - j);
    const int s = j % kColsStages;
    note_load(ld_issued, ld_par, s, static_cast<uint32_t>(j / kColsStages));
    mbar_arrive_expect_tx(&bars[warp][s], kColsInBytes);
    tma_load_2d(s_in + s * kColsInBytes, &tm_x, &bars[warp][s], c0, b * 128);
  };
  if (lane == 0) {
    for (int j = 0; j < kColsStages && j < nseq; ++j) issue(j);
  }

  bool failed = false;
  float m0 = 0.f, m1 = 0.f;   // this lane's column maxima (pass 1)
  float r0 = 0.f, r1 = 0.f;   // quantisation multipliers (pass 2)

  for (int j = 0; j < nseq; ++j) {
    if (j == nmine) {
      // End of pass 1 for this warp: fold the two row parities, publish to the CTA.
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 16));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 16));
      if (h == 0) {
        atomicMax(&s_part[2 * pcol], __float_as_uint(m0));
        atomicMax(&s_part[2 * pcol + 1], __float_as_uint(m1));
      }
      break;  // pass 2 continues after the cluster-wide reduction below
    }
    const int s = j % kColsStages;
    const uint32_t ph = (j / kColsStages) & 1u;
    const bool ok = mbar_wait(&bars[warp][s], ph, kSiteRotqColsLoad);
    if (__any_sync(0xffffffffu, !ok)) { failed = true; break; }
    const uint32_t* blkw = reinterpret_cast<const uint32_t*>(s_in + s * kColsInBytes);
    float2 v[64];
    {
      const int b = first + step * j;
      cols_load_fwht<EXT>(blkw, pcol, h, v, EXT && p.ex.signs ? p.ex.signs + static_cast<int64_t>(b) * 128 : nullptr);
    }
    __syncwarp();
    if (lane == 0 && j + kColsStages < nseq) issue(j + kColsStages);
    cols_fwht_rest(v);
    const float2 mm = absmax64_cols(v);
    m0 = fmaxf(m0, mm.x);
    m1 = fmaxf(m1, mm.y);
  }
  // Cluster-wide column maxima through distributed shared memory.
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  if (threadIdx.x < kColsStrip) {
    uint32_t mx = 0u;
    for (uint32_t r = 0; r < csize; ++r) {
      const uint32_t v = ld_shared_cluster_u32(map_to_rank(&s_part[threadIdx.x], r));
      mx = mx > v ? mx : v;
    }
    const float cm = __uint_as_float(mx);
    s_colmax[threadIdx.x] = cm;
    const int64_t col = c0 + threadIdx.x;
    if (crank == 0 && col < p.cols) p.scales[col] = cm * p.scale_mult;
  }
  __syncthreads();
  cluster_arrive();  // this CTA no longer reads remote shared memory

  {
    const float cm0 = s_colmax[2 * pcol], cm1 = s_colmax[2 * pcol + 1];
    r0 = cm0 > 0.f ? __fdiv_rn(p.qmax, cm0) : 0.f;
    r1 = cm1 > 0.f ? __fdiv_rn(p.qmax, cm1) : 0.f;
  }

  // Pass 2.  The codes of a block go into the input stage it was read from;
  // the other stage held the previous block, whose codes were stored from it
  // at the end of the previous iteration: once that store has read them, the
  // stage is refilled with the next block.  (The first two pass-2 blocks were
  // requested during pass 1.)
  for (int j = nmine; j < nseq && !failed; ++j) {
    const int s = j % kColsStages;
    const uint32_t ph = (j / kColsStages) & 1u;
    const bool ok = mbar_wait(&bars[warp][s], ph, kSiteRotqColsLoad);
    if (__any_sync(0xffffffffu, !ok)) { failed = true; break; }
    const uint32_t* blkw = reinterpret_cast<const uint32_t*>(s_in + s * kColsInBytes);
    float2 v[64];
    const int bq = first + step * (2 * nmine - 1 - j);
    if (EXT) prefetch_block_rand(p.ex.rand, p.ex.ld_rand, static_cast<int64_t>(bq) * 128, c0, p.cols, lane);
    cols_load_fwht<EXT>(blkw, pcol, h, v, EXT && p.ex.signs ? p.ex.signs + static_cast<int64_t>(bq) * 128 : nullptr);
    __syncwarp();
    cols_fwht_rest(v);
    if (lane == 0 && j > nmine && j + 1 < nseq) {
      bulk_wait_read<0>();
      issue(j + 1);
    }
    uint8_t* s_codes = s_in + s * kColsInBytes;  // every lane has read this stage (warp sync above)
    {
      const bool col_ok = c0 + 2 * pcol < p.cols;
      const uint16_t* rnd = EXT && p.ex.rand && col_ok
                                ? p.ex.rand + static_cast<int64_t>(bq) * 128 * p.ex.ld_rand + c0 + 2 * pcol
                                : nullptr;
      cols_write_codes<QT, EXT>(s_codes, v, r0, r1, pcol, h, rnd, p.ex.ld_rand);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&tm_q, s_codes, c0, bq * 128);
      bulk_commit();
    }
  }
  if (lane == 0) {
    drain_loads(bars[warp], kColsStages, ld_issued, ld_par, kSiteRotqColsDrain);
    bulk_wait<0>();
  }
  cluster_wait();  // every CTA of the cluster is done reading this CTA's s_part
}


// ------------------------------------------------------------------------------------------
// rotq_cols_1pass: rotation along dimension 0 when a 32-column strip's
// 128-row blocks split over a cluster of at most 16 CTAs of NW <= 4 warps, one
// block per warp (R = CL * NW * 128 <= 8192 rows).  Every rotated value stays
// in registers while the column maxima are reduced, so the input is read once
// and the codes written once.  The codes of a strip go into the input stage
// that strip was read from (the store has read them before the stage is
// refilled), so a warp holds 16 KB of shared memory and three 4-warp CTAs fit
// on an SM.
//
// Column-max reduction per strip: warps -> CTA with shared-memory atomics and
// one CTA barrier; then the CTA's 32 partial maxima (128 bytes) go to every
// cluster CTA's slot [rank] with 16-byte st.async stores that complete bytes
// on that CTA's mbarrier; each CTA waits on its own mbarrier for CL * 128
// bytes and takes the max over the CL slots.  No cluster barrier or memory
// fence in the loop.  Two slot buffers alternate over strips: a peer writes
// strip k+2 only after every CTA has sent strip k+1, which each CTA does only
// after it has read strip k.  The cluster is persistent over strips; each warp
// keeps its block of the next strip in flight with TMA.
// ------------------------------------------------------------------------------------------
struct RotqCols1Params {
  float* scales;
  int64_t cols;
  int strips;  // ceil(cols / 32)
  float qmax;
  float scale_mult;  // 1 / (qmax * sqrt(128))
  RotqExtras ex;     // EXT = 1 only
};

enum : unsigned int { kSiteRotqCols1Load = 0x202, kSiteRotqCols1Reduce = 0x203, kSiteRotqCols1Drain = 0x205 };

template <int QT, int NW, int EXT>
__global__ void __launch_bounds__(NW * 32, EXT ? 8 / NW : 12 / NW)
    rotq_cols_1pass_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_q,
                           RotqCols1Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t bars[NW][2];                            // TMA loads, per warp and stage
  __shared__ uint64_t red_bar[2];                             // partial vectors received, per buffer
  __shared__ uint32_t s_red[2][kColsStrip];                   // this CTA's column maxima (fp32 bits)
  __shared__ __align__(16) uint32_t s_slot[2][16][kColsStrip];  // every cluster CTA's maxima

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int pcol = lane & 15;
  const int h = lane >> 4;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const int blk = static_cast<int>(crank) * NW + warp;  // this warp's 128-row block
  const uint32_t slot_bytes = csize * kColsStrip * 4;

  uint8_t* s_in = smem + warp * (2 * kColsInBytes);

  if (threadIdx.x < 2 * kColsStrip) (&s_red[0][0])[threadIdx.x] = 0u;
  if (lane == 0) {
    mbar_init(&bars[warp][0], 1);
    mbar_init(&bars[warp][1], 1);
  }
  if (threadIdx.x == 0) {
    mbar_init(&red_bar[0], 1);
    mbar_init(&red_bar[1], 1);
  }
  fence_mbar_init();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&red_bar[0], slot_bytes);  // armed for strips 0 and 1
    mbar_arrive_expect_tx(&red_bar[1], slot_bytes);
  }
  cluster_arrive();  // every peer is running and initialised before the first remote store
  cluster_wait();
  griddep_wait();
  griddep_launch_dependents();

  const int first = blockIdx.y;
  const int step = gridDim.y;
  const int nmine = first < p.strips ? (p.strips - first + step - 1) / step : 0;

  uint32_t ld_issued = 0, ld_par = 0;  // loads issued per stage, for the drain at the end
  auto issue = [&](int k) {
    const int st = k & 1;
    note_load(ld_issued, ld_par, st, static_cast<uint32_t>(k >> 1));
    mbar_arrive_expect_tx(&bars[warp][st], kColsInBytes);
    tma_load_2d(s_in + st * kColsInBytes, &tm_x, &bars[warp][st], (first + k * step) * kColsStrip, blk * 128);
  };
  if (lane == 0) {
    if (nmine > 0) issue(0);
    if (nmine > 1) issue(1);
  }

  bool dead = false;  // a wait ran out: stop waiting, still send every partial
  for (int k = 0; k < nmine; ++k) {
    const int c0 = (first + k * step) * kColsStrip;
    const int par = k & 1;
    if (EXT) prefetch_block_rand(p.ex.rand, p.ex.ld_rand, static_cast<int64_t>(blk) * 128, c0, p.cols, lane);
    float2 v[64];
    if (!dead) {
      const bool ok = mbar_wait(&bars[warp][par], (k >> 1) & 1, kSiteRotqCols1Load);
      dead = __any_sync(0xffffffffu, !ok);
    }
    if (!dead) {
      cols_load_fwht<EXT>(reinterpret_cast<const uint32_t*>(s_in + par * kColsInBytes), pcol, h, v,
                          EXT && p.ex.signs ? p.ex.signs + static_cast<int64_t>(blk) * 128 : nullptr);
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = make_float2(0.f, 0.f);
    }
    __syncwarp();
    cols_fwht_rest(v);
    // The other stage held strip k - 1, whose codes were stored from it at the
    // end of the previous iteration: once that store has read them, refill it.
    if (lane == 0 && !dead && k >= 1 && k + 1 < nmine) {
      bulk_wait_read<0>();
      issue(k + 1);
    }
    const float2 mm = absmax64_cols(v);
    float m0 = mm.x, m1 = mm.y;
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 16));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 16));
    if (h == 0) {
      atomicMax(&s_red[par][2 * pcol], __float_as_uint(m0));
      atomicMax(&s_red[par][2 * pcol + 1], __float_as_uint(m1));
    }
    __syncthreads();
    if (threadIdx.x < kColsStrip / 4) {
      // 4 columns per thread, 16 bytes to every cluster CTA's slot [crank].
      uint4 vec = *reinterpret_cast<const uint4*>(&s_red[par][4 * threadIdx.x]);
      *reinterpret_cast<uint4*>(&s_red[par][4 * threadIdx.x]) = make_uint4(0u, 0u, 0u, 0u);  // for strip k + 2
      for (uint32_t r = 0; r < csize; ++r)
        st_async_v4(map_to_rank(&s_slot[par][crank][4 * threadIdx.x], r), vec, map_to_rank(&red_bar[par], r));
    }
    if (!dead) {
      const bool ok = mbar_wait_cluster(&red_bar[par], (k >> 1) & 1, kSiteRotqCols1Reduce);
      dead = __any_sync(0xffffffffu, !ok);
    }
    uint32_t u0 = 0u, u1 = 0u;
    for (uint32_t r = 0; r < csize; ++r) {
      const uint2 pr = *reinterpret_cast<const uint2*>(&s_slot[par][r][2 * pcol]);
      u0 = max(u0, pr.x);
      u1 = max(u1, pr.y);
    }
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&red_bar[par], slot_bytes);  // re-armed for strip k + 2
    const float cm0 = __uint_as_float(u0), cm1 = __uint_as_float(u1);
    const float r0 = cm0 > 0.f ? __fdiv_rn(p.qmax, cm0) : 0.f;
    const float r1 = cm1 > 0.f ? __fdiv_rn(p.qmax, cm1) : 0.f;
    if (crank == 0 && warp == 0 && h == 0) {
      if (c0 + 2 * pcol < p.cols) p.scales[c0 + 2 * pcol] = cm0 * p.scale_mult;
      if (c0 + 2 * pcol + 1 < p.cols) p.scales[c0 + 2 * pcol + 1] = cm1 * p.scale_mult;
    }
    uint8_t* s_codes = s_in + par * kColsInBytes;  // every lane has read this stage (warp sync above)
    {
      const bool col_ok = c0 + 2 * pcol < p.cols;
      const uint16_t* rnd = EXT && p.ex.rand && col_ok
                                ? p.ex.rand + static_cast<int64_t>(blk) * 128 * p.ex.ld_rand + c0 + 2 * pcol
                                : nullptr;
      cols_write_codes<QT, EXT>(s_codes, v, r0, r1, pcol, h, rnd, p.ex.ld_rand);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&tm_q, s_codes, c0, blk * 128);
      bulk_commit();
    }
  }
  if (lane == 0) {
    drain_loads(bars[warp], 2, ld_issued, ld_par, kSiteRotqCols1Drain);
    bulk_wait<0>();
  }
  __syncthreads();
  cluster_arrive();  // no CTA leaves while a peer could still store into its shared memory
  cluster_wait();
}

// ------------------------------------------------------------------------------------------
// rotq_cols_tm: rotation along dimension 0 (one scale per column, up to 32768
// rows) with each strip's rotated values parked in tensor memory while the
// cluster reduces the column maxima.
//
// A 32-column strip's 128-row blocks are spread over a cluster of CL CTAs of
// NW warps, BW blocks per warp.  A warp brings a block in by TMA (two-stage
// ring, loads two blocks ahead), rotates it in registers (lane layout of
// cols_load_fwht), writes the fp32 values to its own tensor-memory lanes
// (tcgen05.st, 128 columns per block) and folds its column maxima into the
// CTA's partial vector with shared-memory atomics.  The warp that completes the
// CTA's count for the strip sends the partial vector (128 bytes) to every
// cluster CTA with st.async, completing bytes on that CTA's mbarrier.  No warp
// waits for another warp of its CTA.
//
// SLOTS = 2: tensor memory holds two strips.  A warp rotates strip k, sends,
// and only then waits for strip k - 1's maxima (which had the whole rotation
// of strip k to arrive), reads strip k - 1 back (tcgen05.ld), quantises it and
// stores its codes by TMA from a code tile of its own.  SLOTS = 1 (taller
// matrices, two blocks per warp): one strip, quantised after its own maxima.
//
// Buffers reused across strips, and why each reuse is safe:
//   s_red[k % 2], s_cnt[k % 2]  -- a warp contributes to strip k + 2 only after
//       it has waited for strip k's maxima, which include this CTA's own
//       strip-k message, sent after the last contributor cleared the buffer.
//   s_slot[k % 4], red_bar[k % 4] -- a peer sends strip k + 4 only after its
//       wait for strip k + 2, which needs this CTA's strip-k + 2 message, sent
//       after every warp here has finished strip k (read its slots; thread 0
//       re-armed the barrier).
//   tensor-memory slot k % SLOTS -- written in strip k + SLOTS by the same warp
//       that read it back (program order, after tcgen05.wait::ld).
// ------------------------------------------------------------------------------------------
struct RotqColsTmParams {
  float* scales;
  int64_t cols;
  int strips;   // ceil(cols / 32)
  int nblocks;  // padded rows / 128
  float qmax;
  float scale_mult;  // 1 / (qmax * sqrt(128))
  RotqExtras ex;     // EXT = 1 only
};

enum : unsigned int { kSiteRotqColsTmLoad = 0x211, kSiteRotqColsTmReduce = 0x212, kSiteRotqColsTmDrain = 0x213 };

constexpr int kColsTmSlotBufs = 4;
constexpr int kColsCodeBytes = 128 * kColsStrip;  // one 128 x 32 code tile

// Dynamic shared memory of rotq_cols_tm: per warp two input stages and two
// code tiles, plus alignment slack.
constexpr size_t cols_tm_smem(int nw) { return static_cast<size_t>(nw) * (2 * kColsInBytes + 2 * kColsCodeBytes) + 128; }

template <int NW, int SLOTS, int BW>
constexpr uint32_t cols_tm_tmem_cols() { return static_cast<uint32_t>(SLOTS * (NW / 4) * BW * 128); }

template <int QT, int NW, int SLOTS, int BW, int EXT = 0>
__global__ void __launch_bounds__(NW * 32, 1)
    rotq_cols_tm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_q,
                        RotqColsTmParams p) {
  static_assert(NW % 4 == 0 && (SLOTS == 1 || SLOTS == 2), "warps come in groups of four tensor-memory quadrants");
  constexpr uint32_t kTmemCols = cols_tm_tmem_cols<NW, SLOTS, BW>();
  static_assert(kTmemCols == 256 || kTmemCols == 512, "tensor-memory allocation must be a power of two");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t ld_bar[NW][2];                                        // TMA loads, per warp and stage
  __shared__ uint64_t red_bar[kColsTmSlotBufs];                             // cluster maxima received
  __shared__ uint32_t s_red[2][kColsStrip];                                 // this CTA's partial maxima
  __shared__ uint32_t s_cnt[2];                                             // warps done with the strip
  __shared__ __align__(16) uint32_t s_slot[kColsTmSlotBufs][16][kColsStrip];  // every cluster CTA's maxima
  __shared__ uint32_t s_tmem;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int pcol = lane & 15;
  const int h = lane >> 4;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const uint32_t slot_bytes = csize * kColsStrip * 4;

  uint8_t* s_in = smem + warp * (2 * kColsInBytes);
  uint8_t* s_code = smem + NW * (2 * kColsInBytes) + warp * (2 * kColsCodeBytes);

  if (threadIdx.x < 2 * kColsStrip) (&s_red[0][0])[threadIdx.x] = 0u;
  if (threadIdx.x < 2) s_cnt[threadIdx.x] = 0u;
  if (lane == 0) {
    mbar_init(&ld_bar[warp][0], 1);
    mbar_init(&ld_bar[warp][1], 1);
  }
  if (threadIdx.x == 0)
    for (int b = 0; b < kColsTmSlotBufs; ++b) mbar_init(&red_bar[b], 1);
  fence_mbar_init();
  if (warp == 0) {
    tmem_alloc(&s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0)
    for (int b = 0; b < kColsTmSlotBufs; ++b) mbar_arrive_expect_tx(&red_bar[b], slot_bytes);  // strips 0..3
  cluster_arrive();  // every peer is running and initialised before the first remote store
  cluster_wait();
  griddep_wait();
  // Every CTA has its tensor memory before a dependent grid may launch (whose
  // CTAs could otherwise hold tensor memory while waiting for this grid).
  griddep_launch_dependents();

  const uint32_t tmem_base = s_tmem;
  const uint32_t t_lane = static_cast<uint32_t>(32 * (warp % 4)) << 16;
  const int wp = warp / 4;
  const int blk0 = (static_cast<int>(crank) * NW + warp) * BW;  // this warp's first block of every strip
  const int nvalid = max(0, min(BW, p.nblocks - blk0));
  const int first = blockIdx.y;
  const int step = gridDim.y;
  const int nmine = first < p.strips ? (p.strips - first + step - 1) / step : 0;
  const int nitems = nmine * nvalid;  // (strip, block) items of this warp, in order

  uint32_t ld_issued = 0, ld_par = 0;
  auto issue = [&](int i) {
    const int k = i / nvalid, j = i % nvalid;  // called only when nvalid > 0
    const int st = i & 1;
    note_load(ld_issued, ld_par, st, static_cast<uint32_t>(i >> 1));
    mbar_arrive_expect_tx(&ld_bar[warp][st], kColsInBytes);
    tma_load_2d(s_in + st * kColsInBytes, &tm_x, &ld_bar[warp][st], (first + k * step) * kColsStrip,
                (blk0 + j) * 128);
  };
  if (lane == 0) {
    if (nitems > 0) issue(0);
    if (nitems > 1) issue(1);
  }

  bool dead = false;  // a wait ran out: stop waiting, keep sending so that peers do not wait on this CTA
  int ncodes = 0;     // code tiles written by this warp (they alternate)

  auto rotate_strip = [&](int k) {
    const int par = k & 1;
    float m0 = 0.f, m1 = 0.f;
    for (int j = 0; j < nvalid; ++j) {
      const int i = k * nvalid + j;
      const int st = i & 1;
      if (EXT)
        prefetch_block_rand(p.ex.rand, p.ex.ld_rand, static_cast<int64_t>(blk0 + j) * 128,
                            (first + k * step) * kColsStrip, p.cols, lane);
      float2 v[64];
      if (!dead) {
        const bool ok = mbar_wait(&ld_bar[warp][st], (i >> 1) & 1, kSiteRotqColsTmLoad);
        dead = __any_sync(0xffffffffu, !ok);
      }
      if (!dead) {
        cols_load_fwht<EXT>(reinterpret_cast<const uint32_t*>(s_in + st * kColsInBytes), pcol, h, v,
                            EXT && p.ex.signs ? p.ex.signs + static_cast<int64_t>(blk0 + j) * 128 : nullptr);
      } else {
#pragma unroll
        for (int q = 0; q < 64; ++q) v[q] = make_float2(0.f, 0.f);
      }
      __syncwarp();  // every lane has read the stage
      if (lane == 0 && !dead && i + 2 < nitems) issue(i + 2);
      cols_fwht_rest(v);
      const float2 mm = absmax64_cols(v);
      m0 = fmaxf(m0, mm.x);
      m1 = fmaxf(m1, mm.y);
      const uint32_t col = static_cast<uint32_t>((((SLOTS == 2 ? par : 0) * (NW / 4) + wp) * BW + j) * 128);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t r[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          r[2 * e] = __float_as_uint(v[16 * q + e].x);
          r[2 * e + 1] = __float_as_uint(v[16 * q + e].y);
        }
        tmem_st_32x32b_x32(tmem_base + t_lane + col + 32 * q, r);
      }
    }
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 16));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 16));
    if (h == 0 && nvalid > 0) {
      atomicMax(&s_red[par][2 * pcol], __float_as_uint(m0));
      atomicMax(&s_red[par][2 * pcol + 1], __float_as_uint(m1));
    }
    __syncwarp();
    uint32_t last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&s_cnt[par], 1u) == static_cast<uint32_t>(NW - 1) ? 1u : 0u;
      if (last) __threadfence_block();
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __syncwarp();
      // Lane (c, r0): 16-byte chunk c = lane & 7 of the 32 maxima, to cluster
      // ranks r0 = lane >> 3, r0 + 4, ...
      const int c = lane & 7;
      const volatile uint32_t* sr = &s_red[par][4 * c];
      const uint4 vec = make_uint4(sr[0], sr[1], sr[2], sr[3]);
      __syncwarp();  // every lane has read the vector before it is cleared for strip k + 2
      if (lane < 8) *reinterpret_cast<uint4*>(&s_red[par][4 * lane]) = make_uint4(0u, 0u, 0u, 0u);
      if (lane == 0) s_cnt[par] = 0u;
      __syncwarp();
      const int b4 = k & (kColsTmSlotBufs - 1);
      for (uint32_t r = static_cast<uint32_t>(lane >> 3); r < csize; r += 4)
        st_async_v4(map_to_rank(&s_slot[b4][crank][4 * c], r), vec, map_to_rank(&red_bar[b4], r));
    }
  };

  auto quantise_strip = [&](int k) {
    const int b4 = k & (kColsTmSlotBufs - 1);
    if (!dead) {
      const bool ok = mbar_wait_cluster(&red_bar[b4], (k >> 2) & 1, kSiteRotqColsTmReduce);
      dead = __any_sync(0xffffffffu, !ok);
    }
    uint32_t u0 = 0u, u1 = 0u;
    for (uint32_t r = 0; r < csize; ++r) {
      const uint2 pr = *reinterpret_cast<const uint2*>(&s_slot[b4][r][2 * pcol]);
      u0 = max(u0, pr.x);
      u1 = max(u1, pr.y);
    }
    __syncwarp();
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&red_bar[b4], slot_bytes);  // armed for strip k + 4
    const float cm0 = __uint_as_float(u0), cm1 = __uint_as_float(u1);
    const float r0 = cm0 > 0.f ? __fdiv_rn(p.qmax, cm0) : 0.f;
    const float r1 = cm1 > 0.f ? __fdiv_rn(p.qmax, cm1) : 0.f;
    const int c0 = (first + k * step) * kColsStrip;
    if (crank == 0 && warp == 0 && h == 0) {
      if (c0 + 2 * pcol < p.cols) p.scales[c0 + 2 * pcol] = cm0 * p.scale_mult;
      if (c0 + 2 * pcol + 1 < p.cols) p.scales[c0 + 2 * pcol + 1] = cm1 * p.scale_mult;
    }
    if (nvalid > 0) tmem_st_wait();  // this warp's stores of the strip have landed
    for (int j = 0; j < nvalid; ++j) {
      const uint32_t col = static_cast<uint32_t>((((SLOTS == 2 ? (k & 1) : 0) * (NW / 4) + wp) * BW + j) * 128);
      // The block's 128 columns in four loads and one wait (one round trip).
      uint32_t r[4][32];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld_32x32b_x32(tmem_base + t_lane + col + 32 * q, r[q]);
      tmem_ld_wait();
      float2 v[64];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        reg_fence32(r[q]);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          v[16 * q + e] = make_float2(__uint_as_float(r[q][2 * e]), __uint_as_float(r[q][2 * e + 1]));
      }
      uint8_t* tile = s_code + (ncodes & 1) * kColsCodeBytes;
      if (lane == 0) bulk_wait_read<1>();  // the store that last read this tile is done with it
      __syncwarp();
      {
        const bool col_ok = c0 + 2 * pcol < p.cols;
        const uint16_t* rnd = EXT && p.ex.rand && col_ok
                                  ? p.ex.rand + static_cast<int64_t>(blk0 + j) * 128 * p.ex.ld_rand + c0 + 2 * pcol
                                  : nullptr;
        cols_write_codes<QT, EXT>(tile, v, r0, r1, pcol, h, rnd, p.ex.ld_rand);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tm_q, tile, c0, (blk0 + j) * 128);
        bulk_commit();
      }
      ++ncodes;
    }
  };

  for (int k = 0; k < nmine; ++k) {
    rotate_strip(k);
    if (SLOTS == 2) {
      if (k >= 1) quantise_strip(k - 1);
    } else {
      quantise_strip(k);
    }
  }
  if (SLOTS == 2 && nmine >= 1) quantise_strip(nmine - 1);

  if (lane == 0) {
    drain_loads(ld_bar[warp], 2, ld_issued, ld_par, kSiteRotqColsTmDrain);
    bulk_wait<0>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, kTmemCols);
  cluster_arrive();  // no CTA leaves while a peer could still store into its shared memory
  cluster_wait();
}

// ------------------------------------------------------------------------------------------
// rotq_cols_grouped: rotation along dimension 0 with group-wise scales, one per
// `group` (64 or 128) consecutive rows of a column.  A group never leaves a
// 128-row block, so every warp works alone: persistent warps walk the (block,
// strip) items in order, each a 128 x 32 tile brought in by TMA through a
// two-stage ring per warp, rotated in registers (lane layout of
// cols_load_fwht), its group maxima taken over the two lanes that share a
// column pair, and its codes written into the consumed stage and stored by TMA.
// ------------------------------------------------------------------------------------------
struct RotqColsGrParams {
  float* scales;  // [rows_p / group][cols]
  int64_t cols;
  int strips;     // ceil(cols / 32)
  int nblocks;    // rows_p / 128
  int group;      // 64 or 128
  float qmax;
  float scale_mult;  // 1 / (qmax * sqrt(128))
};

enum : unsigned int { kSiteRotqColsGrLoad = 0x204, kSiteRotqColsGrDrain = 0x206 };

// Column-wise max |v| over 32 float2 (x and y are two columns), as trees.
__device__ __forceinline__ float2 absmax32_cols(const float2* v) {
  float mx[16], my[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    mx[i] = fmaxf(fabsf(v[2 * i].x), fabsf(v[2 * i + 1].x));
    my[i] = fmaxf(fabsf(v[2 * i].y), fabsf(v[2 * i + 1].y));
  }
#pragma unroll
  for (int w = 8; w >= 1; w /= 2) {
#pragma unroll
    for (int i = 0; i < w; ++i) {
      mx[i] = fmaxf(mx[i], mx[i + w]);
      my[i] = fmaxf(my[i], my[i + w]);
    }
  }
  return make_float2(mx[0], my[0]);
}

template <int QT>
__global__ void __launch_bounds__(128, 3)
    rotq_cols_grouped_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_q,
                             RotqColsGrParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t bars[4][2];

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int pcol = lane & 15;
  const int h = lane >> 4;
  uint8_t* s_in = smem + warp * (2 * kColsInBytes);

  if (lane == 0) {
    mbar_init(&bars[warp][0], 1);
    mbar_init(&bars[warp][1], 1);
  }
  fence_mbar_init();
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();

  const int64_t items = static_cast<int64_t>(p.nblocks) * p.strips;
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * 4 + warp;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * 4;
  const int64_t nmine = wid < items ? (items - wid + nw - 1) / nw : 0;

  uint32_t ld_issued = 0, ld_par = 0;  // loads issued per stage, for the drain at the end
  auto issue = [&](int64_t k) {
    const int64_t it = wid + k * nw;
    const int b = static_cast<int>(it / p.strips), sidx = static_cast<int>(it % p.strips);
    const int st = static_cast<int>(k & 1);
    note_load(ld_issued, ld_par, st, static_cast<uint32_t>(k >> 1));
    mbar_arrive_expect_tx(&bars[warp][st], kColsInBytes);
    tma_load_2d(s_in + st * kColsInBytes, &tm_x, &bars[warp][st], sidx * kColsStrip, b * 128);
  };
  if (lane == 0) {
    if (nmine > 0) issue(0);
    if (nmine > 1) issue(1);
  }

  const bool g64 = p.group == 64;
  bool dead = false;  // a load wait ran out: stop waiting and loading
  for (int64_t k = 0; k < nmine; ++k) {
    const int par = static_cast<int>(k & 1);
    const int64_t it = wid + k * nw;
    const int b = static_cast<int>(it / p.strips);
    const int c0 = static_cast<int>(it % p.strips) * kColsStrip;
    float2 v[64];
    if (!dead) {
      const bool ok = mbar_wait(&bars[warp][par], static_cast<uint32_t>((k >> 1) & 1), kSiteRotqColsGrLoad);
      dead = __any_sync(0xffffffffu, !ok);
    }
    if (!dead) {
      cols_load_fwht<0>(reinterpret_cast<const uint32_t*>(s_in + par * kColsInBytes), pcol, h, v);
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = make_float2(0.f, 0.f);
    }
    __syncwarp();
    cols_fwht_rest(v);
    // The other stage held item k - 1, whose codes were stored from it at the
    // end of the previous iteration: once that store has read them, refill it.
    if (lane == 0 && !dead && k >= 1 && k + 1 < nmine) {
      bulk_wait_read<0>();
      issue(k + 1);
    }
    // Rows 0..63 of the block are the lane's pairs 0..31, rows 64..127 pairs 32..63.
    float2 lo = absmax32_cols(v), hi = absmax32_cols(v + 32);
    lo.x = fmaxf(lo.x, __shfl_xor_sync(0xffffffffu, lo.x, 16));
    lo.y = fmaxf(lo.y, __shfl_xor_sync(0xffffffffu, lo.y, 16));
    hi.x = fmaxf(hi.x, __shfl_xor_sync(0xffffffffu, hi.x, 16));
    hi.y = fmaxf(hi.y, __shfl_xor_sync(0xffffffffu, hi.y, 16));
    if (!g64) {
      lo = make_float2(fmaxf(lo.x, hi.x), fmaxf(lo.y, hi.y));
      hi = lo;
    }
    const float rl0 = lo.x > 0.f ? __fdiv_rn(p.qmax, lo.x) : 0.f, rl1 = lo.y > 0.f ? __fdiv_rn(p.qmax, lo.y) : 0.f;
    const float rh0 = hi.x > 0.f ? __fdiv_rn(p.qmax, hi.x) : 0.f, rh1 = hi.y > 0.f ? __fdiv_rn(p.qmax, hi.y) : 0.f;
    const int col = c0 + 2 * pcol;
    if (h == 0 && col < p.cols) {  // cols % 8 == 0: both columns of the pair are in range
      if (g64) {
        float* s0 = p.scales + static_cast<int64_t>(2 * b) * p.cols + col;
        s0[0] = lo.x * p.scale_mult;
        s0[1] = lo.y * p.scale_mult;
        s0[p.cols] = hi.x * p.scale_mult;
        s0[p.cols + 1] = hi.y * p.scale_mult;
      } else {
        float* s0 = p.scales + static_cast<int64_t>(b) * p.cols + col;
        s0[0] = lo.x * p.scale_mult;
        s0[1] = lo.y * p.scale_mult;
      }
    }
    uint8_t* s_codes = s_in + par * kColsInBytes;  // every lane has read this stage (warp sync above)
#pragma unroll
    for (int c = 0; c < 4; ++c)  // pairs 16c .. 16c + 15 = rows 32c .. 32c + 31
      cols_write_codes16<QT, 0>(s_codes, v + 16 * c, 16 * c, c < 2 ? rl0 : rh0, c < 2 ? rl1 : rh1, pcol, h,
                                nullptr, 0);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&tm_q, s_codes, c0, b * 128);
      bulk_commit();
    }
  }
  if (lane == 0) {
    drain_loads(bars[warp], 2, ld_issued, ld_par, kSiteRotqColsGrDrain);
    bulk_wait<0>();
  }
}

// ------------------------------------------------------------------------------------------
// rotq_cols_split: the dimension-0 rotation split at the column maxima, for a
// matrix whose rows are spread over several devices (each holds whole 128-row
// blocks).  MODE 0: the per-column maxima of the unnormalised transform,
// max |H x| over this device's rows, merged into amax[] with atomicMax (the
// caller zeroes it; one device's vector is then reduced with the others').
// MODE 1: codes and scales from given per-column maxima (the maxima over
// every device's rows): the same rotation, multipliers qmax / amax and codes
// as the single-device kernels, so the codes are those of the whole matrix.
// Independent warps over the (128-row block, 32-column strip) items, lane
// layout of cols_load_fwht, two-stage TMA ring per warp.
// ------------------------------------------------------------------------------------------
struct RotqColsSplitParams {
  float* amax;          // MODE 0: [cols] maxima out (fp32 bits, atomicMax); MODE 1: [cols] maxima in
  float* scales;        // MODE 1: [cols] scales out (amax * scale_mult)
  int64_t cols;
  int strips;           // ceil(cols / 32)
  int nblocks;          // rows_p / 128
  float qmax;
  float scale_mult;     // 1 / (qmax * sqrt(128))
};

enum : unsigned int { kSiteRotqColsSplitLoad = 0x221, kSiteRotqColsSplitDrain = 0x222 };

template <int QT, int MODE>
__global__ void __launch_bounds__(128, 3)
    rotq_cols_split_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_q,
                           RotqColsSplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t bars[4][2];

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int pcol = lane & 15;
  const int h = lane >> 4;
  uint8_t* s_in = smem + warp * (2 * kColsInBytes);

  if (lane == 0) {
    mbar_init(&bars[warp][0], 1);
    mbar_init(&bars[warp][1], 1);
  }
  fence_mbar_init();
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();

  const int64_t items = static_cast<int64_t>(p.nblocks) * p.strips;
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * 4 + warp;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * 4;
  const int64_t nmine = wid < items ? (items - wid + nw - 1) / nw : 0;

  uint32_t ld_issued = 0, ld_par = 0;
  auto issue = [&](int64_t k) {
    const int64_t it = wid + k * nw;
    const int b = static_cast<int>(it / p.strips), sidx = static_cast<int>(it % p.strips);
    const int st = static_cast<int>(k & 1);
    note_load(ld_issued, ld_par, st, static_cast<uint32_t>(k >> 1));
    mbar_arrive_expect_tx(&bars[warp][st], kColsInBytes);
    tma_load_2d(s_in + st * kColsInBytes, &tm_x, &bars[warp][st], sidx * kColsStrip, b * 128);
  };
  if (lane == 0) {
    if (nmine > 0) issue(0);
    if (nmine > 1) issue(1);
  }

  bool dead = false;
  for (int64_t k = 0; k < nmine; ++k) {
    const int par = static_cast<int>(k & 1);
    const int64_t it = wid + k * nw;
    const int b = static_cast<int>(it / p.strips);
    const int c0 = static_cast<int>(it % p.strips) * kColsStrip;
    const int col = c0 + 2 * pcol;
    float2 v[64];
    if (!dead) {
      const bool ok = mbar_wait(&bars[warp][par], static_cast<uint32_t>((k >> 1) & 1), kSiteRotqColsSplitLoad);
      dead = __any_sync(0xffffffffu, !ok);
    }
    if (!dead) {
      cols_load_fwht<0>(reinterpret_cast<const uint32_t*>(s_in + par * kColsInBytes), pcol, h, v);
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = make_float2(0.f, 0.f);
    }
    __syncwarp();
    if (MODE == 0) {
      // The stage is free once read: refill it with item k + 2 now.
      if (lane == 0 && !dead && k + 2 < nmine) issue(k + 2);
      cols_fwht_rest(v);
      const float2 mm = absmax64_cols(v);
      const float m0 = fmaxf(mm.x, __shfl_xor_sync(0xffffffffu, mm.x, 16));
      const float m1 = fmaxf(mm.y, __shfl_xor_sync(0xffffffffu, mm.y, 16));
      if (h == 0) {
        unsigned int* am = reinterpret_cast<unsigned int*>(p.amax);
        if (col < p.cols) atomicMax(am + col, __float_as_uint(m0));
        if (col + 1 < p.cols) atomicMax(am + col + 1, __float_as_uint(m1));
      }
    } else {
      cols_fwht_rest(v);
      // The other stage held item k - 1, whose codes were stored from it at
      // the end of the previous iteration: once that store has read them, refill it.
      if (lane == 0 && !dead && k >= 1 && k + 1 < nmine) {
        bulk_wait_read<0>();
        issue(k + 1);
      }
      const float cm0 = col < p.cols ? __ldg(p.amax + col) : 0.f;
      const float cm1 = col + 1 < p.cols ? __ldg(p.amax + col + 1) : 0.f;
      const float r0 = cm0 > 0.f ? __fdiv_rn(p.qmax, cm0) : 0.f;
      const float r1 = cm1 > 0.f ? __fdiv_rn(p.qmax, cm1) : 0.f;
      if (b == 0 && h == 0) {
        if (col < p.cols) p.scales[col] = cm0 * p.scale_mult;
        if (col + 1 < p.cols) p.scales[col + 1] = cm1 * p.scale_mult;
      }
      uint8_t* s_codes = s_in + par * kColsInBytes;  // every lane has read this stage (warp sync above)
      cols_write_codes<QT>(s_codes, v, r0, r1, pcol, h);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tm_q, s_codes, c0, b * 128);
        bulk_commit();
      }
    }
  }
  if (lane == 0) {
    drain_loads(bars[warp], 2, ld_issued, ld_par, kSiteRotqColsSplitDrain);
    bulk_wait<0>();
  }
}

}  // namespace halo
