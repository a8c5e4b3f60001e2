// halo.cu -- C ABI (include/halo.h): validation, tensor-map encoding and launch
// orchestration for the rotate+quantise kernels and the tcgen05 GEMM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/halo.h"
#include "qgemm.cuh"
#include "qgemm_grouped.cuh"
#include "rotq.cuh"

using namespace halo;

// Scratch of halo_linear_fwd_noalloc: codes and scales of X and W live here
// instead of in a caller workspace.  Host code must not use this name as an
// address (it is a host-side stand-in); the device address comes from
// cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[HALO_NOALLOC_SCRATCH_BYTES];

namespace {

thread_local int g_last_cuda_error = 0;
thread_local char g_last_detail[256] = "";

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  std::atomic<bool> ready{false};  // set last, with release order, once the rest is filled in
  bool supported = false;
  int sm_count = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

halo_status_t cuda_fail(cudaError_t e, const char* what) {
  g_last_cuda_error = static_cast<int>(e);
  snprintf(g_last_detail, sizeof g_last_detail, "%s: %s", what, cudaGetErrorString(e));
  return HALO_ERR_CUDA;
}

#define HALO_CUDA(call)                                  \
  do {                                                   \
    cudaError_t e_ = (call);                             \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call);  \
  } while (0)

// Let a kernel use all the dynamic shared memory it may: the opt-in limit
// minus its static shared memory.
template <typename K>
cudaError_t set_smem_attr(K kernel, int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin - static_cast<int>(fa.sharedSizeBytes));
}

typedef void (*RowsKernel)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                           RotqRowsParams);
typedef void (*Cols1Kernel)(const CUtensorMap, const CUtensorMap, RotqCols1Params);
typedef void (*Cols2Kernel)(const CUtensorMap, const CUtensorMap, RotqColsParams);

// `ext`: the instantiation that reads the variants' optional inputs (signs,
// random bits); the plain path is compiled without them.
template <int PAD>
RowsKernel rows_kernel_grouped_for(int blk, int qtype) {
  if (blk == 128) return qtype == HALO_Q_INT8 ? rotq_rows_kernel<128, 0, 0, PAD, 1> : rotq_rows_kernel<128, 1, 0, PAD, 1>;
  return qtype == HALO_Q_INT8 ? rotq_rows_kernel<256, 0, 0, PAD, 1> : rotq_rows_kernel<256, 1, 0, PAD, 1>;
}

template <int PAD>
RowsKernel rows_kernel_for(int blk, int qtype, bool ext) {
  if (qtype == kQtDual)
    return blk == 128 ? rotq_rows_kernel<128, kQtDual, 0, PAD> : rotq_rows_kernel<256, kQtDual, 0, PAD>;
  if (blk == 128) {
    if (qtype == HALO_Q_INT8) return ext ? rotq_rows_kernel<128, 0, 1, PAD> : rotq_rows_kernel<128, 0, 0, PAD>;
    return ext ? rotq_rows_kernel<128, 1, 1, PAD> : rotq_rows_kernel<128, 1, 0, PAD>;
  }
  if (qtype == HALO_Q_INT8) return ext ? rotq_rows_kernel<256, 0, 1, PAD> : rotq_rows_kernel<256, 0, 0, PAD>;
  return ext ? rotq_rows_kernel<256, 1, 1, PAD> : rotq_rows_kernel<256, 1, 0, PAD>;
}

// qtype kQtDual (2): INT8 and E4M3 codes from one read (plain path only).
// pad: the row length is not a multiple of the block.
// grouped: group-wise scales (qtype INT8 / E4M3, plain path only).
RowsKernel rows_kernel(int blk, int qtype, bool ext, bool pad, bool grouped = false) {
  if (grouped) return pad ? rows_kernel_grouped_for<1>(blk, qtype) : rows_kernel_grouped_for<0>(blk, qtype);
  return pad ? rows_kernel_for<1>(blk, qtype, ext) : rows_kernel_for<0>(blk, qtype, ext);
}

typedef void (*ColsGrKernel)(const CUtensorMap, const CUtensorMap, RotqColsGrParams);

template <int QT, int EXT>
Cols1Kernel cols_1pass_for(int nw) {
  switch (nw) {
    case 1: return rotq_cols_1pass_kernel<QT, 1, EXT>;
    case 2: return rotq_cols_1pass_kernel<QT, 2, EXT>;
    case 3: return rotq_cols_1pass_kernel<QT, 3, EXT>;
    default: return rotq_cols_1pass_kernel<QT, 4, EXT>;
  }
}

Cols1Kernel cols_1pass_kernel(int qtype, int nw, bool ext) {
  if (qtype == HALO_Q_INT8) return ext ? cols_1pass_for<0, 1>(nw) : cols_1pass_for<0, 0>(nw);
  return ext ? cols_1pass_for<1, 1>(nw) : cols_1pass_for<1, 0>(nw);
}

// Dimension-0 rotation with the rotated values parked in tensor memory, one
// 8-warp CTA per SM (all of its tensor memory), clusters of as few CTAs as
// the column needs so that clusters pack the GPCs' SMs:
// variant 0 (<= 128 blocks of 128 rows): one block per warp, two strips in
// tensor memory (cluster = blocks / 8); variant 1 (<= 256 blocks): two blocks
// per warp, one strip (cluster = blocks / 16).
typedef void (*ColsTmKernel)(const CUtensorMap, const CUtensorMap, RotqColsTmParams);
constexpr int kColsTmVariants = 2;
constexpr int kColsTmWarps[kColsTmVariants] = {8, 8};
constexpr int kColsTmBlocksPerCta[kColsTmVariants] = {8, 16};

template <int QT, int EXT>
ColsTmKernel cols_tm_for(int variant) {
  return variant == 0 ? rotq_cols_tm_kernel<QT, 8, 2, 1, EXT> : rotq_cols_tm_kernel<QT, 8, 1, 2, EXT>;
}

// ext: random signs and / or stochastic rounding (RotqExtras).
ColsTmKernel cols_tm_kernel(int qtype, int variant, bool ext) {
  if (qtype == HALO_Q_INT8) return ext ? cols_tm_for<0, 1>(variant) : cols_tm_for<0, 0>(variant);
  return ext ? cols_tm_for<1, 1>(variant) : cols_tm_for<1, 0>(variant);
}

typedef void (*ColsSplitKernel)(const CUtensorMap, const CUtensorMap, RotqColsSplitParams);

ColsSplitKernel cols_split_kernel(int qtype, int mode) {
  if (mode == 0) return rotq_cols_split_kernel<0, 0>;  // maxima only: no codes, the type does not matter
  return qtype == HALO_Q_INT8 ? rotq_cols_split_kernel<0, 1> : rotq_cols_split_kernel<1, 1>;
}

Cols2Kernel cols_2pass_kernel(int qtype, bool ext) {
  if (qtype == HALO_Q_INT8) return ext ? rotq_cols_kernel<0, 1> : rotq_cols_kernel<0, 0>;
  return ext ? rotq_cols_kernel<1, 1> : rotq_cols_kernel<1, 0>;
}

// One-time per-device set-up: architecture check, SM count, kernel attributes,
// driver entry point for tensor-map encoding.
halo_status_t device_setup(int* dev_out) {
  int dev = 0;
  HALO_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return HALO_ERR_UNSUPPORTED;
  *dev_out = dev;
  DeviceInfo& d = g_dev[dev];
  if (d.ready.load(std::memory_order_acquire)) return d.supported ? HALO_OK : HALO_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (d.ready.load(std::memory_order_relaxed)) return d.supported ? HALO_OK : HALO_ERR_UNSUPPORTED;
  int major = 0, minor = 0;
  HALO_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  HALO_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  HALO_CUDA(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev));
  d.supported = (major == 10 && minor == 0);
  if (d.supported) {
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      HALO_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
      if (q != cudaDriverEntryPointSuccess || !fn) {
        snprintf(g_last_detail, sizeof g_last_detail, "cuTensorMapEncodeTiled entry point not found");
        return HALO_ERR_CUDA;
      }
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    int optin = 0;
    HALO_CUDA(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    HALO_CUDA(set_smem_attr(rotq_cols_grouped_kernel<0>, optin));
    HALO_CUDA(set_smem_attr(rotq_cols_grouped_kernel<1>, optin));
    HALO_CUDA(set_smem_attr(qgemm_grouped_kernel<0>, optin));
    HALO_CUDA(set_smem_attr(qgemm_grouped_kernel<1>, optin));
    HALO_CUDA(set_smem_attr(rotq_rows_pair_kernel<0>, optin));
    HALO_CUDA(set_smem_attr(rotq_rows_pair_kernel<1>, optin));
    for (int pad = 0; pad < 2; ++pad) {
      for (int qt = 0; qt < 2; ++qt) {
        HALO_CUDA(set_smem_attr(rows_kernel(128, qt, false, pad, true), optin));
        HALO_CUDA(set_smem_attr(rows_kernel(256, qt, false, pad, true), optin));
      }
      HALO_CUDA(set_smem_attr(rows_kernel(128, kQtDual, false, pad), optin));
      HALO_CUDA(set_smem_attr(rows_kernel(256, kQtDual, false, pad), optin));
      for (int e = 0; e < 2; ++e) {
        for (int qt = 0; qt < 2; ++qt) {
          HALO_CUDA(set_smem_attr(rows_kernel(128, qt, e, pad), optin));
          HALO_CUDA(set_smem_attr(rows_kernel(256, qt, e, pad), optin));
        }
      }
    }
    HALO_CUDA(set_smem_attr(cols_split_kernel(0, 0), optin));
    HALO_CUDA(set_smem_attr(cols_split_kernel(0, 1), optin));
    HALO_CUDA(set_smem_attr(cols_split_kernel(1, 1), optin));
    for (int qt = 0; qt < 2; ++qt) {
      for (int v = 0; v < kColsTmVariants; ++v) {
        for (int e = 0; e < 2; ++e) {
          HALO_CUDA(set_smem_attr(cols_tm_kernel(qt, v, e), optin));
          HALO_CUDA(cudaFuncSetAttribute(cols_tm_kernel(qt, v, e), cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
        }
      }
    }
    for (int e = 0; e < 2; ++e) {
      for (int qt = 0; qt < 2; ++qt) {
        HALO_CUDA(set_smem_attr(cols_2pass_kernel(qt, e), optin));
        for (int nw = 1; nw <= 4; ++nw) {
          HALO_CUDA(set_smem_attr(cols_1pass_kernel(qt, nw, e), optin));
          HALO_CUDA(cudaFuncSetAttribute(cols_1pass_kernel(qt, nw, e),
                                         cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
        }
      }
    }
    HALO_CUDA(set_smem_attr(qgemm_kernel<0>, optin));
    HALO_CUDA(set_smem_attr(qgemm_kernel<1>, optin));
    HALO_CUDA(set_smem_attr(qgemm_pair_kernel<0, 0>, optin));
    HALO_CUDA(set_smem_attr(qgemm_pair_kernel<0, 1>, optin));
    HALO_CUDA(set_smem_attr(qgemm_pair_kernel<1, 0>, optin));
    HALO_CUDA(set_smem_attr(qgemm_pair_kernel<1, 1>, optin));
  }
  d.ready.store(true, std::memory_order_release);
  return d.supported ? HALO_OK : HALO_ERR_UNSUPPORTED;
}

// Device address of g_noalloc_scratch, one per device, set on the first
// halo_linear_fwd_noalloc call made with that device current.
// Read without the lock on the fast path, so atomic: a thread that sees a
// non-null address (acquire) also sees the set-up that produced it (release).
std::atomic<void*> g_noalloc_ptr[kMaxDevices] = {};

halo_status_t noalloc_setup(int dev, void** out) {
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    p = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
      HALO_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
      g_noalloc_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return HALO_OK;
}

// Launch configuration with programmatic dependent launch on (each kernel's
// prologue may overlap the previous kernel's tail; the kernels wait with
// griddepcontrol.wait before touching global memory) and an optional cluster
// shape.  Use in place: cfg points into this object.
struct Launch {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  Launch(dim3 grid, dim3 block, size_t smem, cudaStream_t stream, int cluster_x) {
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 0) {
      attr[n].id = cudaLaunchAttributeClusterDimension;
      attr[n].val.clusterDim.x = cluster_x;
      attr[n].val.clusterDim.y = 1;
      attr[n].val.clusterDim.z = 1;
      ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }



halo_status_t encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
                     const cuuint64_t* strides_bytes, const cuuint32_t* box, CUtensorMapSwizzle sw) {
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides_bytes, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = 10000 + static_cast<int>(r);
    snprintf(g_last_detail, sizeof g_last_detail,
             "cuTensorMapEncodeTiled(rank %d, dims %llu x %llu, box %u x %u) failed with CUresult %d", rank,
             static_cast<unsigned long long>(dims[0]), static_cast<unsigned long long>(dims[1]), box[0], box[1],
             static_cast<int>(r));
    return HALO_ERR_CUDA;
  }
  return HALO_OK;
}

// Failure-path self-test: one thread waits, with the given bound, on an
// mbarrier that nothing ever completes; the wait runs out, records its site
// in the device error word and returns (no trap, no hang).
enum : unsigned int { kSiteSelftest = 0xF01 };

__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, kSiteSelftest, limit_ns);
}

// n rounded up to a multiple of b (the zero-padded length of a rotated dimension).
int64_t pad_to(int64_t n, int64_t b) { return (n + b - 1) / b * b; }

// ------------------------------------------------------------------------ rotq launches
// Rows of 193..256 whole 128-element chunks (whole blocks of 128, one output):
// each row split over a cluster of two CTAs of 4 warps (rotq_rows_pair_kernel).
bool rows_pair_applies(int64_t cols, int blk, int qtype, bool ext, int group) {
  if (blk != 128 || ext || group != 0 || (qtype != HALO_Q_INT8 && qtype != HALO_Q_E4M3) || cols % 128 != 0)
    return false;
  const int64_t nb = cols / 128;
  return nb > 192 && nb <= 256 && nb % 2 == 0;
}

halo_status_t launch_rotq_rows_pair(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int qtype, void* q,
                                    int64_t ld_q, float* scales, cudaStream_t stream, int dev) {
  const int nb = static_cast<int>(cols / 128);
  const int h = nb / 2;
  CUtensorMap tm_x, tm_q;
  {
    // [rows][nb][128] with a 136-element inner box: the 8 elements past each
    // chunk are out of range and arrive as zeros (a 272-byte slot per thread).
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(nb), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(ld_x) * 2};
    cuuint32_t box[3] = {kRowsInSlot / 2, static_cast<cuuint32_t>(h), 1};
    halo_status_t st = encode(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, x, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  {
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(nb), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(ld_q)};
    cuuint32_t box[3] = {kRowsOutSlot, static_cast<cuuint32_t>(h), 1};
    halo_status_t st = encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  RotqRowsPairParams p;
  p.scales = scales;
  p.rows = rows;
  p.h = h;
  p.qmax = qtype == HALO_Q_E4M3 ? 448.f : 127.f;
  p.scale_mult = static_cast<float>(1.0 / (static_cast<double>(p.qmax) * sqrt(128.0)));
  auto kern = qtype == HALO_Q_INT8 ? rotq_rows_pair_kernel<0> : rotq_rows_pair_kernel<1>;
  // Persistent: as many two-CTA clusters as fit at once, each looping over rows.
  Launch L(dim3(2), dim3(128), 2 * kRowsPairStageBytes + 128, stream, 2);
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &L.cfg) != cudaSuccess || max_clusters < 1) {
    (void)cudaGetLastError();
    max_clusters = g_dev[dev].sm_count;
  }
  L.cfg.gridDim = dim3(static_cast<unsigned>(2 * std::min<int64_t>(rows, max_clusters)));
  HALO_CUDA(cudaLaunchKernelEx(&L.cfg, kern, tm_x, tm_q, p));
  return HALO_OK;
}

// qtype kQtDual: q / ld_q / scales take the INT8 output, q2 / ld_q2 / scales2
// the E4M3 one (unused otherwise).
halo_status_t launch_rotq_rows(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int blk, int qtype,
                               void* q, int64_t ld_q, float* scales, const RotqExtras& ex, bool ext,
                               cudaStream_t stream, int dev, void* q2 = nullptr, int64_t ld_q2 = 0,
                               float* scales2 = nullptr, int group = 0) {
  const bool dual = qtype == kQtDual;
  if (!dual && rows_pair_applies(cols, blk, qtype, ext, group))
    return launch_rotq_rows_pair(x, rows, cols, ld_x, qtype, q, ld_q, scales, stream, dev);
  // A row of `cols` elements is zero-padded to whole blocks: nb 128-element
  // chunks, of which nbt are whole in the input and one more (tail > 0
  // elements) is partial; chunks past that are all zero.
  const int nb = static_cast<int>(pad_to(cols, blk) / 128);
  const int nbt = static_cast<int>(cols / 128);
  const int tail = static_cast<int>(cols % 128);
  // A row group of ceil(nb / 32) warps owns one row at a time; 4 warps per
  // CTA when a group fits in 4, else one group per CTA (up to 8 warps).
  const int gw = (nb + 31) / 32;
  const int groups = gw <= 4 ? 4 / gw : 1;
  const int threads = groups * gw * 32;

  CUtensorMap tm_x, tm_xt, tm_q, tm_q2;
  if (tail) {
    // The partial chunk: a 2-D view of X, one 128-element box per row.
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_x) * 2};
    cuuint32_t box[2] = {128, 1};
    halo_status_t st = encode(&tm_xt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  if (nbt > 0) {
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(nbt), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(ld_x) * 2};
    cuuint32_t box[3] = {kRowsInSlot / 2, static_cast<cuuint32_t>(nbt), 1};
    halo_status_t st = encode(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, x, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  } else {
    tm_x = tm_xt;  // never read: the kernel issues no 3-D load when nbt == 0
  }
  if (!tail) tm_xt = tm_x;  // never read
  {
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(nb), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(ld_q)};
    cuuint32_t box[3] = {kRowsOutSlot, static_cast<cuuint32_t>(nb), 1};
    halo_status_t st = encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
    tm_q2 = tm_q;
    if (dual) {
      strides[1] = static_cast<cuuint64_t>(ld_q2);
      st = encode(&tm_q2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (st != HALO_OK) return st;
    }
  }
  const bool pad = tail != 0 || nbt != nb;
  // Code tiles of their own (two rows in flight ahead), or, for one output
  // when that fits more CTAs on an SM, codes written into the consumed input
  // stage (one row in flight ahead).
  const size_t smem_tiles = static_cast<size_t>(groups) * rows_group_smem(gw, dual ? 2 : 1, pad) + 128;  // + alignment slack
  const size_t smem_in_stage = static_cast<size_t>(groups) * rows_group_smem(gw, 0, pad) + 128;

  RotqRowsParams p;
  p.scales = scales;
  p.rows = rows;
  p.nb = nb;
  p.nbt = nbt;
  p.tail = tail;
  p.gw = gw;
  p.groups = groups;
  p.qmax = qtype == HALO_Q_E4M3 ? 448.f : 127.f;
  p.scale_mult = static_cast<float>(1.0 / (static_cast<double>(p.qmax) * sqrt(static_cast<double>(blk))));
  p.ex = ex;
  p.scales2 = scales2;
  p.scale_mult2 = static_cast<float>(1.0 / (448.0 * sqrt(static_cast<double>(blk))));
  p.group = group;

  RowsKernel kern = rows_kernel(blk, qtype, ext, pad, group != 0);
  int per_sm = 0, per_sm_in_stage = 0;
  HALO_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem_tiles));
  if (!dual) HALO_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm_in_stage, kern, threads, smem_in_stage));
  const bool in_stage = per_sm_in_stage > per_sm;
  const size_t smem = in_stage ? smem_in_stage : smem_tiles;
  p.out_tiles = in_stage ? 0 : (dual ? 2 : 1);
  if (in_stage) per_sm = per_sm_in_stage;
  if (per_sm < 1) per_sm = 1;
  const int64_t ctas_needed = (rows + groups - 1) / groups;
  const int grid = static_cast<int>(std::min<int64_t>(ctas_needed, static_cast<int64_t>(g_dev[dev].sm_count) * per_sm));
  Launch L(dim3(grid), dim3(threads), smem, stream, 0);
  HALO_CUDA(cudaLaunchKernelEx(&L.cfg, kern, tm_x, tm_xt, tm_q, tm_q2, p));
  return HALO_OK;
}

// Single pass when the 128-row blocks of a column strip split evenly over a
// cluster of at most 16 CTAs with at most 4 warps each (R <= 8192 rows).
halo_status_t launch_rotq_cols_1pass(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int qtype, void* q,
                                     int64_t ld_q, float* scales, const RotqExtras& ex, bool ext,
                                     cudaStream_t stream, int nw, int cl, int dev) {
  const int strips = static_cast<int>((cols + kColsStrip - 1) / kColsStrip);
  CUtensorMap tm_x, tm_q;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_x) * 2};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(pad_to(rows, 128))};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_q)};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  RotqCols1Params p;
  p.scales = scales;
  p.cols = cols;
  p.strips = strips;
  p.qmax = qtype == HALO_Q_INT8 ? 127.f : 448.f;
  p.scale_mult = static_cast<float>(1.0 / (static_cast<double>(p.qmax) * sqrt(128.0)));
  p.ex = ex;
  Cols1Kernel kern = cols_1pass_kernel(qtype, nw, ext);

  // Persistent: as many clusters as fit at once (each loops over strips).
  Launch L(dim3(cl, 1, 1), dim3(32 * nw), static_cast<size_t>(nw) * (2 * kColsInBytes) + 128, stream, cl);
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &L.cfg) != cudaSuccess || max_clusters < 1) {
    (void)cudaGetLastError();
    max_clusters = std::max(1, g_dev[dev].sm_count / cl);
  }
  L.cfg.gridDim = dim3(cl, std::min(strips, max_clusters), 1);
  HALO_CUDA(cudaLaunchKernelEx(&L.cfg, kern, tm_x, tm_q, p));
  return HALO_OK;
}

// Rotation along dimension 0 of up to 256 blocks of 128 rows, the rotated
// values parked in tensor memory across the cluster's column-max reduction
// (rotq_cols_tm_kernel).  One CTA per SM for the 8-warp variants (all of the
// SM's tensor memory), two for the 4-warp one.
halo_status_t launch_rotq_cols_tm(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int qtype, void* q,
                                  int64_t ld_q, float* scales, const RotqExtras& ex, bool ext, cudaStream_t stream,
                                  int variant, int nblocks, int dev) {
  const int strips = static_cast<int>((cols + kColsStrip - 1) / kColsStrip);
  const int cl = (nblocks + kColsTmBlocksPerCta[variant] - 1) / kColsTmBlocksPerCta[variant];
  CUtensorMap tm_x, tm_q;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_x) * 2};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(pad_to(rows, 128))};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_q)};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  RotqColsTmParams p;
  p.scales = scales;
  p.cols = cols;
  p.strips = strips;
  p.nblocks = nblocks;
  p.qmax = qtype == HALO_Q_INT8 ? 127.f : 448.f;
  p.scale_mult = static_cast<float>(1.0 / (static_cast<double>(p.qmax) * sqrt(128.0)));
  p.ex = ex;
  ColsTmKernel kern = cols_tm_kernel(qtype, variant, ext);
  // Persistent: as many clusters as fit at once (each loops over strips).
  Launch L(dim3(cl, 1, 1), dim3(32 * kColsTmWarps[variant]), cols_tm_smem(kColsTmWarps[variant]), stream, cl);
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &L.cfg) != cudaSuccess || max_clusters < 1) {
    (void)cudaGetLastError();
    max_clusters = std::max(1, g_dev[dev].sm_count / cl);
  }
  L.cfg.gridDim = dim3(cl, std::min(strips, max_clusters), 1);
  HALO_CUDA(cudaLaunchKernelEx(&L.cfg, kern, tm_x, tm_q, p));
  return HALO_OK;
}

halo_status_t launch_rotq_cols(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int qtype, void* q,
                               int64_t ld_q, float* scales, const RotqExtras& ex, bool ext, cudaStream_t stream,
                               int dev) {
  // Rows past the input (zero padding to whole 128-row blocks) are outside the
  // input tensor map and arrive as zeros; the codes cover the padded rows.
  const int nblocks = static_cast<int>(pad_to(rows, 128) / 128);
  // Up to 8192 rows: the single-pass kernel with the strip in registers (most
  // warps per CTA, up to 4, at most 16 CTAs per cluster).  8193..16384 rows:
  // the strip parked in tensor memory, which reads the input once where the
  // register kernel would need two passes.  Taller: two passes.  (Measured on
  // this pool, isolated: 8192 x 8192 69.6 us in registers against 71.7 us in
  // tensor memory; 16384 x 4096 73.7 us in tensor memory against 84.0 us in
  // two passes; 28672 x 8192 243.7 us in two passes against 280.6 us.)
  for (int nw = 4; nw >= 1; --nw) {
    if (nblocks % nw == 0 && nblocks / nw <= 16)
      return launch_rotq_cols_1pass(x, rows, cols, ld_x, qtype, q, ld_q, scales, ex, ext, stream, nw, nblocks / nw,
                                    dev);
  }
  if (nblocks <= 16 * kColsTmBlocksPerCta[0])
    return launch_rotq_cols_tm(x, rows, cols, ld_x, qtype, q, ld_q, scales, ex, ext, stream, 0, nblocks, dev);
  // Taller matrices: the two-pass kernel (column maxima first, then codes).
  int cl = 8;
  while (cl > 1 && cl > nblocks) cl /= 2;
  const int warps = std::max(1, std::min(4, (nblocks + cl - 1) / cl));
  const int strips = static_cast<int>((cols + kColsStrip - 1) / kColsStrip);

  CUtensorMap tm_x, tm_q;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_x) * 2};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(pad_to(rows, 128))};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_q)};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  RotqColsParams p;
  p.scales = scales;
  p.cols = cols;
  p.nblocks = nblocks;
  p.warps = warps;
  p.qmax = qtype == HALO_Q_INT8 ? 127.f : 448.f;
  p.scale_mult = static_cast<float>(1.0 / (static_cast<double>(p.qmax) * sqrt(128.0)));
  p.ex = ex;
  const size_t smem = static_cast<size_t>(warps) * (kColsStages * kColsInBytes) + 128;

  Launch L(dim3(cl, strips, 1), dim3(32 * warps), smem, stream, cl);
  HALO_CUDA(cudaLaunchKernelEx(&L.cfg, cols_2pass_kernel(qtype, ext), tm_x, tm_q, p));
  return HALO_OK;
}

// Dimension-0 rotation with group-wise scales: independent warps over the
// (128-row block, 32-column strip) items; scales [rows_p / group][cols].
halo_status_t launch_rotq_cols_grouped(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int qtype, void* q,
                                       int64_t ld_q, float* scales, int group, cudaStream_t stream, int dev) {
  CUtensorMap tm_x, tm_q;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_x) * 2};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(pad_to(rows, 128))};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_q)};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  RotqColsGrParams p;
  p.scales = scales;
  p.cols = cols;
  p.strips = static_cast<int>((cols + kColsStrip - 1) / kColsStrip);
  p.nblocks = static_cast<int>(pad_to(rows, 128) / 128);
  p.group = group;
  p.qmax = qtype == HALO_Q_INT8 ? 127.f : 448.f;
  p.scale_mult = static_cast<float>(1.0 / (static_cast<double>(p.qmax) * sqrt(128.0)));
  ColsGrKernel kern = qtype == HALO_Q_INT8 ? rotq_cols_grouped_kernel<0> : rotq_cols_grouped_kernel<1>;
  const size_t smem = 4 * (2 * kColsInBytes) + 128;
  int per_sm = 0;
  HALO_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 128, smem));
  if (per_sm < 1) per_sm = 1;
  const int64_t items = static_cast<int64_t>(p.nblocks) * p.strips;
  const int grid = static_cast<int>(std::min<int64_t>((items + 3) / 4, static_cast<int64_t>(g_dev[dev].sm_count) * per_sm));
  Launch L(dim3(grid), dim3(128), smem, stream, 0);
  HALO_CUDA(cudaLaunchKernelEx(&L.cfg, kern, tm_x, tm_q, p));
  return HALO_OK;
}

// Dimension-0 rotation split at the column maxima (rotq_cols_split_kernel):
// mode 0 merges this matrix's per-column maxima into amax (zeroed here first),
// mode 1 writes codes and scales from given maxima.  Independent warps over
// the (128-row block, 32-column strip) items.
halo_status_t launch_rotq_cols_split(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int qtype, int mode,
                                     float* amax, void* q, int64_t ld_q, float* scales, cudaStream_t stream,
                                     int dev) {
  CUtensorMap tm_x, tm_q;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_x) * 2};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  }
  if (mode == 1) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(pad_to(rows, 128))};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_q)};
    cuuint32_t box[2] = {kColsStrip, 128};
    halo_status_t st = encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != HALO_OK) return st;
  } else {
    tm_q = tm_x;  // never used: mode 0 stores no codes
    HALO_CUDA(cudaMemsetAsync(amax, 0, static_cast<size_t>(cols) * sizeof(float), stream));
  }
  RotqColsSplitParams p;
  p.amax = amax;
  p.scales = scales;
  p.cols = cols;
  p.strips = static_cast<int>((cols + kColsStrip - 1) / kColsStrip);
  p.nblocks = static_cast<int>(pad_to(rows, 128) / 128);
  p.qmax = qtype == HALO_Q_INT8 ? 127.f : 448.f;
  p.scale_mult = static_cast<float>(1.0 / (static_cast<double>(p.qmax) * sqrt(128.0)));
  ColsSplitKernel kern = cols_split_kernel(qtype, mode);
  const size_t smem = 4 * (2 * kColsInBytes) + 128;
  int per_sm = 0;
  HALO_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 128, smem));
  if (per_sm < 1) per_sm = 1;
  const int64_t items = static_cast<int64_t>(p.nblocks) * p.strips;
  const int grid = static_cast<int>(std::min<int64_t>((items + 3) / 4, static_cast<int64_t>(g_dev[dev].sm_count) * per_sm));
  Launch L(dim3(grid), dim3(128), smem, stream, 0);
  HALO_CUDA(cudaLaunchKernelEx(&L.cfg, kern, tm_x, tm_q, p));
  return HALO_OK;
}

// GEMM with group-wise scales: 128 x 128 tiles, one CTA per SM, persistent.
// Scale of (row i, group G) of a K-major operand [outer, K]: s[i * K/g + G];
// of an MN-major operand [K, outer]: s[G * outer + i].
halo_status_t launch_qgemm_grouped(const void* a, const float* sa, int a_mn, int64_t ld_a, const void* b,
                                   const float* sb, int b_mn, int64_t ld_b, int64_t m, int64_t n, int64_t k,
                                   int group, int qtype, void* c, int otype, int64_t ld_c, cudaStream_t stream,
                                   int dev) {
  CUtensorMap tm_a, tm_b;
  const CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(a_mn ? m : k), static_cast<cuuint64_t>(a_mn ? k : m)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_a)};
    cuuint32_t box[2] = {128, 128};
    halo_status_t st = encode(&tm_a, dt, 2, a, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != HALO_OK) return st;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(b_mn ? n : k), static_cast<cuuint64_t>(b_mn ? k : n)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_b)};
    cuuint32_t box[2] = {128, 128};
    halo_status_t st = encode(&tm_b, dt, 2, b, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != HALO_OK) return st;
  }
  GroupedGemmParams p;
  p.m = static_cast<int>(m);
  p.n = static_cast<int>(n);
  p.k = static_cast<int>(k);
  p.group = group;
  p.tiles_m = static_cast<int>((m + kGgBM - 1) / kGgBM);
  p.tiles_n = static_cast<int>((n + kGgBN - 1) / kGgBN);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.a_mn = a_mn;
  p.b_mn = b_mn;
  uint32_t idesc = 0;
  if (qtype == HALO_Q_INT8)
    idesc |= (2u << 4) | (1u << 7) | (1u << 10);  // s32 accumulate, signed 8-bit A and B
  else
    idesc |= (1u << 4);                           // f32 accumulate, E4M3 A and B
  idesc |= static_cast<uint32_t>(a_mn) << 15;
  idesc |= static_cast<uint32_t>(b_mn) << 16;
  idesc |= static_cast<uint32_t>(kGgBN >> 3) << 17;
  idesc |= static_cast<uint32_t>(kGgBM >> 4) << 24;
  p.idesc = idesc;
  const int64_t ng = k / group;
  p.sa = sa;
  p.sa_row = a_mn ? 1 : ng;
  p.sa_grp = a_mn ? m : 1;
  p.sb = sb;
  p.sb_row = b_mn ? 1 : ng;
  p.sb_grp = b_mn ? n : 1;
  p.c = c;
  p.ldc = ld_c;
  p.out_bf16 = otype == HALO_OUT_BF16;
  const int grid = std::min(p.num_tiles, g_dev[dev].sm_count);
  Launch L(dim3(grid), dim3(kGgThreads), kGgSmemBytes, stream, 0);
  if (qtype == HALO_Q_INT8)
    HALO_CUDA(cudaLaunchKernelEx(&L.cfg, qgemm_grouped_kernel<0>, tm_a, tm_b, p));
  else
    HALO_CUDA(cudaLaunchKernelEx(&L.cfg, qgemm_grouped_kernel<1>, tm_a, tm_b, p));
  return HALO_OK;
}

// ------------------------------------------------------------------------ GEMM launch
halo_status_t launch_qgemm(const void* a, const float* sa, int a_mn, int64_t ld_a, const void* b, const float* sb,
                           int b_mn, int64_t ld_b, int64_t m, int64_t n, int64_t k, int qtype, void* c, int otype,
                           int64_t ld_c, cudaStream_t stream, int dev) {
  CUtensorMap tm_a, tm_b;
  const CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  {
    cuuint64_t dims[2];
    if (a_mn) {
      dims[0] = static_cast<cuuint64_t>(m);
      dims[1] = static_cast<cuuint64_t>(k);
    } else {
      dims[0] = static_cast<cuuint64_t>(k);
      dims[1] = static_cast<cuuint64_t>(m);
    }
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_a)};
    cuuint32_t box[2] = {128, 128};
    halo_status_t st = encode(&tm_a, dt, 2, a, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != HALO_OK) return st;
  }
  {
    cuuint64_t dims[2];
    cuuint32_t box[2];
    if (b_mn) {
      dims[0] = static_cast<cuuint64_t>(n);
      dims[1] = static_cast<cuuint64_t>(k);
      box[0] = 128;
      box[1] = 128;
    } else {
      dims[0] = static_cast<cuuint64_t>(k);
      dims[1] = static_cast<cuuint64_t>(n);
      box[0] = 128;
      box[1] = m > 128 ? 128 : 256;  // the pair kernel loads 128 N indices per CTA
    }
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_b)};
    halo_status_t st = encode(&tm_b, dt, 2, b, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != HALO_OK) return st;
  }
  // 256 x 256 tiles on SM pairs unless M is too small to fill a pair.
  const bool use_pair = m > 128;
  GemmParams p;
  p.m = static_cast<int>(m);
  p.n = static_cast<int>(n);
  p.k = static_cast<int>(k);
  const int bm = use_pair ? 256 : kGemmBM;
  p.tiles_m = static_cast<int>((m + bm - 1) / bm);
  p.tiles_n = static_cast<int>((n + kGemmBN - 1) / kGemmBN);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.a_mn = a_mn;
  p.b_mn = b_mn;
  p.group_m = kGemmGroupM;
  // Instruction descriptor: D format (bits 4-5), A/B formats (7-9, 10-12),
  // A/B major (15, 16), N >> 3 (17-22), M >> 4 (24-28).
  uint32_t idesc = 0;
  if (qtype == HALO_Q_INT8)
    idesc |= (2u << 4) | (1u << 7) | (1u << 10);  // s32 accumulate, signed 8-bit A and B
  else
    idesc |= (1u << 4);                           // f32 accumulate, E4M3 A and B
  idesc |= static_cast<uint32_t>(a_mn) << 15;
  idesc |= static_cast<uint32_t>(b_mn) << 16;
  idesc |= static_cast<uint32_t>(kGemmBN >> 3) << 17;
  idesc |= static_cast<uint32_t>(bm >> 4) << 24;  // M of one MMA: 128 per CTA, 256 per pair
  p.idesc = idesc;
  p.sa = sa;
  p.sb = sb;
  p.c = c;
  p.ldc = ld_c;
  p.out_bf16 = otype == HALO_OUT_BF16;
  if (!use_pair) {
    const int grid = std::min(p.num_tiles, g_dev[dev].sm_count);
    Launch L(dim3(grid), dim3(kGemmThreads), kGemmSmemBytes, stream, 0);
    if (qtype == HALO_Q_INT8)
      HALO_CUDA(cudaLaunchKernelEx(&L.cfg, qgemm_kernel<0>, tm_a, tm_b, p));
    else
      HALO_CUDA(cudaLaunchKernelEx(&L.cfg, qgemm_kernel<1>, tm_a, tm_b, p));
    return HALO_OK;
  }
  const int pairs = std::min(p.num_tiles, g_dev[dev].sm_count / 2);
  // The output as a tensor for the bulk-store epilogue: 32 rows x 128 bytes
  // per copy, 128-byte swizzle (the layout the epilogue writes).
  const bool bf16_out = otype == HALO_OUT_BF16;
  CUtensorMap tm_c;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(m)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_c) * (bf16_out ? 2 : 4)};
    cuuint32_t box[2] = {bf16_out ? 64u : 32u, 32u};
    halo_status_t st = encode(&tm_c, bf16_out ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                              c, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != HALO_OK) return st;
  }
  typedef void (*PairKernel)(const CUtensorMap, const CUtensorMap, const CUtensorMap, GemmParams);
  const PairKernel kern = qtype == HALO_Q_INT8 ? (bf16_out ? qgemm_pair_kernel<0, 1> : qgemm_pair_kernel<0, 0>)
                                              : (bf16_out ? qgemm_pair_kernel<1, 1> : qgemm_pair_kernel<1, 0>);
  Launch L(dim3(2 * pairs), dim3(kGemmThreads), kPairSmemBytes, stream, 2);
  HALO_CUDA(cudaLaunchKernelEx(&L.cfg, kern, tm_a, tm_b, tm_c, p));
  return HALO_OK;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool valid_qtype(int q) { return q == HALO_Q_INT8 || q == HALO_Q_E4M3; }
bool valid_otype(int o) { return o == HALO_OUT_FP32 || o == HALO_OUT_BF16; }

halo_status_t check_hadamard_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int axis, int blk,
                                      int qtype, const void* q, int64_t ld_q, const float* scales) {
  if (!x || !q || !scales) return HALO_ERR_NULL;
  if (!valid_qtype(qtype) || (axis != HALO_AXIS_COLS && axis != HALO_AXIS_ROWS)) return HALO_ERR_DTYPE;
  if (blk != 128 && blk != 256) return HALO_ERR_BLOCK;
  if (axis == HALO_AXIS_ROWS && blk != 128) return HALO_ERR_BLOCK;
  if (rows <= 0 || cols <= 0 || ld_x < cols || ld_q < cols) return HALO_ERR_SHAPE;
  // A rotated length that is not a multiple of blk is zero-padded; the codes
  // cover the padded length.
  if (axis == HALO_AXIS_COLS && (pad_to(cols, blk) > 32768 || ld_q < pad_to(cols, blk))) return HALO_ERR_SHAPE;
  if (axis == HALO_AXIS_ROWS && cols % 8 != 0) return HALO_ERR_SHAPE;
  if (rows > (int64_t(1) << 31) - 1 || cols > (int64_t(1) << 31) - 1) return HALO_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(q) || !aligned16(scales) || (ld_x * 2) % 16 != 0 || ld_q % 16 != 0)
    return HALO_ERR_ALIGN;
  return HALO_OK;
}

halo_status_t check_extras(const int8_t* signs, const uint16_t* rand_bits, int64_t ld_rand, int64_t cols,
                           int axis, int blk) {
  if (signs && !aligned16(signs)) return HALO_ERR_ALIGN;
  if (rand_bits) {
    if (ld_rand < (axis == HALO_AXIS_COLS ? pad_to(cols, blk) : cols)) return HALO_ERR_SHAPE;
    if (!aligned16(rand_bits) || (ld_rand * 2) % 16 != 0) return HALO_ERR_ALIGN;
  }
  return HALO_OK;
}

halo_status_t check_qgemm(const void* a, const float* sa, int a_major, int64_t ld_a, const void* b,
                          const float* sb, int b_major, int64_t ld_b, int64_t m, int64_t n, int64_t k, int qtype,
                          const void* c, int otype, int64_t ld_c) {
  if (!a || !sa || !b || !sb || !c) return HALO_ERR_NULL;
  if (!valid_qtype(qtype) || !valid_otype(otype)) return HALO_ERR_DTYPE;
  if ((a_major != HALO_MAJOR_K && a_major != HALO_MAJOR_MN) || (b_major != HALO_MAJOR_K && b_major != HALO_MAJOR_MN))
    return HALO_ERR_DTYPE;
  if (m <= 0 || n <= 0 || k <= 0) return HALO_ERR_SHAPE;
  if (m > (int64_t(1) << 31) - 1 || n > (int64_t(1) << 31) - 1) return HALO_ERR_SHAPE;
  if (qtype == HALO_Q_INT8 && k > 133144) return HALO_ERR_SHAPE;
  if (k > (int64_t(1) << 31) - 1) return HALO_ERR_SHAPE;
  if (ld_a < (a_major == HALO_MAJOR_K ? k : m) || ld_b < (b_major == HALO_MAJOR_K ? k : n) || ld_c < n)
    return HALO_ERR_SHAPE;
  const int64_t esz = otype == HALO_OUT_FP32 ? 4 : 2;
  if (!aligned16(a) || !aligned16(b) || !aligned16(c) || !aligned16(sa) || !aligned16(sb) || ld_a % 16 != 0 ||
      ld_b % 16 != 0 || (ld_c * esz) % 16 != 0)
    return HALO_ERR_ALIGN;
  return HALO_OK;
}

// Workspace layout (each region 256-byte aligned):
//   fwd: Xq[M*K] Wq[N*K] sx[M] sw[N]
//   bwd: dYq_rows[M*N] Wq_cols[N*K] s_dy_rows[M] s_w_cols[K]
//        dYq_cols[M*N] Xq_cols[M*K] s_dy_cols[N] s_x_cols[K]
struct WsLayout {
  size_t off[8];
  size_t total;
};

// Scratch of the linear layers: codes and scales of both operands of each GEMM,
// the contraction dimension zero-padded to whole blocks (fwd: K to blk; dX: N
// to 128; dW: M to 128).
// group > 0: group-wise scales, one per `group` positions of the contraction
// dimension instead of one per operand row.
WsLayout ws_layout(int64_t m, int64_t n, int64_t k, int which, int blk, int group = 0) {
  WsLayout L = {};
  size_t sizes[8];
  int cnt;
  auto ngroups = [&](int64_t len) { return static_cast<size_t>(group ? len / group : 1); };
  if (which == 0) {
    const int64_t kp = pad_to(k, blk);
    sizes[0] = size_t(m) * kp;
    sizes[1] = size_t(n) * kp;
    sizes[2] = size_t(m) * ngroups(kp) * 4;
    sizes[3] = size_t(n) * ngroups(kp) * 4;
    cnt = 4;
  } else {
    const int64_t np = pad_to(n, 128), mp = pad_to(m, 128);
    sizes[0] = size_t(m) * np;
    sizes[1] = size_t(np) * k;
    sizes[2] = size_t(m) * ngroups(np) * 4;
    sizes[3] = size_t(k) * ngroups(np) * 4;
    sizes[4] = size_t(mp) * n;
    sizes[5] = size_t(mp) * k;
    sizes[6] = size_t(n) * ngroups(mp) * 4;
    sizes[7] = size_t(k) * ngroups(mp) * 4;
    cnt = 8;
  }
  size_t off = 0;
  for (int i = 0; i < cnt; ++i) {
    L.off[i] = off;
    off = align_up(off + sizes[i], 256);
  }
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

const char* halo_status_string(int status) {
  switch (status) {
    case HALO_OK: return "HALO_OK";
    case HALO_ERR_NULL: return "HALO_ERR_NULL: a required pointer is NULL";
    case HALO_ERR_SHAPE: return "HALO_ERR_SHAPE: invalid or unsupported size";
    case HALO_ERR_BLOCK: return "HALO_ERR_BLOCK: unsupported Hadamard block size";
    case HALO_ERR_ALIGN: return "HALO_ERR_ALIGN: pointer or stride alignment";
    case HALO_ERR_DTYPE: return "HALO_ERR_DTYPE: unknown qtype / otype / axis / major";
    case HALO_ERR_WORKSPACE: return "HALO_ERR_WORKSPACE: workspace missing or too small";
    case HALO_ERR_CUDA: return "HALO_ERR_CUDA: a CUDA call failed";
    case HALO_ERR_TIMEOUT: return "HALO_ERR_TIMEOUT: a kernel's bounded wait ran out";
    case HALO_ERR_UNSUPPORTED: return "HALO_ERR_UNSUPPORTED: device is not sm_100 (B200)";
    default: return "HALO: unknown status";
  }
}

int halo_last_cuda_error(void) { return g_last_cuda_error; }

const char* halo_last_error_detail(void) { return g_last_detail; }

halo_status_t halo_device_error(int* where) {
  HALO_CUDA(cudaDeviceSynchronize());
  unsigned int site = 0, zero = 0;
  HALO_CUDA(cudaMemcpyFromSymbol(&site, g_error_site, sizeof(site)));
  if (site != 0) HALO_CUDA(cudaMemcpyToSymbol(g_error_site, &zero, sizeof(zero)));
  if (where) *where = static_cast<int>(site);
  return site ? HALO_ERR_TIMEOUT : HALO_OK;
}

halo_status_t halo_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns <= 0 || static_cast<unsigned long long>(limit_ns) > kWaitLimitNs) return HALO_ERR_SHAPE;
  int dev = 0;
  halo_status_t st = device_setup(&dev);
  if (st != HALO_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<unsigned long long>(limit_ns));
  HALO_CUDA(cudaGetLastError());
  return HALO_OK;
}

size_t halo_workspace_size(int64_t m, int64_t n, int64_t k, int which) {
  if (m <= 0 || n <= 0 || k <= 0 || (which != 0 && which != 1)) return 0;
  // forward: enough for either block size (K padded to 256 is the larger)
  return ws_layout(m, n, k, which, which == 0 ? 256 : 128).total;
}

halo_status_t halo_hadamard_quantize_ex(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x, int axis,
                                        int blk, int qtype, const int8_t* signs, const uint16_t* rand_bits,
                                        int64_t ld_rand, void* q_out, int64_t ld_q, float* scales_out,
                                        void* stream) {
  halo_status_t st = check_hadamard_quantize(x_bf16, rows, cols, ld_x, axis, blk, qtype, q_out, ld_q, scales_out);
  if (st != HALO_OK) return st;
  if ((st = check_extras(signs, rand_bits, ld_rand, cols, axis, blk)) != HALO_OK) return st;
  int dev = 0;
  st = device_setup(&dev);
  if (st != HALO_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RotqExtras ex;
  ex.signs = signs;
  ex.rand = rand_bits;
  ex.ld_rand = rand_bits ? ld_rand : 0;
  const bool ext = signs != nullptr || rand_bits != nullptr;
  if (axis == HALO_AXIS_COLS)
    return launch_rotq_rows(x_bf16, rows, cols, ld_x, blk, qtype, q_out, ld_q, scales_out, ex, ext, s, dev);
  return launch_rotq_cols(x_bf16, rows, cols, ld_x, qtype, q_out, ld_q, scales_out, ex, ext, s, dev);
}

halo_status_t halo_hadamard_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x, int axis,
                                     int blk, int qtype, void* q_out, int64_t ld_q, float* scales_out,
                                     void* stream) {
  return halo_hadamard_quantize_ex(x_bf16, rows, cols, ld_x, axis, blk, qtype, nullptr, nullptr, 0, q_out, ld_q,
                                   scales_out, stream);
}

halo_status_t halo_hadamard_quantize_both(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x, int blk,
                                          int qtype, void* q_rows, int64_t ld_qr, float* scales_rows, void* q_cols,
                                          int64_t ld_qc, float* scales_cols, void* stream) {
  // Every argument of both rotations is checked before either is launched.
  halo_status_t st = check_hadamard_quantize(x_bf16, rows, cols, ld_x, HALO_AXIS_COLS, blk, qtype, q_rows, ld_qr,
                                             scales_rows);
  if (st != HALO_OK) return st;
  if ((st = check_hadamard_quantize(x_bf16, rows, cols, ld_x, HALO_AXIS_ROWS, 128, qtype, q_cols, ld_qc,
                                    scales_cols)) != HALO_OK)
    return st;
  // Back to back on the stream: the second rotation reads X while the first
  // has just brought it through L2.
  if ((st = halo_hadamard_quantize(x_bf16, rows, cols, ld_x, HALO_AXIS_COLS, blk, qtype, q_rows, ld_qr, scales_rows,
                                   stream)) != HALO_OK)
    return st;
  return halo_hadamard_quantize(x_bf16, rows, cols, ld_x, HALO_AXIS_ROWS, 128, qtype, q_cols, ld_qc, scales_cols,
                                stream);
}

halo_status_t halo_hadamard_quantize_dual(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x, int blk,
                                          void* q_int8, int64_t ld_q8, float* scales_int8, void* q_e4m3,
                                          int64_t ld_qf8, float* scales_e4m3, void* stream) {
  halo_status_t st = check_hadamard_quantize(x_bf16, rows, cols, ld_x, HALO_AXIS_COLS, blk, HALO_Q_INT8, q_int8,
                                             ld_q8, scales_int8);
  if (st != HALO_OK) return st;
  st = check_hadamard_quantize(x_bf16, rows, cols, ld_x, HALO_AXIS_COLS, blk, HALO_Q_E4M3, q_e4m3, ld_qf8,
                               scales_e4m3);
  if (st != HALO_OK) return st;
  int dev = 0;
  st = device_setup(&dev);
  if (st != HALO_OK) return st;
  RotqExtras ex;
  ex.signs = nullptr;
  ex.rand = nullptr;
  ex.ld_rand = 0;
  return launch_rotq_rows(x_bf16, rows, cols, ld_x, blk, kQtDual, q_int8, ld_q8, scales_int8, ex, false,
                          static_cast<cudaStream_t>(stream), dev, q_e4m3, ld_qf8, scales_e4m3);
}

halo_status_t halo_hadamard_quantize_grouped(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x,
                                             int axis, int blk, int group, int qtype, void* q_out, int64_t ld_q,
                                             float* scales_out, void* stream) {
  halo_status_t st = check_hadamard_quantize(x_bf16, rows, cols, ld_x, axis, blk, qtype, q_out, ld_q, scales_out);
  if (st != HALO_OK) return st;
  if (group != 64 && group != 128) return HALO_ERR_BLOCK;
  int dev = 0;
  st = device_setup(&dev);
  if (st != HALO_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (axis == HALO_AXIS_COLS) {
    RotqExtras ex;
    ex.signs = nullptr;
    ex.rand = nullptr;
    ex.ld_rand = 0;
    return launch_rotq_rows(x_bf16, rows, cols, ld_x, blk, qtype, q_out, ld_q, scales_out, ex, false, s, dev,
                            nullptr, 0, nullptr, group);
  }
  return launch_rotq_cols_grouped(x_bf16, rows, cols, ld_x, qtype, q_out, ld_q, scales_out, group, s, dev);
}

halo_status_t halo_hadamard_colmax(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x, int blk,
                                   float* amax_out, void* stream) {
  // The checks of halo_hadamard_quantize along dimension 0 (amax_out stands in
  // for the codes and scales, which this call does not write).
  halo_status_t st = check_hadamard_quantize(x_bf16, rows, cols, ld_x, HALO_AXIS_ROWS, blk, HALO_Q_INT8, amax_out,
                                             cols + (16 - cols % 16) % 16, amax_out);
  if (st != HALO_OK) return st;
  int dev = 0;
  if ((st = device_setup(&dev)) != HALO_OK) return st;
  return launch_rotq_cols_split(x_bf16, rows, cols, ld_x, HALO_Q_INT8, 0, amax_out, nullptr, 0, nullptr,
                                static_cast<cudaStream_t>(stream), dev);
}

halo_status_t halo_hadamard_quantize_colmax(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x, int blk,
                                            int qtype, const float* amax, void* q_out, int64_t ld_q,
                                            float* scales_out, void* stream) {
  halo_status_t st = check_hadamard_quantize(x_bf16, rows, cols, ld_x, HALO_AXIS_ROWS, blk, qtype, q_out, ld_q,
                                             scales_out);
  if (st != HALO_OK) return st;
  if (!amax) return HALO_ERR_NULL;
  if (!aligned16(amax)) return HALO_ERR_ALIGN;
  int dev = 0;
  if ((st = device_setup(&dev)) != HALO_OK) return st;
  return launch_rotq_cols_split(x_bf16, rows, cols, ld_x, qtype, 1, const_cast<float*>(amax), q_out, ld_q,
                                scales_out, static_cast<cudaStream_t>(stream), dev);
}

halo_status_t halo_qgemm_grouped(const void* a_q, const float* s_a, int a_major, int64_t ld_a, const void* b_q,
                                 const float* s_b, int b_major, int64_t ld_b, int64_t m, int64_t n, int64_t k,
                                 int group, int qtype, void* c, int otype, int64_t ld_c, void* stream) {
  halo_status_t st = check_qgemm(a_q, s_a, a_major, ld_a, b_q, s_b, b_major, ld_b, m, n, k, qtype, c, otype, ld_c);
  if (st != HALO_OK) return st;
  if (group != 64 && group != 128) return HALO_ERR_BLOCK;
  if (k % 128 != 0) return HALO_ERR_SHAPE;
  int dev = 0;
  st = device_setup(&dev);
  if (st != HALO_OK) return st;
  return launch_qgemm_grouped(a_q, s_a, a_major, ld_a, b_q, s_b, b_major, ld_b, m, n, k, group, qtype, c, otype,
                              ld_c, static_cast<cudaStream_t>(stream), dev);
}

size_t halo_workspace_size_grouped(int64_t m, int64_t n, int64_t k, int group, int which) {
  if (m <= 0 || n <= 0 || k <= 0 || (which != 0 && which != 1) || (group != 64 && group != 128)) return 0;
  return ws_layout(m, n, k, which, which == 0 ? 256 : 128, group).total;
}

halo_status_t halo_qgemm(const void* a_q, const float* s_a, int a_major, int64_t ld_a, const void* b_q,
                         const float* s_b, int b_major, int64_t ld_b, int64_t m, int64_t n, int64_t k, int qtype,
                         void* c, int otype, int64_t ld_c, void* stream) {
  halo_status_t st = check_qgemm(a_q, s_a, a_major, ld_a, b_q, s_b, b_major, ld_b, m, n, k, qtype, c, otype, ld_c);
  if (st != HALO_OK) return st;
  int dev = 0;
  st = device_setup(&dev);
  if (st != HALO_OK) return st;
  return launch_qgemm(a_q, s_a, a_major, ld_a, b_q, s_b, b_major, ld_b, m, n, k, qtype, c, otype, ld_c,
                      static_cast<cudaStream_t>(stream), dev);
}

// The linear layers with per-row scales (group 0) or group-wise scales.
static halo_status_t quantize_op(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int axis, int blk,
                                 int group, int qtype, void* q, int64_t ld_q, float* s, void* stream) {
  return group ? halo_hadamard_quantize_grouped(x, rows, cols, ld_x, axis, blk, group, qtype, q, ld_q, s, stream)
               : halo_hadamard_quantize(x, rows, cols, ld_x, axis, blk, qtype, q, ld_q, s, stream);
}

static halo_status_t gemm_op(const void* a, const float* sa, int a_major, int64_t ld_a, const void* b,
                             const float* sb, int b_major, int64_t ld_b, int64_t m, int64_t n, int64_t k, int group,
                             int qtype, void* c, int otype, int64_t ld_c, void* stream) {
  return group ? halo_qgemm_grouped(a, sa, a_major, ld_a, b, sb, b_major, ld_b, m, n, k, group, qtype, c, otype,
                                    ld_c, stream)
               : halo_qgemm(a, sa, a_major, ld_a, b, sb, b_major, ld_b, m, n, k, qtype, c, otype, ld_c, stream);
}

static halo_status_t linear_fwd_impl(const void* x_bf16, const void* w_bf16, int64_t m, int64_t n, int64_t k,
                                     int blk, int group, int qtype, void* y, int otype, void* ws, size_t ws_bytes,
                                     void* stream) {
  if (!x_bf16 || !w_bf16 || !y) return HALO_ERR_NULL;
  if (!valid_qtype(qtype) || !valid_otype(otype)) return HALO_ERR_DTYPE;
  if (blk != 128 && blk != 256) return HALO_ERR_BLOCK;
  if (group != 0 && group != 64 && group != 128) return HALO_ERR_BLOCK;
  if (m <= 0 || n <= 0 || k <= 0 || pad_to(k, blk) > 32768) return HALO_ERR_SHAPE;
  if (!ws) return HALO_ERR_WORKSPACE;
  const WsLayout L = ws_layout(m, n, k, 0, blk, group);
  if (ws_bytes < L.total) return HALO_ERR_WORKSPACE;
  const int64_t esz = otype == HALO_OUT_FP32 ? 4 : 2;
  if (!aligned16(x_bf16) || !aligned16(w_bf16) || !aligned16(y) || !aligned16(ws) || (n * esz) % 16 != 0 ||
      k % 8 != 0)
    return HALO_ERR_ALIGN;
  const int64_t kp = pad_to(k, blk);  // K zero-padded to whole blocks
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  uint8_t* xq = w8 + L.off[0];
  uint8_t* wq = w8 + L.off[1];
  float* sx = reinterpret_cast<float*>(w8 + L.off[2]);
  float* sw = reinterpret_cast<float*>(w8 + L.off[3]);
  halo_status_t st;
  if ((st = quantize_op(x_bf16, m, k, k, HALO_AXIS_COLS, blk, group, qtype, xq, kp, sx, stream)) != HALO_OK) return st;
  if ((st = quantize_op(w_bf16, n, k, k, HALO_AXIS_COLS, blk, group, qtype, wq, kp, sw, stream)) != HALO_OK) return st;
  return gemm_op(xq, sx, HALO_MAJOR_K, kp, wq, sw, HALO_MAJOR_K, kp, m, n, kp, group, qtype, y, otype, n, stream);
}

halo_status_t halo_linear_fwd(const void* x_bf16, const void* w_bf16, int64_t m, int64_t n, int64_t k, int blk,
                              int qtype, void* y, int otype, void* ws, size_t ws_bytes, void* stream) {
  return linear_fwd_impl(x_bf16, w_bf16, m, n, k, blk, 0, qtype, y, otype, ws, ws_bytes, stream);
}

halo_status_t halo_linear_fwd_grouped(const void* x_bf16, const void* w_bf16, int64_t m, int64_t n, int64_t k,
                                      int blk, int group, int qtype, void* y, int otype, void* ws, size_t ws_bytes,
                                      void* stream) {
  if (group != 64 && group != 128) return HALO_ERR_BLOCK;
  return linear_fwd_impl(x_bf16, w_bf16, m, n, k, blk, group, qtype, y, otype, ws, ws_bytes, stream);
}

halo_status_t halo_linear_fwd_noalloc(const void* x_bf16, const void* w_bf16, int64_t m, int64_t n, int64_t k,
                                      int blk, int qtype, void* y, int otype, void* stream) {
  // Argument checks of halo_linear_fwd and the scratch limit come first, so
  // that nothing touches the device on input this call would reject.
  if (!x_bf16 || !w_bf16 || !y) return HALO_ERR_NULL;
  if (!valid_qtype(qtype) || !valid_otype(otype)) return HALO_ERR_DTYPE;
  if (blk != 128 && blk != 256) return HALO_ERR_BLOCK;
  if (m <= 0 || n <= 0 || k <= 0 || pad_to(k, blk) > 32768) return HALO_ERR_SHAPE;
  const int64_t esz = otype == HALO_OUT_FP32 ? 4 : 2;
  if (!aligned16(x_bf16) || !aligned16(w_bf16) || !aligned16(y) || (n * esz) % 16 != 0 || k % 8 != 0)
    return HALO_ERR_ALIGN;
  const size_t need = ws_layout(m, n, k, 0, blk).total;
  if (need > HALO_NOALLOC_SCRATCH_BYTES) {
    snprintf(g_last_detail, sizeof g_last_detail,
             "halo_linear_fwd_noalloc: these sizes need %zu bytes of scratch, the library's static array holds %llu",
             need, static_cast<unsigned long long>(HALO_NOALLOC_SCRATCH_BYTES));
    return HALO_ERR_WORKSPACE;
  }
  int dev = 0;
  halo_status_t st = device_setup(&dev);
  if (st != HALO_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_setup(dev, &scratch)) != HALO_OK) return st;
  return halo_linear_fwd(x_bf16, w_bf16, m, n, k, blk, qtype, y, otype, scratch, HALO_NOALLOC_SCRATCH_BYTES, stream);
}

static halo_status_t linear_bwd_impl(const void* dy_bf16, const void* x_bf16, const void* w_bf16, int64_t m,
                                     int64_t n, int64_t k, int blk, int group, int qtype, void* dx, int otype_dx,
                                     void* dw, int otype_dw, void* ws, size_t ws_bytes, void* stream) {
  if (!dy_bf16 || (!dx && !dw)) return HALO_ERR_NULL;
  if (dx && !w_bf16) return HALO_ERR_NULL;
  if (dw && !x_bf16) return HALO_ERR_NULL;
  if (!valid_qtype(qtype) || (dx && !valid_otype(otype_dx)) || (dw && !valid_otype(otype_dw))) return HALO_ERR_DTYPE;
  if (blk != 128) return HALO_ERR_BLOCK;
  if (group != 0 && group != 64 && group != 128) return HALO_ERR_BLOCK;
  if (m <= 0 || n <= 0 || k <= 0) return HALO_ERR_SHAPE;
  if (dx && (pad_to(n, blk) > 32768 || k % 16 != 0)) return HALO_ERR_SHAPE;
  if (dw && (n % 16 != 0 || k % 16 != 0)) return HALO_ERR_SHAPE;
  if (!ws) return HALO_ERR_WORKSPACE;
  const WsLayout L = ws_layout(m, n, k, 1, blk, group);
  if (ws_bytes < L.total) return HALO_ERR_WORKSPACE;
  if (!aligned16(dy_bf16) || (x_bf16 && !aligned16(x_bf16)) || (w_bf16 && !aligned16(w_bf16)) ||
      (dx && !aligned16(dx)) || (dw && !aligned16(dw)) || !aligned16(ws))
    return HALO_ERR_ALIGN;
  if (dx && (k * (otype_dx == HALO_OUT_FP32 ? 4 : 2)) % 16 != 0) return HALO_ERR_ALIGN;
  if (n % 8 != 0) return HALO_ERR_ALIGN;  // dY's rows: a multiple of 16 bytes
  if (dw && (k * (otype_dw == HALO_OUT_FP32 ? 4 : 2)) % 16 != 0) return HALO_ERR_ALIGN;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  halo_status_t st;
  // With both products, dY is rotated both ways back to back (the second
  // rotation reads it from L2 when it fits there), before W and X.
  const bool both = dx && dw && group == 0;
  if (both && (st = halo_hadamard_quantize_both(dy_bf16, m, n, n, blk, qtype, w8 + L.off[0], pad_to(n, blk),
                                                reinterpret_cast<float*>(w8 + L.off[2]), w8 + L.off[4], n,
                                                reinterpret_cast<float*>(w8 + L.off[6]), stream)) != HALO_OK)
    return st;
  if (dx) {
    uint8_t* dyq = w8 + L.off[0];
    uint8_t* wq = w8 + L.off[1];
    float* sdy = reinterpret_cast<float*>(w8 + L.off[2]);
    float* sw = reinterpret_cast<float*>(w8 + L.off[3]);
    // dX[M,K] = dY[M,N] W[N,K]: contraction over N (zero-padded to np).
    const int64_t np = pad_to(n, blk);
    if (!both &&
        (st = quantize_op(dy_bf16, m, n, n, HALO_AXIS_COLS, blk, group, qtype, dyq, np, sdy, stream)) != HALO_OK)
      return st;
    if ((st = quantize_op(w_bf16, n, k, k, HALO_AXIS_ROWS, blk, group, qtype, wq, k, sw, stream)) != HALO_OK)
      return st;
    if ((st = gemm_op(dyq, sdy, HALO_MAJOR_K, np, wq, sw, HALO_MAJOR_MN, k, m, k, np, group, qtype, dx, otype_dx, k,
                      stream)) != HALO_OK)
      return st;
  }
  if (dw) {
    uint8_t* dyq = w8 + L.off[4];
    uint8_t* xq = w8 + L.off[5];
    float* sdy = reinterpret_cast<float*>(w8 + L.off[6]);
    float* sx = reinterpret_cast<float*>(w8 + L.off[7]);
    // dW[N,K] = dY^T[N,M] X[M,K]: contraction over M (tokens, zero-padded to mp).
    const int64_t mp = pad_to(m, blk);
    if (!both &&
        (st = quantize_op(dy_bf16, m, n, n, HALO_AXIS_ROWS, blk, group, qtype, dyq, n, sdy, stream)) != HALO_OK)
      return st;
    if ((st = quantize_op(x_bf16, m, k, k, HALO_AXIS_ROWS, blk, group, qtype, xq, k, sx, stream)) != HALO_OK)
      return st;
    if ((st = gemm_op(dyq, sdy, HALO_MAJOR_MN, n, xq, sx, HALO_MAJOR_MN, k, n, k, mp, group, qtype, dw, otype_dw, k,
                      stream)) != HALO_OK)
      return st;
  }
  return HALO_OK;
}

halo_status_t halo_linear_bwd(const void* dy_bf16, const void* x_bf16, const void* w_bf16, int64_t m, int64_t n,
                              int64_t k, int blk, int qtype, void* dx, int otype_dx, void* dw, int otype_dw,
                              void* ws, size_t ws_bytes, void* stream) {
  return linear_bwd_impl(dy_bf16, x_bf16, w_bf16, m, n, k, blk, 0, qtype, dx, otype_dx, dw, otype_dw, ws, ws_bytes,
                         stream);
}

halo_status_t halo_linear_bwd_grouped(const void* dy_bf16, const void* x_bf16, const void* w_bf16, int64_t m,
                                      int64_t n, int64_t k, int blk, int group, int qtype, void* dx, int otype_dx,
                                      void* dw, int otype_dw, void* ws, size_t ws_bytes, void* stream) {
  if (group != 64 && group != 128) return HALO_ERR_BLOCK;
  return linear_bwd_impl(dy_bf16, x_bf16, w_bf16, m, n, k, blk, group, qtype, dx, otype_dx, dw, otype_dw, ws,
                         ws_bytes, stream);
}

}  // extern "C"
