// Host side of the C ABI declared in include/convrot.h: argument checks,
// TMA tensor-map encoding, launch configuration, and the composition of the
// W8A8 ConvRot linear and the expert-choice MoE block from the kernels.
//
// All kernels live in this one translation unit (the device error word is a
// single __device__ variable without relocatable device code).

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "convrot.h"
#include "common.cuh"
#include "gemm_tcgen05.cuh"
#include "lowbit.cuh"
#include "rotquant.cuh"
#include "routing.cuh"

using namespace convrot;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  bool supported = false;
  int sm_count = 0;
  // how many CTAs (single-CTA kernel) and CTA pairs (pair kernel) of the
  // requantising SwiGLU GEMM can be resident at once: its grid never exceeds
  // them, since its tiles wait for one another
  int rq_ctas = 0;
  int rq_pairs = 0;
  // CTA pairs of the low-bit GEMM that can be resident at once
  int lb_pairs = 0;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

template <int EPI, bool BT>
void set_gemm_attr() {
  cudaFuncSetAttribute(gemm_s8_tcgen05_kernel<EPI, BT>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<EPI>::kSmem1);
  cudaFuncSetAttribute(gemm_s8_tcgen05_pair_kernel<EPI, BT>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<EPI>::kSmem2);
}

template <int BITS, int EPI>
void set_lowbit_attr() {
  cudaFuncSetAttribute(gemm_lowbit_tcgen05_kernel<BITS, EPI, false, false>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, lb::kSmemMax);
  cudaFuncSetAttribute(gemm_lowbit_tcgen05_kernel<BITS, EPI, false, true>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, lb::kSmemMax);
  cudaFuncSetAttribute(gemm_lowbit_tcgen05_kernel<BITS, EPI, true, false>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, lb::kSmemMax);
}

template <int BITS>
void set_lowbit_attrs() {
  set_lowbit_attr<BITS, kLbF32>();
  set_lowbit_attr<BITS, kLbBf16>();
  set_lowbit_attr<BITS, kLbSwiglu>();
}

// every GEMM instantiation the entry points launch
template <bool BT>
void set_gemm_attrs() {
  set_gemm_attr<kEpiI32, BT>();
  set_gemm_attr<kEpiBf16, BT>();
  set_gemm_attr<kEpiSwiglu, BT>();
  set_gemm_attr<kEpiScatter, BT>();
  set_gemm_attr<kEpiSwigluRq, BT>();
}

// Co-resident CTAs / CTA pairs of the requantising SwiGLU GEMM on this device.
int swiglu_rq_residency(int sms, int* ctas, int* pairs) {
  using Cfg = EpiCfg<kEpiSwigluRq>;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
          &per_sm, gemm_s8_tcgen05_kernel<kEpiSwigluRq, true>, Cfg::kThreads, Cfg::kSmem1) !=
      cudaSuccess)
    return CONVROT_ERR_CUDA;
  *ctas = per_sm * sms;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2 * (unsigned)(sms / 2));
  lc.blockDim = dim3(Cfg::kThreads);
  lc.dynamicSmemBytes = Cfg::kSmem2;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  lc.attrs = &attr;
  lc.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, gemm_s8_tcgen05_pair_kernel<kEpiSwigluRq, true>,
                                     &lc) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  *pairs = clusters;
  return CONVROT_OK;
}

// Co-resident CTA pairs of the low-bit GEMM on this device.
int lowbit_pair_residency(int sms, int* pairs) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2 * (unsigned)(sms / 2));
  lc.blockDim = dim3(lb::kThreads);
  lc.dynamicSmemBytes = lb::kSmemMax;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  lc.attrs = &attr;
  lc.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters,
                                     gemm_lowbit_tcgen05_kernel<6, kLbSwiglu, true, false>,
                                     &lc) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  *pairs = clusters;
  return CONVROT_OK;
}

// Per-device one-time setup: capability check, SM count, kernel attributes.
int device_setup(int* sm_count) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return CONVROT_ERR_UNSUPPORTED_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return CONVROT_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return CONVROT_ERR_UNSUPPORTED_DEVICE;
    }
    d.supported = (major == 10 && minor == 0);
    d.sm_count = sms;
    if (d.supported) {
      set_gemm_attrs<false>();
      set_gemm_attrs<true>();
      set_lowbit_attrs<4>();
      set_lowbit_attrs<6>();
      if (cudaGetLastError() != cudaSuccess) return CONVROT_ERR_CUDA;
      if (swiglu_rq_residency(sms, &d.rq_ctas, &d.rq_pairs) != CONVROT_OK ||
          lowbit_pair_residency(sms, &d.lb_pairs) != CONVROT_OK) {
        cudaGetLastError();
        return CONVROT_ERR_CUDA;
      }
    }
    d.ready = true;
  }
  if (!d.supported) return CONVROT_ERR_UNSUPPORTED_DEVICE;
  if (sm_count) *sm_count = d.sm_count;
  return CONVROT_OK;
}

// Co-resident CTA pairs of the low-bit GEMM on the current device; 0 before
// device_setup.
int lowbit_pair_capacity() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  return g_dev[dev].lb_pairs;
}

// Co-resident CTAs (pairs = false) or CTA pairs of the requantising SwiGLU
// GEMM on the current device; 0 before device_setup.
int swiglu_rq_capacity(bool pairs) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  return pairs ? g_dev[dev].rq_pairs : g_dev[dev].rq_ctas;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool valid_group(int g) { return g == 1 || g == 4 || g == 16 || g == 64 || g == 256; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// The name of the last CUDA error an entry point of this thread saw.
thread_local const char* g_last_cuda_error = "none";

int cuda_failed(cudaError_t e) {
  g_last_cuda_error = cudaGetErrorName(e);
  cudaGetLastError();
  return CONVROT_ERR_CUDA;
}

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? CONVROT_OK : cuda_failed(e);
}

// Launches `kern` on `st`; `pdl` adds programmatic stream serialization (the
// kernel may start while its predecessor on the stream finishes; it waits for
// it with griddepcontrol.wait), `cluster_x` > 1 a cluster dimension.
template <typename... KArgs, typename... Args>
int launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                  bool pdl, int cluster_x, Args... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  lc.attrs = attr;
  lc.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&lc, kern, args...);
  if (e != cudaSuccess) return cuda_failed(e);
  return CONVROT_OK;
}

// --------------------------------------------------------------- rotquant --
// 3-D byte view {128, K * esize / 128, rows} of a row-major [rows, K] matrix,
// box = `box_rows` whole rows, 128-byte swizzle (see rotquant_tma_kernel).
int encode_rows_sw128(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows,
                      uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CONVROT_ERR_CUDA;
  const cuuint64_t dims[3] = {128, row_bytes / 128, rows};
  const cuuint64_t strides[2] = {128, row_bytes};
  const cuuint32_t box[3] = {128, (cuuint32_t)(row_bytes / 128), box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// grid_cap > 0: when the rows need more CTAs than fit on the device at once,
// run at most grid_cap persistent CTAs (the MoE call keeps SMs free for the
// routing kernels that run beside the activation rotation).
template <typename InT, int G, int SEG>
int launch_rq_tma(const void* x, int64_t rows, int K, int8_t* q, float* s, RqOut out,
                   cudaStream_t st, bool pdl, int64_t grid_cap, bool wait_at_end) {
  constexpr int kRowsPerWarp = 32 / SEG;
  const uint64_t row_bytes = (uint64_t)K * sizeof(InT);
  CUtensorMap tm;
  if (encode_rows_sw128(&tm, x, row_bytes, (uint64_t)rows, kRowsPerWarp) != CONVROT_OK)
    return CONVROT_ERR_CUDA;
  const int slot_bytes = (int)((kRowsPerWarp * row_bytes + 1023) / 1024 * 1024);
  int slots = (int)((110 * 1024) / ((int64_t)kRqTmaWarps * slot_bytes));
  slots = std::max(2, std::min(kRqMaxSlots, slots));
  const size_t smem = 1024 + (size_t)kRqTmaWarps * slots * (slot_bytes + 8) + kRqTmaWarps * 4;
  auto kern = rotquant_tma_kernel<InT, G, SEG>;
  int sms = 0;
  device_setup(&sms);
  // the attribute and the occupancy for this shared-memory size, once per device
  struct Residency {
    size_t smem = 0;
    int per_sm = 0;
  };
  static Residency cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CONVROT_ERR_CUDA;
  int per_sm = 0;
  {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    Residency& r = cached[dev];
    if (r.smem != smem) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kRqTmaWarps * 32, smem) !=
              cudaSuccess ||
          n < 1) {
        cudaGetLastError();
        n = 1;
      }
      r.smem = smem;
      r.per_sm = n;
    }
    per_sm = r.per_sm;
  }
  const int64_t units = (rows + kRowsPerWarp - 1) / kRowsPerWarp;
  const int64_t ctas = (units + kRqTmaWarps - 1) / kRqTmaWarps;
  int64_t grid = std::min<int64_t>(ctas, (int64_t)per_sm * std::max(sms, 1));
  if (grid_cap > 0 && ctas > grid) grid = std::min(grid, grid_cap);
  return launch_kernel(kern, dim3((unsigned)grid), dim3(kRqTmaWarps * 32), smem, st, pdl, 1, tm,
                       rows, K, slots, slot_bytes, q, s, out, wait_at_end ? 1 : 0);
}

template <typename InT, int G>
int launch_rq(const void* x, int64_t rows, int K, int8_t* q, float* s, RqOut out,
               cudaStream_t st, bool pdl, int64_t grid_cap, bool wait_at_end) {
  // K % 64 == 0, K <= 2048: one warp segment of SEG lanes per row, 64
  // elements per lane (G = 256 needs at least the four lanes of one group)
  if (K % 64 == 0 && K <= 2048) {
    const int lanes = K / 64;
    if (lanes <= 1 && G < 256) return launch_rq_tma<InT, G, (G < 256 ? 1 : 4)>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
    if (lanes <= 2 && G < 256) return launch_rq_tma<InT, G, (G < 256 ? 2 : 4)>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
    if (lanes <= 4) return launch_rq_tma<InT, G, 4>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
    if (lanes <= 8) return launch_rq_tma<InT, G, 8>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
    if (lanes <= 16) return launch_rq_tma<InT, G, 16>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
    return launch_rq_tma<InT, G, 32>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
  }
  const int nch = K / 16;
  int tpr;
  if (nch <= 32) {
    tpr = 1;
    while (tpr < nch) tpr <<= 1;
  } else {
    tpr = (nch + 31) / 32 * 32;
  }
  // whole rows per CTA: a CTA never holds threads beyond rpc * tpr
  const int rpc = std::max(1, kRqThreads / tpr);
  const int threads = rpc * tpr;
  const int64_t groups = (rows + rpc - 1) / rpc;
  // persistent: as many CTAs as fit on the device at once
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotquant_kernel<InT, G>, threads, 0) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  int sms = 0;
  device_setup(&sms);
  const int64_t grid = std::min<int64_t>(groups, (int64_t)per_sm * std::max(sms, 1));
  return launch_kernel(rotquant_kernel<InT, G>, dim3((unsigned)grid), dim3(threads), 0, st, pdl, 1,
                       reinterpret_cast<const InT*>(x), rows, K, tpr, q, s, out);
}

template <typename InT>
int dispatch_rq(int group, const void* x, int64_t rows, int K, int8_t* q, float* s, RqOut out,
                cudaStream_t st, bool pdl, int64_t grid_cap, bool wait_at_end) {
  switch (group) {
    case 1: return launch_rq<InT, 1>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
    case 4: return launch_rq<InT, 4>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
    case 16: return launch_rq<InT, 16>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
    case 64: return launch_rq<InT, 64>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
    default: return launch_rq<InT, 256>(x, rows, K, q, s, out, st, pdl, grid_cap, wait_at_end);
  }
}

int check_rq_args(const void* x, int x_dtype, int64_t rows, int64_t K, int group, const int8_t* q,
                  const float* s) {
  if (x_dtype != CONVROT_DTYPE_BF16 && x_dtype != CONVROT_DTYPE_F32) return CONVROT_ERR_INVALID_ARG;
  if (rows < 0 || rows >= ((int64_t)1 << 31)) return CONVROT_ERR_INVALID_ARG;
  if (!valid_group(group)) return CONVROT_ERR_INVALID_ARG;
  if (K < 16 || K > 16384 || K % 16 != 0 || K % group != 0) return CONVROT_ERR_INVALID_ARG;
  if (rows > 0 && (!x || !q || !s)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(x) || !al16(q) || !al16(s)) return CONVROT_ERR_MISALIGNED;
  return CONVROT_OK;
}

int rotquant_impl(const void* x, int x_dtype, int64_t rows, int64_t K, int group, int8_t* q,
                  float* s, cudaStream_t st, RqOut out = RqOut{0, 1, 1, 1}, bool pdl = false,
                  int64_t grid_cap = 0, bool wait_at_end = false) {
  if (rows == 0) return CONVROT_OK;
  const int rc = (x_dtype == CONVROT_DTYPE_BF16)
                     ? dispatch_rq<__nv_bfloat16>(group, x, rows, (int)K, q, s, out, st, pdl,
                                                  grid_cap, wait_at_end)
                     : dispatch_rq<float>(group, x, rows, (int)K, q, s, out, st, pdl, grid_cap,
                                          wait_at_end);
  if (rc != CONVROT_OK) return rc;
  return launch_status();
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// The offline weight quantiser: fp64 rotation and quotients (the definition
// exactly), one persistent CTA per row at a time, the row in shared memory.
template <int G>
int launch_rq_f64(const void* w, int64_t rows, int K, int8_t* q, float* s, RqOut out,
                  cudaStream_t st) {
  auto kern = rotquant_f64_kernel<G>;
  const size_t smem = (size_t)K * sizeof(double);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return CONVROT_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRq64Threads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  int sms = 0;
  device_setup(&sms);
  const int64_t grid = std::min<int64_t>(rows, (int64_t)per_sm * std::max(sms, 1));
  return launch_kernel(kern, dim3((unsigned)grid), dim3(kRq64Threads), smem, st, false, 1,
                       reinterpret_cast<const __nv_bfloat16*>(w), rows, K, q, s, out);
}

int quantize_weights_impl(const void* w, int64_t rows, int64_t K, int group, int8_t* q, float* s,
                          cudaStream_t st, RqOut out) {
  if (rows == 0) return CONVROT_OK;
  int rc;
  switch (group) {
    case 1: rc = launch_rq_f64<1>(w, rows, (int)K, q, s, out, st); break;
    case 4: rc = launch_rq_f64<4>(w, rows, (int)K, q, s, out, st); break;
    case 16: rc = launch_rq_f64<16>(w, rows, (int)K, q, s, out, st); break;
    case 64: rc = launch_rq_f64<64>(w, rows, (int)K, q, s, out, st); break;
    default: rc = launch_rq_f64<256>(w, rows, (int)K, q, s, out, st); break;
  }
  if (rc != CONVROT_OK) return rc;
  return launch_status();
}

// Bytes of the tiled weight format for n_mats matrices of `rows` x K.
int64_t tiled_bytes(int64_t n_mats, int64_t rows, int64_t K) {
  return n_mats * cdiv(rows, 128) * cdiv(K, 128) * 16384;
}

// ------------------------------------------------------------------ GEMM --
int encode_3d_i8(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint64_t groups,
                 uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CONVROT_ERR_CUDA;
  const cuuint64_t dims[3] = {K, rows, groups};
  const cuuint64_t strides[2] = {K, K * rows};
  const cuuint32_t box[3] = {(cuuint32_t)gemm::BK, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CONVROT_OK : CONVROT_ERR_CUDA;
}

int check_gemm_shape(const int8_t* a, const int8_t* b, int64_t G, int64_t M, int64_t NB,
                     int64_t K) {
  if (G < 0 || M < 0 || NB < 0 || K < 16) return CONVROT_ERR_INVALID_ARG;
  if (G >= ((int64_t)1 << 31) || M >= ((int64_t)1 << 31) || NB >= ((int64_t)1 << 31))
    return CONVROT_ERR_INVALID_ARG;
  if (K % 16 != 0 || K >= ((int64_t)1 << 31) || NB % 16 != 0) return CONVROT_ERR_INVALID_ARG;
  if (K * 127 * 127 >= ((int64_t)1 << 31)) return CONVROT_ERR_INVALID_ARG;  // int32 accumulator
  if (G * M > 0 && (!a || !b)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(a) || !al16(b)) return CONVROT_ERR_MISALIGNED;
  return CONVROT_OK;
}

int encode_tiled_b(CUtensorMap* map, const void* base, uint64_t kb_count, uint64_t row_blocks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CONVROT_ERR_CUDA;
  const cuuint64_t dims[4] = {128, 128, kb_count, row_blocks};
  const cuuint64_t strides[3] = {128, 16384, 16384 * kb_count};
  const cuuint32_t box[4] = {128, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// Units (CTAs, or CTA pairs) the requantising SwiGLU GEMM runs `tiles` tiles
// on, n_blocks of them per row block; 0 when the device cannot keep enough of
// them resident for the tiles of a row block to meet.
// The same for a given capacity of co-resident units (a pure host rule).
int64_t rq_units_for(int64_t tiles, int64_t n_blocks, int64_t cap) {
  if (tiles <= 0 || n_blocks <= 0) return 0;
  if (tiles <= cap) return tiles;
  if (cap < n_blocks) return 0;
  // a whole number of row blocks per wave: the tiles of a row block then run
  // side by side instead of one wave apart
  return cap / n_blocks * n_blocks;
}

int64_t swiglu_rq_units(int64_t tiles, int64_t n_blocks, bool pairs, int sms) {
  const int64_t cap = std::min<int64_t>(pairs ? sms / 2 : sms, swiglu_rq_capacity(pairs));
  return rq_units_for(tiles, n_blocks, cap);
}

// Whether the gate/up GEMM over G groups of M rows (tiled weights, F h
// columns) can requantise h in its epilogue on this device.
bool swiglu_rq_fits(int64_t G, int64_t M, int64_t F, int sms) {
  const bool pairs = M > gemm::BM && sms >= 2;
  const int64_t n_blocks = cdiv(F, gemm::BN / 2);
  const int64_t tiles = G * cdiv(M, pairs ? gemm2::BM : gemm::BM) * n_blocks;
  return swiglu_rq_units(tiles, n_blocks, pairs, sms) > 0;
}

// Bytes of the fused h requantisation's synchronisation scratch for G groups
// of M rows: the row maxima [G*M] (fp32 bits), then at a 256-byte boundary
// the tile arrivals of every 128-row slab [G*(ceil(M/128)+1)], one abort
// word, and each group's count of published tiles [G] (read by a streamed
// down GEMM). All zero before the GEMM starts.
size_t swiglu_rq_sync_bytes(int64_t G, int64_t M) {
  const size_t rows = (size_t)G * (size_t)M;
  const size_t counters = (size_t)G * (size_t)(cdiv(M, 128) + 1) + 1 + (size_t)G;
  return ((rows * 4 + 255) & ~(size_t)255) + counters * 4;
}

// The published-tile counters of that scratch.
int* swiglu_rq_done_words(char* sync, int64_t G, int64_t M) {
  const size_t rows = (size_t)G * (size_t)M;
  return reinterpret_cast<int*>(sync + ((rows * 4 + 255) & ~(size_t)255)) +
         G * (cdiv(M, 128) + 1) + 1;
}

// NB = rows of one B matrix per group (2F for SwiGLU). With BT the B operand
// is in the tiled weight format: for SwiGLU each group holds a gate matrix and
// an up matrix of F rows, each padded to 128-row blocks.
template <int EPI, bool BT>
int launch_gemm(const int8_t* a, const int8_t* b, int64_t G, int64_t M, int64_t NB, int64_t K,
                int64_t n_out, GemmArgs args, cudaStream_t st, bool pdl = false) {
  int sms = 0;
  int rc = device_setup(&sms);
  if (rc != CONVROT_OK) return rc;
  if (G == 0 || M == 0 || n_out == 0) return CONVROT_OK;
  CUtensorMap ta, tb;
  const uint32_t box_a = (uint32_t)std::min<int64_t>(gemm::BM, M);
  uint32_t box_b;
  if ((rc = encode_3d_i8(&ta, a, (uint64_t)K, (uint64_t)M, (uint64_t)G, box_a)) != CONVROT_OK)
    return rc;
  if (BT) {
    const int64_t blocks = epi_is_swiglu(EPI) ? cdiv(n_out, 128) : cdiv(NB, 128);
    const int64_t per_group = epi_is_swiglu(EPI) ? 2 * blocks : blocks;
    args.b_blocks = (int)blocks;
    box_b = 128;
    if ((rc = encode_tiled_b(&tb, b, (uint64_t)cdiv(K, 128), (uint64_t)(G * per_group))) !=
        CONVROT_OK)
      return rc;
  } else {
    box_b = (uint32_t)std::min<int64_t>(gemm::BN / 2, NB);
    if ((rc = encode_3d_i8(&tb, b, (uint64_t)K, (uint64_t)NB, (uint64_t)G, box_b)) != CONVROT_OK)
      return rc;
  }
  args.G = (int)G;
  args.M = (int)M;
  args.NB = (int)NB;
  args.K = (int)K;
  args.n_out = (int)n_out;
  // CTA pairs (M = 256 tiles) once a group has more than 128 rows and the
  // weight boxes are whole 128-row blocks
  const bool pairs = M > gemm::BM && box_b == 128 && sms >= 2;
  // The requantising SwiGLU epilogue: tiles n-block fastest, the grid within
  // what can be resident at once and, when it cannot hold every tile, at
  // least one row block's n_blocks tiles (its tiles wait for one another).
  args.nb_fast = EPI == kEpiSwigluRq ? 1 : 0;
  const int64_t n_tile = epi_is_swiglu(EPI) ? gemm::BN / 2 : gemm::BN;
  args.n_blocks = (int)cdiv(n_out, n_tile);
  args.k_blocks = (int)cdiv(K, gemm::BK);
  auto resident_units = [&](int64_t tiles, int64_t units) -> int64_t {
    if (EPI != kEpiSwigluRq) return std::min<int64_t>(tiles, units);
    return swiglu_rq_units(tiles, args.n_blocks, pairs, sms);
  };
  if (pairs) {
    args.m_blocks = (int)cdiv(M, gemm2::BM);
    args.slabs = 2 * args.m_blocks;
    const int64_t tiles = G * args.m_blocks * args.n_blocks;
    if (tiles >= ((int64_t)1 << 30)) return CONVROT_ERR_INVALID_ARG;
    args.num_tiles = (int)tiles;
    args.box_bytes = 2 * (128 + 128) * gemm::BK;  // both CTAs' A and B boxes
    const int64_t n_pairs = resident_units(tiles, sms / 2);
    if (n_pairs < 1) return CONVROT_ERR_INVALID_ARG;
    const int grid = 2 * (int)n_pairs;
    if ((rc = launch_kernel(gemm_s8_tcgen05_pair_kernel<EPI, BT>, dim3(grid),
                            dim3(EpiCfg<EPI>::kThreads), EpiCfg<EPI>::kSmem2, st, pdl, 2, ta, tb,
                            args)) != CONVROT_OK)
      return rc;
    return launch_status();
  }
  args.m_blocks = (int)cdiv(M, gemm::BM);
  args.slabs = args.m_blocks;
  args.a_lane0 = M <= 64 ? 64 : 0;
  const int64_t tiles = G * args.m_blocks * args.n_blocks;
  if (tiles >= ((int64_t)1 << 31)) return CONVROT_ERR_INVALID_ARG;
  args.num_tiles = (int)tiles;
  args.box_bytes = (int)((box_a + 2 * box_b) * gemm::BK);  // A and B boxes of one stage
  const int grid = (int)resident_units(tiles, sms);
  if (grid < 1) return CONVROT_ERR_INVALID_ARG;
  if ((rc = launch_kernel(gemm_s8_tcgen05_kernel<EPI, BT>, dim3(grid), dim3(EpiCfg<EPI>::kThreads),
                          EpiCfg<EPI>::kSmem1, st, pdl, 1, ta, tb, args)) != CONVROT_OK)
    return rc;
  return launch_status();
}

template <int EPI>
int launch_gemm_layout(int b_layout, const int8_t* a, const int8_t* b, int64_t G, int64_t M,
                       int64_t NB, int64_t K, int64_t n_out, GemmArgs args, cudaStream_t st) {
  if (b_layout == CONVROT_LAYOUT_TILES)
    return launch_gemm<EPI, true>(a, b, G, M, NB, K, n_out, args, st);
  return launch_gemm<EPI, false>(a, b, G, M, NB, K, n_out, args, st);
}

int topc_impl(const float* s_t, int64_t T, int E, int64_t C, int32_t* idx, float* w,
              int32_t* slot, cudaStream_t st, bool pdl = false) {
  if (E == 0 || (C == 0 && slot == nullptr)) return CONVROT_OK;
  // scores held in registers when T <= 16 per thread; the general kernel
  // re-reads them from memory on every pass
  const int per_thread = (int)((T + kTopcThreads - 1) / kTopcThreads);
  auto kern = topc_kernel;
  if (per_thread <= 1)
    kern = topc_reg_kernel<1>;
  else if (per_thread <= 2)
    kern = topc_reg_kernel<2>;
  else if (per_thread <= 4)
    kern = topc_reg_kernel<4>;
  else if (per_thread <= 8)
    kern = topc_reg_kernel<8>;
  else if (per_thread <= 16)
    kern = topc_reg_kernel<16>;
  const int rc = launch_kernel(kern, dim3(E), dim3(kTopcThreads), 0, st, pdl, 1, s_t, (int)T,
                               (int)C, idx, w, slot);
  if (rc != CONVROT_OK) return rc;
  return launch_status();
}

template <int NJ>
int launch_combine(const void* z, const float* s_t, const int32_t* slot, int E, int64_t T,
                   int64_t C, int64_t d, void* y, int sms, cudaStream_t st, bool pdl) {
  auto kern = combine_tokens_kernel<NJ>;
  // tokens per CTA: the smallest power of two in [1, 32] for which the whole
  // grid is resident at once (measured on B200 at T = 2048: one wave of 4
  // tokens per CTA beats 3.5 waves of single tokens by 4 us, as every later
  // wave would repeat the list building after the GEMM has finished)
  static std::atomic<int> resident[kMaxDevices][4];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CONVROT_ERR_CUDA;
  std::atomic<int>& cached = resident[dev][NJ == 1 ? 0 : NJ == 2 ? 1 : NJ == 4 ? 2 : 3];
  int per_sm = cached.load(std::memory_order_relaxed);
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kCombThreads,
                                                      combine_tokens_smem(E, 1)) != cudaSuccess) {
      cudaGetLastError();
      return CONVROT_ERR_CUDA;
    }
    cached.store(per_sm, std::memory_order_relaxed);
  }
  const int64_t capacity = std::max<int64_t>(1, (int64_t)std::max(per_sm, 1) * std::max(sms, 1));
  int tpc = 1;
  while (tpc < 32 && cdiv(T, tpc) > capacity) tpc <<= 1;
  const size_t smem = combine_tokens_smem(E, tpc);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return CONVROT_ERR_CUDA;
  const int64_t grid = (T + tpc - 1) / tpc;
  return launch_kernel(kern, dim3((unsigned)grid), dim3(kCombThreads), smem, st, pdl, 1,
                       reinterpret_cast<const __nv_bfloat16*>(z), s_t, slot, E, (int)T, (int)C,
                       (int)d, tpc, reinterpret_cast<__nv_bfloat16*>(y));
}

// E <= 256 (checked by the entry points)
int combine_impl(const void* z, const float* s_t, const int32_t* slot, int E, int64_t T, int64_t C,
                 int64_t d, void* y, int sms, cudaStream_t st, bool pdl = false) {
  if (T == 0) return CONVROT_OK;
  int rc;
  if (E <= 32)
    rc = launch_combine<1>(z, s_t, slot, E, T, C, d, y, sms, st, pdl);
  else if (E <= 64)
    rc = launch_combine<2>(z, s_t, slot, E, T, C, d, y, sms, st, pdl);
  else if (E <= 128)
    rc = launch_combine<4>(z, s_t, slot, E, T, C, d, y, sms, st, pdl);
  else
    rc = launch_combine<8>(z, s_t, slot, E, T, C, d, y, sms, st, pdl);
  if (rc != CONVROT_OK) return rc;
  return launch_status();
}

template <int NJ>
void launch_softmax(const void* logits, int64_t T, int E, float* s_t, cudaStream_t st) {
  const int64_t grid = (T + kSmTokens - 1) / kSmTokens;
  router_softmax_kernel<NJ><<<(unsigned)grid, 32 * kSmTokens,
                              (size_t)E * kSmTokens * sizeof(float), st>>>(
      reinterpret_cast<const __nv_bfloat16*>(logits), (int)T, E, s_t);
}

// E <= 256 (checked by the entry points): NJ = ceil(E / 32) experts per lane
int softmax_impl(const void* logits, int64_t T, int E, float* s_t, cudaStream_t st) {
  if (T == 0) return CONVROT_OK;
  switch ((E + 31) / 32) {
    case 1: launch_softmax<1>(logits, T, E, s_t, st); break;
    case 2: launch_softmax<2>(logits, T, E, s_t, st); break;
    case 3: launch_softmax<3>(logits, T, E, s_t, st); break;
    case 4: launch_softmax<4>(logits, T, E, s_t, st); break;
    case 5: launch_softmax<5>(logits, T, E, s_t, st); break;
    case 6: launch_softmax<6>(logits, T, E, s_t, st); break;
    case 7: launch_softmax<7>(logits, T, E, s_t, st); break;
    default: launch_softmax<8>(logits, T, E, s_t, st); break;
  }
  return launch_status();
}

int gather_impl(const int8_t* src, const float* s_src, int64_t n_src, const int32_t* idx,
                int64_t n_rows, int64_t K, int8_t* dst, float* s_dst, cudaStream_t st,
                uint32_t* zero = nullptr, int64_t n_zero = 0, bool pdl = false) {
  if (n_rows == 0) return CONVROT_OK;
  const int64_t grid = (n_rows + 7) / 8;
  const int rc = launch_kernel(gather_rows_kernel, dim3((unsigned)grid), dim3(256), 0, st, pdl, 1,
                               src, s_src, n_src, idx, n_rows, (int)K, dst, s_dst, zero, n_zero);
  if (rc != CONVROT_OK) return rc;
  return launch_status();
}

int convert_impl(const float* x, int64_t n, void* y, int sms, cudaStream_t st) {
  if (n == 0) return CONVROT_OK;
  const int64_t n4 = n / 4;
  const int64_t grid = std::min<int64_t>((n4 + 255) / 256, (int64_t)sms * 8);
  f32_to_bf16_kernel<<<(unsigned)grid, 256, 0, st>>>(x, n4,
                                                     reinterpret_cast<__nv_bfloat16*>(y));
  return launch_status();
}

// ---------------------------------------------------------------- low-bit --
inline bool valid_bits(int bits) { return bits == 4 || bits == 6; }

int lowbit_tile_bytes(int bits) {
  return bits == 4 ? LbFmt<4>::kTileBytes : LbFmt<6>::kTileBytes;
}

// Bytes of the b-bit weight format for `rows` x K (rows % 128 == 0, K % 64 == 0).
int64_t lowbit_bytes(int64_t rows, int64_t K, int bits) {
  return (rows / 128) * (K / 64) * (int64_t)lowbit_tile_bytes(bits);
}

template <int G, int BITS>
int launch_lowbit_quant(const void* w, int64_t rows, int K, uint8_t* out, float* s,
                        cudaStream_t st) {
  auto kern = lowbit_quant_f64_kernel<G, BITS>;
  const size_t smem = (size_t)K * sizeof(double);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return CONVROT_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kLbQuantThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  int sms = 0;
  device_setup(&sms);
  const int64_t grid = std::min<int64_t>(rows, (int64_t)per_sm * std::max(sms, 1));
  return launch_kernel(kern, dim3((unsigned)grid), dim3(kLbQuantThreads), smem, st, false, 1,
                       reinterpret_cast<const __nv_bfloat16*>(w), rows, K, out, s);
}

template <int BITS>
int lowbit_quant_group(const void* w, int64_t rows, int K, int group, uint8_t* out, float* s,
                       cudaStream_t st) {
  switch (group) {
    case 1: return launch_lowbit_quant<1, BITS>(w, rows, K, out, s, st);
    case 4: return launch_lowbit_quant<4, BITS>(w, rows, K, out, s, st);
    case 16: return launch_lowbit_quant<16, BITS>(w, rows, K, out, s, st);
    case 64: return launch_lowbit_quant<64, BITS>(w, rows, K, out, s, st);
    default: return launch_lowbit_quant<256, BITS>(w, rows, K, out, s, st);
  }
}

// 3-D view {K, rows, groups} of int8 activation codes, box {64 codes,
// box_rows rows, 1}, no swizzle (the converters read it row by row).
int encode_act_i8(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint64_t groups,
                  uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CONVROT_ERR_CUDA;
  const cuuint64_t dims[3] = {K, rows, groups};
  const cuuint64_t strides[2] = {K, K * rows};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// Tokens per tile when the caller leaves it open: one tile of all the tokens
// up to 64, else 128 (the MMA's M; rows past the tile's tokens are not
// widened and their accumulator rows are not read).
int lowbit_auto_nt(int64_t M) {
  return M <= 64 ? (int)std::max<int64_t>(16, cdiv(M, 16) * 16) : lb::kMaxNt;
}

int check_lowbit_gemm(const int8_t* x, const void* wq, int64_t G, int64_t M, int64_t N,
                      int64_t K, int bits, int tile_tokens) {
  if (!valid_bits(bits)) return CONVROT_ERR_INVALID_ARG;
  if (G < 0 || M < 0 || N < 0 || K < 64 || K > 16384 || K % 64 != 0 || N % 256 != 0)
    return CONVROT_ERR_INVALID_ARG;
  if (G >= ((int64_t)1 << 31) || M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) ||
      G * M >= ((int64_t)1 << 31) || G * N >= ((int64_t)1 << 31))
    return CONVROT_ERR_INVALID_ARG;
  if (tile_tokens != 0 && (tile_tokens < 16 || tile_tokens > lb::kMaxNt || tile_tokens % 16))
    return CONVROT_ERR_INVALID_ARG;
  if (G * M > 0 && N > 0 && (!x || !wq)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(x) || !al16(wq)) return CONVROT_ERR_MISALIGNED;
  return CONVROT_OK;
}

template <int BITS, int EPI>
int launch_lowbit_gemm(const int8_t* x, const float* s_x, const uint8_t* wq, const float* s_w,
                       int64_t G, int64_t M, int64_t N, int64_t K, int tile_tokens, void* out,
                       cudaStream_t st, bool pdl = false) {
  int sms = 0;
  int rc = device_setup(&sms);
  if (rc != CONVROT_OK) return rc;
  if (G == 0 || M == 0 || N == 0) return CONVROT_OK;
  // more than one tile of tokens per group: CTA pairs, each decoded weight
  // serving the 256 tokens of both CTAs
  const int pairs = lowbit_pair_capacity();
  const bool pair = tile_tokens == 0 && M > lb::kMaxNt && pairs > 0;
  LowbitArgs a{};
  a.G = (int)G;
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.n_out = (int)(EPI == kLbSwiglu ? N / 2 : N);
  a.nt = pair ? lb::kMaxNt : tile_tokens > 0 ? tile_tokens : lowbit_auto_nt(M);
  a.box_rows = (int)std::min<int64_t>(a.nt, M);
  a.t_blocks = (int)cdiv(M, pair ? 2 * a.nt : a.nt);
  a.w_blocks = (int)(N / 256);
  a.k_blocks = (int)(K / 64);
  const int64_t tiles = G * a.w_blocks * a.t_blocks;
  if (tiles >= ((int64_t)1 << 31)) return CONVROT_ERR_INVALID_ARG;
  a.num_tiles = (int)tiles;
  a.raw_stages = lb::raw_stages<BITS>(a.nt, pair);
  a.wq = wq;
  a.s_w = s_w;
  a.s_x = s_x;
  a.out = out;
  CUtensorMap tx;
  if ((rc = encode_act_i8(&tx, x, (uint64_t)K, (uint64_t)M, (uint64_t)G, (uint32_t)a.box_rows)) !=
      CONVROT_OK)
    return rc;
  if (pair) {
    const int grid = 2 * (int)std::min<int64_t>(tiles, pairs);
    rc = launch_kernel(gemm_lowbit_tcgen05_kernel<BITS, EPI, true, false>, dim3(grid),
                       dim3(lb::kThreads), lb::smem_bytes<BITS>(a.nt, true), st, pdl, 2, tx, a);
  } else {
    // up to 64 tokens per tile: M = 64 instructions
    const int grid = (int)std::min<int64_t>(tiles, sms);
    if (a.nt <= 64)
      rc = launch_kernel(gemm_lowbit_tcgen05_kernel<BITS, EPI, false, true>, dim3(grid),
                         dim3(lb::kThreads), lb::smem_bytes<BITS>(a.nt, false), st, pdl, 1, tx, a);
    else
      rc = launch_kernel(gemm_lowbit_tcgen05_kernel<BITS, EPI, false, false>, dim3(grid),
                         dim3(lb::kThreads), lb::smem_bytes<BITS>(a.nt, false), st, pdl, 1, tx, a);
  }
  if (rc != CONVROT_OK) return rc;
  return launch_status();
}

template <int EPI>
int launch_lowbit_bits(int bits, const int8_t* x, const float* s_x, const void* wq,
                       const float* s_w, int64_t G, int64_t M, int64_t N, int64_t K,
                       int tile_tokens, void* out, cudaStream_t st, bool pdl = false) {
  const uint8_t* w = reinterpret_cast<const uint8_t*>(wq);
  if (bits == 4)
    return launch_lowbit_gemm<4, EPI>(x, s_x, w, s_w, G, M, N, K, tile_tokens, out, st, pdl);
  return launch_lowbit_gemm<6, EPI>(x, s_x, w, s_w, G, M, N, K, tile_tokens, out, st, pdl);
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

// ===================================================================== ABI ==
extern "C" {

int convrot_abi_version(void) { return 3; }

const char* convrot_last_cuda_error(void) { return g_last_cuda_error; }

const char* convrot_status_string(int status) {
  switch (status) {
    case CONVROT_OK: return "ok";
    case CONVROT_ERR_INVALID_ARG: return "invalid argument";
    case CONVROT_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs sm_100)";
    case CONVROT_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case CONVROT_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case CONVROT_ERR_CUDA: return "CUDA error";
    case CONVROT_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int convrot_device_check(void) { return device_setup(nullptr); }

int convrot_check_device_error(void* stream, unsigned* flags) {
  int rc = device_setup(nullptr);
  if (rc != CONVROT_OK) return rc;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return CONVROT_ERR_CUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  if (flags) *flags = v;
  return v ? CONVROT_ERR_TIMEOUT : CONVROT_OK;
}

int convrot_wait_selftest(unsigned long long limit_ns, int* result_dev, void* stream) {
  int rc = device_setup(nullptr);
  if (rc != CONVROT_OK) return rc;
  if (!result_dev || limit_ns > 10000000000ull) return CONVROT_ERR_INVALID_ARG;
  wait_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(limit_ns, result_dev);
  return launch_status();
}

int convrot_count_wait_selftest(unsigned long long limit_ns, int* words_dev, int* result_dev,
                                void* stream) {
  int rc = device_setup(nullptr);
  if (rc != CONVROT_OK) return rc;
  if (!words_dev || !result_dev || limit_ns > 10000000000ull) return CONVROT_ERR_INVALID_ARG;
  count_wait_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(limit_ns, words_dev, result_dev);
  return launch_status();
}

int64_t convrot_swiglu_rq_units(int64_t tiles, int64_t n_blocks, int64_t capacity) {
  if (tiles < 0 || n_blocks < 0 || capacity < 0) return -1;
  return rq_units_for(tiles, n_blocks, capacity);
}

int convrot_rotquant(const void* x, int x_dtype, int64_t rows, int64_t K, int group, int8_t* q,
                     float* scale, void* stream) {
  int rc = check_rq_args(x, x_dtype, rows, K, group, q, scale);
  if (rc != CONVROT_OK) return rc;
  if ((rc = device_setup(nullptr)) != CONVROT_OK) return rc;
  return rotquant_impl(x, x_dtype, rows, K, group, q, scale, as_stream(stream));
}

int convrot_quantize_weights(const void* w_bf16, int64_t rows, int64_t K, int group, int8_t* w_q,
                             float* row_scale, void* stream) {
  int rc = check_rq_args(w_bf16, CONVROT_DTYPE_BF16, rows, K, group, w_q, row_scale);
  if (rc != CONVROT_OK) return rc;
  if ((rc = device_setup(nullptr)) != CONVROT_OK) return rc;
  return quantize_weights_impl(w_bf16, rows, K, group, w_q, row_scale, as_stream(stream),
                               RqOut{0, 1, 1, 1});
}

int64_t convrot_tiled_weight_bytes(int64_t n_mats, int64_t rows, int64_t K) {
  if (n_mats < 0 || rows < 0 || K < 0) return -1;
  return tiled_bytes(n_mats, rows, K);
}

int convrot_quantize_weights_tiled(const void* w_bf16, int64_t n_mats, int64_t rows, int64_t K,
                                   int group, int8_t* w_tiled, float* row_scale, void* stream) {
  if (n_mats < 0 || rows < 0 || n_mats * rows >= ((int64_t)1 << 31)) return CONVROT_ERR_INVALID_ARG;
  int rc = check_rq_args(w_bf16, CONVROT_DTYPE_BF16, n_mats * rows, K, group, w_tiled, row_scale);
  if (rc != CONVROT_OK) return rc;
  if ((rc = device_setup(nullptr)) != CONVROT_OK) return rc;
  if (n_mats * rows == 0) return CONVROT_OK;
  cudaStream_t st = as_stream(stream);
  // padding rows and K columns of the last tiles read as zero codes
  if (cudaMemsetAsync(w_tiled, 0, (size_t)tiled_bytes(n_mats, rows, K), st) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  const RqOut out{1, rows, (int)cdiv(rows, 128), (int)cdiv(K, 128)};
  return quantize_weights_impl(w_bf16, n_mats * rows, K, group, w_tiled, row_scale, st, out);
}

int convrot_router_softmax(const void* logits_bf16, int64_t T, int E, float* s_t, void* stream) {
  if (T < 0 || T >= ((int64_t)1 << 31) || E < 1 || E > 256) return CONVROT_ERR_INVALID_ARG;
  if (T > 0 && (!logits_bf16 || !s_t)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(logits_bf16) || !al16(s_t)) return CONVROT_ERR_MISALIGNED;
  int rc = device_setup(nullptr);
  if (rc != CONVROT_OK) return rc;
  return softmax_impl(logits_bf16, T, E, s_t, as_stream(stream));
}

int convrot_topc(const float* s_t, int64_t T, int E, int64_t C, int32_t* idx, float* w,
                 int32_t* slot, void* stream) {
  if (T < 0 || T >= ((int64_t)1 << 31) || E < 0 || E > 65535 || C < 0 || C > T)
    return CONVROT_ERR_INVALID_ARG;
  if (C > 0 && E > 0 && (!s_t || !idx || !w)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(s_t) || !al16(idx) || !al16(w) || !al16(slot)) return CONVROT_ERR_MISALIGNED;
  int rc = device_setup(nullptr);
  if (rc != CONVROT_OK) return rc;
  return topc_impl(s_t, T, E, C, idx, w, slot, as_stream(stream));
}

int convrot_combine_rows(const void* z_bf16, const float* s_t, const int32_t* slot, int E,
                         int64_t T, int64_t C, int64_t d, void* y_bf16, void* stream) {
  if (E < 1 || E > 256 || T < 0 || T >= ((int64_t)1 << 31) || C < 0 || C > T || d < 8 ||
      d > 8192 || d % 8 != 0 || (int64_t)E * C >= ((int64_t)1 << 31))
    return CONVROT_ERR_INVALID_ARG;
  if (T > 0 && (!slot || !s_t || !y_bf16 || (C > 0 && !z_bf16))) return CONVROT_ERR_INVALID_ARG;
  if (!al16(z_bf16) || !al16(s_t) || !al16(slot) || !al16(y_bf16)) return CONVROT_ERR_MISALIGNED;
  int sms = 0;
  int rc = device_setup(&sms);
  if (rc != CONVROT_OK) return rc;
  return combine_impl(z_bf16, s_t, slot, E, T, C, d, y_bf16, sms, as_stream(stream));
}

int convrot_gather_rows(const int8_t* src, const float* s_src, int64_t n_src, const int32_t* idx,
                        int64_t n_rows, int64_t K, int8_t* dst, float* s_dst, void* stream) {
  if (n_src < 0 || n_rows < 0 || K < 16 || K % 16 != 0 || K >= ((int64_t)1 << 31))
    return CONVROT_ERR_INVALID_ARG;
  if (n_rows > 0 && (!src || !s_src || !idx || !dst || !s_dst || n_src == 0))
    return CONVROT_ERR_INVALID_ARG;
  if (!al16(src) || !al16(dst)) return CONVROT_ERR_MISALIGNED;
  int rc = device_setup(nullptr);
  if (rc != CONVROT_OK) return rc;
  return gather_impl(src, s_src, n_src, idx, n_rows, K, dst, s_dst, as_stream(stream));
}

int convrot_i8_gemm_i32(const int8_t* a, const int8_t* b, int b_layout, int64_t G, int64_t M,
                        int64_t N, int64_t K, int32_t* d, void* stream) {
  if (b_layout != CONVROT_LAYOUT_ROWS && b_layout != CONVROT_LAYOUT_TILES)
    return CONVROT_ERR_INVALID_ARG;
  int rc = check_gemm_shape(a, b, G, M, N, K);
  if (rc != CONVROT_OK) return rc;
  if (G * M * N > 0 && !d) return CONVROT_ERR_INVALID_ARG;
  if (!al16(d)) return CONVROT_ERR_MISALIGNED;
  GemmArgs args{};
  args.out = d;
  return launch_gemm_layout<kEpiI32>(b_layout, a, b, G, M, N, K, N, args, as_stream(stream));
}

int convrot_i8_gemm_bf16(const int8_t* a, const float* s_a, const int8_t* b, const float* s_b,
                         int b_layout, int64_t G, int64_t M, int64_t N, int64_t K, void* y_bf16,
                         void* stream) {
  if (b_layout != CONVROT_LAYOUT_ROWS && b_layout != CONVROT_LAYOUT_TILES)
    return CONVROT_ERR_INVALID_ARG;
  int rc = check_gemm_shape(a, b, G, M, N, K);
  if (rc != CONVROT_OK) return rc;
  if (G * M * N > 0 && (!s_a || !s_b || !y_bf16)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(s_a) || !al16(s_b) || !al16(y_bf16)) return CONVROT_ERR_MISALIGNED;
  GemmArgs args{};
  args.s_a = s_a;
  args.s_b = s_b;
  args.out = y_bf16;
  return launch_gemm_layout<kEpiBf16>(b_layout, a, b, G, M, N, K, N, args, as_stream(stream));
}

int convrot_i8_gemm_swiglu(const int8_t* a, const float* s_a, const int8_t* b, const float* s_b,
                           int b_layout, int64_t G, int64_t M, int64_t F, int64_t K, float* h,
                           void* stream) {
  if (b_layout != CONVROT_LAYOUT_ROWS && b_layout != CONVROT_LAYOUT_TILES)
    return CONVROT_ERR_INVALID_ARG;
  if (F < 0 || F % 16 != 0) return CONVROT_ERR_INVALID_ARG;
  int rc = check_gemm_shape(a, b, G, M, 2 * F, K);
  if (rc != CONVROT_OK) return rc;
  if (G * M * F > 0 && (!s_a || !s_b || !h)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(s_a) || !al16(s_b) || !al16(h)) return CONVROT_ERR_MISALIGNED;
  GemmArgs args{};
  args.s_a = s_a;
  args.s_b = s_b;
  args.out = h;
  return launch_gemm_layout<kEpiSwiglu>(b_layout, a, b, G, M, 2 * F, K, F, args,
                                        as_stream(stream));
}

size_t convrot_swiglu_rq_sync_bytes(int64_t G, int64_t M) {
  if (G < 0 || M < 0) return 0;
  return swiglu_rq_sync_bytes(G, M);
}

int convrot_i8_gemm_swiglu_rq(const int8_t* a, const float* s_a, const int8_t* b,
                              const float* s_b, int b_layout, int64_t G, int64_t M, int64_t F,
                              int64_t K, int g_h, int8_t* h_q, float* s_h, void* sync,
                              size_t sync_bytes, void* stream) {
  if (b_layout != CONVROT_LAYOUT_ROWS && b_layout != CONVROT_LAYOUT_TILES)
    return CONVROT_ERR_INVALID_ARG;
  if (F < 0 || F % 16 != 0 || F % g_h != 0) return CONVROT_ERR_INVALID_ARG;
  if (g_h != 1 && g_h != 4 && g_h != 16 && g_h != 64) return CONVROT_ERR_INVALID_ARG;
  int rc = check_gemm_shape(a, b, G, M, 2 * F, K);
  if (rc != CONVROT_OK) return rc;
  if (G * M * F > 0 && (!s_a || !s_b || !h_q || !s_h || !sync)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(s_a) || !al16(s_b) || !al16(h_q) || !al16(s_h) || !al16(sync))
    return CONVROT_ERR_MISALIGNED;
  if (G * M * F == 0) return device_setup(nullptr);
  if (sync_bytes < swiglu_rq_sync_bytes(G, M)) return CONVROT_ERR_WORKSPACE_TOO_SMALL;
  if ((rc = device_setup(nullptr)) != CONVROT_OK) return rc;
  cudaStream_t st = as_stream(stream);
  if (cudaMemsetAsync(sync, 0, swiglu_rq_sync_bytes(G, M), st) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  GemmArgs args{};
  args.s_a = s_a;
  args.s_b = s_b;
  args.out = h_q;
  args.g_h = g_h;
  args.s_h = s_h;
  args.hmax = reinterpret_cast<unsigned*>(sync);
  args.rsync = reinterpret_cast<int*>(reinterpret_cast<char*>(sync) +
                                      (((size_t)G * (size_t)M * 4 + 255) & ~(size_t)255));
  return launch_gemm_layout<kEpiSwigluRq>(b_layout, a, b, G, M, 2 * F, K, F, args, st);
}

int convrot_i8_gemm_scatter(const int8_t* a, const float* s_a, const int8_t* b, const float* s_b,
                            int b_layout, const int32_t* idx, const float* w, int64_t G, int64_t M,
                            int64_t N, int64_t K, float* out32, int64_t T, void* stream) {
  if (b_layout != CONVROT_LAYOUT_ROWS && b_layout != CONVROT_LAYOUT_TILES)
    return CONVROT_ERR_INVALID_ARG;
  int rc = check_gemm_shape(a, b, G, M, N, K);
  if (rc != CONVROT_OK) return rc;
  if (T < 0) return CONVROT_ERR_INVALID_ARG;
  if (G * M * N > 0 && (!s_a || !s_b || !idx || !w || !out32 || T == 0))
    return CONVROT_ERR_INVALID_ARG;
  if (!al16(s_a) || !al16(s_b) || !al16(out32)) return CONVROT_ERR_MISALIGNED;
  GemmArgs args{};
  args.s_a = s_a;
  args.s_b = s_b;
  args.out = out32;
  args.idx = idx;
  args.w = w;
  if (T >= ((int64_t)1 << 31)) return CONVROT_ERR_INVALID_ARG;
  args.out_rows = (int)T;
  return launch_gemm_layout<kEpiScatter>(b_layout, a, b, G, M, N, K, N, args, as_stream(stream));
}

int convrot_f32_to_bf16(const float* x, int64_t n, void* y_bf16, void* stream) {
  if (n < 0 || n % 4 != 0) return CONVROT_ERR_INVALID_ARG;
  if (n > 0 && (!x || !y_bf16)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(x) || ((uintptr_t)y_bf16 & 7u) != 0) return CONVROT_ERR_MISALIGNED;
  int sms = 0;
  int rc = device_setup(&sms);
  if (rc != CONVROT_OK) return rc;
  return convert_impl(x, n, y_bf16, sms, as_stream(stream));
}

size_t convrot_linear_workspace_size(int64_t M, int64_t K) {
  if (M < 0 || K < 0) return 0;
  return align256((size_t)M * (size_t)K) + align256((size_t)M * sizeof(float));
}

int w8a8_convrot_linear(const void* x_bf16, int64_t M, int64_t K, const int8_t* w_q,
                        const float* w_scale, int64_t N, int group, void* y_bf16, void* workspace,
                        size_t ws_bytes, void* stream) {
  int rc = check_rq_args(x_bf16, CONVROT_DTYPE_BF16, M, K, group, (const int8_t*)workspace,
                         (const float*)workspace);
  if (rc != CONVROT_OK) return rc;
  if ((rc = check_gemm_shape(w_q, w_q, 1, M, N, K)) != CONVROT_OK) return rc;
  if (M > 0 && N > 0 && (!w_scale || !y_bf16 || !workspace)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(w_scale) || !al16(y_bf16) || !al16(workspace)) return CONVROT_ERR_MISALIGNED;
  if (ws_bytes < convrot_linear_workspace_size(M, K)) return CONVROT_ERR_WORKSPACE_TOO_SMALL;
  if ((rc = device_setup(nullptr)) != CONVROT_OK) return rc;
  if (M == 0 || N == 0) return CONVROT_OK;
  cudaStream_t st = as_stream(stream);
  int8_t* x_q = reinterpret_cast<int8_t*>(workspace);
  float* s_x = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                        align256((size_t)M * (size_t)K));
  if ((rc = rotquant_impl(x_bf16, CONVROT_DTYPE_BF16, M, K, group, x_q, s_x, st)) != CONVROT_OK)
    return rc;
  GemmArgs args{};
  args.s_a = s_x;
  args.s_b = w_scale;
  args.out = y_bf16;
  return launch_gemm<kEpiBf16, false>(x_q, w_q, 1, M, N, K, N, args, st);
}

int moe_workspace_layout(int64_t T, int64_t d, int64_t f, int E, int64_t C,
                         convrot_moe_layout_t* lay) {
  if (!lay || T < 0 || d < 0 || f < 0 || E < 0 || C < 0) return CONVROT_ERR_INVALID_ARG;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t ec = (size_t)E * (size_t)C;
  lay->x_q = take((size_t)T * d);
  lay->s_x = take((size_t)T * 4);
  lay->s_t = take((size_t)E * T * 4);
  lay->idx = take(ec * 4);
  lay->w = take(ec * 4);
  lay->x_g = take(ec * d);
  lay->s_g = take(ec * 4);
  lay->h = take(ec * f * 4);
  lay->h_q = take(ec * f);
  lay->s_h = take(ec * 4);
  lay->hsync = take(swiglu_rq_sync_bytes(E, C));
  lay->slot = take((size_t)E * T * 4);
  lay->z = take(ec * d * 2);
  lay->total = off;
  return CONVROT_OK;
}

size_t moe_workspace_size(int64_t T, int64_t d, int64_t f, int E, int64_t C) {
  convrot_moe_layout_t lay;
  if (moe_workspace_layout(T, d, f, E, C, &lay) != CONVROT_OK) return 0;
  return lay.total;
}

int moe_expert_choice_forward(const void* x_bf16, const void* logits_bf16, const int8_t* w_gu,
                              const float* s_gu, const int8_t* w_d, const float* s_d, int64_t T,
                              int64_t d, int64_t f, int E, int64_t C, int g_gu, int g_d,
                              void* y_bf16, void* workspace, size_t ws_bytes, void* stream) {
  if (T < 0 || T >= ((int64_t)1 << 31) || E < 1 || E > 256 || C < 0 || C > T)
    return CONVROT_ERR_INVALID_ARG;
  if (!valid_group(g_gu) || !valid_group(g_d)) return CONVROT_ERR_INVALID_ARG;
  if (d < 16 || d > 8192 || d % 16 != 0 || d % g_gu != 0) return CONVROT_ERR_INVALID_ARG;
  if (f < 16 || f > 8192 || f % 16 != 0 || f % g_d != 0) return CONVROT_ERR_INVALID_ARG;
  if ((int64_t)E * C >= ((int64_t)1 << 31)) return CONVROT_ERR_INVALID_ARG;
  if (T > 0 && (!x_bf16 || !logits_bf16 || !w_gu || !s_gu || !w_d || !s_d || !y_bf16 ||
                !workspace))
    return CONVROT_ERR_INVALID_ARG;
  if (!al16(x_bf16) || !al16(logits_bf16) || !al16(w_gu) || !al16(s_gu) || !al16(w_d) ||
      !al16(s_d) || !al16(y_bf16) || !al16(workspace))
    return CONVROT_ERR_MISALIGNED;
  convrot_moe_layout_t lay;
  moe_workspace_layout(T, d, f, E, C, &lay);
  if (ws_bytes < lay.total) return CONVROT_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  int rc = device_setup(&sms);
  if (rc != CONVROT_OK) return rc;
  if (T == 0) return CONVROT_OK;
  cudaStream_t st = as_stream(stream);
  char* ws = reinterpret_cast<char*>(workspace);
  int8_t* x_q = reinterpret_cast<int8_t*>(ws + lay.x_q);
  float* s_x = reinterpret_cast<float*>(ws + lay.s_x);
  float* s_t = reinterpret_cast<float*>(ws + lay.s_t);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + lay.idx);
  float* w = reinterpret_cast<float*>(ws + lay.w);
  int8_t* x_g = reinterpret_cast<int8_t*>(ws + lay.x_g);
  float* s_g = reinterpret_cast<float*>(ws + lay.s_g);
  float* h = reinterpret_cast<float*>(ws + lay.h);
  int8_t* h_q = reinterpret_cast<int8_t*>(ws + lay.h_q);
  float* s_h = reinterpret_cast<float*>(ws + lay.s_h);
  int32_t* slot = reinterpret_cast<int32_t*>(ws + lay.slot);
  void* z = ws + lay.z;

  // One stream, every kernel after the first launched with programmatic
  // stream serialization, in the order 1. softmax, 2. top-C, 3. x rotation,
  // 4. gather, ...: top-C waits for the softmax before reading its scores;
  // the x rotation reads only X, so it runs beside the routing from the start
  // and waits for top-C only before it exits (its completion implies top-C's);
  // the gather then waits for the rotation and has both its inputs.
  // 1. router softmax
  if ((rc = softmax_impl(logits_bf16, T, E, s_t, st)) != CONVROT_OK) return rc;
  // 2. expert-choice top-C (+ each token's slot per expert)
  if ((rc = topc_impl(s_t, T, E, C, idx, w, slot, st, true)) != CONVROT_OK) return rc;
  // 3. rotate + quantise the tokens once (the gate/up rotation is expert-independent);
  // a rotation longer than one round of resident CTAs runs on at most 1.5
  // CTAs per SM, which the top-C CTAs beside it leave room for (measured on
  // B200 at T=8192: -6 us against two CTAs per SM, whose last CTAs start
  // only as top-C ends)
  if ((rc = rotquant_impl(x_bf16, CONVROT_DTYPE_BF16, T, d, g_gu, x_q, s_x, st, RqOut{0, 1, 1, 1},
                          true, sms + sms / 2, true)) != CONVROT_OK)
    return rc;
  if (C > 0) {
    // h is rotated and requantised inside the gate/up GEMM's epilogue when its
    // groups fit one thread (g_d <= 64) and the device holds enough of the
    // GEMM's CTAs at once; otherwise h goes through HBM in fp32 and the
    // rotation kernel
    const bool fused_h = g_d <= 64 && swiglu_rq_fits(E, C, f, sms);
    char* hsync = ws + lay.hsync;
    // 4. gather each expert's token codes (and clear the fused epilogue's
    // synchronisation words)
    if ((rc = gather_impl(x_q, s_x, T, idx, (int64_t)E * C, d, x_g, s_g, st,
                          fused_h ? reinterpret_cast<uint32_t*>(hsync) : nullptr,
                          fused_h ? (int64_t)(swiglu_rq_sync_bytes(E, C) / 4) : 0, true)) !=
        CONVROT_OK)
      return rc;
    GemmArgs a1{};
    a1.s_a = s_g;
    a1.s_b = s_gu;
    GemmArgs a2{};  // the down projection to the experts' BF16 outputs
    a2.s_a = s_h;
    a2.s_b = s_d;
    a2.out = z;
    if (fused_h) {
      // 5 + 6. gate/up GEMM: dequant, SwiGLU, rotation (g_d) and requantisation;
      // each tile publishes its expert's h codes (done) for the down GEMM
      a1.out = h_q;
      a1.g_h = g_d;
      a1.s_h = s_h;
      a1.hmax = reinterpret_cast<unsigned*>(hsync);
      a1.rsync = reinterpret_cast<int*>(hsync + align256((size_t)E * (size_t)C * 4));
      a1.done = swiglu_rq_done_words(hsync, E, C);
      const bool pairs1 = C > gemm::BM && sms >= 2;  // as launch_gemm decides
      const int64_t mb1 = cdiv(C, pairs1 ? gemm2::BM : gemm::BM);
      const int64_t slabs1 = pairs1 ? 2 * mb1 : mb1;
      a2.done = a1.done;
      a2.done_target = (int)((pairs1 ? 2 : 1) * mb1 * cdiv(f, gemm::BN / 2));
      a2.done_abort = a1.rsync + E * slabs1;
      if ((rc = launch_gemm<kEpiSwigluRq, true>(x_g, w_gu, E, C, 2 * f, d, f, a1, st, true)) !=
          CONVROT_OK)
        return rc;
    } else {
      // 5. gate/up GEMM with dequant + SwiGLU
      a1.out = h;
      if ((rc = launch_gemm<kEpiSwiglu, true>(x_g, w_gu, E, C, 2 * f, d, f, a1, st, true)) !=
          CONVROT_OK)
        return rc;
      // 6. rotate (g_d) + requantise h per row
      if ((rc = rotquant_impl(h, CONVROT_DTYPE_F32, (int64_t)E * C, f, g_d, h_q, s_h, st,
                              RqOut{0, 1, 1, 1}, true)) != CONVROT_OK)
        return rc;
    }
    // 7. down GEMM; after the fused requantisation it is streamed: each
    // expert's tiles start once that expert's h codes are published, so the
    // down GEMM's CTAs take over SMs as the gate/up GEMM's CTAs leave instead
    // of after its last tile
    if ((rc = launch_gemm<kEpiBf16, true>(h_q, w_d, E, C, d, f, d, a2, st, true)) != CONVROT_OK)
      return rc;
  }
  // 8. per token: router-weighted fp32 sum over its experts in ascending
  // order, one bf16 rounding
  return combine_impl(z, s_t, slot, E, T, C, d, y_bf16, sms, st, C > 0);
}

// ---------------------------------------------------------------- low-bit --
int64_t convrot_lowbit_weight_bytes(int64_t rows, int64_t K, int bits) {
  if (!valid_bits(bits) || rows < 0 || K < 0 || rows % 128 != 0 || K % 64 != 0) return -1;
  return lowbit_bytes(rows, K, bits);
}

int convrot_quantize_weights_lowbit(const void* w_bf16, int64_t rows, int64_t K, int group,
                                    int bits, void* w_packed, float* row_scale, void* stream) {
  if (!valid_bits(bits) || !valid_group(group)) return CONVROT_ERR_INVALID_ARG;
  if (rows < 0 || rows >= ((int64_t)1 << 31) || rows % 128 != 0) return CONVROT_ERR_INVALID_ARG;
  if (K < 64 || K > 16384 || K % 64 != 0 || K % group != 0) return CONVROT_ERR_INVALID_ARG;
  if (rows > 0 && (!w_bf16 || !w_packed || !row_scale)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(w_bf16) || !al16(w_packed)) return CONVROT_ERR_MISALIGNED;
  int rc = device_setup(nullptr);
  if (rc != CONVROT_OK) return rc;
  if (rows == 0) return CONVROT_OK;
  cudaStream_t st = as_stream(stream);
  uint8_t* out = reinterpret_cast<uint8_t*>(w_packed);
  rc = bits == 4 ? lowbit_quant_group<4>(w_bf16, rows, (int)K, group, out, row_scale, st)
                 : lowbit_quant_group<6>(w_bf16, rows, (int)K, group, out, row_scale, st);
  if (rc != CONVROT_OK) return rc;
  return launch_status();
}

int convrot_lowbit_gemm(const int8_t* x_q, const float* s_x, const void* w_packed,
                        const float* row_scale, int64_t G, int64_t M, int64_t N, int64_t K,
                        int bits, int epilogue, int tile_tokens, void* out, void* stream) {
  int rc = check_lowbit_gemm(x_q, w_packed, G, M, N, K, bits, tile_tokens);
  if (rc != CONVROT_OK) return rc;
  if (epilogue < CONVROT_LOWBIT_F32 || epilogue > CONVROT_LOWBIT_SWIGLU)
    return CONVROT_ERR_INVALID_ARG;
  if (G * M > 0 && N > 0 && (!row_scale || !out || (epilogue != CONVROT_LOWBIT_F32 && !s_x)))
    return CONVROT_ERR_INVALID_ARG;
  if (!al16(out) || !al16(row_scale)) return CONVROT_ERR_MISALIGNED;
  cudaStream_t st = as_stream(stream);
  switch (epilogue) {
    case CONVROT_LOWBIT_F32:
      return launch_lowbit_bits<kLbF32>(bits, x_q, s_x, w_packed, row_scale, G, M, N, K,
                                        tile_tokens, out, st);
    case CONVROT_LOWBIT_BF16:
      return launch_lowbit_bits<kLbBf16>(bits, x_q, s_x, w_packed, row_scale, G, M, N, K,
                                         tile_tokens, out, st);
    default:
      return launch_lowbit_bits<kLbSwiglu>(bits, x_q, s_x, w_packed, row_scale, G, M, N, K,
                                           tile_tokens, out, st);
  }
}

int lowbit_convrot_linear(const void* x_bf16, int64_t M, int64_t K, const void* w_packed,
                          const float* row_scale, int64_t N, int group, int bits, void* y_bf16,
                          void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_rq_args(x_bf16, CONVROT_DTYPE_BF16, M, K, group, (const int8_t*)workspace,
                         (const float*)workspace);
  if (rc != CONVROT_OK) return rc;
  if ((rc = check_lowbit_gemm((const int8_t*)workspace, w_packed, 1, M, N, K, bits, 0)) !=
      CONVROT_OK)
    return rc;
  if (M > 0 && N > 0 && (!row_scale || !y_bf16 || !workspace)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(y_bf16) || !al16(workspace) || !al16(row_scale)) return CONVROT_ERR_MISALIGNED;
  if (ws_bytes < convrot_linear_workspace_size(M, K)) return CONVROT_ERR_WORKSPACE_TOO_SMALL;
  if ((rc = device_setup(nullptr)) != CONVROT_OK) return rc;
  if (M == 0 || N == 0) return CONVROT_OK;
  cudaStream_t st = as_stream(stream);
  int8_t* x_q = reinterpret_cast<int8_t*>(workspace);
  float* s_x = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                        align256((size_t)M * (size_t)K));
  if ((rc = rotquant_impl(x_bf16, CONVROT_DTYPE_BF16, M, K, group, x_q, s_x, st)) != CONVROT_OK)
    return rc;
  return launch_lowbit_bits<kLbBf16>(bits, x_q, s_x, w_packed, row_scale, 1, M, N, K, 0, y_bf16,
                                     st, true);
}

int moe_expert_choice_forward_lowbit(const void* x_bf16, const void* logits_bf16,
                                     const void* w_gu, const float* s_gu, const void* w_d,
                                     const float* s_d, int64_t T, int64_t d, int64_t f, int E,
                                     int64_t C, int g_gu, int g_d, int bits, void* y_bf16,
                                     void* workspace, size_t ws_bytes, void* stream) {
  if (!valid_bits(bits)) return CONVROT_ERR_INVALID_ARG;
  if (T < 0 || T >= ((int64_t)1 << 31) || E < 1 || E > 256 || C < 0 || C > T)
    return CONVROT_ERR_INVALID_ARG;
  if (!valid_group(g_gu) || !valid_group(g_d)) return CONVROT_ERR_INVALID_ARG;
  if (d < 256 || d > 8192 || d % 256 != 0 || d % g_gu != 0) return CONVROT_ERR_INVALID_ARG;
  if (f < 128 || f > 8192 || f % 128 != 0 || f % g_d != 0) return CONVROT_ERR_INVALID_ARG;
  if ((int64_t)E * C >= ((int64_t)1 << 31)) return CONVROT_ERR_INVALID_ARG;
  if (T > 0 && (!x_bf16 || !logits_bf16 || !w_gu || !s_gu || !w_d || !s_d || !y_bf16 ||
                !workspace))
    return CONVROT_ERR_INVALID_ARG;
  if (!al16(x_bf16) || !al16(logits_bf16) || !al16(w_gu) || !al16(s_gu) || !al16(w_d) ||
      !al16(s_d) || !al16(y_bf16) || !al16(workspace))
    return CONVROT_ERR_MISALIGNED;
  convrot_moe_layout_t lay;
  moe_workspace_layout(T, d, f, E, C, &lay);
  if (ws_bytes < lay.total) return CONVROT_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  int rc = device_setup(&sms);
  if (rc != CONVROT_OK) return rc;
  if (T == 0) return CONVROT_OK;
  cudaStream_t st = as_stream(stream);
  char* ws = reinterpret_cast<char*>(workspace);
  int8_t* x_q = reinterpret_cast<int8_t*>(ws + lay.x_q);
  float* s_x = reinterpret_cast<float*>(ws + lay.s_x);
  float* s_t = reinterpret_cast<float*>(ws + lay.s_t);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + lay.idx);
  float* w = reinterpret_cast<float*>(ws + lay.w);
  int8_t* x_g = reinterpret_cast<int8_t*>(ws + lay.x_g);
  float* s_g = reinterpret_cast<float*>(ws + lay.s_g);
  float* h = reinterpret_cast<float*>(ws + lay.h);
  int8_t* h_q = reinterpret_cast<int8_t*>(ws + lay.h_q);
  float* s_h = reinterpret_cast<float*>(ws + lay.s_h);
  int32_t* slot = reinterpret_cast<int32_t*>(ws + lay.slot);
  void* z = ws + lay.z;
  // the int8 block's schedule (see moe_expert_choice_forward) with the
  // low-bit GEMMs and h through HBM in fp32 and the rotation kernel
  if ((rc = softmax_impl(logits_bf16, T, E, s_t, st)) != CONVROT_OK) return rc;
  if ((rc = topc_impl(s_t, T, E, C, idx, w, slot, st, true)) != CONVROT_OK) return rc;
  if ((rc = rotquant_impl(x_bf16, CONVROT_DTYPE_BF16, T, d, g_gu, x_q, s_x, st, RqOut{0, 1, 1, 1},
                          true, sms + sms / 2, true)) != CONVROT_OK)
    return rc;
  if (C > 0) {
    if ((rc = gather_impl(x_q, s_x, T, idx, (int64_t)E * C, d, x_g, s_g, st, nullptr, 0, true)) !=
        CONVROT_OK)
      return rc;
    if ((rc = launch_lowbit_bits<kLbSwiglu>(bits, x_g, s_g, w_gu, s_gu, E, C, 2 * f, d, 0, h, st,
                                            true)) != CONVROT_OK)
      return rc;
    if ((rc = rotquant_impl(h, CONVROT_DTYPE_F32, (int64_t)E * C, f, g_d, h_q, s_h, st,
                            RqOut{0, 1, 1, 1}, true)) != CONVROT_OK)
      return rc;
    if ((rc = launch_lowbit_bits<kLbBf16>(bits, h_q, s_h, w_d, s_d, E, C, d, f, 0, z, st, true)) !=
        CONVROT_OK)
      return rc;
  }
  return combine_impl(z, s_t, slot, E, T, C, d, y_bf16, sms, st, C > 0);
}

}  // extern "C"

// ======================================================= no-allocation ==
// Scratch of w8a8_convrot_linear_noalloc: activation codes then token scales,
// one file-scope device array reserved on every GPU that loads the library.
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[CONVROT_NOALLOC_MAX_CODES + CONVROT_NOALLOC_MAX_ROWS * sizeof(float)];

namespace {

struct NoAllocSlot {
  bool ready = false;
  void* ptr = nullptr;
};
NoAllocSlot g_noalloc_slot[kMaxDevices];
std::mutex g_noalloc_mu;

// Whether p is device (or managed) memory that the current device can use as
// its own: allocated on it, or managed.
bool on_current_device(const void* p) {
  int dev = 0;
  cudaPointerAttributes at;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (at.type == cudaMemoryTypeManaged) return true;
  return at.type == cudaMemoryTypeDevice && at.device == dev;
}

// Device address of the scratch array for the current device, looked up once
// per device (host code cannot use the array's name as a device pointer).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return CONVROT_ERR_UNSUPPORTED_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocSlot& slot = g_noalloc_slot[dev];
  if (!slot.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return CONVROT_ERR_CUDA;
    }
    slot.ptr = p;
    slot.ready = true;
  }
  *out = slot.ptr;
  return CONVROT_OK;
}

}  // namespace

extern "C" int w8a8_convrot_linear_noalloc(const void* x_bf16, int64_t M, int64_t K,
                                           const int8_t* w_q, const float* w_scale, int64_t N,
                                           int group, void* y_bf16, void* stream) {
  int rc = check_rq_args(x_bf16, CONVROT_DTYPE_BF16, M, K, group, w_q, w_scale);
  if (rc != CONVROT_OK) return rc;
  if ((rc = check_gemm_shape(w_q, w_q, 1, M, N, K)) != CONVROT_OK) return rc;
  if (M > 0 && N > 0 && (!w_scale || !y_bf16)) return CONVROT_ERR_INVALID_ARG;
  if (!al16(w_scale) || !al16(y_bf16)) return CONVROT_ERR_MISALIGNED;
  // K <= 16384 and M < 2^31 hold here, so M * K cannot overflow
  if (M > CONVROT_NOALLOC_MAX_ROWS || M * K > (int64_t)CONVROT_NOALLOC_MAX_CODES)
    return CONVROT_ERR_WORKSPACE_TOO_SMALL;
  if ((rc = device_setup(nullptr)) != CONVROT_OK) return rc;
  // the scratch is the current device's: the caller's buffers must be there too
  if (M > 0 && N > 0 && (!on_current_device(x_bf16) || !on_current_device(y_bf16)))
    return CONVROT_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch)) != CONVROT_OK) return rc;
  if (M == 0 || N == 0) return CONVROT_OK;
  cudaStream_t st = as_stream(stream);
  int8_t* x_q = reinterpret_cast<int8_t*>(scratch);
  float* s_x = reinterpret_cast<float*>(reinterpret_cast<char*>(scratch) + CONVROT_NOALLOC_MAX_CODES);
  if ((rc = rotquant_impl(x_bf16, CONVROT_DTYPE_BF16, M, K, group, x_q, s_x, st)) != CONVROT_OK)
    return rc;
  GemmArgs args{};
  args.s_a = s_x;
  args.s_b = w_scale;
  args.out = y_bf16;
  return launch_gemm<kEpiBf16, false>(x_q, w_q, 1, M, N, K, N, args, st);
}
