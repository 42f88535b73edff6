// host_util.cuh - host-side helpers shared by the C ABI translation units:
// the tensor-map encoder (driver entry point fetched through the runtime, so
// the library links no libcuda), alignment checks, the current device and
// its SM count, and the one-time per-device kernel set-up.  Host code only.
#pragma once

#include <atomic>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "gdla.h"

namespace gdla_host {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Resolved once; immutable afterwards (C++11 guarantees thread-safe init).
inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Devices whose ordinal fits the 64-bit masks below get their one-time
// kernel set-up and attribute queries cached; others redo them per call.
constexpr int kCachedDevices = 64;

inline int current_device(int *dev) {
  return cudaGetDevice(dev) == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}

// Number of SMs of the current device (queried once per device).
inline int sm_count(int *sms) {
  static std::atomic<int> cache[kCachedDevices];
  int dev = 0;
  if (current_device(&dev) != GDLA_OK) return GDLA_ERR_CUDA;
  if (dev >= 0 && dev < kCachedDevices) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) {
      *sms = c;
      return GDLA_OK;
    }
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return GDLA_ERR_CUDA;
  if (dev >= 0 && dev < kCachedDevices) cache[dev].store(n, std::memory_order_relaxed);
  *sms = n;
  return GDLA_OK;
}

// One-time set-up of kernel `Kern` on the current device: its dynamic
// shared-memory limit and, when `want_regs` > 0, the check that the build
// uses exactly that many registers per thread (kernels that re-split their
// register pool with setmaxnreg are only sound for the count they were
// written for).  Both are properties of the device context and the binary,
// so they are done once per device; two threads racing here only repeat
// idempotent work.
template <auto Kern>
inline int prepare_kernel(uint32_t smem, int want_regs) {
  static std::atomic<uint64_t> ready{0};
  int dev = 0;
  if (current_device(&dev) != GDLA_OK) return GDLA_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < kCachedDevices) ? (1ull << dev) : 0ull;
  if (bit && (ready.load(std::memory_order_acquire) & bit)) return GDLA_OK;
  if (cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return GDLA_ERR_CUDA;
  if (want_regs > 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, Kern) != cudaSuccess) return GDLA_ERR_CUDA;
    if (fa.numRegs != want_regs) return GDLA_ERR_UNSUPPORTED;
  }
  if (bit) ready.fetch_or(bit, std::memory_order_release);
  return GDLA_OK;
}

// Row-major bf16 tensor of `rank` dims given innermost-first; box innermost-first.
inline bool make_map(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
              const uint32_t *box) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  cuuint64_t gdim[5];
  cuuint64_t gstride[4];
  cuuint32_t bdim[5];
  cuuint32_t estride[5];
  uint64_t stride = 2;  // bytes
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
    if (i > 0) gstride[i - 1] = stride;
    stride *= dims[i];
  }
  const CUresult r =
      fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
         const_cast<void *>(base), gdim, gstride, bdim, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace gdla_host
