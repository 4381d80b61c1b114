// runtime.h -- host-side helpers shared by the TokenGate launchers: error detail,
// the per-device status word, SM count and TMA tensor-map encoding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "tokengate.h"

namespace tg {

constexpr int kMaxDevices = 64;

// Record a printf-style detail for tg_last_error_detail() and return ``st``.
tg_status fail(tg_status st, const char *fmt, ...);

// Clear the calling thread's detail (start of every API call).
void clear_detail();

// An NVTX range around one C-ABI call on the calling host thread (visible in a
// timeline profiler; a no-op when no tool is attached).
struct ApiRange {
  explicit ApiRange(const char *name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
  ApiRange(const ApiRange &) = delete;
  ApiRange &operator=(const ApiRange &) = delete;
};

// First statement of every C-ABI entry point: clears the thread's error detail and
// opens the call's NVTX range (closed when the call returns).
#define TG_API_ENTRY()   \
  ::tg::clear_detail(); \
  const ::tg::ApiRange tg_api_range_(__func__)

// Per-device one-time set-up (kernel attributes, symbol addresses) that host threads
// may reach concurrently.  The first caller on a device runs ``setup(dev)`` under a
// library-wide lock and publishes the flag; later callers only read it.  A set-up
// that fails is not published, so the next call runs it again.
struct PerDevice {
  std::atomic<bool> done[kMaxDevices];
};
std::mutex &setup_mutex();

// ``device`` (optional) receives the current device's ordinal.
template <typename F>
tg_status once_per_device(PerDevice &flags, F &&setup, int *device = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fail(TG_ERR_CUDA, "no current CUDA device (or device ordinal >= %d)", kMaxDevices);
  if (device) *device = dev;
  if (flags.done[dev].load(std::memory_order_acquire)) return TG_OK;
  std::lock_guard<std::mutex> lock(setup_mutex());
  if (flags.done[dev].load(std::memory_order_relaxed)) return TG_OK;
  const tg_status st = setup(dev);
  if (st == TG_OK) flags.done[dev].store(true, std::memory_order_release);
  return st;
}

// Device address of the current device's status word (the kernels OR bits into it).
// Returns nullptr (and records a detail) if the address cannot be obtained.
uint32_t *device_error_word();

// Number of SMs of the current device (cached per device).
int sm_count();

// Map a pending CUDA error after a launch to TG_ERR_CUDA.
tg_status check_launch(const char *what);

// Encode a tiled TMA descriptor; strides_bytes has rank-1 entries (dimension 0 is dense).
// Returns false (with a detail recorded) on failure.
bool encode_tmap(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base,
                 const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                 CUtensorMapSwizzle swizzle);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch with programmatic stream serialization: the kernel may begin while the
// previous kernel on the stream drains; it must call pdl_wait() before touching
// global memory.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace tg
