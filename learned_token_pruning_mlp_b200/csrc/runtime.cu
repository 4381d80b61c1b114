// runtime.cu -- host-side plumbing of the TokenGate C ABI: status strings, the
// per-thread error detail, the per-device status word the kernels report
// device-side conditions into, SM counts and TMA descriptor encoding.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "ptx.cuh"
#include "runtime.h"

// Sticky per-device status word (bits TG_DEVERR_*).  Kernels receive its address.
__device__ uint32_t g_tg_status_word;

namespace tg {

namespace {
thread_local char t_detail[512];

std::mutex g_mu;
uint32_t *g_word_addr[kMaxDevices];
int g_sms[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}
}  // namespace

void clear_detail() { t_detail[0] = 0; }

std::mutex &setup_mutex() {
  static std::mutex mu;
  return mu;
}

tg_status fail(tg_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_detail, sizeof t_detail, fmt, ap);
  va_end(ap);
  return st;
}

uint32_t *device_error_word() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) {
    fail(TG_ERR_CUDA, "no current CUDA device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_word_addr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_tg_status_word);
    if (e != cudaSuccess) {
      fail(TG_ERR_CUDA, "cudaGetSymbolAddress(status word): %s", cudaGetErrorString(e));
      return nullptr;
    }
    g_word_addr[dev] = static_cast<uint32_t *>(p);
  }
  return g_word_addr[dev];
}

int sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

tg_status check_launch(const char *what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return TG_OK;
}

bool encode_tmap(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base, const uint64_t *dims,
                 const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swizzle) {
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_encode) {
      void *fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
        fail(TG_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
        return false;
      }
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
  }
  cuuint64_t d[5];
  cuuint64_t s[4];
  cuuint32_t b[5];
  cuuint32_t es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) s[i] = strides_bytes[i];
  }
  const CUresult r = g_encode(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void *>(base), d, s, b, es,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(TG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return false;
  }
  return true;
}

}  // namespace tg

// A kernel that waits on an mbarrier nothing ever arrives on, with a caller-chosen
// limit, so that the bounded-wait path can be exercised without hanging a GPU.
__global__ void tg_wait_probe_kernel(uint64_t limit_ns, uint32_t *err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    tg::mbar_init(tg::smem_addr(&bar), 1);
    tg::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!tg::mbar_wait(tg::smem_addr(&bar), 0, &abort_flag, limit_ns)) tg::set_device_error(err, TG_DEVERR_TIMEOUT);
    // release the barrier so the CTA leaves nothing pending
    tg::mbar_arrive(tg::smem_addr(&bar));
  }
}

extern "C" {

int tg_abi_version(void) { return TG_ABI_VERSION; }

const char *tg_status_string(tg_status st) {
  switch (st) {
    case TG_OK: return "TG_OK";
    case TG_ERR_INVALID_ARG: return "TG_ERR_INVALID_ARG";
    case TG_ERR_UNSUPPORTED: return "TG_ERR_UNSUPPORTED";
    case TG_ERR_ALIGNMENT: return "TG_ERR_ALIGNMENT";
    case TG_ERR_CUDA: return "TG_ERR_CUDA";
  }
  return "TG_ERR_UNKNOWN";
}

const char *tg_last_error_detail(void) { return tg::t_detail; }

tg_status tg_get_device_error(tg_stream stream, uint32_t *bits) {
  TG_API_ENTRY();
  if (!bits) return tg::fail(TG_ERR_INVALID_ARG, "bits is NULL");
  *bits = 0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, g_tg_status_word, sizeof v);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "reading status word: %s", cudaGetErrorString(e));
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbol(g_tg_status_word, &zero, sizeof zero);
  if (e != cudaSuccess) return tg::fail(TG_ERR_CUDA, "clearing status word: %s", cudaGetErrorString(e));
  *bits = v;
  return TG_OK;
}

tg_status tg_probe_wait_timeout(int64_t limit_ns, tg_stream stream) {
  TG_API_ENTRY();
  if (limit_ns <= 0 || limit_ns > 2000000000LL)
    return tg::fail(TG_ERR_INVALID_ARG, "limit_ns must be in (0, 2e9]");
  uint32_t *err = tg::device_error_word();
  if (!err) return TG_ERR_CUDA;
  tg_wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_ns), err);
  return tg::check_launch("tg_wait_probe_kernel");
}

}  // extern "C"
