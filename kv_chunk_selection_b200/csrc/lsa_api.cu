// Library-wide entry points of liblsa: status strings, version, the device
// status word, and the per-device facts the launchers need.
#include <mutex>

#include "lsa_common.cuh"
#include "lsa_runtime.cuh"

// One status word per device context.  Kernels OR LSA_DEV_ERR_* bits into it.
__device__ unsigned g_lsa_device_status;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
lsa::EncodeTiledFn g_encode = nullptr;
bool g_encode_tried = false;

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return (dev >= 0 && dev < kMaxDevices) ? dev : -1;
}
}  // namespace

unsigned* lsa_device_status_ptr() {
  const int dev = current_device();
  if (dev < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lsa_device_status) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_status_ptr[dev] = static_cast<unsigned*>(p);
  }
  return g_status_ptr[dev];
}

namespace lsa {

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return -1;
    }
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

EncodeTiledFn tensor_map_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode_tried) {
    g_encode_tried = true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    } else {
      cudaGetLastError();
    }
  }
  return g_encode;
}

}  // namespace lsa

namespace {
// Self-test of the bounded waits every kernel relies on: mode 0 waits on an
// mbarrier that nothing will complete, mode 1 on a device flag (complete when
// the caller has set it).  A wait that runs out sets LSA_DEV_ERR_TIMEOUT and
// the kernel returns normally, leaving the context usable.
__global__ void selftest_wait_kernel(int mode, const int* flag, unsigned long long limit_ns, unsigned* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    lsa::mbar_init(&bar, 1);
    abort_flag = 0;
    lsa::mbar_fence_init();
  }
  __syncthreads();
  bool ok;
  if (mode == 0) ok = lsa::mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns);
  else ok = lsa::flag_wait_bounded(flag, limit_ns);
  if (!ok && threadIdx.x == 0) lsa::set_status(status, LSA_DEV_ERR_TIMEOUT);
}
}  // namespace

extern "C" {

int lsa_selftest_bounded_wait(int mode, const int* flag, unsigned int limit_us, void* stream) {
  if (mode != 0 && mode != 1) return LSA_ERR_INVALID_ARG;
  if (mode == 1 && !flag) return LSA_ERR_INVALID_ARG;
  if (limit_us == 0 || limit_us > 2000000u) return LSA_ERR_INVALID_ARG;
  if (lsa::device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      mode, flag, static_cast<unsigned long long>(limit_us) * 1000ull, lsa_device_status_ptr());
  return lsa::launch_status();
}

const char* lsa_status_string(int status) {
  switch (status) {
    case LSA_OK: return "LSA_OK";
    case LSA_ERR_INVALID_ARG: return "LSA_ERR_INVALID_ARG";
    case LSA_ERR_UNSUPPORTED_SHAPE: return "LSA_ERR_UNSUPPORTED_SHAPE";
    case LSA_ERR_WORKSPACE: return "LSA_ERR_WORKSPACE";
    case LSA_ERR_CUDA: return "LSA_ERR_CUDA";
    case LSA_ERR_NOT_PINNED: return "LSA_ERR_NOT_PINNED";
    case LSA_ERR_MISALIGNED: return "LSA_ERR_MISALIGNED";
    case LSA_ERR_NO_DEVICE: return "LSA_ERR_NO_DEVICE";
    default: return "LSA_ERR_UNKNOWN";
  }
}

int lsa_version(void) { return 100; }

int lsa_read_device_status(void* stream, unsigned int* bits) {
  if (!bits) return LSA_ERR_INVALID_ARG;
  unsigned* d = lsa_device_status_ptr();
  if (!d) return LSA_ERR_NO_DEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned h = 0;
  if (cudaMemcpyAsync(&h, d, sizeof(unsigned), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess || cudaMemsetAsync(d, 0, sizeof(unsigned), s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  *bits = h;
  return LSA_OK;
}

}  // extern "C"
