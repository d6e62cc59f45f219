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

extern "C" {

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
