// Per-device status word, wait limit, status strings and size helpers.
#include <mutex>

#include "common.cuh"

namespace fp4 {

// One word per device (each device that loads the library gets its own copy
// of this module variable).  Kernels record the first device-side error here.
static __device__ unsigned int g_status_word;

static std::mutex g_mu;
static DeviceCtx g_ctx[64];
static bool g_init[64];
static uint64_t g_wait_limit_override = 0;

const DeviceCtx *device_ctx() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_init[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_ctx[dev].status = static_cast<unsigned int *>(p);
    g_init[dev] = true;
  }
  g_ctx[dev].wait_limit_ns = g_wait_limit_override ? g_wait_limit_override : 2000000000ull;
  return &g_ctx[dev];
}

}  // namespace fp4

extern "C" {

const char *fp4_status_string(fp4_status s) {
  switch (s) {
    case FP4_OK: return "FP4_OK";
    case FP4_ERR_INVALID_ARG: return "FP4_ERR_INVALID_ARG";
    case FP4_ERR_ALIGNMENT: return "FP4_ERR_ALIGNMENT";
    case FP4_ERR_UNSUPPORTED_SHAPE: return "FP4_ERR_UNSUPPORTED_SHAPE";
    case FP4_ERR_RANGE: return "FP4_ERR_RANGE";
    case FP4_ERR_BAD_EXPERT: return "FP4_ERR_BAD_EXPERT";
    case FP4_ERR_WORKSPACE: return "FP4_ERR_WORKSPACE";
    case FP4_ERR_DEVICE_TIMEOUT: return "FP4_ERR_DEVICE_TIMEOUT";
    case FP4_ERR_CUDA: return "FP4_ERR_CUDA";
  }
  return "FP4_ERR_UNKNOWN";
}

size_t fp4_sf_tiled_bytes(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0 || cols % 64) return 0;
  return (size_t)(((rows + 127) / 128) * 128) * (size_t)(cols / 16);
}

size_t fp4_quantize_workspace_size(void) { return 256; }

fp4_status fp4_get_device_status(fp4_stream_t stream) {
  const fp4::DeviceCtx *ctx = fp4::device_ctx();
  if (!ctx) return FP4_ERR_CUDA;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FP4_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, ctx->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return FP4_ERR_CUDA;
  unsigned int zero = 0;
  if (cudaMemcpy(ctx->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return FP4_ERR_CUDA;
  return static_cast<fp4_status>(v);
}

void fp4_set_wait_limit_ns(uint64_t ns) {
  std::lock_guard<std::mutex> lk(fp4::g_mu);
  fp4::g_wait_limit_override = ns;
}

}  // extern "C"
