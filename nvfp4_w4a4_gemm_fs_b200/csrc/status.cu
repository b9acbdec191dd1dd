// Status strings, per-thread last-error detail and small ABI helpers.
#include "common.cuh"

namespace fs {

static thread_local std::string g_last_error;

void set_last_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

fs_status fail(fs_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

fs_status cuda_status(cudaError_t e, const char* what) {
  return fail(FS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

int sm_count() {
  static PerDevice<int> cache;
  int n = 0;
  const int dev = current_device();
  if (cache.get(dev, &n, [dev](int* v) {
        return cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && *v > 0;
      }))
    return n;
  return 148;
}

fs_status set_max_dynamic_smem(PerDevice<int>& cache, const void* kernel, int bytes, const char* who) {
  int done = 0;
  cudaError_t err = cudaSuccess;
  if (cache.get(current_device(), &done, [&](int* v) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        *v = 1;
        return err == cudaSuccess;
      }))
    return FS_OK;
  if (err != cudaSuccess) return cuda_status(err, who);
  return fail(FS_ERR_CUDA, "%s: no current device", who);
}

}  // namespace fs

extern "C" {

const char* fs_status_string(fs_status s) {
  switch (s) {
    case FS_OK: return "FS_OK";
    case FS_ERR_INVALID_ARGUMENT: return "FS_ERR_INVALID_ARGUMENT";
    case FS_ERR_UNSUPPORTED: return "FS_ERR_UNSUPPORTED";
    case FS_ERR_CUDA: return "FS_ERR_CUDA";
    case FS_ERR_RANGE: return "FS_ERR_RANGE";
    case FS_ERR_TIMEOUT: return "FS_ERR_TIMEOUT";
  }
  return "FS_ERR_UNKNOWN";
}

const char* fs_last_error(void) { return fs::g_last_error.c_str(); }

const char* fs_version(void) { return "foursight-splicegemm 0.1 (sm_100a)"; }

int32_t fs_side_cols(int32_t p) { return p < 0 ? 0 : fs::side_cols(p); }

int32_t fs_compact_cols(int32_t K, int32_t p) {
  return (K < 0 || p < 0 || p > K) ? 0 : static_cast<int32_t>(fs::round_up(K - p, 256));
}

int64_t fs_sf_bytes(int64_t R, int32_t K) { return (R < 0 || K < 0) ? 0 : fs::sf_bytes(R, K); }

int64_t fs_grouped_rows(int64_t max_rows, int32_t E) {
  return (max_rows < 0 || E < 0) ? 0 : fs::round_up(max_rows, 128) + 128 * static_cast<int64_t>(E);
}

}  // extern "C"
