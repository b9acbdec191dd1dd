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

int64_t fs_sf_bytes(int64_t R, int32_t K) { return (R < 0 || K < 0) ? 0 : fs::sf_bytes(R, K); }

int64_t fs_grouped_rows(int64_t max_rows, int32_t E) {
  return (max_rows < 0 || E < 0) ? 0 : fs::round_up(max_rows, 128) + 128 * static_cast<int64_t>(E);
}

}  // extern "C"
