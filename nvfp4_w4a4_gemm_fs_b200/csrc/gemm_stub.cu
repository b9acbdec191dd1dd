// Placeholder GEMM entry points (replaced by the tensor-core and decode kernels).
#include "common.cuh"
using namespace fs;
struct fs_plan_s { int N, K, p_max; uint32_t opts; uint32_t* err; };
extern "C" fs_status fs_plan_create(fs_plan* out, int32_t N, int32_t K, int32_t p_max, uint32_t opts) { return fail(FS_ERR_UNSUPPORTED, "not built"); }
extern "C" fs_status fs_plan_destroy(fs_plan plan) { return FS_OK; }
extern "C" fs_status fs_plan_check(fs_plan plan, void* stream) { return FS_OK; }
extern "C" fs_status fs_splice_gemm(fs_plan plan, int64_t M, int32_t p, const uint8_t* xq, const uint8_t* sfx, const uint16_t* xs, const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws, const float* alpha, void* Y, int64_t ldy, void* stream) { return fail(FS_ERR_UNSUPPORTED, "not built"); }
extern "C" fs_status fs_splice_gemm_grouped(fs_plan plan, int32_t E, const int64_t* row_offsets, int64_t max_rows, int32_t p, const uint8_t* xq, const uint8_t* sfx, const uint16_t* xs, const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws, const float* alpha, void* Y, int64_t ldy, void* stream) { return fail(FS_ERR_UNSUPPORTED, "not built"); }
