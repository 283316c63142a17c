// seedlm_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/seedlm.h"

// Bounds-checked build (-DSEEDLM_CHECK=1, `python -m
// prng_seeded_decompress_b200.build --check`): every memory index a kernel
// computes is compared with the extent its arguments (or its shared-memory
// layout) define before the access; a violation sets the kernel file's check
// flag, which seedlm_device_error reports, and the access is skipped.  In
// normal builds the checks compile to nothing.
#ifndef SEEDLM_CHECK
#define SEEDLM_CHECK 0
#endif
#if SEEDLM_CHECK
#define SEEDLM_IN_BOUNDS(flag, idx, extent)                                              \
  (((unsigned long long)(idx) < (unsigned long long)(extent)) ? true                     \
                                                              : (atomicOr(&(flag), 1u), false))
// One check flag per kernel file, with a host reader that clears it.
#define SEEDLM_CHECK_FLAG(name)                                                          \
  namespace {                                                                            \
  __device__ unsigned int g_check_flag;                                                  \
  }                                                                                      \
  int read_and_clear_check_##name(unsigned int* out) {                                   \
    unsigned int v = 0, zero = 0;                                                        \
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_check_flag, sizeof(v));                 \
    if (err == cudaSuccess && v) err = cudaMemcpyToSymbol(g_check_flag, &zero, sizeof(zero)); \
    *out = v;                                                                            \
    return record_cuda_error(err);                                                       \
  }
// Code that only the checked build compiles (extents computed for the checks).
#define SEEDLM_CHECK_ONLY(...) __VA_ARGS__
// Bytes of dynamic shared memory the running kernel was launched with.
__device__ __forceinline__ unsigned int seedlm_dynamic_smem_bytes() {
  unsigned int r;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}
#else
#define SEEDLM_IN_BOUNDS(flag, idx, extent) true
#define SEEDLM_CHECK_ONLY(...)
#define SEEDLM_CHECK_FLAG(name)                                                          \
  int read_and_clear_check_##name(unsigned int* out) {                                   \
    *out = 0;                                                                            \
    return 0;                                                                            \
  }
#endif

namespace seedlm {

int read_and_clear_check_gemv(unsigned int* out);
int read_and_clear_check_decompress(unsigned int* out);
int read_and_clear_check_gemm_tc(unsigned int* out);
int read_and_clear_check_encode(unsigned int* out);
int read_and_clear_check_dense(unsigned int* out);
int read_and_clear_check_gemm_cc(unsigned int* out);
int read_and_clear_check_gemv_amort(unsigned int* out);

struct DeviceInfo {
  int device;
  int num_sms;
  int max_smem_optin;  // bytes of dynamic shared memory a block may opt into
  int cc_major, cc_minor;
};

// Properties of the current device (cached per device); SEEDLM_OK or an error.
int current_device_info(DeviceInfo* out);

// Argument checks shared by every entry point: p is a multiple of a bytes;
// the format is one the kernels support and self-consistent (SEEDLM_OK,
// SEEDLM_EINVAL or SEEDLM_EUNSUPPORTED); the record (and, for (12,4),
// exponent) planes are present and aligned when the matrix is not empty.
bool aligned(const void* p, uintptr_t a);
int check_format(const seedlm_format* f);
int check_planes(const seedlm_format* f, const uint32_t* rec, const uint8_t* eplane);

// Records err as this thread's last CUDA error; SEEDLM_OK or SEEDLM_ECUDA.
int record_cuda_error(cudaError_t err);
// Counts one kernel launch (process-wide).
void count_launch();
// Lets `kernel` use all the dynamic shared memory the device allows; done once
// per kernel and device, outside any stream capture the caller may start later.
int allow_max_smem(const void* kernel, const DeviceInfo& dev);

// Shared memory the GEMV kernel needs for f on dev (0: its tables do not fit).
size_t gemv_smem_bytes(const seedlm_format& f, const DeviceInfo& dev);
int read_and_clear_gemv_error(unsigned int* out);
// Tall 3-bit matrices (at least 128 rows per SM, at most 256): the GEMV with
// the x-dependent part of every block's dot taken from per-column-block
// tables (gemv_amort.cu).
bool gemv_amort_applies(const seedlm_format& f, const DeviceInfo& dev);
int launch_gemv_amort(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                      const uint16_t* x, int is_bf16, float* y, cudaStream_t stream,
                      const DeviceInfo& dev);
int read_and_clear_amort_error(unsigned int* out);
int launch_gemv(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                const uint16_t* x, int is_bf16, float* y, cudaStream_t stream,
                const DeviceInfo& dev);
// n (<= 8) GEMVs of one format (same C) in one launch; every entry non-empty.
int launch_gemv_batch(int n, const seedlm_format* const* f, const uint32_t* const* rec,
                      const uint8_t* const* eplane, const uint16_t* const* x, int is_bf16,
                      float* const* y, cudaStream_t stream, const DeviceInfo& dev);
int launch_decompress(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                      float* W, int64_t ldw, cudaStream_t stream, const DeviceInfo& dev);
int launch_dense_gemv_f16(int rows, int cols, const uint16_t* W, int64_t ldw, const uint16_t* x,
                          float* y, cudaStream_t stream, const DeviceInfo& dev);
// Largest batch of one tensor-core GEMM pass (the MMA's largest N); more
// rows are run as consecutive passes.
constexpr int kGemmPassRows = 256;
int64_t gemm_tc_workspace_bytes(const seedlm_format& f, int M, const DeviceInfo& dev);
int launch_gemm_tc(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                   const uint16_t* X, int is_bf16, int M, float* Y, void* workspace,
                   int64_t workspace_bytes, cudaStream_t stream, const DeviceInfo& dev);
int read_and_clear_tc_error(unsigned int* out);
// 2 <= M <= kGemmCcMaxRows rows of X run on the CUDA cores (gemm_cc.cu): the
// rebuilt weights feed M packed FMAs each, with no workspace.
constexpr int kGemmCcMaxRows = 4;
bool gemm_cc_applies(const seedlm_format& f, int M);
int launch_gemm_cc(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                   const uint16_t* X, int is_bf16, int M, float* Y, cudaStream_t stream,
                   const DeviceInfo& dev);
int read_and_clear_cc_error(unsigned int* out);
int read_and_clear_encode_error(unsigned int* out);
int launch_wait_timeout(uint64_t limit_ns, cudaStream_t stream);
int launch_bounds_check(int64_t index, int64_t extent, cudaStream_t stream);
int launch_encode(const seedlm_format& f, const float* W, int64_t ldw, uint32_t* rec,
                  uint8_t* eplane, double* err, cudaStream_t stream, const DeviceInfo& dev);

}  // namespace seedlm
