// seedlm_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/seedlm.h"

namespace seedlm {

struct DeviceInfo {
  int device;
  int num_sms;
  int max_smem_optin;  // bytes of dynamic shared memory a block may opt into
  int cc_major, cc_minor;
};

// Properties of the current device (cached per device); SEEDLM_OK or an error.
int current_device_info(DeviceInfo* out);

// Records err as this thread's last CUDA error; SEEDLM_OK or SEEDLM_ECUDA.
int record_cuda_error(cudaError_t err);
// Counts one kernel launch (process-wide).
void count_launch();
// Lets `kernel` use all the dynamic shared memory the device allows; done once
// per kernel and device, outside any stream capture the caller may start later.
int allow_max_smem(const void* kernel, const DeviceInfo& dev);

// Shared memory the GEMV needs for f within max_smem bytes (0: x does not fit).
size_t gemv_smem_bytes(const seedlm_format& f, int max_smem);
int launch_gemv(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                const uint16_t* x, int is_bf16, float* y, cudaStream_t stream,
                const DeviceInfo& dev);
int launch_decompress(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                      float* W, int64_t ldw, cudaStream_t stream, const DeviceInfo& dev);
int launch_dense_gemv_f16(int rows, int cols, const uint16_t* W, int64_t ldw, const uint16_t* x,
                          float* y, cudaStream_t stream, const DeviceInfo& dev);
int64_t gemm_tc_workspace_bytes(const seedlm_format& f, int M, const DeviceInfo& dev);
int launch_gemm_tc(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                   const uint16_t* X, int is_bf16, int M, float* Y, void* workspace,
                   int64_t workspace_bytes, cudaStream_t stream, const DeviceInfo& dev);
int read_and_clear_tc_error(unsigned int* out);
int launch_wait_timeout(uint64_t limit_ns, cudaStream_t stream);
int launch_encode(const seedlm_format& f, const float* W, int64_t ldw, uint32_t* rec,
                  uint8_t* eplane, double* err, cudaStream_t stream);

}  // namespace seedlm
