// abi.cu -- the extern "C" entry points of libseedlm.so: argument checks,
// per-device setup and dispatch to the kernels.  See include/seedlm.h for the
// contract of every function.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "seedlm_internal.h"

namespace seedlm {

namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<int64_t> g_launches{0};

constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_ready[kMaxDevices] = {};

int device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return record_cuda_error(err);
  if (dev < 0 || dev >= kMaxDevices) return SEEDLM_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (!g_dev_ready[dev]) {
    DeviceInfo d{};
    d.device = dev;
    if ((err = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev)) !=
            cudaSuccess ||
        (err = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                      dev)) != cudaSuccess ||
        (err = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) !=
            cudaSuccess ||
        (err = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) !=
            cudaSuccess)
      return record_cuda_error(err);
    // The kernels are built for sm_100a only.
    if (d.cc_major != 10 || d.cc_minor != 0) return SEEDLM_EUNSUPPORTED;
    g_dev[dev] = d;
    g_dev_ready[dev] = true;
  }
  *out = g_dev[dev];
  return SEEDLM_OK;
}

}  // namespace

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_format(const seedlm_format* f) {
  if (!f) return SEEDLM_EINVAL;
  const bool c8 = f->C == 8 && f->P == 3 && f->K == 16;
  const bool c12 = f->C == 12 && f->P == 4 && f->K == 16;
  if (!c8 && !c12) return SEEDLM_EUNSUPPORTED;
  if (f->rows < 0 || f->cols < 0) return SEEDLM_EINVAL;
  if (f->nb != (f->cols + f->C - 1) / f->C) return SEEDLM_EINVAL;
  if (f->rec_pitch < f->nb || f->rec_pitch % 4 != 0) return SEEDLM_EINVAL;
  if (c12 && f->e_pitch < (f->nb + 1) / 2) return SEEDLM_EINVAL;
  return SEEDLM_OK;
}

int check_planes(const seedlm_format* f, const uint32_t* rec, const uint8_t* eplane) {
  if (f->rows == 0 || f->nb == 0) return SEEDLM_OK;
  if (!rec || !aligned(rec, 16)) return SEEDLM_EINVAL;
  if (f->P == 4 && !eplane) return SEEDLM_EINVAL;
  return SEEDLM_OK;
}

int record_cuda_error(cudaError_t err) {
  if (err == cudaSuccess) return SEEDLM_OK;
  g_last_cuda_error = (int)err;
  return SEEDLM_ECUDA;
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int current_device_info(DeviceInfo* out) { return device_info(out); }

int allow_max_smem(const void* kernel, const DeviceInfo& dev) {
  static std::mutex m;
  static std::set<std::pair<const void*, int>> done;
  std::lock_guard<std::mutex> lock(m);
  if (done.count({kernel, dev.device})) return SEEDLM_OK;
  cudaError_t err =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dev.max_smem_optin);
  if (err != cudaSuccess) return record_cuda_error(err);
  done.insert({kernel, dev.device});
  return SEEDLM_OK;
}

}  // namespace seedlm

using namespace seedlm;

namespace {

// Workspace of seedlm_gemm: the larger of a full pass and the last pass.
int64_t gemm_any_workspace(const seedlm_format& f, int M, const DeviceInfo& dev) {
  if (M == 1 && gemv_smem_bytes(f, dev) > 0) return 0;  // the GEMV
  if (gemm_cc_applies(f, M)) return 0;                  // the CUDA-core kernel
  const int full = M < kGemmPassRows ? M : kGemmPassRows;
  int64_t need = gemm_tc_workspace_bytes(f, full, dev);
  const int last = M % kGemmPassRows;
  if (M > kGemmPassRows && last) {
    const int64_t l = gemm_tc_workspace_bytes(f, last, dev);
    if (l > need) need = l;
  }
  return need;
}

}  // namespace

extern "C" {

int seedlm_init(void) {
  DeviceInfo d;
  return device_info(&d);
}

int seedlm_decompress(const seedlm_format* fmt, const uint32_t* rec, const uint8_t* eplane,
                      float* W, int64_t ldw, seedlm_stream stream) {
  int rc = check_format(fmt);
  if (rc) return rc;
  if ((rc = check_planes(fmt, rec, eplane))) return rc;
  if (fmt->rows == 0 || fmt->cols == 0) return SEEDLM_OK;
  if (!W || !aligned(W, 4) || ldw < fmt->cols) return SEEDLM_EINVAL;
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  return launch_decompress(*fmt, rec, eplane, W, ldw, (cudaStream_t)stream, dev);
}

int seedlm_gemv(const seedlm_format* fmt, const uint32_t* rec, const uint8_t* eplane,
                const void* x, int x_dtype, float* y, seedlm_stream stream) {
  int rc = check_format(fmt);
  if (rc) return rc;
  if ((rc = check_planes(fmt, rec, eplane))) return rc;
  if (x_dtype != SEEDLM_F16 && x_dtype != SEEDLM_BF16) return SEEDLM_EINVAL;
  if (fmt->rows == 0) return SEEDLM_OK;
  if (!y || !aligned(y, 4)) return SEEDLM_EINVAL;
  if (fmt->cols > 0 && (!x || !aligned(x, 2))) return SEEDLM_EINVAL;
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  if (fmt->cols == 0)
    return record_cuda_error(
        cudaMemsetAsync(y, 0, (size_t)fmt->rows * sizeof(float), (cudaStream_t)stream));
  return launch_gemv(*fmt, rec, eplane, static_cast<const uint16_t*>(x),
                     x_dtype == SEEDLM_BF16, y, (cudaStream_t)stream, dev);
}

int seedlm_gemv_batch(int32_t n, const seedlm_format* fmts, const uint32_t* const* recs,
                      const uint8_t* const* eplanes, const void* const* xs, int x_dtype,
                      float* const* ys, seedlm_stream stream) {
  if (n < 0 || n > 8 || (n > 0 && (!fmts || !recs || !xs || !ys))) return SEEDLM_EINVAL;
  if (x_dtype != SEEDLM_F16 && x_dtype != SEEDLM_BF16) return SEEDLM_EINVAL;
  int rc;
  for (int k = 0; k < n; ++k) {
    const seedlm_format* f = &fmts[k];
    if ((rc = check_format(f))) return rc;
    if (f->C != fmts[0].C) return SEEDLM_EUNSUPPORTED;
    if ((rc = check_planes(f, recs[k], eplanes ? eplanes[k] : nullptr))) return rc;
    if (f->rows == 0) continue;
    if (!ys[k] || !aligned(ys[k], 4)) return SEEDLM_EINVAL;
    if (f->cols > 0 && (!xs[k] || !aligned(xs[k], 2))) return SEEDLM_EINVAL;
  }
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  const seedlm_format* f[8];
  const uint32_t* r[8];
  const uint8_t* e[8];
  const uint16_t* x[8];
  float* y[8];
  int m = 0;
  for (int k = 0; k < n; ++k) {
    if (fmts[k].rows == 0) continue;
    if (fmts[k].cols == 0) {
      if ((rc = record_cuda_error(cudaMemsetAsync(ys[k], 0, (size_t)fmts[k].rows * sizeof(float),
                                                  (cudaStream_t)stream))))
        return rc;
      continue;
    }
    f[m] = &fmts[k];
    r[m] = recs[k];
    e[m] = eplanes ? eplanes[k] : nullptr;
    x[m] = static_cast<const uint16_t*>(xs[k]);
    y[m] = ys[k];
    ++m;
  }
  return launch_gemv_batch(m, f, r, e, x, x_dtype == SEEDLM_BF16, y, (cudaStream_t)stream, dev);
}

int seedlm_gemm_smallM(const seedlm_format* fmt, const uint32_t* rec, const uint8_t* eplane,
                       const void* X, int x_dtype, int M, float* Y, void* workspace,
                       int64_t workspace_bytes, seedlm_stream stream) {
  int rc = check_format(fmt);
  if (rc) return rc;
  if ((rc = check_planes(fmt, rec, eplane))) return rc;
  if (x_dtype != SEEDLM_F16 && x_dtype != SEEDLM_BF16) return SEEDLM_EINVAL;
  if (M < 1 || M > 64 || workspace_bytes < 0) return SEEDLM_EINVAL;
  if (fmt->rows == 0) return SEEDLM_OK;
  if (!Y || !aligned(Y, 4)) return SEEDLM_EINVAL;
  if (fmt->cols > 0 && (!X || !aligned(X, 2))) return SEEDLM_EINVAL;
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  if (fmt->cols == 0)
    return record_cuda_error(
        cudaMemsetAsync(Y, 0, (size_t)M * fmt->rows * sizeof(float), (cudaStream_t)stream));
  const uint16_t* Xh = static_cast<const uint16_t*>(X);
  // M = 1 runs the GEMV unless x is too wide for its shared memory, 2 to 4
  // rows the CUDA-core kernel, more rows the tensor cores.
  if (M == 1 && gemv_smem_bytes(*fmt, dev) > 0)
    return launch_gemv(*fmt, rec, eplane, Xh, x_dtype == SEEDLM_BF16, Y, (cudaStream_t)stream,
                       dev);
  if (gemm_cc_applies(*fmt, M))
    return launch_gemm_cc(*fmt, rec, eplane, Xh, x_dtype == SEEDLM_BF16, M, Y, (cudaStream_t)stream,
                          dev);
  return launch_gemm_tc(*fmt, rec, eplane, Xh, x_dtype == SEEDLM_BF16, M, Y, workspace,
                        workspace_bytes, (cudaStream_t)stream, dev);
}

int64_t seedlm_gemm_smallM_workspace_bytes(const seedlm_format* fmt, int M) {
  if (check_format(fmt) || M < 1 || M > 64) return SEEDLM_EINVAL;
  if (fmt->rows == 0 || fmt->cols == 0) return 0;
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  if (M == 1 && gemv_smem_bytes(*fmt, dev) > 0) return 0;  // the GEMV
  if (gemm_cc_applies(*fmt, M)) return 0;                  // the CUDA-core kernel
  return gemm_tc_workspace_bytes(*fmt, M, dev);
}

int seedlm_gemm(const seedlm_format* fmt, const uint32_t* rec, const uint8_t* eplane, const void* X,
                int x_dtype, int M, float* Y, void* workspace, int64_t workspace_bytes,
                seedlm_stream stream) {
  int rc = check_format(fmt);
  if (rc) return rc;
  if ((rc = check_planes(fmt, rec, eplane))) return rc;
  if (x_dtype != SEEDLM_F16 && x_dtype != SEEDLM_BF16) return SEEDLM_EINVAL;
  if (M < 1 || workspace_bytes < 0) return SEEDLM_EINVAL;
  if (fmt->rows == 0) return SEEDLM_OK;
  if (!Y || !aligned(Y, 4)) return SEEDLM_EINVAL;
  if (fmt->cols > 0 && (!X || !aligned(X, 2))) return SEEDLM_EINVAL;
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  const cudaStream_t st = (cudaStream_t)stream;
  if (fmt->cols == 0)
    return record_cuda_error(cudaMemsetAsync(Y, 0, (size_t)M * fmt->rows * sizeof(float), st));
  const uint16_t* Xh = static_cast<const uint16_t*>(X);
  const int is_bf16 = x_dtype == SEEDLM_BF16;
  if (M == 1 && gemv_smem_bytes(*fmt, dev) > 0)
    return launch_gemv(*fmt, rec, eplane, Xh, is_bf16, Y, st, dev);
  if (gemm_cc_applies(*fmt, M)) return launch_gemm_cc(*fmt, rec, eplane, Xh, is_bf16, M, Y, st, dev);
  if (workspace_bytes < gemm_any_workspace(*fmt, M, dev)) return SEEDLM_EINVAL;
  // Passes of up to kGemmPassRows rows of X, one after the other on the
  // stream, sharing the workspace (each pass leaves its counters at zero).
  for (int m0 = 0; m0 < M; m0 += kGemmPassRows) {
    const int mc = M - m0 < kGemmPassRows ? M - m0 : kGemmPassRows;
    rc = launch_gemm_tc(*fmt, rec, eplane, Xh + (size_t)m0 * fmt->cols, is_bf16, mc,
                        Y + (size_t)m0 * fmt->rows, workspace, workspace_bytes, st, dev);
    if (rc) return rc;
  }
  return SEEDLM_OK;
}

int64_t seedlm_gemm_workspace_bytes(const seedlm_format* fmt, int M) {
  if (check_format(fmt) || M < 1) return SEEDLM_EINVAL;
  if (fmt->rows == 0 || fmt->cols == 0) return 0;
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  return gemm_any_workspace(*fmt, M, dev);
}

int seedlm_encode(const seedlm_format* fmt, const float* W, int64_t ldw, uint32_t* rec,
                  uint8_t* eplane, double* err, seedlm_stream stream) {
  int rc = check_format(fmt);
  if (rc) return rc;
  if ((rc = check_planes(fmt, rec, eplane))) return rc;
  if (fmt->rows == 0 || fmt->cols == 0) return SEEDLM_OK;
  if (!W || !aligned(W, 4) || ldw < fmt->cols) return SEEDLM_EINVAL;
  if (err && !aligned(err, 8)) return SEEDLM_EINVAL;
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  return launch_encode(*fmt, W, ldw, rec, eplane, err, (cudaStream_t)stream, dev);
}

int seedlm_selftest_wait_timeout(int64_t limit_ns, seedlm_stream stream) {
  if (limit_ns < 1000 || limit_ns > 100000000) return SEEDLM_EINVAL;
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  return launch_wait_timeout((uint64_t)limit_ns, (cudaStream_t)stream);
}

int seedlm_selftest_bounds_check(int64_t index, int64_t extent, seedlm_stream stream) {
  if (index < 0 || extent < 0) return SEEDLM_EINVAL;
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  return launch_bounds_check(index, extent, (cudaStream_t)stream);
}

int seedlm_device_error(int* flag) {
  if (!flag) return SEEDLM_EINVAL;
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  unsigned int v = 0;
  if ((rc = read_and_clear_tc_error(&v))) return rc;
  int out = v ? 1 : 0;
  if ((rc = read_and_clear_encode_error(&v))) return rc;
  if (v) out |= 1;
  if ((rc = read_and_clear_gemv_error(&v))) return rc;
  if (v) out |= 1;
  if ((rc = read_and_clear_cc_error(&v))) return rc;
  if (v) out |= 1;
  if ((rc = read_and_clear_amort_error(&v))) return rc;
  if (v) out |= 1;
  // Bounds violations recorded by a checked build (always 0 otherwise).
  int (*const readers[])(unsigned int*) = {read_and_clear_check_gemv, read_and_clear_check_decompress,
                                           read_and_clear_check_gemm_tc, read_and_clear_check_encode,
                                           read_and_clear_check_dense, read_and_clear_check_gemm_cc,
                                           read_and_clear_check_gemv_amort};
  for (auto read : readers) {
    unsigned int c = 0;
    if ((rc = read(&c))) return rc;
    if (c) out |= 2;
  }
  *flag = out;
  return SEEDLM_OK;
}

int seedlm_checked_build(void) { return SEEDLM_CHECK ? 1 : 0; }

int seedlm_dense_gemv_f16(int32_t rows, int32_t cols, const uint16_t* W, int64_t ldw,
                          const uint16_t* x, float* y, seedlm_stream stream) {
  if (rows < 0 || cols < 0 || ldw < cols || ldw % 8 != 0) return SEEDLM_EINVAL;
  if (rows == 0) return SEEDLM_OK;
  if (!y || !aligned(y, 4)) return SEEDLM_EINVAL;
  if (cols > 0 && (!W || !aligned(W, 16) || !x || !aligned(x, 2))) return SEEDLM_EINVAL;
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  if (cols == 0)
    return record_cuda_error(
        cudaMemsetAsync(y, 0, (size_t)rows * sizeof(float), (cudaStream_t)stream));
  return launch_dense_gemv_f16(rows, cols, W, ldw, x, y, (cudaStream_t)stream, dev);
}

int64_t seedlm_row_bytes_ideal(const seedlm_format* fmt) {
  if (check_format(fmt)) return -1;
  const int64_t bits = (int64_t)(fmt->K + 4 * fmt->P + 4) * fmt->nb;
  return (bits + 7) / 8;
}

int64_t seedlm_row_bytes_stored(const seedlm_format* fmt) {
  if (check_format(fmt)) return -1;
  return 4 * (int64_t)fmt->rec_pitch + (fmt->P == 4 ? (int64_t)fmt->e_pitch : 0);
}

const char* seedlm_strerror(int code) {
  switch (code) {
    case SEEDLM_OK: return "success";
    case SEEDLM_EINVAL: return "invalid argument (null or misaligned pointer, bad size or field)";
    case SEEDLM_EUNSUPPORTED: return "unsupported format, size or device";
    case SEEDLM_ECUDA: return "a CUDA call failed (see seedlm_last_cuda_error)";
    default: return "unknown error code";
  }
}

int seedlm_last_cuda_error(void) { return g_last_cuda_error; }

int64_t seedlm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void seedlm_shutdown(void) {}

}  // extern "C"
