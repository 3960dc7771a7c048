// qmm_api.cu -- the extern "C" entry points of libqmm.so: argument validation
// (host only, before any CUDA call), device checks and dispatch to the
// kernel launchers. The operations themselves are defined in include/qmm.h.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "qmm_internal.h"

namespace qmm {

static thread_local std::string t_last_error;

qmm_status set_error(qmm_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

qmm_status cuda_check(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return QMM_OK;
  return set_error(QMM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
DevInfo g_dev[kMaxDevices];
bool g_dev_known[kMaxDevices];

// Attributes of the current device (queried once per device, then cached).
qmm_status current_device(DevInfo *out) {
  int d = -1;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return cuda_check(e, "cudaGetDevice");
  if (d < 0 || d >= kMaxDevices) return set_error(QMM_ERR_DEVICE, "device ordinal %d out of range", d);
  {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (!g_dev_known[d]) {
      DevInfo info;
      info.device = d;
      e = cudaDeviceGetAttribute(&info.cc_major, cudaDevAttrComputeCapabilityMajor, d);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&info.cc_minor, cudaDevAttrComputeCapabilityMinor, d);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, d);
      if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&info.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, d);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&info.l2_bytes, cudaDevAttrL2CacheSize, d);
      if (e != cudaSuccess) return cuda_check(e, "cudaDeviceGetAttribute");
      g_dev[d] = info;
      g_dev_known[d] = true;
    }
    *out = g_dev[d];
  }
  if (out->cc_major != 10 || out->cc_minor != 0)
    return set_error(QMM_ERR_DEVICE, "device %d has compute capability %d.%d; this library is built for sm_100a (10.0)",
                     d, out->cc_major, out->cc_minor);
  return QMM_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Common checks of (M, N, K, block). `max_m` < 0 means unbounded M.
qmm_status check_shape(const char *fn, int64_t M, int64_t N, int64_t K, int block, int64_t max_m) {
  if (block != QMM_BLOCK) return set_error(QMM_ERR_BLOCK, "%s: block=%d, only 32 is supported", fn, block);
  if (M < 0 || N < 0 || K < 0)
    return set_error(QMM_ERR_SHAPE, "%s: negative size M=%lld N=%lld K=%lld", fn, (long long)M, (long long)N,
                     (long long)K);
  if (K % QMM_BLOCK != 0) return set_error(QMM_ERR_SHAPE, "%s: K=%lld is not a multiple of 32", fn, (long long)K);
  if (K > QMM_MAX_K) return set_error(QMM_ERR_SHAPE, "%s: K=%lld exceeds %d", fn, (long long)K, QMM_MAX_K);
  if (max_m >= 0 && M > max_m)
    return set_error(QMM_ERR_SHAPE, "%s: M=%lld exceeds %lld", fn, (long long)M, (long long)max_m);
  if (N > (int64_t(1) << 40)) return set_error(QMM_ERR_SHAPE, "%s: N=%lld too large", fn, (long long)N);
  return QMM_OK;
}

qmm_status check_ptr(const char *fn, const char *name, const void *p, bool needed, uintptr_t align) {
  if (!needed) return QMM_OK;
  if (p == nullptr) return set_error(QMM_ERR_NULL, "%s: %s is NULL", fn, name);
  if (!aligned(p, align))
    return set_error(QMM_ERR_ALIGN, "%s: %s=%p is not %u-byte aligned", fn, name, p, (unsigned)align);
  return QMM_OK;
}

#define QMM_TRY(expr)                  \
  do {                                 \
    qmm_status _st = (expr);           \
    if (_st != QMM_OK) return _st;     \
  } while (0)

qmm_status zero_fill(float *Y, int64_t count, cudaStream_t s) {
  return cuda_check(cudaMemsetAsync(Y, 0, static_cast<size_t>(count) * sizeof(float), s), "cudaMemsetAsync");
}

}  // namespace

static qmm_status q8_gemv_impl(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X,
                               float *Y, qmm_stream_t stream, uint32_t user_flags) {
  const char *fn = "qmm_q8_gemv";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, N, K, block, QMM_MAX_DECODE_M));
  if (user_flags & ~uint32_t(QMM_FLAG_EARLY_WEIGHTS))
    return set_error(QMM_ERR_SHAPE, "%s: unknown flags 0x%x", fn, user_flags);
  if (M == 0 || N == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "W", W, K > 0, 16));
  QMM_TRY(check_ptr(fn, "X", X, K > 0, 16));
  QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return zero_fill(Y, M * N, s);
  uint32_t flags = kLaunchPdl | ((user_flags & QMM_FLAG_EARLY_WEIGHTS) ? kPrefetchBeforeWait : 0u);
  return launch_q8_gemv(dev, static_cast<int>(M), N, static_cast<int>(K), W, X, Y, s, flags);
}

static qmm_status quantize_q8_0_impl(int64_t M, int64_t K, int block, const float *X, void *XB, qmm_stream_t stream) {
  const char *fn = "qmm_quantize_act_q8_0";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, 0, K, block, -1));
  if (M == 0 || K == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "X", X, true, 16));
  QMM_TRY(check_ptr(fn, "XB", XB, true, 16));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  return launch_quantize_act_q8_0(dev, M, static_cast<int>(K), X, static_cast<uint8_t *>(XB),
                                  reinterpret_cast<cudaStream_t>(stream), kLaunchPdl);
}

static qmm_status q8q8_q8_0_impl(int64_t M, int64_t N, int64_t K, int block, const void *W, const void *XB, float *Y,
                                 uint32_t user_flags, qmm_stream_t stream) {
  const char *fn = "qmm_q8q8_gemv_q8_0";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, N, K, block, QMM_MAX_DECODE_M));
  if (user_flags & ~uint32_t(QMM_FLAG_EARLY_WEIGHTS))
    return set_error(QMM_ERR_SHAPE, "%s: unknown flags 0x%x", fn, user_flags);
  if (M == 0 || N == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "W", W, K > 0, 16));
  QMM_TRY(check_ptr(fn, "XB", XB, K > 0, 16));
  QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return zero_fill(Y, M * N, s);
  uint32_t flags = kLaunchPdl | ((user_flags & QMM_FLAG_EARLY_WEIGHTS) ? kPrefetchBeforeWait : 0u);
  return launch_q8q8_gemv_q8_0(dev, static_cast<int>(M), N, static_cast<int>(K), W, static_cast<const uint8_t *>(XB),
                               Y, s, flags);
}

static qmm_status auto_impl(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X, float *Y,
                            int8_t *QX, float *DX, uint32_t user_flags, qmm_stream_t stream) {
  const char *fn = "qmm_q8_gemv_auto";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, N, K, block, QMM_MAX_DECODE_M));
  if (user_flags & ~uint32_t(QMM_FLAG_EARLY_WEIGHTS))
    return set_error(QMM_ERR_SHAPE, "%s: unknown flags 0x%x", fn, user_flags);
  if (M == 0 || N == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "W", W, K > 0, 16));
  QMM_TRY(check_ptr(fn, "X", X, K > 0, 16));
  QMM_TRY(check_ptr(fn, "QX", QX, K > 0, 16));
  QMM_TRY(check_ptr(fn, "DX", DX, K > 0, 4));
  QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return zero_fill(Y, M * N, s);
  uint32_t flags = kLaunchPdl | ((user_flags & QMM_FLAG_EARLY_WEIGHTS) ? kPrefetchBeforeWait : 0u);
  return launch_q8_gemv_auto(dev, static_cast<int>(M), N, static_cast<int>(K), W, X, Y, QX, DX, s, flags);
}

static qmm_status multi_impl(int64_t M, int64_t K, int block, int nproj, const int64_t *N, const void *const *W,
                             const float *X, float *const *Y, uint32_t user_flags, qmm_stream_t stream) {
  const char *fn = "qmm_q8_gemv_multi";
  t_last_error.clear();
  if (nproj < 1 || nproj > QMM_MAX_PROJ) return set_error(QMM_ERR_SHAPE, "%s: nproj=%d outside 1..%d", fn, nproj, QMM_MAX_PROJ);
  if (!N || !W || !Y) return set_error(QMM_ERR_NULL, "%s: N, W and Y arrays are required", fn);
  if (user_flags & ~uint32_t(QMM_FLAG_EARLY_WEIGHTS))
    return set_error(QMM_ERR_SHAPE, "%s: unknown flags 0x%x", fn, user_flags);
  int64_t n[QMM_MAX_PROJ];
  const void *w[QMM_MAX_PROJ];
  float *y[QMM_MAX_PROJ];
  int k = 0;
  for (int i = 0; i < nproj; ++i) {
    QMM_TRY(check_shape(fn, M, N[i], K, block, QMM_MAX_DECODE_M));
    if (N[i] == 0 || M == 0) continue;
    QMM_TRY(check_ptr(fn, "W[i]", W[i], K > 0, 16));
    QMM_TRY(check_ptr(fn, "Y[i]", Y[i], true, 4));
    n[k] = N[i];
    w[k] = W[i];
    y[k] = Y[i];
    ++k;
  }
  if (k == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "X", X, K > 0, 16));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) {
    for (int i = 0; i < k; ++i) QMM_TRY(zero_fill(y[i], M * n[i], s));
    return QMM_OK;
  }
  uint32_t flags = kLaunchPdl | ((user_flags & QMM_FLAG_EARLY_WEIGHTS) ? kPrefetchBeforeWait : 0u);
  return launch_q8_gemv_multi(dev, static_cast<int>(M), static_cast<int>(K), k, n, w, X, y, s, flags);
}

static qmm_status quantize_impl(int64_t M, int64_t K, int block, const float *X, int8_t *QX, float *DX,
                                qmm_stream_t stream) {
  const char *fn = "qmm_quantize_act_q8";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, 0, K, block, -1));
  if (M == 0 || K == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "X", X, true, 16));
  QMM_TRY(check_ptr(fn, "QX", QX, true, 16));
  QMM_TRY(check_ptr(fn, "DX", DX, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  return launch_quantize_act_q8(dev, M, static_cast<int>(K), X, QX, DX, reinterpret_cast<cudaStream_t>(stream),
                                kLaunchPdl);
}

static qmm_status q8q8_impl(int64_t M, int64_t N, int64_t K, int block, const void *W, const int8_t *QX,
                            const float *DX, float *Y, int32_t *isum, qmm_stream_t stream, uint32_t user_flags) {
  const char *fn = isum ? "qmm_q8q8_block_dots" : "qmm_q8q8_gemv";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, N, K, block, QMM_MAX_DECODE_M));
  if (user_flags & ~uint32_t(QMM_FLAG_EARLY_WEIGHTS))
    return set_error(QMM_ERR_SHAPE, "%s: unknown flags 0x%x", fn, user_flags);
  if (M == 0 || N == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "W", W, K > 0, 16));
  QMM_TRY(check_ptr(fn, "QX", QX, K > 0, 16));
  if (isum) {
    QMM_TRY(check_ptr(fn, "isum", isum, K > 0, 4));
  } else {
    QMM_TRY(check_ptr(fn, "DX", DX, K > 0, 4));
    QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  }
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return isum ? QMM_OK : zero_fill(Y, M * N, s);
  if (isum) return launch_q8q8_block_dots(dev, static_cast<int>(M), N, static_cast<int>(K), W, QX, nullptr, isum, s);
  uint32_t flags = kLaunchPdl | ((user_flags & QMM_FLAG_EARLY_WEIGHTS) ? kPrefetchBeforeWait : 0u);
  return launch_q8q8_gemv(dev, static_cast<int>(M), N, static_cast<int>(K), W, QX, DX, Y, s, flags);
}

static qmm_status q8q8_fused_impl(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X,
                                  int8_t *QX, float *DX, float *Y, qmm_stream_t stream, uint32_t user_flags) {
  const char *fn = "qmm_q8q8_gemv_fused";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, N, K, block, QMM_MAX_DECODE_M));
  if (user_flags & ~uint32_t(QMM_FLAG_EARLY_WEIGHTS))
    return set_error(QMM_ERR_SHAPE, "%s: unknown flags 0x%x", fn, user_flags);
  if (M == 0 || N == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "W", W, K > 0, 16));
  QMM_TRY(check_ptr(fn, "X", X, K > 0, 16));
  QMM_TRY(check_ptr(fn, "QX", QX, K > 0, 16));
  QMM_TRY(check_ptr(fn, "DX", DX, K > 0, 4));
  QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return zero_fill(Y, M * N, s);
  uint32_t flags = kLaunchPdl | ((user_flags & QMM_FLAG_EARLY_WEIGHTS) ? kPrefetchBeforeWait : 0u);
  return launch_q8q8_gemv_fused(dev, static_cast<int>(M), N, static_cast<int>(K), W, X, QX, DX, Y, s, flags);
}

static qmm_status fused_dots_impl(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X,
                                  int8_t *QX, float *DX, float *Y, int32_t *isum, qmm_stream_t stream) {
  const char *fn = "qmm_q8q8_gemv_fused_dots";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, N, K, block, QMM_MAX_DECODE_M));
  if (M == 0 || N == 0 || K == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "W", W, true, 16));
  QMM_TRY(check_ptr(fn, "X", X, true, 16));
  QMM_TRY(check_ptr(fn, "QX", QX, true, 16));
  QMM_TRY(check_ptr(fn, "DX", DX, true, 4));
  QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  QMM_TRY(check_ptr(fn, "isum", isum, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  return launch_q8q8_gemv_fused_dots(dev, static_cast<int>(M), N, static_cast<int>(K), W, X, QX, DX, Y, isum,
                                     reinterpret_cast<cudaStream_t>(stream));
}

static qmm_status dots_q8_0_impl(int64_t M, int64_t N, int64_t K, int block, const void *W, const void *XB,
                                 int32_t *isum, qmm_stream_t stream) {
  const char *fn = "qmm_q8q8_block_dots_q8_0";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, N, K, block, QMM_MAX_DECODE_M));
  if (M == 0 || N == 0 || K == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "W", W, true, 16));
  QMM_TRY(check_ptr(fn, "XB", XB, true, 16));
  QMM_TRY(check_ptr(fn, "isum", isum, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  return launch_q8q8_block_dots(dev, static_cast<int>(M), N, static_cast<int>(K), W, nullptr,
                                static_cast<const uint8_t *>(XB), isum, reinterpret_cast<cudaStream_t>(stream));
}

static qmm_status withheld_impl(int kernel, int64_t M, int64_t N, int64_t K, int block, const void *W, const void *X,
                                float *Y, uint64_t wait_ns, qmm_stream_t stream) {
  const char *fn = "qmm_test_withheld_copy";
  t_last_error.clear();
  if (kernel != 0 && kernel != 1) return set_error(QMM_ERR_SHAPE, "%s: kernel=%d, expected 0 or 1", fn, kernel);
  QMM_TRY(check_shape(fn, M, N, K, block, kernel == 0 ? QMM_MAX_DECODE_M : 32));
  if (M < 1 || N < 1 || K < 32) return set_error(QMM_ERR_SHAPE, "%s: M, N must be >= 1 and K >= 32", fn);
  if (wait_ns < 1000 || wait_ns > 2000000000ull)
    return set_error(QMM_ERR_SHAPE, "%s: wait_ns=%llu outside 1e3 .. 2e9", fn, (unsigned long long)wait_ns);
  QMM_TRY(check_ptr(fn, "W", W, true, 16));
  QMM_TRY(check_ptr(fn, "X", X, true, 16));
  QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (kernel == 0)
    return launch_q8_gemv_withheld(dev, static_cast<int>(M), N, static_cast<int>(K), W, static_cast<const float *>(X), Y,
                                   wait_ns, s);
  return launch_prefill_small_withheld(dev, QMM_Q8_0, M, N, static_cast<int>(K), W, static_cast<const uint16_t *>(X), Y,
                                       wait_ns, s);
}

static qmm_status q4_gemv_impl(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X, float *Y,
                               uint32_t user_flags, qmm_stream_t stream) {
  const char *fn = "qmm_q4_gemv";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, N, K, block, QMM_MAX_DECODE_M));
  if (user_flags & ~uint32_t(QMM_FLAG_EARLY_WEIGHTS))
    return set_error(QMM_ERR_SHAPE, "%s: unknown flags 0x%x", fn, user_flags);
  if (M == 0 || N == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "W", W, K > 0, 16));
  QMM_TRY(check_ptr(fn, "X", X, K > 0, 16));
  QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return zero_fill(Y, M * N, s);
  uint32_t flags = kLaunchPdl | ((user_flags & QMM_FLAG_EARLY_WEIGHTS) ? kPrefetchBeforeWait : 0u);
  return launch_q4_gemv(dev, static_cast<int>(M), N, static_cast<int>(K), W, X, Y, s, flags);
}

static qmm_status gateup_impl(int64_t M, int64_t N, int64_t K, int block, const void *Wg, const void *Wu,
                              const float *X, float *G, float *U, float *Y, qmm_stream_t stream, bool unfused,
                              uint32_t user_flags) {
  const char *fn = unfused ? "qmm_q4_gateup_unfused" : "qmm_q4_swiglu_gateup";
  t_last_error.clear();
  QMM_TRY(check_shape(fn, M, N, K, block, QMM_MAX_DECODE_M));
  if (user_flags & ~uint32_t(QMM_FLAG_EARLY_WEIGHTS))
    return set_error(QMM_ERR_SHAPE, "%s: unknown flags 0x%x", fn, user_flags);
  if (M == 0 || N == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "Wg", Wg, K > 0, 16));
  QMM_TRY(check_ptr(fn, "Wu", Wu, K > 0, 16));
  QMM_TRY(check_ptr(fn, "X", X, K > 0, 16));
  QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  if (unfused) {
    QMM_TRY(check_ptr(fn, "G", G, true, 4));
    QMM_TRY(check_ptr(fn, "U", U, true, 4));
  }
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) {
    if (unfused) {
      QMM_TRY(zero_fill(G, M * N, s));
      QMM_TRY(zero_fill(U, M * N, s));
    }
    return zero_fill(Y, M * N, s);
  }
  if (unfused)
    return launch_q4_gateup_unfused(dev, static_cast<int>(M), N, static_cast<int>(K), Wg, Wu, X, G, U, Y, s);
  uint32_t flags = kLaunchPdl | ((user_flags & QMM_FLAG_EARLY_WEIGHTS) ? kPrefetchBeforeWait : 0u);
  return launch_q4_gateup(dev, static_cast<int>(M), N, static_cast<int>(K), Wg, Wu, X, Y, s, flags);
}

static qmm_status prefill_impl(int wtype, int64_t M, int64_t N, int64_t K, int block, const void *W,
                               const uint16_t *X, float *Y, qmm_stream_t stream, uint32_t user_flags) {
  const char *fn = "qmm_quant_matmul_prefill";
  t_last_error.clear();
  if (wtype != QMM_Q8_0 && wtype != QMM_Q4_0) return set_error(QMM_ERR_DTYPE, "%s: unknown weight type %d", fn, wtype);
  QMM_TRY(check_shape(fn, M, N, K, block, -1));
  if (M > (int64_t(1) << 24)) return set_error(QMM_ERR_SHAPE, "%s: M=%lld too large", fn, (long long)M);
  if (user_flags & ~uint32_t(QMM_FLAG_EARLY_WEIGHTS))
    return set_error(QMM_ERR_SHAPE, "%s: unknown flags 0x%x", fn, user_flags);
  if (M == 0 || N == 0) return QMM_OK;
  QMM_TRY(check_ptr(fn, "W", W, K > 0, 16));
  QMM_TRY(check_ptr(fn, "X", X, K > 0, 16));
  QMM_TRY(check_ptr(fn, "Y", Y, true, 4));
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return zero_fill(Y, M * N, s);
  const uint32_t flags = kLaunchPdl | ((user_flags & QMM_FLAG_EARLY_WEIGHTS) ? kPrefetchBeforeWait : 0u);
  return launch_prefill(dev, wtype, M, N, static_cast<int>(K), W, X, Y, s, flags);
}

}  // namespace qmm

using namespace qmm;

extern "C" {

QMM_API qmm_status qmm_q8_gemv(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X,
                               float *Y, qmm_stream_t stream) {
  return q8_gemv_impl(M, N, K, block, W, X, Y, stream, 0u);
}

QMM_API qmm_status qmm_q8_gemv_ex(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X,
                                  float *Y, uint32_t flags, qmm_stream_t stream) {
  return q8_gemv_impl(M, N, K, block, W, X, Y, stream, flags);
}

QMM_API qmm_status qmm_quantize_act_q8_0(int64_t M, int64_t K, int block, const float *X, void *XB,
                                         qmm_stream_t stream) {
  return quantize_q8_0_impl(M, K, block, X, XB, stream);
}

QMM_API qmm_status qmm_q8q8_gemv_q8_0(int64_t M, int64_t N, int64_t K, int block, const void *W, const void *XB,
                                      float *Y, uint32_t flags, qmm_stream_t stream) {
  return q8q8_q8_0_impl(M, N, K, block, W, XB, Y, flags, stream);
}

QMM_API qmm_status qmm_q8_gemv_auto(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X,
                                    float *Y, int8_t *QX, float *DX, uint32_t flags, qmm_stream_t stream) {
  return auto_impl(M, N, K, block, W, X, Y, QX, DX, flags, stream);
}

QMM_API qmm_status qmm_q8_gemv_multi(int64_t M, int64_t K, int block, int nproj, const int64_t *N,
                                     const void *const *W, const float *X, float *const *Y, uint32_t flags,
                                     qmm_stream_t stream) {
  return multi_impl(M, K, block, nproj, N, W, X, Y, flags, stream);
}

QMM_API qmm_status qmm_quantize_act_q8(int64_t M, int64_t K, int block, const float *X, int8_t *QX, float *DX,
                                       qmm_stream_t stream) {
  return quantize_impl(M, K, block, X, QX, DX, stream);
}

QMM_API qmm_status qmm_q8q8_gemv(int64_t M, int64_t N, int64_t K, int block, const void *W, const int8_t *QX,
                                 const float *DX, float *Y, qmm_stream_t stream) {
  return q8q8_impl(M, N, K, block, W, QX, DX, Y, nullptr, stream, 0u);
}

QMM_API qmm_status qmm_q8q8_gemv_ex(int64_t M, int64_t N, int64_t K, int block, const void *W, const int8_t *QX,
                                    const float *DX, float *Y, uint32_t flags, qmm_stream_t stream) {
  return q8q8_impl(M, N, K, block, W, QX, DX, Y, nullptr, stream, flags);
}

QMM_API qmm_status qmm_q8q8_gemv_fused(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X,
                                       int8_t *QX, float *DX, float *Y, uint32_t flags, qmm_stream_t stream) {
  return q8q8_fused_impl(M, N, K, block, W, X, QX, DX, Y, stream, flags);
}

QMM_API qmm_status qmm_q8q8_block_dots(int64_t M, int64_t N, int64_t K, int block, const void *W, const int8_t *QX,
                                       int32_t *isum, qmm_stream_t stream) {
  return q8q8_impl(M, N, K, block, W, QX, nullptr, nullptr, isum, stream, 0u);
}

QMM_API qmm_status qmm_q8q8_gemv_fused_dots(int64_t M, int64_t N, int64_t K, int block, const void *W,
                                            const float *X, int8_t *QX, float *DX, float *Y, int32_t *isum,
                                            qmm_stream_t stream) {
  return fused_dots_impl(M, N, K, block, W, X, QX, DX, Y, isum, stream);
}

QMM_API qmm_status qmm_q8q8_block_dots_q8_0(int64_t M, int64_t N, int64_t K, int block, const void *W, const void *XB,
                                            int32_t *isum, qmm_stream_t stream) {
  return dots_q8_0_impl(M, N, K, block, W, XB, isum, stream);
}

QMM_API qmm_status qmm_test_withheld_copy(int kernel, int64_t M, int64_t N, int64_t K, int block, const void *W,
                                          const void *X, float *Y, uint64_t wait_ns, qmm_stream_t stream) {
  return withheld_impl(kernel, M, N, K, block, W, X, Y, wait_ns, stream);
}

QMM_API qmm_status qmm_q4_swiglu_gateup(int64_t M, int64_t N, int64_t K, int block, const void *Wg, const void *Wu,
                                        const float *X, float *Y, qmm_stream_t stream) {
  return gateup_impl(M, N, K, block, Wg, Wu, X, nullptr, nullptr, Y, stream, false, 0u);
}

QMM_API qmm_status qmm_q4_swiglu_gateup_ex(int64_t M, int64_t N, int64_t K, int block, const void *Wg,
                                           const void *Wu, const float *X, float *Y, uint32_t flags,
                                           qmm_stream_t stream) {
  return gateup_impl(M, N, K, block, Wg, Wu, X, nullptr, nullptr, Y, stream, false, flags);
}

QMM_API qmm_status qmm_q4_gemv(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X, float *Y,
                               uint32_t flags, qmm_stream_t stream) {
  return q4_gemv_impl(M, N, K, block, W, X, Y, flags, stream);
}

QMM_API qmm_status qmm_q4_gateup_unfused(int64_t M, int64_t N, int64_t K, int block, const void *Wg, const void *Wu,
                                         const float *X, float *G, float *U, float *Y, qmm_stream_t stream) {
  return gateup_impl(M, N, K, block, Wg, Wu, X, G, U, Y, stream, true, 0u);
}

QMM_API qmm_status qmm_quant_matmul_prefill(int wtype, int64_t M, int64_t N, int64_t K, int block, const void *W,
                                            const uint16_t *X, float *Y, qmm_stream_t stream) {
  return prefill_impl(wtype, M, N, K, block, W, X, Y, stream, 0u);
}

QMM_API qmm_status qmm_quant_matmul_prefill_ex(int wtype, int64_t M, int64_t N, int64_t K, int block, const void *W,
                                               const uint16_t *X, float *Y, uint32_t flags, qmm_stream_t stream) {
  return prefill_impl(wtype, M, N, K, block, W, X, Y, stream, flags);
}

QMM_API qmm_status qmm_prefill_plan(int wtype, int64_t M, int64_t N, int64_t K, int block, int32_t *plan) {
  const char *fn = "qmm_prefill_plan";
  t_last_error.clear();
  if (plan == nullptr) return set_error(QMM_ERR_NULL, "%s: plan is NULL", fn);
  if (wtype != QMM_Q8_0 && wtype != QMM_Q4_0) return set_error(QMM_ERR_DTYPE, "%s: unknown weight type %d", fn, wtype);
  QMM_TRY(check_shape(fn, M, N, K, block, -1));
  if (M < 1 || N < 1 || K < 32) return set_error(QMM_ERR_SHAPE, "%s: M, N must be >= 1 and K >= 32", fn);
  if (M > (int64_t(1) << 24)) return set_error(QMM_ERR_SHAPE, "%s: M=%lld too large", fn, (long long)M);
  DevInfo dev;
  QMM_TRY(current_device(&dev));
  PrefillPlan pl{};
  QMM_TRY(launch_prefill(dev, wtype, M, N, static_cast<int>(K), nullptr, nullptr, nullptr, nullptr, 0u, &pl));
  plan[0] = pl.mt;
  plan[1] = pl.split;
  plan[2] = pl.stages;
  plan[3] = pl.ctas;
  plan[4] = pl.kind;
  return QMM_OK;
}

QMM_API const char *qmm_last_error_string(void) { return t_last_error.c_str(); }

QMM_API const char *qmm_version(void) { return "qmm 0.1.0 sm_100a"; }

QMM_API qmm_status qmm_device_status(uint32_t *bits) {
  if (bits == nullptr) return set_error(QMM_ERR_NULL, "qmm_device_status: bits is NULL");
  *bits = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_check(e, "cudaDeviceSynchronize");
  uint32_t b = 0;
  e = q8_gemv_status(&b);
  if (e != cudaSuccess) return cuda_check(e, "status read");
  *bits |= b;
  e = q4_gateup_status(&b);
  if (e != cudaSuccess) return cuda_check(e, "status read");
  *bits |= b;
  e = prefill_status(&b);
  if (e != cudaSuccess) return cuda_check(e, "status read");
  *bits |= b;
  if (*bits) return set_error(QMM_ERR_DEVICE_CHECK, "qmm_device_status: a kernel recorded a failure (bits 0x%x)", *bits);
  return QMM_OK;
}

}  // extern "C"
