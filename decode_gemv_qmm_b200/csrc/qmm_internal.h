// qmm_internal.h -- host-side declarations shared by the C-ABI layer and the
// kernel files (launchers, device info, error recording). Not installed.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/qmm.h"

namespace qmm {

struct DevInfo {
  int device = -1;
  int sms = 0;
  int cc_major = 0, cc_minor = 0;
  int smem_optin = 0;  // max dynamic shared memory per block (opt-in)
  int l2_bytes = 0;
};

// Once-per-device flags for a kernel's attribute set-up (devices 0..63; others
// always read as done, and their launches use the default attributes).
// Concurrent first calls may both run the set-up, which is idempotent; the
// flags themselves are atomic, so the check is free of data races.
struct DeviceFlags {
  std::atomic<bool> f[64];
  bool done(int dev) const { return dev < 0 || dev >= 64 || f[dev].load(std::memory_order_acquire); }
  void set(int dev) {
    if (dev >= 0 && dev < 64) f[dev].store(true, std::memory_order_release);
  }
};

// Launch options carried from the entry points to the launchers.
enum : uint32_t {
  kLaunchPdl = 1u,            // launch with programmatic stream serialization
  kPrefetchBeforeWait = 2u,   // stream W before the preceding grid has finished
};

// Record an error message for qmm_last_error_string() and return `st`.
qmm_status set_error(qmm_status st, const char *fmt, ...);
// Translate a CUDA error (cudaSuccess -> QMM_OK).
qmm_status cuda_check(cudaError_t e, const char *what);

// ---- launchers (arguments already validated; sizes > 0) -------------------
qmm_status launch_q8_gemv(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X,
                          float *Y, cudaStream_t stream, uint32_t flags);

// Per-K choice between the fused Q8xQ8 form (short rows) and the fp32 GEMV.
qmm_status launch_q8_gemv_auto(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X, float *Y,
                               int8_t *QX, float *DX, cudaStream_t stream, uint32_t flags);
// nproj (<= 4) projections of the same X in one launch where the shape allows.
qmm_status launch_q8_gemv_multi(const DevInfo &dev, int M, int K, int nproj, const int64_t *N, const void *const *W,
                                const float *X, float *const *Y, cudaStream_t stream, uint32_t flags);

qmm_status launch_q8q8_gemv(const DevInfo &dev, int M, int64_t N, int K, const void *W, const int8_t *QX,
                            const float *DX, float *Y, cudaStream_t stream, uint32_t flags);
// The exact block dots of the streaming Q8xQ8 kernel (activations as QX codes,
// or as Q8_0 blocks XB when XB is set).
qmm_status launch_q8q8_block_dots(const DevInfo &dev, int M, int64_t N, int K, const void *W, const int8_t *QX,
                                  const uint8_t *XB, int32_t *isum, cudaStream_t stream);
// launch_q8q8_gemv_fused with the exact block dots written to isum as well.
qmm_status launch_q8q8_gemv_fused_dots(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X,
                                       int8_t *QX, float *DX, float *Y, int32_t *isum, cudaStream_t stream);
// Failure-path test: the streaming fp32 GEMV with the given wait limit and the
// first weight stage of CTA 0 withheld.
qmm_status launch_q8_gemv_withheld(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X,
                                   float *Y, uint64_t wait_ns, cudaStream_t stream);
qmm_status launch_q8q8_gemv_fused(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X,
                                  int8_t *QX, float *DX, float *Y, cudaStream_t stream, uint32_t flags);
qmm_status launch_quantize_act_q8_0(const DevInfo &dev, int64_t M, int K, const float *X, uint8_t *XB,
                                    cudaStream_t stream, uint32_t flags);
qmm_status launch_q8q8_gemv_q8_0(const DevInfo &dev, int M, int64_t N, int K, const void *W, const uint8_t *XB,
                                 float *Y, cudaStream_t stream, uint32_t flags);
qmm_status launch_quantize_act_q8(const DevInfo &dev, int64_t M, int K, const float *X, int8_t *QX, float *DX,
                                  cudaStream_t stream, uint32_t flags);

qmm_status launch_q4_gateup(const DevInfo &dev, int M, int64_t N, int K, const void *Wg, const void *Wu,
                            const float *X, float *Y, cudaStream_t stream, uint32_t flags);
// One Q4_0 projection Y = X . dequant(W)^T: M = 1 with K a multiple of 256 on
// the integer tensor-core GEMV (q8_gemv.cu), otherwise the gate/up kernel with
// one matrix.
qmm_status launch_q4_gemv(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X, float *Y,
                          cudaStream_t stream, uint32_t flags);
// The M = 1 Q4_0 GEMV on the integer tensor-core kernel; false when the shape
// does not suit it (then nothing was launched).
bool launch_q4_gemv_digits(const DevInfo &dev, int64_t N, int K, const void *W, const float *X, float *Y,
                           cudaStream_t stream, uint32_t flags, qmm_status *out);
qmm_status launch_q4_gateup_unfused(const DevInfo &dev, int M, int64_t N, int K, const void *Wg, const void *Wu,
                                    const float *X, float *G, float *U, float *Y, cudaStream_t stream);

// The tiling launch_prefill picks: tokens per tile, K ranges per tile
// (cluster size), MMA stages in flight (0 for the small-M kernel), CTAs of the
// launch, and the kernel (0: tcgen05 tiles, 1: small-M mma.sync).
struct PrefillPlan {
  int mt, split, stages, ctas, kind;
};
// With `plan` set, only the tiling is computed (nothing is launched).
qmm_status launch_prefill(const DevInfo &dev, int wtype, int64_t M, int64_t N, int K, const void *W,
                          const uint16_t *X, float *Y, cudaStream_t stream, uint32_t flags,
                          PrefillPlan *plan = nullptr);

// Failure-path test: the small-M prefill kernel with the given wait limit and
// CTA 0's weight copy withheld (QMM_ERR_SHAPE if the shape does not take it).
qmm_status launch_prefill_small_withheld(const DevInfo &dev, int wtype, int64_t M, int64_t N, int K, const void *W,
                                         const uint16_t *X, float *Y, uint64_t wait_ns, cudaStream_t stream);

// Device status word of each kernel file: read and clear (synchronous).
cudaError_t q8_gemv_status(uint32_t *bits);
cudaError_t q4_gateup_status(uint32_t *bits);
cudaError_t prefill_status(uint32_t *bits);

}  // namespace qmm
