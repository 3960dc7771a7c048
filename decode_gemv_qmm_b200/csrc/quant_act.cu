// quant_act.cu -- per-32-block Q8 quantisation of fp32 activations.
//
// The activation-quantisation step of the Q8xQ8 path ("Lumen v0.4.0 --
// shape-aware VNNI/fp32 hybrid dispatch", section "Phase 7.M -- Q8xQ8 AVX2 int
// dot"). For each block of 32 consecutive activations of a row:
//   amax = max_j |x_j|;  d = amax / 127   (IEEE binary32 division);
//   q_j  = round-half-away-from-zero(x_j / d) (IEEE binary32 division),
//          clamped to [-127, 127];  d == 0 gives all-zero codes.
// Codes and scales are bit-exact functions of X (no reciprocal, no fast math).
// A second kernel writes the ggml-compatible form: Q8_0 blocks (fp16 scale,
// then the codes) with ggml's rule, codes round(x_j * (1 / d)).
//
// One warp per block: lane j owns x_j, the block maximum is one warp-wide
// integer max over the bit patterns of |x_j| (non-negative floats order like
// their bits), and the warp writes its 32 codes as one coalesced 32-byte store.
#include <algorithm>

#include "qmm_common.cuh"
#include "qmm_internal.h"

namespace qmm {
namespace {

__global__ void __launch_bounds__(256) quantize_act_q8_kernel(const float *__restrict__ X, int8_t *__restrict__ QX,
                                                               float *__restrict__ DX, int64_t nblocks) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t b = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; b < nblocks; b += nwarps) {
    const float x = __ldg(X + b * 32 + lane);
    const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(x))));
    const float d = q8_act_scale(amax);
    QX[b * 32 + lane] = static_cast<int8_t>(q8_act_code(x, d));
    if (lane == 0) DX[b] = d;
  }
}

// Activations as Q8_0 blocks (34 bytes: fp16 d, then 32 int8 codes) with the
// ggml reference rule: d = amax / 127, id = 1 / d (0 when d == 0), q_j =
// round-half-away(x_j * id) -- each an IEEE binary32 operation -- and d stored
// as binary16 rounded to nearest even. |x_j * id| < 127.5, so the clamp never
// acts. One warp per block; lane j writes code j, lane 0 the scale.
__global__ void __launch_bounds__(256) quantize_act_q8_0_kernel(const float *__restrict__ X, uint8_t *__restrict__ XB,
                                                                 int64_t nblocks) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t b = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; b < nblocks; b += nwarps) {
    const float x = __ldg(X + b * 32 + lane);
    const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(x))));
    const float d = __fdiv_rn(amax, 127.0f);
    const float id = d != 0.0f ? __fdiv_rn(1.0f, d) : 0.0f;
    float r = roundf(__fmul_rn(x, id));
    r = fminf(fmaxf(r, -127.0f), 127.0f);
    uint8_t *blk = XB + b * 34;
    blk[2 + lane] = static_cast<uint8_t>(static_cast<int8_t>(static_cast<int>(r)));
    if (lane == 0) *reinterpret_cast<uint16_t *>(blk) = __half_as_ushort(__float2half_rn(d));
  }
}

}  // namespace

qmm_status launch_quantize_act_q8_0(const DevInfo &dev, int64_t M, int K, const float *X, uint8_t *XB,
                                    cudaStream_t stream, uint32_t flags) {
  const int64_t nblocks = M * (K / 32);
  const int threads = 256;
  const int64_t want = (nblocks + (threads / 32) - 1) / (threads / 32);
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(dev.sms) * 16));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, quantize_act_q8_0_kernel, X, XB, nblocks), "quantize_act_q8_0 launch");
}

qmm_status launch_quantize_act_q8(const DevInfo &dev, int64_t M, int K, const float *X, int8_t *QX, float *DX,
                                  cudaStream_t stream, uint32_t flags) {
  const int64_t nblocks = M * (K / 32);
  const int threads = 256;
  const int64_t want = (nblocks + (threads / 32) - 1) / (threads / 32);
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(dev.sms) * 16));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, quantize_act_q8_kernel, X, QX, DX, nblocks), "quantize_act_q8 launch");
}

}  // namespace qmm
