// q8_gemv.cu -- decode GEMV / small-M matmul on Q8_0 blocks, fp32 activations.
//
// Operation ("Lumen v0.2.0 -- Q8-native decode", section "Phase 7.D --
// Q8-native fused matmul"): the weights stay in the native Q8_0 block layout;
// each block's fp16 scale d is broadcast over its 32 int8 codes, the K
// direction is reduced block by block in fp32 and one output per row is
// written. No dequantised copy of W exists anywhere.
//
//   Y[m][n] = sum_b d[n][b] * sum_j q[n][b][j] * X[m][32b + j]
//
// B200 design (HBM-bound stream of 34-byte blocks):
//  * Each CTA owns a contiguous range of rows, i.e. a contiguous byte range of
//    W. One thread streams it through a ring of shared-memory stages with 1-D
//    bulk copies (cp.async.bulk, completion on an mbarrier). Copies are widened
//    to 16-byte boundaries; the <16-byte tail of the whole matrix is copied
//    with plain loads so nothing past the end of W is read.
//  * Lane l of a warp owns block column c = 32*window + l and keeps the 32
//    activations of that column in registers for the whole kernel; warps of a
//    CTA split the K blocks into 32-column windows (split-K across warps) and
//    the rows of a stage. A lane reads its block from shared memory with nine
//    aligned 32-bit loads and funnel shifts (blocks are only 2-byte aligned).
//  * int8 -> fp32 without a conversion instruction: the code byte (biased by
//    128) is placed in the mantissa of 2^23 with one byte-permute, and one
//    packed fp32x2 add removes 2^23 + 128 exactly. The products use packed
//    fp32x2 FMAs. Each block is summed in four fp32 chains, scaled by d,
//    then reduced across the warp (shuffles) and across windows (shared
//    memory) in a fixed order, so results are deterministic.
//  * Programmatic dependent launch: with the "early weights" option the ring
//    is filled before griddepcontrol.wait (W must not be written by the
//    preceding kernel); X and Y are touched only after it.
#include <algorithm>

#include "qmm_common.cuh"
#include "qmm_internal.h"

namespace qmm {
namespace {

static __device__ uint32_t g_q8_gemv_status;

constexpr int kMaxWarps = 16;
constexpr int kMaxStages = 8;
constexpr int kStageTarget = 32 * 1024;  // bytes of W per stage (aim)
constexpr int kSmemBudget = 100 * 1024;  // two CTAs of consecutive launches fit one SM
constexpr int kBarBytes = 128;           // mbarrier area at the start of shared memory

struct Params {
  const uint8_t *W;
  const float *X;
  float *Y;
  int64_t N;
  int64_t row_bytes;
  int64_t total_bytes;
  int M, K, KB;
  int grid;
  int rows_chunk;
  int stages;
  int stage_bytes;
  int stage_off;
  int cg;  // 32-column windows = ceil(KB / 32)
  int cs;  // column slots (warps side by side along K)
  int rs;  // row slots (warps side by side along N)
  int prefetch_before_wait;
};

// d * sum_j q_j x_j for one Q8_0 block at `blk` (2-byte aligned, shared memory).
template <int MP>
__device__ __forceinline__ void q8_block_dot(const uint8_t *blk, const float2 (&x2)[MP][16],
                                             float (&out)[MP]) {
  const uint32_t mis = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(blk)) & 2u;
  const uint32_t *wp = reinterpret_cast<const uint32_t *>(blk - mis);
  uint32_t w[9];
#pragma unroll
  for (int k = 0; k < 9; ++k) w[k] = wp[k];
  const uint32_t r8 = mis << 3;  // 0 or 16: bit offset of d inside w[0]
  const float d = half_bits_to_float(__funnelshift_rc(w[0], w[1], r8));
  const uint32_t sh = 16u + r8;  // 16 or 32: bit offset of qs inside (w[i+1]:w[i])
  const float2 neg_bias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
  float2 acc[MP][2];
#pragma unroll
  for (int m = 0; m < MP; ++m) acc[m][0] = acc[m][1] = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t q4 = __funnelshift_rc(w[i], w[i + 1], sh) ^ 0x80808080u;  // bytes q + 128
    float2 f01 = make_float2(__uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7440u)),
                             __uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7441u)));
    float2 f23 = make_float2(__uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7442u)),
                             __uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7443u)));
    f01 = __fadd2_rn(f01, neg_bias);  // exact: 2^23 + 128 + q - (2^23 + 128) = q
    f23 = __fadd2_rn(f23, neg_bias);
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      acc[m][0] = __ffma2_rn(f01, x2[m][2 * i], acc[m][0]);
      acc[m][1] = __ffma2_rn(f23, x2[m][2 * i + 1], acc[m][1]);
    }
  }
#pragma unroll
  for (int m = 0; m < MP; ++m)
    out[m] = d * ((acc[m][0].x + acc[m][0].y) + (acc[m][1].x + acc[m][1].y));
}

template <int MP>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) q8_gemv_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  float *red = reinterpret_cast<float *>(smem + kBarBytes);
  uint8_t *stage_mem = smem + p.stage_off;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.x) * p.N / p.grid;
  const int64_t r_end = static_cast<int64_t>(blockIdx.x + 1) * p.N / p.grid;
  const int nrows = static_cast<int>(r_end - r_begin);
  const int nchunks = (nrows + p.rows_chunk - 1) / p.rows_chunk;
  const int S = p.stages;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // Producer (thread 0): copy the bytes of chunk `c` into stage c % S.
  uint64_t policy = 0;
  int issued = 0;
  auto issue = [&](int c) {
    const int s = c % S;
    const int64_t r0 = r_begin + static_cast<int64_t>(c) * p.rows_chunk;
    const int64_t r1 = min(r0 + p.rows_chunk, r_end);
    const int64_t b0 = r0 * p.row_bytes, b1 = r1 * p.row_bytes;
    const int64_t a0 = b0 & ~int64_t(15);
    int64_t a1 = (b1 + 15) & ~int64_t(15);
    const int64_t lim = p.total_bytes & ~int64_t(15);
    uint8_t *dst = stage_mem + static_cast<int64_t>(s) * p.stage_bytes;
    if (a1 > lim) {  // last chunk of W: bytes past the last 16-byte boundary by hand
      for (int64_t t = lim; t < b1; ++t) dst[t - a0] = p.W[t];
      a1 = lim;
    }
    const uint32_t bytes = static_cast<uint32_t>(a1 - a0);
    mbar_arrive_expect_tx(&full[s], bytes);
    if (bytes) bulk_g2s(dst, p.W + a0, bytes, &full[s], policy);
  };
  const int prologue = min(S, nchunks);
  if (p.prefetch_before_wait) {
    if (tid == 0) {
      policy = l2_evict_first_policy();
      for (; issued < prologue; ++issued) issue(issued);
    }
    pdl_wait();
  } else {
    pdl_wait();
    if (tid == 0) {
      policy = l2_evict_first_policy();
      for (; issued < prologue; ++issued) issue(issued);
    }
  }
  pdl_launch_dependents();

  const int cs_w = warp % p.cs, rs_w = warp / p.cs;
  float2 x2[MP][16];
  auto load_x = [&](int m0, int cw) {
    const int c = cw * 32 + lane;
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      if (c < p.KB && m0 + m < p.M) {
        const float4 *src =
            reinterpret_cast<const float4 *>(p.X + static_cast<int64_t>(m0 + m) * p.K + c * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 v = __ldg(src + j);
          x2[m][2 * j] = make_float2(v.x, v.y);
          x2[m][2 * j + 1] = make_float2(v.z, v.w);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) x2[m][j] = make_float2(0.f, 0.f);
      }
    }
  };
  const bool x_cached = (p.cg == p.cs) && (p.M <= MP);
  if (x_cached) load_x(0, cs_w);

  bool bad = false;
  int chunk = 0;
  for (; chunk < nchunks; ++chunk) {
    const int s = chunk % S;
    const bool ok = mbar_wait(&full[s], static_cast<uint32_t>(chunk / S) & 1u);
    if (!ok) bad = true;
    const int64_t r0 = r_begin + static_cast<int64_t>(chunk) * p.rows_chunk;
    const int rows = static_cast<int>(min(static_cast<int64_t>(p.rows_chunk), r_end - r0));
    const int64_t byte0 = r0 * p.row_bytes;
    const uint8_t *base = stage_mem + static_cast<int64_t>(s) * p.stage_bytes + (byte0 & 15);
    float *redb = red + (chunk & 1) * p.M * p.cg * p.rows_chunk;
    if (ok) {
      for (int m0 = 0; m0 < p.M; m0 += MP) {
        for (int cw = cs_w; cw < p.cg; cw += p.cs) {
          if (!x_cached) load_x(m0, cw);
          const int c = cw * 32 + lane;
          const bool act = c < p.KB;
          for (int rl = rs_w; rl < rows; rl += p.rs) {
            float part[MP];
            if (act) {
              q8_block_dot<MP>(base + static_cast<int64_t>(rl) * p.row_bytes + 34 * c, x2, part);
            } else {
#pragma unroll
              for (int m = 0; m < MP; ++m) part[m] = 0.f;
            }
#pragma unroll
            for (int m = 0; m < MP; ++m) {
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) part[m] += __shfl_xor_sync(0xffffffffu, part[m], o);
            }
            if (lane == 0) {
#pragma unroll
              for (int m = 0; m < MP; ++m) {
                if (m0 + m < p.M) {
                  if (p.cg == 1)
                    p.Y[static_cast<int64_t>(m0 + m) * p.N + r0 + rl] = part[m];
                  else
                    redb[((m0 + m) * p.cg + cw) * p.rows_chunk + rl] = part[m];
                }
              }
            }
          }
        }
      }
    }
    if (__syncthreads_or(bad)) break;  // uniform exit if any thread gave up
    if (tid == 0 && issued < nchunks) {
      issue(issued);  // refill the stage everyone just finished with
      ++issued;
    }
    if (p.cg > 1) {  // sum the windows of each row in a fixed order
      for (int t = tid; t < p.M * rows; t += blockDim.x) {
        const int m = t / rows, rl = t - m * rows;
        const float *src = redb + m * p.cg * p.rows_chunk + rl;
        float v = src[0];
        for (int cw = 1; cw < p.cg; ++cw) v += src[cw * p.rows_chunk];
        p.Y[static_cast<int64_t>(m) * p.N + r0 + rl] = v;
      }
    }
  }
  if (chunk < nchunks && tid == 0) {  // error path: record, then drain copies in flight
    atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
    for (int c = chunk; c < issued; ++c)
      if (!mbar_wait(&full[c % S], static_cast<uint32_t>(c / S) & 1u))
        atomicOr(&g_q8_gemv_status, kDevTimeoutDrain);
  }
}

int align_up(int64_t v, int a) { return static_cast<int>((v + a - 1) / a * a); }

}  // namespace

qmm_status launch_q8_gemv(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X,
                          float *Y, cudaStream_t stream, uint32_t flags) {
  Params p{};
  p.W = static_cast<const uint8_t *>(W);
  p.X = X;
  p.Y = Y;
  p.N = N;
  p.M = M;
  p.K = K;
  p.KB = K / 32;
  p.row_bytes = 34ll * p.KB;
  p.total_bytes = N * p.row_bytes;
  p.cg = (p.KB + 31) / 32;
  p.cs = std::min(p.cg, kMaxWarps);
  p.rs = std::max(1, kMaxWarps / p.cs);
  const int threads = p.cs * p.rs * 32;
  p.grid = static_cast<int>(std::min<int64_t>(N, dev.sms));
  const int64_t rows_max = (N + p.grid - 1) / p.grid;
  int64_t rc = std::max<int64_t>(1, kStageTarget / p.row_bytes);
  if (rc >= p.rs) rc = rc / p.rs * p.rs;
  rc = std::min<int64_t>(rc, rows_max);
  p.rows_chunk = static_cast<int>(rc);
  // data + up to 15 bytes of alignment slack in front + over-read of the last block
  p.stage_bytes = align_up(rc * p.row_bytes + 32, 128);
  const int64_t nchunks_max = (rows_max + rc - 1) / rc;
  int S = std::max(1, kSmemBudget / p.stage_bytes);
  S = static_cast<int>(std::min<int64_t>({S, kMaxStages, nchunks_max}));
  p.stages = S;
  const int red_bytes = p.cg > 1 ? 2 * M * p.cg * p.rows_chunk * 4 : 0;
  p.stage_off = kBarBytes + align_up(red_bytes, 128);
  const size_t smem = static_cast<size_t>(p.stage_off) + static_cast<size_t>(S) * p.stage_bytes;
  if (smem > static_cast<size_t>(dev.smem_optin))
    return set_error(QMM_ERR_SHAPE, "q8_gemv: K=%d needs %zu bytes of shared memory", K, smem);
  p.prefetch_before_wait = (flags & kPrefetchBeforeWait) ? 1 : 0;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (M == 1) {
    e = cudaFuncSetAttribute(q8_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, q8_gemv_kernel<1>, p);
  } else {
    e = cudaFuncSetAttribute(q8_gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, q8_gemv_kernel<2>, p);
  }
  return cuda_check(e, "q8_gemv launch");
}

cudaError_t q8_gemv_status(uint32_t *bits) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(bits, g_q8_gemv_status, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_q8_gemv_status, &zero, sizeof(uint32_t));
  return e;
}

}  // namespace qmm
