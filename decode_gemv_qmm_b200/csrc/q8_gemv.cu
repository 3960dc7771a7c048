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
// The same streaming kernel also runs the Q8xQ8 variant ("Lumen v0.4.0 --
// shape-aware VNNI/fp32 hybrid dispatch", section "Phase 7.M -- Q8xQ8 AVX2 int
// dot"): activations quantised to int8 per 32-block (scale DX); each block's
// dot of weight codes and activation codes is an exact int32 (eight dp4a
// steps over 4-byte words), scaled by d_w * d_x in fp32:
//
//   isum[m][n][b] = sum_j q[n][b][j] * QX[m][32b + j]   (exact)
//   Y[m][n]       = sum_b (d[n][b] * DX[m][b]) * isum[m][n][b]
//
// B200 design (a stream of 34-byte blocks; HBM-bound when the integer pipe
// keeps up):
//  * Each CTA owns a contiguous range of rows = a contiguous byte range of W.
//    A producer warp streams it through a ring of shared-memory stages with
//    1-D bulk copies (cp.async.bulk, completion counted on a "full" mbarrier);
//    consumer warps release a stage through an "empty" mbarrier, so warps
//    never wait for each other. Copies are widened to 16-byte boundaries; the
//    <16-byte tail of the whole matrix is copied with plain loads so nothing
//    past the end of W is read.
//  * Lane l of a consumer warp owns block column c = 32*window + l and keeps
//    the 32 activations of that column in registers; consumer warps split the
//    K blocks into 32-column windows (split-K across warps) and the rows of a
//    stage. A lane reads its 2-byte-aligned block with nine aligned 32-bit
//    shared loads and funnel shifts.
//  * int8 -> fp32 without a conversion instruction: the code byte (biased by
//    128) is placed in the mantissa of 2^23 by one byte-permute, and a packed
//    fp32x2 add removes 2^23 + 128 exactly; products use packed fp32x2 FMAs.
//    (On sm_100 the byte permute issues at half rate, so it bounds the
//    kernel; everything else is kept off the integer pipe where possible.)
//  * A warp processes RG rows at a time (independent chains for latency
//    hiding) and reduces their partial sums across lanes with one
//    reduce-scatter butterfly. Windows of a row are summed by the producer
//    warp in a fixed order, so results are deterministic.
//  * Programmatic dependent launch: with the "early weights" option the ring
//    is filled before griddepcontrol.wait (W must not be written by the
//    preceding kernel); X and Y are touched only after it. The CTA footprint
//    is small enough for two launches to share an SM.
//  * In Q8xQ8 mode the activations may also come as ggml Q8_0 blocks (fp16
//    scale and codes interleaved), read with half-word loads.
//
// The file also holds the M = 1 kernels that launch_q8_gemv prefers when the
// shape suits them (each described where it is defined): the fp32
// register-resident kernel, the tensor-core resident kernel, the integer
// tensor-core streaming kernel (which also serves several projections of one
// activation vector in one launch), and the fused Q8xQ8 resident kernel that
// quantises the activations itself.
#include <algorithm>
#include <type_traits>

#include "qmm_common.cuh"
#include "qmm_internal.h"
#include "qmm_tmap.h"

namespace qmm {
namespace {

static __device__ uint32_t g_q8_gemv_status;

constexpr int kMaxStages = 8;
constexpr int kStageTarget = 16 * 1024;  // bytes of W per stage (aim)
constexpr int kSmemBudget = 96 * 1024;   // two CTAs of consecutive launches fit one SM
constexpr int kBarBytes = 256;           // full[8] + empty[8] mbarriers
constexpr int kMaxConsumerWarps = 16;
constexpr int kPanelBytes = 32 * 1024;  // activation panel kept in shared memory up to this size (256 rows)
constexpr int64_t kMmaMinSliceWeights = 16384;  // per-CTA weights above which M = 1 uses tensor cores
constexpr int kMmaMaxK = 2048;  // longer rows: the per-CTA activation split costs more than it saves

enum : int { kModeF32 = 0, kModeQ8 = 1, kModeQ8Dots = 2 };

struct alignas(64) Params {
  CUtensorMap xmap;  // X viewed as (M*K/32) rows of 128 bytes, 128-byte swizzle
  const uint8_t *W;
  const float *X;    // fp32 activations (kModeF32)
  const int8_t *QX;  // int8 activation codes (kModeQ8, kModeQ8Dots)
  const float *DX;   // per-block activation scales (kModeQ8)
  const uint8_t *XB; // kModeQ8 alternative to QX / DX: activations as Q8_0 blocks (fp16 scale)
  float *Y;
  int32_t *isum;     // block dots out (kModeQ8Dots)
  int64_t N;
  int64_t row_bytes;
  int64_t total_bytes;
  int M, K, KB;
  int grid;
  int rows_chunk;
  int stages;
  int stage_bytes;
  int stage_off;
  int xs_off;  // byte offset of the activation panel in shared memory (0 = no panel)
  int xs_rows;  // rows of 32 activations in the panel (M * K / 32)
  int xs_bytes;  // panel bytes
  int cg;  // 32-column windows = ceil(KB / 32)
  int cs;  // column slots (consumer warps side by side along K)
  int rs;  // row slots (consumer warps side by side along N)
  int prefetch_before_wait;
  // failure-path test only (defaults: kWaitLimitNs, 0): the limit of every
  // barrier wait, and whether CTA 0 withholds the copy of its first weight stage
  uint64_t wait_ns;
  int withhold;
};

// Convert four int8 codes (one 32-bit word) and multiply-accumulate them
// against four activations held as two float2 pairs.
__device__ __forceinline__ void fma4(uint32_t qword, const float2 &x01, const float2 &x23, float2 &a01,
                                     float2 &a23) {
  const float2 neg_bias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
  const uint32_t q4 = qword ^ 0x80808080u;                        // bytes q + 128
  float2 f01 = make_float2(__uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7440u)),
                           __uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7441u)));
  float2 f23 = make_float2(__uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7442u)),
                           __uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7443u)));
  f01 = __fadd2_rn(f01, neg_bias);  // exact: 2^23 + 128 + q - (2^23 + 128) = q
  f23 = __fadd2_rn(f23, neg_bias);
  a01 = __ffma2_rn(f01, x01, a01);
  a23 = __ffma2_rn(f23, x23, a23);
}

// d * sum_j q_j x_j of one Q8_0 block at shared address `sa` (2-byte aligned)
// for MP activation rows. Each 4-weight word feeds its own accumulator pair;
// the pairs are summed in a fixed tree, which keeps the dependent chain short.
template <int MP>
__device__ __forceinline__ void q8_block_dot(uint32_t sa, const float2 (&x2)[MP][16], float (&out)[MP]) {
  const uint32_t mis = sa & 2u;
  const uint32_t wa = sa - mis;
  uint32_t w[9];
#pragma unroll
  for (int k = 0; k < 9; ++k) w[k] = lds_u32(wa + 4 * k);
  const uint32_t r8 = mis << 3;  // 0 or 16: bit offset of d inside w[0]
  const float d = half_bits_to_float(__funnelshift_rc(w[0], w[1], r8));
  const uint32_t sh = 16u + r8;  // 16 or 32: bit offset of qs inside (w[i+1]:w[i])
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    float2 a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      a[i] = b[i] = make_float2(0.f, 0.f);
      fma4(__funnelshift_rc(w[i], w[i + 1], sh), x2[m][2 * i], x2[m][2 * i + 1], a[i], b[i]);
    }
#pragma unroll
    for (int st = 1; st < 8; st *= 2) {
#pragma unroll
      for (int i = 0; i < 8; i += 2 * st) {
        a[i] = __fadd2_rn(a[i], a[i + st]);
        b[i] = __fadd2_rn(b[i], b[i + st]);
      }
    }
    const float2 t = __fadd2_rn(a[0], b[0]);
    out[m] = d * (t.x + t.y);
  }
}

// Exact int32 dot of one Q8_0 block's codes with MP rows of int8 activation
// codes (eight 4-byte words each); also returns the block's scale d.
template <int MP>
__device__ __forceinline__ float q8q8_block_isum(uint32_t sa, const uint32_t (&qx)[MP][8], int (&isum)[MP]) {
  const uint32_t mis = sa & 2u;
  const uint32_t wa = sa - mis;
  uint32_t w[9];
#pragma unroll
  for (int k = 0; k < 9; ++k) w[k] = lds_u32(wa + 4 * k);
  const uint32_t r8 = mis << 3;
  const float d = half_bits_to_float(__funnelshift_rc(w[0], w[1], r8));
  const uint32_t sh = 16u + r8;
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    int s0 = 0, s1 = 0;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      s0 = __dp4a(static_cast<int>(__funnelshift_rc(w[i], w[i + 1], sh)), static_cast<int>(qx[m][i]), s0);
      s1 = __dp4a(static_cast<int>(__funnelshift_rc(w[i + 1], w[i + 2], sh)), static_cast<int>(qx[m][i + 1]), s1);
    }
    isum[m] = s0 + s1;  // |isum| <= 32 * 128 * 128 = 2^19: exact
  }
  return d;
}

// Reduce V per-lane values over the 32 lanes with a reduce-scatter butterfly:
// afterwards lane l holds the total of value index vidx(l) (V in {1, 2, 4}).
template <int V>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[V], int lane) {
  if constexpr (V == 4) {
    const bool hi16 = lane & 16;
    float k0 = hi16 ? v[2] : v[0], k1 = hi16 ? v[3] : v[1];
    const float s0 = hi16 ? v[0] : v[2], s1 = hi16 ? v[1] : v[3];
    k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    const bool hi8 = lane & 8;
    float k = hi8 ? k1 : k0;
    k += __shfl_xor_sync(0xffffffffu, hi8 ? k0 : k1, 8);
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
    return k;  // value index ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1)
  } else if constexpr (V == 2) {
    const bool hi16 = lane & 16;
    float k = hi16 ? v[1] : v[0];
    k += __shfl_xor_sync(0xffffffffu, hi16 ? v[0] : v[1], 16);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
    return k;  // value index (lane >> 4) & 1
  } else {
    float k = v[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
    return k;
  }
}
template <int V>
__device__ __forceinline__ int scatter_index(int lane) {
  if constexpr (V == 4) return ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
  if constexpr (V == 2) return (lane >> 4) & 1;
  return 0;
}
template <int V>
__device__ __forceinline__ bool scatter_writer(int lane) {
  if constexpr (V == 4) return (lane & 7) == 0;
  if constexpr (V == 2) return (lane & 15) == 0;
  return lane == 0;
}

// MODE: activation kind; MP activation rows per pass (1 or 2); RG weight rows
// per warp step.
template <int MODE, int MP, int RG>
__global__ void __launch_bounds__((kMaxConsumerWarps + 1) * 32) q8_gemv_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + kMaxStages;
  uint64_t *xbar = empty + kMaxStages;
  float *red = reinterpret_cast<float *>(smem + kBarBytes);
  uint8_t *stage_mem = smem + p.stage_off;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nconsumer = p.cs * p.rs;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.x) * p.N / p.grid;
  const int64_t r_end = static_cast<int64_t>(blockIdx.x + 1) * p.N / p.grid;
  const int nrows = static_cast<int>(r_end - r_begin);
  const int nchunks = (nrows + p.rows_chunk - 1) / p.rows_chunk;
  const int S = p.stages;
  const int red_stride = p.M * p.cg * p.rows_chunk;  // floats of partials per stage

  // Let the next launch in the stream start its prologue (weight prefetch) as
  // soon as SM resources allow; its own griddepcontrol.wait still orders it.
  pdl_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], nconsumer);
    }
    mbar_init(xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint64_t policy = 0, policy_x = 0;
    if constexpr (MODE != kModeF32) policy_x = l2_evict_last_policy();
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
      if (p.withhold && blockIdx.x == 0 && c == 0) return;  // failure-path test: stage 0 never fills
      mbar_arrive_expect_tx(&full[s], bytes);
      if (bytes) bulk_g2s(dst, p.W + a0, bytes, &full[s], policy);
    };
    // Sum the window partials of chunk c (all consumers have released it).
    auto finish = [&](int c) {
      if (p.cg == 1 || MODE == kModeQ8Dots) return;
      const int s = c % S;
      const int64_t r0 = r_begin + static_cast<int64_t>(c) * p.rows_chunk;
      const int rows = static_cast<int>(min(static_cast<int64_t>(p.rows_chunk), r_end - r0));
      const float *rb = red + s * red_stride;
      for (int t = lane; t < p.M * rows; t += 32) {
        const int m = t / rows, rl = t - m * rows;
        const float *src = rb + m * p.cg * p.rows_chunk + rl;
        float v = src[0];
        for (int cw = 1; cw < p.cg; ++cw) v += src[cw * p.rows_chunk];
        p.Y[static_cast<int64_t>(m) * p.N + r0 + rl] = v;
      }
    };
    // The activation panel: one 2-D TMA load with the 128-byte swizzle, issued
    // as soon as the preceding grid has finished (X may be its output).
    // (int8 activation codes: one plain bulk copy of the M x K bytes.)
    auto issue_x = [&]() {
      if (p.xs_off) {
        mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(p.xs_bytes));
        if constexpr (MODE == kModeF32)
          tma_load_2d(smem + p.xs_off, &p.xmap, 0, 0, xbar);
        else
          bulk_g2s(smem + p.xs_off, p.QX, static_cast<uint32_t>(p.xs_bytes), xbar, policy_x);
      }
    };
    const int prologue = min(S, nchunks);
    if (p.prefetch_before_wait) {
      if (lane == 0) {
        policy = l2_evict_first_policy();
        for (int c = 0; c < prologue; ++c) issue(c);
      }
      pdl_wait();
      if (lane == 0) issue_x();
    } else {
      pdl_wait();
      if (lane == 0) {
        issue_x();
        policy = l2_evict_first_policy();
        for (int c = 0; c < prologue; ++c) issue(c);
      }
    }
    bool ok = true;
    int issued = prologue;
    for (int c = 0; c < nchunks && ok; ++c) {
      // chunk c is released once every consumer warp arrived on empty[c % S]
      ok = mbar_wait(&empty[c % S], static_cast<uint32_t>(c / S) & 1u, p.wait_ns);
      if (!ok) break;
      __syncwarp();
      finish(c);
      __syncwarp();
      if (lane == 0 && issued < nchunks) {
        issue(issued);
        ++issued;
      }
    }
    if (!ok && lane == 0) {  // error path: record, then drain copies still in flight
      atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
      for (int c = max(0, issued - S); c < issued; ++c)
        if (!mbar_wait(&full[c % S], static_cast<uint32_t>(c / S) & 1u, p.wait_ns))
          atomicOr(&g_q8_gemv_status, kDevTimeoutDrain);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  pdl_wait();
  const int cwarp = warp - 1;
  const int cs_w = cwarp % p.cs, rs_w = cwarp / p.cs;
  // Activation panel (when present): row r = m * KB + c holds the 32
  // activations of block column c of token m; the TMA's 128-byte swizzle puts
  // 16-byte unit u of row r at unit u ^ (r & 7), so the eight lanes of a
  // shared-memory phase (consecutive c) read eight different bank groups.
  const bool xs = p.xs_off != 0;
  const uint32_t xs_sa = smem_u32(smem) + p.xs_off;
  if (xs && !mbar_wait(xbar, 0, p.wait_ns)) {
    if (lane == 0) atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
    return;
  }
  // Per-lane activations of its block column: fp32 values, or int8 codes
  // (eight words) and the block's activation scale.
  float2 x2[MP][16];
  uint32_t qx[MP][8];
  float dxr[MP];
  auto load_x = [&](int m0, int cw) {
    const int c = cw * 32 + lane;
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      const bool valid = c < p.KB && m0 + m < p.M;
      if constexpr (MODE == kModeF32) {
        if (valid) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int row = (m0 + m) * p.KB + c;
            const float4 v = xs ? lds_f4(xs_sa + 16u * (row * 8 + (j ^ (row & 7))))
                                : __ldg(reinterpret_cast<const float4 *>(p.X + static_cast<int64_t>(m0 + m) * p.K) + 8 * c + j);
            x2[m][2 * j] = make_float2(v.x, v.y);
            x2[m][2 * j + 1] = make_float2(v.z, v.w);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) x2[m][j] = make_float2(0.f, 0.f);
        }
      } else {
        if (valid && p.XB) {
          // a Q8_0 activation block: the fp16 scale, then the 32 codes as 16
          // half-words (2-byte aligned: exactly the block's 34 bytes are read)
          const uint16_t *bp =
              reinterpret_cast<const uint16_t *>(p.XB + (static_cast<int64_t>(m0 + m) * p.KB + c) * 34);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            qx[m][j] = static_cast<uint32_t>(__ldg(bp + 1 + 2 * j)) | (static_cast<uint32_t>(__ldg(bp + 2 + 2 * j)) << 16);
          dxr[m] = half_bits_to_float(__ldg(bp));
        } else if (valid) {
          const int64_t off = static_cast<int64_t>(m0 + m) * p.K + 32 * c;
          uint4 lo, hi;
          if (xs) {
            lo = lds_u4(xs_sa + static_cast<uint32_t>(off));
            hi = lds_u4(xs_sa + static_cast<uint32_t>(off) + 16u);
          } else {
            lo = __ldg(reinterpret_cast<const uint4 *>(p.QX + off));
            hi = __ldg(reinterpret_cast<const uint4 *>(p.QX + off) + 1);
          }
          qx[m][0] = lo.x; qx[m][1] = lo.y; qx[m][2] = lo.z; qx[m][3] = lo.w;
          qx[m][4] = hi.x; qx[m][5] = hi.y; qx[m][6] = hi.z; qx[m][7] = hi.w;
          dxr[m] = (MODE == kModeQ8) ? __ldg(p.DX + static_cast<int64_t>(m0 + m) * p.KB + c) : 0.f;
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) qx[m][j] = 0u;
          dxr[m] = 0.f;
        }
      }
    }
  };
  const bool x_cached = (p.cg == p.cs) && (p.M <= MP);
  if (x_cached) load_x(0, cs_w);

  for (int c = 0; c < nchunks; ++c) {
    const int s = c % S;
    if (!mbar_wait(&full[s], static_cast<uint32_t>(c / S) & 1u, p.wait_ns)) {
      if (lane == 0) atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
      return;  // the producer times out on this warp's missing arrival and drains
    }
    const int64_t r0 = r_begin + static_cast<int64_t>(c) * p.rows_chunk;
    const int rows = static_cast<int>(min(static_cast<int64_t>(p.rows_chunk), r_end - r0));
    const uint32_t base = smem_u32(stage_mem) + s * p.stage_bytes + static_cast<uint32_t>((r0 * p.row_bytes) & 15);
    float *rb = red + s * red_stride;
    for (int m0 = 0; m0 < p.M; m0 += MP) {
      for (int cw = cs_w; cw < p.cg; cw += p.cs) {
        if (!x_cached) load_x(m0, cw);
        const int col = cw * 32 + lane;
        const bool act = col < p.KB;
        // Lanes past the last block column and rows past the chunk compute on a
        // valid in-bounds block and discard the result: no branch, so the RG
        // block dots of a step can be interleaved by the scheduler.
        const uint32_t col_off = 34u * static_cast<uint32_t>(act ? col : p.KB - 1);
        for (int rl = rs_w * RG; rl < rows; rl += p.rs * RG) {
          float part[RG * MP];
#pragma unroll
          for (int g = 0; g < RG; ++g) {
            const bool ok = act && rl + g < rows;
            const int row = min(rl + g, rows - 1);
            const uint32_t sa = base + static_cast<uint32_t>(row * p.row_bytes) + col_off;
            float o[MP];
            if constexpr (MODE == kModeF32) {
              q8_block_dot<MP>(sa, x2, o);
            } else {
              int is[MP];
              const float d = q8q8_block_isum<MP>(sa, qx, is);
#pragma unroll
              for (int m = 0; m < MP; ++m) {
                if constexpr (MODE == kModeQ8Dots) {
                  if (ok && m0 + m < p.M)
                    p.isum[((static_cast<int64_t>(m0 + m) * p.N) + r0 + rl + g) * p.KB + col] = is[m];
                  o[m] = 0.f;
                } else {
                  o[m] = (d * dxr[m]) * static_cast<float>(is[m]);
                }
              }
            }
#pragma unroll
            for (int m = 0; m < MP; ++m) part[g * MP + m] = ok ? o[m] : 0.f;
          }
          if constexpr (MODE == kModeQ8Dots) continue;
          const float tot = warp_reduce_scatter<RG * MP>(part, lane);
          if (scatter_writer<RG * MP>(lane)) {
            const int v = scatter_index<RG * MP>(lane);
            const int g = v / MP, m = m0 + v % MP;
            if (rl + g < rows && m < p.M) {
              if (p.cg == 1)
                p.Y[static_cast<int64_t>(m) * p.N + r0 + rl + g] = tot;
              else
                rb[(m * p.cg + cw) * p.rows_chunk + rl + g] = tot;
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}


// ---------------------------------------------------------------------------
// Resident variant (M = 1, small weight slices): a chain of dependent decode
// GEMVs is latency-bound, and only the FMAs need the activations. So a CTA
// loads its whole weight slice (before griddepcontrol.wait when allowed),
// decodes every block it owns into registers as exact fp32 codes (plus the
// block scale), and after the activations arrive does only packed FMAs, one
// multiply by d per block, one reduce-scatter and the store. With four rows a
// warp (long rows) the codes are held as exact fp16 pairs instead, half the
// registers, and widened to fp32 after the wait (the products are the same).
//
// Warp (window cw, row slot k) owns block column 32*cw + lane of rows
// r_begin + k + U*... (U rows, stride wpw); windows of a row are added by the
// CTA in window order. Deterministic.

struct alignas(64) RParams {
  CUtensorMap xmap;  // X as K/32 rows of 128 bytes, 128-byte swizzle
  const uint8_t *W;
  float *Y;
  int64_t N;
  int64_t row_bytes;
  int64_t total_bytes;
  int K, KB;
  int grid;
  int cg;    // 32-column windows
  int wpw;   // warps per window
  int xs_off;      // swizzled activation panel (1024-aligned)
  int red_off;     // window partials (cg > 1)
  int w_off;       // raw weight slice
  int max_rows;    // rows per CTA upper bound
  int prefetch_before_wait;
  // fused Q8xQ8 only: the CTA's quantised activations, and where CTA 0 also writes them
  int qx_off, dx_off;
  int8_t *QXo;
  float *DXo;
  int32_t *isum;  // fused Q8xQ8, dump instance only: the exact block dots, N x K/32
};

template <int U>
// At most 112 registers for U = 4: 320 threads x 112 fit one SM beside a CTA
// of the tensor-core resident kernel (224 x 128), so the down projection can
// start and fetch its weights while the preceding up projection runs.
__global__ void __maxnreg__(U == 4 ? 112 : 128)
q8_gemv_resident_kernel(const __grid_constant__ RParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *wbar = reinterpret_cast<uint64_t *>(smem);
  uint64_t *xbar = wbar + 1;
  float *red = reinterpret_cast<float *>(smem + p.red_off);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.x) * p.N / p.grid;
  const int64_t r_end = static_cast<int64_t>(blockIdx.x + 1) * p.N / p.grid;
  const int rows = static_cast<int>(r_end - r_begin);
  const int64_t b0 = r_begin * p.row_bytes, b1 = r_end * p.row_bytes;
  const int64_t a0 = b0 & ~int64_t(15);

  pdl_launch_dependents();
  if (tid == 0) {
    mbar_init(wbar, 1);
    mbar_init(xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue_w = [&]() {
    int64_t a1 = (b1 + 15) & ~int64_t(15);
    const int64_t lim = p.total_bytes & ~int64_t(15);
    uint8_t *dst = smem + p.w_off;
    if (a1 > lim) {  // bytes past the last 16-byte boundary of W by hand
      for (int64_t t = lim; t < b1; ++t) dst[t - a0] = p.W[t];
      a1 = lim;
    }
    const uint32_t bytes = static_cast<uint32_t>(a1 - a0);
    mbar_arrive_expect_tx(wbar, bytes);
    const uint64_t pol = l2_evict_first_policy();
    constexpr uint32_t kPiece = 8192;  // several copies in flight
    for (uint32_t o = 0; o < bytes; o += kPiece)
      bulk_g2s(dst + o, p.W + a0 + o, min(kPiece, bytes - o), wbar, pol);
  };
  auto issue_x = [&]() {
    mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(p.KB) * 128u);
    tma_load_2d(smem + p.xs_off, &p.xmap, 0, 0, xbar);
  };
  if (tid == 0) {
    if (p.prefetch_before_wait) {
      issue_w();
      pdl_wait();
      issue_x();
    } else {
      pdl_wait();
      issue_x();
      issue_w();
    }
  }

  // ---- decode the owned blocks into registers (does not need X)
  const int cw = warp % p.cg, k = warp / p.cg;
  const int col = cw * 32 + lane;
  const bool act = col < p.KB;
  const uint32_t wbase = smem_u32(smem + p.w_off) + static_cast<uint32_t>(b0 - a0);
  // U = 4 (long rows, 168 registers with fp32 codes): the codes are kept as
  // exact fp16 pairs, half the registers, widened to fp32 after the wait
  constexpr bool kH = U == 4;
  float2 wq[kH ? 1 : U][16];
  uint32_t wh[kH ? U : 1][16];
  float wd[U];
  bool ok = mbar_wait(wbar, 0);
  if (!ok && lane == 0) atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int rl = k + u * p.wpw;
    if (ok && act && rl < rows) {
      const uint32_t sa = wbase + static_cast<uint32_t>(rl * p.row_bytes) + 34u * col;
      const uint32_t mis = sa & 2u, wa = sa - mis;
      uint32_t w[9];
#pragma unroll
      for (int i = 0; i < 9; ++i) w[i] = lds_u32(wa + 4 * i);
      const uint32_t r8 = mis << 3, sh = 16u + r8;
      wd[u] = half_bits_to_float(__funnelshift_rc(w[0], w[1], r8));
      const float2 nb = make_float2(-8388736.0f, -8388736.0f);
      const __half2 k1152 = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t q4 = __funnelshift_rc(w[i], w[i + 1], sh) ^ 0x80808080u;
        if constexpr (kH) {
          // 0x6400 | (q + 128) is 1024 + q + 128 in fp16; minus 1152: q, exact
          uint32_t t01 = __byte_perm(q4, 0x6464u, 0x5140u), t23 = __byte_perm(q4, 0x6464u, 0x5342u);
          __half2 h01 = __hsub2(*reinterpret_cast<__half2 *>(&t01), k1152);
          __half2 h23 = __hsub2(*reinterpret_cast<__half2 *>(&t23), k1152);
          wh[u][2 * i] = *reinterpret_cast<uint32_t *>(&h01);
          wh[u][2 * i + 1] = *reinterpret_cast<uint32_t *>(&h23);
        } else {
          const float2 f01 = make_float2(__uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7440u)),
                                         __uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7441u)));
          const float2 f23 = make_float2(__uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7442u)),
                                         __uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7443u)));
          wq[kH ? 0 : u][2 * i] = __fadd2_rn(f01, nb);  // exact codes q
          wq[kH ? 0 : u][2 * i + 1] = __fadd2_rn(f23, nb);
        }
      }
    } else {
      wd[u] = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if constexpr (kH) wh[u][i] = 0u;
        else wq[kH ? 0 : u][i] = make_float2(0.f, 0.f);
      }
    }
  }

  // ---- activations (after the preceding grid has finished)
  pdl_wait();
  float2 x2[16];
  if (ok && !mbar_wait(xbar, 0)) {
    ok = false;
    if (lane == 0) atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
  }
  if (ok && act) {
    const uint32_t xa = smem_u32(smem + p.xs_off);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 v = lds_f4(xa + 16u * (col * 8 + (j ^ (col & 7))));
      x2[2 * j] = make_float2(v.x, v.y);
      x2[2 * j + 1] = make_float2(v.z, v.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) x2[j] = make_float2(0.f, 0.f);
  }

  // ---- products: four packed accumulators per row, then a fixed tree
  float part[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    float2 a[4];
    auto wv = [&](int i) -> float2 {
      if constexpr (kH) return __half22float2(*reinterpret_cast<const __half2 *>(&wh[u][i]));
      else return wq[kH ? 0 : u][i];
    };
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = __fmul2_rn(wv(i), x2[i]);
#pragma unroll
    for (int i = 4; i < 16; ++i) a[i & 3] = __ffma2_rn(wv(i), x2[i], a[i & 3]);
    const float2 t = __fadd2_rn(__fadd2_rn(a[0], a[1]), __fadd2_rn(a[2], a[3]));
    part[u] = wd[u] * (t.x + t.y);
  }
  if (!ok && tid == 0) {  // error path: give copies still in flight a bounded chance to land
    if (!mbar_wait(wbar, 0) || !mbar_wait(xbar, 0)) atomicOr(&g_q8_gemv_status, kDevTimeoutDrain);
  }
  const float tot = warp_reduce_scatter<U>(part, lane);
  const int ui = scatter_index<U>(lane);
  const int rl = k + ui * p.wpw;
  if (p.cg == 1) {
    if (scatter_writer<U>(lane) && rl < rows) p.Y[r_begin + rl] = tot;
    return;
  }
  if (scatter_writer<U>(lane) && rl < rows) red[cw * p.max_rows + rl] = tot;
  __syncthreads();
  for (int r = tid; r < rows; r += blockDim.x) {
    float v = red[r];
    for (int c = 1; c < p.cg; ++c) v += red[c * p.max_rows + r];
    p.Y[r_begin + r] = v;
  }
}

// ---------------------------------------------------------------------------
// Fused Q8xQ8 resident variant (M = 1): the activation quantisation of
// qmm_quantize_act_q8 done by every CTA into shared memory (same binary32
// operations, so the same codes), then the exact int32 block dots on raw code
// words held in registers. Q8 codes are one byte per weight, so a CTA keeps
// its whole slice as raw words (8 registers per block and row) -- a quarter of
// the fp32 resident form -- loaded and unpacked before the dependency wait; the
// work left after it is the quantisation of X, eight dp4a per block and row,
// one multiply by d_w * d_x, the reductions and the store.
//
//   isum[n][b] = sum_j q[n][b][j] * qx[32b + j]      (exact int32)
//   Y[n]       = sum_b (d[n][b] * dx[b]) * isum[n][b]
//
// Quantisation: eight lanes per 32-block (four activations each, read from
// the 128-byte-swizzled panel), the block maximum by a three-step shuffle max
// over |x| bit patterns, then q8_act_scale / q8_act_code. CTA 0 also writes the
// codes and scales to QX / DX.

// DOTS: the test instance, which also writes every exact block dot to p.isum
// (the arithmetic is the same code).
template <int U, bool DOTS>
__global__ void __launch_bounds__(512, 1) q8q8_resident_kernel(const __grid_constant__ RParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *wbar = reinterpret_cast<uint64_t *>(smem);
  uint64_t *xbar = wbar + 1;
  float *red = reinterpret_cast<float *>(smem + p.red_off);
  uint8_t *qx = smem + p.qx_off;
  float *dx = reinterpret_cast<float *>(smem + p.dx_off);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.x) * p.N / p.grid;
  const int64_t r_end = static_cast<int64_t>(blockIdx.x + 1) * p.N / p.grid;
  const int rows = static_cast<int>(r_end - r_begin);
  const int64_t b0 = r_begin * p.row_bytes, b1 = r_end * p.row_bytes;
  const int64_t a0 = b0 & ~int64_t(15);

  pdl_launch_dependents();
  if (tid == 0) {
    mbar_init(wbar, 1);
    mbar_init(xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue_w = [&]() {
    int64_t a1 = (b1 + 15) & ~int64_t(15);
    const int64_t lim = p.total_bytes & ~int64_t(15);
    uint8_t *dst = smem + p.w_off;
    if (a1 > lim) {  // bytes past the last 16-byte boundary of W by hand
      for (int64_t t = lim; t < b1; ++t) dst[t - a0] = p.W[t];
      a1 = lim;
    }
    const uint32_t bytes = static_cast<uint32_t>(a1 - a0);
    mbar_arrive_expect_tx(wbar, bytes);
    const uint64_t pol = l2_evict_first_policy();
    constexpr uint32_t kPiece = 8192;  // several copies in flight
    for (uint32_t o = 0; o < bytes; o += kPiece)
      bulk_g2s(dst + o, p.W + a0 + o, min(kPiece, bytes - o), wbar, pol);
  };
  auto issue_x = [&]() {
    mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(p.KB) * 128u);
    tma_load_2d(smem + p.xs_off, &p.xmap, 0, 0, xbar);
  };
  if (tid == 0) {
    if (p.prefetch_before_wait) {
      issue_w();
      pdl_wait();
      issue_x();
    } else {
      pdl_wait();
      issue_x();
      issue_w();
    }
  }

  // ---- raw code words and block scales into registers (does not need X)
  const int cw = warp % p.cg, k = warp / p.cg;
  const int col = cw * 32 + lane;
  const bool act = col < p.KB;
  const uint32_t wbase = smem_u32(smem + p.w_off) + static_cast<uint32_t>(b0 - a0);
  uint32_t wc[U][8];
  float wd[U];
  bool ok = mbar_wait(wbar, 0);
  if (!ok && lane == 0) atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int rl = k + u * p.wpw;
    if (ok && act && rl < rows) {
      const uint32_t sa = wbase + static_cast<uint32_t>(rl * p.row_bytes) + 34u * col;
      const uint32_t mis = sa & 2u, wa = sa - mis;
      uint32_t w[9];
#pragma unroll
      for (int i = 0; i < 9; ++i) w[i] = lds_u32(wa + 4 * i);
      const uint32_t r8 = mis << 3, sh = 16u + r8;
      wd[u] = half_bits_to_float(__funnelshift_rc(w[0], w[1], r8));
#pragma unroll
      for (int i = 0; i < 8; ++i) wc[u][i] = __funnelshift_rc(w[i], w[i + 1], sh);
    } else {
      wd[u] = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) wc[u][i] = 0u;
    }
  }

  // ---- activations (after the preceding grid has finished), quantised by the CTA
  pdl_wait();
  if (ok && !mbar_wait(xbar, 0)) {
    ok = false;
    if (lane == 0) atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
  }
  const uint32_t xa = smem_u32(smem + p.xs_off);
  const int units = p.KB * 8;  // (block, unit of four activations)
#pragma unroll 1
  for (int base = warp * 32; base < units; base += blockDim.x) {  // uniform per warp: it shuffles
    const int it = base + lane;
    const int c = it >> 3, u = it & 7;
    const bool have = ok && it < units;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (have) v = lds_f4(xa + 16u * (c * 8 + (u ^ (c & 7))));
    uint32_t m = max(max(__float_as_uint(fabsf(v.x)), __float_as_uint(fabsf(v.y))),
                     max(__float_as_uint(fabsf(v.z)), __float_as_uint(fabsf(v.w))));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
    const float d = q8_act_scale(__uint_as_float(m));
    const uint32_t word = (static_cast<uint32_t>(q8_act_code(v.x, d)) & 0xffu) |
                          ((static_cast<uint32_t>(q8_act_code(v.y, d)) & 0xffu) << 8) |
                          ((static_cast<uint32_t>(q8_act_code(v.z, d)) & 0xffu) << 16) |
                          (static_cast<uint32_t>(q8_act_code(v.w, d)) << 24);
    if (have) {
      *reinterpret_cast<uint32_t *>(qx + 32 * c + 4 * u) = word;
      if (u == 0) dx[c] = d;
      if (blockIdx.x == 0) {  // the codes and scales for the caller
        *reinterpret_cast<uint32_t *>(p.QXo + 32 * c + 4 * u) = word;
        if (u == 0) p.DXo[c] = d;
      }
    }
  }
  __syncthreads();

  // ---- exact int32 block dots, then (d_w * d_x) * isum
  uint32_t qa[8];
  float dxv = 0.f;
  if (ok && act) {
    const uint4 lo = *reinterpret_cast<const uint4 *>(qx + 32 * col);
    const uint4 hi = *reinterpret_cast<const uint4 *>(qx + 32 * col + 16);
    qa[0] = lo.x; qa[1] = lo.y; qa[2] = lo.z; qa[3] = lo.w;
    qa[4] = hi.x; qa[5] = hi.y; qa[6] = hi.z; qa[7] = hi.w;
    dxv = dx[col];
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) qa[i] = 0u;
  }
  float part[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    int s0 = 0, s1 = 0;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      s0 = __dp4a(static_cast<int>(wc[u][i]), static_cast<int>(qa[i]), s0);
      s1 = __dp4a(static_cast<int>(wc[u][i + 1]), static_cast<int>(qa[i + 1]), s1);
    }
    part[u] = (wd[u] * dxv) * static_cast<float>(s0 + s1);  // |isum| <= 2^19: exact in fp32
    if constexpr (DOTS) {
      const int rl = k + u * p.wpw;
      if (ok && act && rl < rows) p.isum[(r_begin + rl) * p.KB + col] = s0 + s1;
    }
  }
  if (!ok && tid == 0) {  // error path: give copies still in flight a bounded chance to land
    if (!mbar_wait(wbar, 0) || !mbar_wait(xbar, 0)) atomicOr(&g_q8_gemv_status, kDevTimeoutDrain);
  }
  const float tot = warp_reduce_scatter<U>(part, lane);
  const int ui = scatter_index<U>(lane);
  const int rl = k + ui * p.wpw;
  if (p.cg == 1) {
    if (scatter_writer<U>(lane) && rl < rows) p.Y[r_begin + rl] = tot;
    return;
  }
  if (scatter_writer<U>(lane) && rl < rows) red[cw * p.max_rows + rl] = tot;
  __syncthreads();
  for (int r = tid; r < rows; r += blockDim.x) {
    float v = red[r];
    for (int c = 1; c < p.cg; ++c) v += red[c * p.max_rows + r];
    p.Y[r_begin + r] = v;
  }
}

// ---------------------------------------------------------------------------
// Tensor-core resident variant (M = 1) for weight slices whose fp32 register
// form would fill the SM: the next launch in the stream could then not start
// streaming its own weights before this one exits. Here the codes are held as
// fp16 (exact for int8), half that footprint, so two consecutive launches
// share an SM and the next one's weights land and are converted while this one
// computes. Every CTA splits the whole activation vector once, so this only
// pays for short rows (measured on B200 in a chain of dependent launches:
// 896 -> 4864 at 2.80 us per GEMV against 3.19 us for the fp32 resident
// kernel; 4864 -> 896 at 4.05 us against 3.38 us, so long rows stay there).
//
//  * mma.m16n8k16 with the weights as A: rows 0..7 of A are the eight rows of
//    a row group at block b, rows 8..15 the same rows at block b + 1. Thread
//    (g, t) holds codes 8t..8t+7 of row g at both blocks; inside a block the k
//    order is free, so with c0 c1 c2 c3 = codes 8t+4s .. 8t+4s+3 (slice s) the
//    register at k = 2t, 2t+1 holds (c0, c2) and the one at k = 2t+8, 2t+9
//    holds (c1, c3). A masked xor puts each biased byte in the mantissa of
//    1024 and one packed fp16 subtraction of 1152 leaves the code exactly.
//  * Activations as B: column 0/1 = hi/lo parts of block b, column 2/3 = those
//    of block b + 1 (columns 4..7 repeat 0..3). Each 32-block is scaled by
//    2^(141 - E_b), E_b the biased exponent of its largest |x|, so its largest
//    element lies in [2^14, 2^15), and split (Veltkamp) into hi with 11
//    significant bits and lo = v - hi, both then rounded to fp16:
//    |v - hi - lo| <= 2^-23 |v| + 2^-25. Products are exact in fp32. The parts
//    are built once per CTA, in place over the activation vector in shared
//    memory, laid out so that each lane reads its B registers with one 16-byte
//    load.
//  * C row g, columns 0 + 1 (thread (g, 0)) is row g's dot with block b;
//    C row g + 8, columns 2 + 3 (thread (g, 1)) the dot with block b + 1. Each
//    adds (dot * d) * 2^(E_b - 141) to its accumulator: dot * d is a normal
//    number and the power-of-two factor costs one rounding, also where the
//    result is subnormal. Threads (g, 0) and (g, 1) are summed and the warps
//    (split-K) are added in warp order. Deterministic.

struct alignas(64) MParams {
  const uint8_t *W;
  const float *X;
  float *Y;
  int64_t N;
  int64_t row_bytes;
  int64_t total_bytes;
  int64_t ngroups;  // ceil(N / 8)
  int K, KB, KBp;   // KBp = KB rounded up to even
  int grid;
  int np;           // block pairs per warp
  int x_off, d_off, e_off, red_off, w_off;  // shared-memory offsets (bytes)
  int prefetch_before_wait;
};

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

// int8 codes in bytes 0 and 2 of w -> fp16x2 (exact).
__device__ __forceinline__ uint32_t codes_even_h2(uint32_t w) {
  const uint32_t biased = (w & 0x00ff00ffu) ^ 0x64806480u;  // 1024 + (code + 128) in each half
  const __half2 k1152 = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
  return h2_bits(__hsub2(*reinterpret_cast<const __half2 *>(&biased), k1152));
}

// Veltkamp split of a pair: hi = the 11 leading bits, lo = v - hi (exact in fp32).
__device__ __forceinline__ void split_pair(float2 v, uint32_t &hi, uint32_t &lo) {
  const float2 c = __fmul2_rn(v, make_float2(8193.0f, 8193.0f));  // (rounded ops: never contracted)
  const float hx = __fsub_rn(c.x, __fsub_rn(c.x, v.x)), hy = __fsub_rn(c.y, __fsub_rn(c.y, v.y));
  hi = h2_bits(__floats2half2_rn(hx, hy));
  lo = h2_bits(__floats2half2_rn(__fsub_rn(v.x, hx), __fsub_rn(v.y, hy)));
}

__device__ __forceinline__ void mma_f16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9},"
      " {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int GM, int NPM>
__global__ void __launch_bounds__(256, 2) q8_gemv_mma_kernel(const __grid_constant__ MParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;  // 16-byte aligned, all the layout needs; kept un-cast so accesses stay LDS/STS
  uint64_t *wbar = reinterpret_cast<uint64_t *>(smem);
  uint64_t *xbar = wbar + 1;
  float *dtab = reinterpret_cast<float *>(smem + p.d_off);  // [group][block][8 rows] scales
  float *ftab = reinterpret_cast<float *>(smem + p.e_off);  // block factors 2^(E_b - 141)
  float *red = reinterpret_cast<float *>(smem + p.red_off); // [warp][group][8 rows] partials
  uint8_t *xtab = smem + p.x_off;                           // activations, then their parts

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3, odd = t & 1;
  const int64_t g_begin = static_cast<int64_t>(blockIdx.x) * p.ngroups / p.grid;
  const int64_t g_end = static_cast<int64_t>(blockIdx.x + 1) * p.ngroups / p.grid;
  const int groups = static_cast<int>(g_end - g_begin);
  const int64_t r_begin = 8 * g_begin;
  const int64_t r_end = min(p.N, 8 * g_end);
  const int rows = static_cast<int>(r_end - r_begin);
  const int64_t b0 = r_begin * p.row_bytes, b1 = r_end * p.row_bytes;
  const int64_t a0 = b0 & ~int64_t(15);

  pdl_launch_dependents();
  if (tid == 0) {
    mbar_init(wbar, 1);
    mbar_init(xbar, 1);
    fence_mbar_init();
  }
  if (p.KBp > p.KB) {  // padding block of an odd block count: zero parts, scales and exponent
    for (int i = tid; i < 32 + 8 * GM; i += blockDim.x) {
      if (i < 32) reinterpret_cast<float *>(xtab + 128 * p.KB)[i] = 0.f;
      else dtab[((i - 32) / 8 * p.KBp + p.KB) * 8 + (i - 32) % 8] = 0.f;
    }
    if (tid == 0) ftab[p.KB] = 0.f;
  }
  __syncthreads();
  auto issue_w = [&]() {
    int64_t a1 = (b1 + 15) & ~int64_t(15);
    const int64_t lim = p.total_bytes & ~int64_t(15);
    uint8_t *dst = smem + p.w_off;
    if (a1 > lim) {  // bytes past the last 16-byte boundary of W by hand
      for (int64_t i = lim; i < b1; ++i) dst[i - a0] = p.W[i];
      a1 = lim;
    }
    const uint32_t bytes = static_cast<uint32_t>(a1 - a0);
    mbar_arrive_expect_tx(wbar, bytes);
    const uint64_t pol = l2_evict_first_policy();
    constexpr uint32_t kPiece = 8192;  // several copies in flight
    for (uint32_t o = 0; o < bytes; o += kPiece)
      bulk_g2s(dst + o, p.W + a0 + o, min(kPiece, bytes - o), wbar, pol);
  };
  auto issue_x = [&]() {
    const uint32_t bytes = static_cast<uint32_t>(p.K) * 4u;
    mbar_arrive_expect_tx(xbar, bytes);
    bulk_g2s(xtab, p.X, bytes, xbar, l2_evict_last_policy());
  };
  if (tid == 0) {
    if (!p.prefetch_before_wait) {
      pdl_wait();
      issue_x();
    }
    issue_w();
  }

  // ---- A fragments (fp16 codes of block pairs) and block scales; independent of X
  const int P = p.KBp / 2;
  const int kp0 = warp * p.np;
  const uint32_t wbase = smem_u32(smem + p.w_off) + static_cast<uint32_t>(b0 - a0);
  uint32_t Wr[NPM][GM][8];
  bool ok = mbar_wait(wbar, 0);
  if (!ok && lane == 0) atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
#pragma unroll
  for (int j = 0; j < NPM; ++j) {
    const int pp = kp0 + j;
    const bool pair_ok = j < p.np && pp < P;
#pragma unroll
    for (int gi = 0; gi < GM; ++gi) {
      const int rl = gi * 8 + g;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int blk = 2 * pp + h;
        uint32_t w0 = 0u, w1 = 0u;
        if (ok && pair_ok && blk < p.KB && rl < rows) {
          const uint32_t blk_a = wbase + static_cast<uint32_t>(rl * p.row_bytes) + 34u * blk;
          const uint32_t ca = blk_a + 2u + 8u * t;  // codes 8t..8t+7 (2-byte aligned)
          const uint32_t mis = ca & 2u, wa = ca - mis, sh = mis << 3;
          const uint32_t v0 = lds_u32(wa), v1 = lds_u32(wa + 4), v2 = lds_u32(wa + 8);
          w0 = __funnelshift_r(v0, v1, sh);
          w1 = __funnelshift_r(v1, v2, sh);
          if (t == 0) dtab[(gi * p.KBp + blk) * 8 + g] = half_bits_to_float(lds_u16(blk_a));
        } else if (pair_ok && blk < p.KB && t == 0) {
          dtab[(gi * p.KBp + blk) * 8 + g] = 0.f;
        }
        Wr[j][gi][0 + h] = codes_even_h2(w0);       // slice 0, k = 2t, 2t+1: codes (0, 2)
        Wr[j][gi][2 + h] = codes_even_h2(w0 >> 8);  // slice 0, k = 2t+8, 2t+9: codes (1, 3)
        Wr[j][gi][4 + h] = codes_even_h2(w1);       // slice 1: codes (4, 6)
        Wr[j][gi][6 + h] = codes_even_h2(w1 >> 8);  // slice 1: codes (5, 7)
      }
    }
  }

  // ---- activations (after the preceding grid): scaled hi/lo parts in place
  pdl_wait();
  if (tid == 0 && p.prefetch_before_wait) issue_x();
  if (ok && !mbar_wait(xbar, 0)) {
    ok = false;
    if (lane == 0) atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
  }
  const int slots = p.KB * 4;  // (block, t): eight activations 8t..8t+7 of a block
#pragma unroll 2
  for (int base = warp * 32; base < slots; base += blockDim.x) {
    const int s = base + lane;
    const bool have = ok && s < slots;
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f), w = u;
    float4 *slot = reinterpret_cast<float4 *>(xtab + 32 * s);
    if (have) {
      u = slot[0];
      w = slot[1];
    }
    uint32_t mb = max(max(max(__float_as_uint(u.x) & 0x7fffffffu, __float_as_uint(u.y) & 0x7fffffffu),
                          max(__float_as_uint(u.z) & 0x7fffffffu, __float_as_uint(u.w) & 0x7fffffffu)),
                      max(max(__float_as_uint(w.x) & 0x7fffffffu, __float_as_uint(w.y) & 0x7fffffffu),
                          max(__float_as_uint(w.z) & 0x7fffffffu, __float_as_uint(w.w) & 0x7fffffffu)));
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
    const int E = max(static_cast<int>(mb >> 23), 1);  // largest |x| of the block < 2^(E - 126)
    const int sh = 141 - E, sh1 = min(sh, 127);
    const float2 s1 = make_float2(__int_as_float((127 + sh1) << 23), __int_as_float((127 + sh1) << 23));
    const float2 s2 = make_float2(__int_as_float((127 + sh - sh1) << 23), __int_as_float((127 + sh - sh1) << 23));
    uint4 hi, lo;
    split_pair(__fmul2_rn(__fmul2_rn(make_float2(u.x, u.z), s1), s2), hi.x, lo.x);  // elements 0, 2
    split_pair(__fmul2_rn(__fmul2_rn(make_float2(u.y, u.w), s1), s2), hi.y, lo.y);  // 1, 3
    split_pair(__fmul2_rn(__fmul2_rn(make_float2(w.x, w.z), s1), s2), hi.z, lo.z);  // 4, 6
    split_pair(__fmul2_rn(__fmul2_rn(make_float2(w.y, w.w), s1), s2), hi.w, lo.w);  // 5, 7
    if (have) {
      uint4 *dst = reinterpret_cast<uint4 *>(xtab + 32 * s);
      dst[0] = hi;
      dst[1] = lo;
      // 2^(E - 141), exact (a subnormal power of two below E = 15)
      if (t == 0) ftab[s >> 2] = E >= 15 ? __int_as_float((E - 14) << 23) : __int_as_float(1 << (E + 8));
    }
  }
  __syncthreads();

  // ---- tensor-core block dots and the scale epilogue
  float acc[GM];
#pragma unroll
  for (int gi = 0; gi < GM; ++gi) acc[gi] = 0.f;
  if (ok) {
#pragma unroll
    for (int j = 0; j < NPM; ++j) {
      const int pp = kp0 + j;
      if (j < p.np && pp < P) {
        // B registers: column g of the (hi b, lo b, hi b+1, lo b+1) pattern
        const uint4 xb =
            *reinterpret_cast<const uint4 *>(xtab + 128 * (2 * pp + ((g >> 1) & 1)) + 32 * t + 16 * (g & 1));
        const int bo = 2 * pp + odd;  // the block whose dot this thread keeps
        const float f = ftab[bo];
#pragma unroll
        for (int gi = 0; gi < GM; ++gi) {
          if (gi < groups) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            mma_f16_16816(c, Wr[j][gi][0], Wr[j][gi][1], Wr[j][gi][2], Wr[j][gi][3], xb.x, xb.y);
            mma_f16_16816(c, Wr[j][gi][4], Wr[j][gi][5], Wr[j][gi][6], Wr[j][gi][7], xb.z, xb.w);
            const float sv = odd ? c[2] + c[3] : c[0] + c[1];
            // (dot * d) is a normal number; one rounding for the power-of-two factor
            acc[gi] = fmaf(sv * dtab[(gi * p.KBp + bo) * 8 + g], f, acc[gi]);
          }
        }
      }
    }
  }
  if (!ok && tid == 0) {  // error path: give copies still in flight a bounded chance to land
    if (!mbar_wait(wbar, 0) || !mbar_wait(xbar, 0)) atomicOr(&g_q8_gemv_status, kDevTimeoutDrain);
  }
#pragma unroll
  for (int gi = 0; gi < GM; ++gi) {
    const float v = acc[gi] + __shfl_xor_sync(0xffffffffu, acc[gi], 1);  // even + odd blocks
    if (t == 0 && gi < groups) red[(warp * GM + gi) * 8 + g] = v;
  }
  __syncthreads();
  const int nw = blockDim.x >> 5;
  for (int r = tid; r < rows; r += blockDim.x) {
    const int gi = r >> 3, rr = r & 7;
    float v = 0.f;
    for (int w = 0; w < nw; ++w) v += red[(w * GM + gi) * 8 + rr];
    p.Y[r_begin + r] = v;
  }
}

// ---------------------------------------------------------------------------
// Integer tensor-core streaming variant (M = 1, K <= 2048, many rows per CTA:
// lm_head-like shapes). The fp32 streaming kernel is ALU-bound in the int8 ->
// fp32 conversion (~2.9 instructions per weight); here the raw int8 codes are
// the A operand of mma.m16n8k32.s8 as they sit in shared memory, so a weight
// costs only its share of the loads.
//
//  * Activations, once per CTA: x_j = M_j 2^(E_j - 150) (24-bit significand)
//    becomes the integer x_int = M_j 2^(E_j - E_b + 38) (rounded to nearest
//    for elements 2^38 below the block's largest exponent E_b), |x_int| <
//    2^62, written as eight balanced base-256 digits in [-128, 127]: the
//    bytes of (x_int + 0x8080..80) xor 0x8080..80. Digit k of the block's
//    activations forms B column k (k order within the block as stored).
//  * C column k = sum_j q_j digit_k(x_j): exact int32 (|C| < 2^20). Thread
//    (g, t) holds digits 2t, 2t+1 of its two rows; C_2t + 256 C_2t+1 is an
//    exact int32 (< 2^28), converted once and scaled by d * 2^(E_b - E + 16t)
//    in fp32 (E the largest E_b of the warp's K slice); the four digit lanes
//    are summed, and the producer scales each slice's partial by 2^(E - 188)
//    and adds the slices in order. Apart from fp32 rounding the activation
//    representation is exact for every element within 2^38 of its block
//    maximum. Each K slice's activations are converted by the warps that use
//    them (a named barrier per slice, no CTA-wide barrier).
//  * Shared-memory layout: a stage is a verbatim copy of consecutive rows
//    (34-byte blocks). MMA rows g and g + 8 of a tile are the tile's rows 2g
//    and 2g + 1: with the 952-byte rows of K = 896 the eight rows 2g start
//    28 banks apart, so every code load of a warp touches 32 distinct banks
//    (consecutive rows put all lanes on even banks, 2- to 3-way conflicts).
//    When rows are 4-byte multiples the codes of odd blocks are word-aligned
//    (two loads per row) and those of even blocks start 2 bytes past a word
//    (four loads and two byte permutes); the loop takes blocks in pairs.
//  * Rows come in 16-row tiles; 32 rows (two tiles) per stage for K <= 1024,
//    16 otherwise. Eight consumer warps split a stage as (tile, K slice); the
//    producer warp sums the K slices of each row in slice order when the
//    stage is released and writes Y. Deterministic.

constexpr int kMaxProj = 4;  // projections of one activation vector per launch

struct alignas(64) DParams {
  // Projections (weight matrix, its rows, output) sharing X; their row chunks
  // form one chunk space, chunk0[s] the first chunk of projection s.
  const uint8_t *Wp[kMaxProj];
  float *Yp[kMaxProj];
  int64_t Np[kMaxProj];
  int64_t chunk0[kMaxProj + 1];
  int nproj;
  const float *X;
  int64_t row_bytes;
  int K, KB;
  int grid;
  int tps;        // 16-row tiles per stage (1 or 2)
  int stages;
  int stage_bytes;
  int tab_off, ftab_off, eb_off, red_off, stage_off;  // shared-memory offsets
  int rows_aligned;  // block starts are even and rows whole words: parity-specialised code loads
  int padded;        // rows copied in groups of 2^lg_sub rows, group g at g * sub_pitch
  int lg_sub, sub_pitch;
  uint8_t rowmap[16];  // MMA row m of a 16-row tile -> row of the tile in memory order
  int wexp;          // power of two of the code scale (Q4_0 codes enter as 16 (q - 8): -4)
  int prefetch_before_wait;
};

constexpr int kDigitWarps = 8;  // consumer warps of a CTA when two CTAs share an SM (16 with one)
constexpr int kMaxSliceBlocks = 32;  // blocks of one K slice (the launcher checks the bound)
constexpr int kTabStride = 36;       // uint2 per block of B registers: 32 lanes + pad (conflict-free stores)

__device__ __forceinline__ void imma_16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9},"
      " {%10, %10, %10, %10};"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// The eight balanced base-256 digits of x_int = x 2^(188 - E_b) (x = M 2^(E - 150):
// exact for elements within 2^38 of the block maximum, rounded to nearest below
// that), as the bytes of (x_int + 0x8080..80) xor 0x8080..80. fa fb = 2^(156 - E_b),
// two normal powers of two. In fp32, every step exact: |x| fa fb = |x_int| / 2^32
// (< 2^30), its integer part is the high word and the fraction times 2^32 the low
// word of |x_int|; the sign is applied in two's complement with the bias added.
__device__ __forceinline__ uint64_t x_digits(float x, float fa, float fb) {
  const float xa = (fabsf(x) * fa) * fb;
  const uint32_t hw = __float2uint_rz(xa);
  const uint32_t lw = __float2uint_rn((xa - truncf(xa)) * 4294967296.0f);
  const uint64_t mag = (static_cast<uint64_t>(hw) << 32) | lw;
  const uint64_t neg = static_cast<uint64_t>(static_cast<int64_t>(static_cast<int32_t>(__float_as_uint(x)) >> 31));
  const uint64_t bias = 0x8080808080808080ull;
  return (((mag ^ neg) + (neg & 1u)) + bias) ^ bias;
}

// WT: QMM_Q8_0 (rows verbatim in shared memory, MMA rows interleaved) or
// QMM_Q4_0 (one GEMV; rows copied in groups placed so that the eight rows of
// an MMA half start on distinct banks; codes widened to 16 (q - 8), the factor
// 16 undone by wexp).
// NW: consumer warps (8 when two CTAs share an SM, 16 when one CTA has it).
template <int TPS, bool MULTI, int WT, int NW>
__global__ void __launch_bounds__((NW + 1) * 32) q8_gemv_digits_kernel(const __grid_constant__ DParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + kMaxStages;
  int *ewt = reinterpret_cast<int *>(empty + kMaxStages);  // [K slice] its largest block exponent
  int *ewp = ewt + 16;                                      // [consumer warp] the same over its units
  uint2 *tab = reinterpret_cast<uint2 *>(smem + p.tab_off);     // [KB][kTabStride]: 32 lanes' B registers + pad
  float *fwt = reinterpret_cast<float *>(smem + p.ftab_off);    // [warp][block of its K slice][t] 2^(E_b - E + 16t)
  int *ebt = reinterpret_cast<int *>(smem + p.eb_off);          // [KB] E_b
  float *red = reinterpret_cast<float *>(smem + p.red_off);     // [stage][kSlices][16 TPS rows]
  uint8_t *stage_mem = smem + p.stage_off;
  constexpr int kRows = 16 * TPS;
  constexpr int kSlices = NW / TPS;
  constexpr uint32_t kBB = WT == QMM_Q8_0 ? 34u : 18u;  // bytes per block

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // Work split: the projection table by whole chunks (a chunk never spans two
  // matrices); one matrix by whole 16-row tiles, so that a CTA may end in a
  // one-tile chunk (half the bytes of a two-tile chunk: the busiest CTAs of a
  // long launch carry half a chunk more, not a whole one). An even split of
  // rows would end every CTA in a ragged chunk that streams nearly as long.
  int64_t c_begin = 0, r_begin = 0, r_end = 0;
  int nchunks;
  if constexpr (MULTI) {
    const int64_t tchunks = p.chunk0[p.nproj];
    c_begin = static_cast<int64_t>(blockIdx.x) * tchunks / p.grid;
    nchunks = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * tchunks / p.grid - c_begin);
  } else {
    const int64_t tiles = (p.Np[0] + 15) / 16;
    r_begin = 16 * (static_cast<int64_t>(blockIdx.x) * tiles / p.grid);
    r_end = min(p.Np[0], 16 * (static_cast<int64_t>(blockIdx.x + 1) * tiles / p.grid));
    nchunks = static_cast<int>((r_end - r_begin + kRows - 1) / kRows);
  }
  const int S = p.stages;
  // chunk c of this CTA: its projection, first row and valid rows
  struct Chunk {
    int proj;
    int64_t r0;
    int rows;
  };
  auto chunk = [&](int c) -> Chunk {
    if constexpr (MULTI) {
      const int64_t gc = c_begin + c;
      int sg = 0;
      while (sg + 1 < p.nproj && gc >= p.chunk0[sg + 1]) ++sg;
      const int64_t r0 = (gc - p.chunk0[sg]) * kRows;
      return {sg, r0, static_cast<int>(min(static_cast<int64_t>(kRows), p.Np[sg] - r0))};
    } else {
      const int64_t r0 = r_begin + static_cast<int64_t>(c) * kRows;
      return {0, r0, static_cast<int>(min(static_cast<int64_t>(kRows), r_end - r0))};
    }
  };

  pdl_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    fence_mbar_init();
  }
  for (int b = tid; b < p.KB; b += blockDim.x) ebt[b] = 1;
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint64_t policy = 0;
    auto issue = [&](int c) {
      const int s = c % S;
      const Chunk ch = chunk(c);
      const uint8_t *W = MULTI ? p.Wp[ch.proj] : p.Wp[0];
      if (p.padded) {  // rows are 16-byte multiples: one copy per group of rows
        uint8_t *dst = stage_mem + static_cast<int64_t>(s) * p.stage_bytes;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(p.row_bytes * ch.rows));
        const int gr = 1 << p.lg_sub;
        for (int r = 0, gi = 0; r < ch.rows; r += gr, ++gi)
          bulk_g2s(dst + gi * p.sub_pitch, W + (ch.r0 + r) * p.row_bytes,
                   static_cast<uint32_t>(p.row_bytes * min(gr, ch.rows - r)), &full[s], policy);
        return;
      }
      const int64_t b0 = ch.r0 * p.row_bytes, b1 = (ch.r0 + ch.rows) * p.row_bytes;
      const int64_t a0 = b0 & ~int64_t(15);
      int64_t a1 = (b1 + 15) & ~int64_t(15);
      const int64_t lim = ((MULTI ? p.Np[ch.proj] : p.Np[0]) * p.row_bytes) & ~int64_t(15);
      uint8_t *dst = stage_mem + static_cast<int64_t>(s) * p.stage_bytes;
      if (a1 > lim) {  // last chunk of a matrix: bytes past its last 16-byte boundary by hand
        for (int64_t t = max(lim, a0); t < b1; ++t) dst[t - a0] = W[t];
        a1 = max(lim, a0);
      }
      const uint32_t bytes = static_cast<uint32_t>(a1 - a0);
      mbar_arrive_expect_tx(&full[s], bytes);
      if (bytes) bulk_g2s(dst, W + a0, bytes, &full[s], policy);
    };
    const int prologue = min(S, nchunks);
    if (lane == 0) {
      policy = l2_evict_first_policy();
      if (!p.prefetch_before_wait) pdl_wait();
      for (int c = 0; c < prologue; ++c) issue(c);
    }
    Chunk ch = nchunks > 0 ? chunk(0) : Chunk{0, 0, 0};
    pdl_wait();
    bool ok = true;
    int issued = prologue;
    float f1[kSlices], f2[kSlices];  // 2^(E_slice - 188) in two exact steps, per K slice
    int s = 0;
    uint32_t ph = 0;
    for (int c = 0; c < nchunks && ok; ++c) {
      ok = mbar_wait(&empty[s], ph);
      if (!ok) break;
      if (c == 0) {  // the slice exponents were written before the consumers' first release
#pragma unroll
        for (int k = 0; k < kSlices; ++k) {
          const int e = ewt[k] - 188 + p.wexp, e1 = max(e, -120);
          f1[k] = __int_as_float((127 + e1) << 23);
          f2[k] = __int_as_float((127 + e - e1) << 23);
        }
      }
      // rows of chunk c: each K slice's partial at its own scale, added in slice order
      const int64_t r0 = ch.r0;
      const int rows = ch.rows;
      float *Y = MULTI ? p.Yp[ch.proj] : p.Yp[0];
      const float *rb = red + s * kSlices * kRows;
      for (int r = lane; r < rows; r += 32) {
        float v = (rb[r] * f1[0]) * f2[0];
#pragma unroll
        for (int k = 1; k < kSlices; ++k) v += (rb[k * kRows + r] * f1[k]) * f2[k];
        Y[r0 + r] = v;
      }
      __syncwarp();
      if (lane == 0 && issued < nchunks) {
        issue(issued);
        ++issued;
      }
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
      if (c + 1 < nchunks) ch = chunk(c + 1);
    }
    if (!ok && lane == 0) {  // error path: record, then drain copies still in flight
      atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
      for (int c = max(0, issued - S); c < issued; ++c)
        if (!mbar_wait(&full[c % S], static_cast<uint32_t>(c / S) & 1u)) atomicOr(&g_q8_gemv_status, kDevTimeoutDrain);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;
  const int tl = cw % TPS, ks = cw / TPS;  // this warp's tile of the stage and K slice
  const int kb0 = ks * p.KB / kSlices, kb1 = (ks + 1) * p.KB / kSlices;
  const int g = lane >> 2, t = lane & 3;
  Chunk ch = nchunks > 0 ? chunk(0) : Chunk{0, 0, 0};
  pdl_wait();
  // One pass over this K slice's activations, shared by its TPS warps: block
  // exponents (the eight units of a block are eight lanes of a warp: a
  // shuffle max), then each unit's digits, transposed into B registers (lane
  // (k, t) of block b holds digit k of activations 4t..4t+3 in word 0 and
  // 16+4t..16+4t+3 in word 1); the slice's largest block exponent E_w.
  int wmaxE = 1;
  const int u_end = 8 * kb1;
  const float4 *X4 = reinterpret_cast<const float4 *>(p.X);
  float4 vn = make_float4(0.f, 0.f, 0.f, 0.f);  // the next pass's activations, loaded a pass ahead
  if (8 * kb0 + 32 * tl + lane < u_end) vn = __ldg(X4 + 8 * kb0 + 32 * tl + lane);
  for (int base = 8 * kb0 + 32 * tl; base < u_end; base += 32 * TPS) {  // warp-uniform: it shuffles
    const int u = base + lane;
    const float4 v = vn;
    vn = make_float4(0.f, 0.f, 0.f, 0.f);
    if (u + 32 * TPS < u_end) vn = __ldg(X4 + u + 32 * TPS);
    uint32_t m = max(max(__float_as_uint(v.x) & 0x7fffffffu, __float_as_uint(v.y) & 0x7fffffffu),
                     max(__float_as_uint(v.z) & 0x7fffffffu, __float_as_uint(v.w) & 0x7fffffffu));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
    const int Eb = max(static_cast<int>(m >> 23), 1);
    wmaxE = max(wmaxE, Eb);
    if (u < u_end) {
      const int b = u >> 3, t = u & 3, h = (u >> 2) & 1;  // activations 4(u & 7) .. 4(u & 7) + 3
      if ((u & 7) == 0) ebt[b] = Eb;
      const int ke = 156 - Eb, ka = min(ke, 127);
      const float fa = __int_as_float((127 + ka) << 23), fb = __int_as_float((127 + ke - ka) << 23);
      const uint64_t d0 = x_digits(v.x, fa, fb), d1 = x_digits(v.y, fa, fb);
      const uint64_t d2 = x_digits(v.z, fa, fb), d3 = x_digits(v.w, fa, fb);
      uint32_t *tb = reinterpret_cast<uint32_t *>(tab + b * kTabStride);
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // digits 0..3, then 4..7
        const uint32_t w0 = static_cast<uint32_t>(d0 >> (32 * half)), w1 = static_cast<uint32_t>(d1 >> (32 * half));
        const uint32_t w2 = static_cast<uint32_t>(d2 >> (32 * half)), w3 = static_cast<uint32_t>(d3 >> (32 * half));
        const uint32_t l01 = __byte_perm(w0, w1, 0x5140u), h01 = __byte_perm(w0, w1, 0x7362u);
        const uint32_t l23 = __byte_perm(w2, w3, 0x5140u), h23 = __byte_perm(w2, w3, 0x7362u);
        const uint32_t dig[4] = {__byte_perm(l01, l23, 0x5410u), __byte_perm(l01, l23, 0x7632u),
                                 __byte_perm(h01, h23, 0x5410u), __byte_perm(h01, h23, 0x7632u)};
#pragma unroll
        for (int k = 0; k < 4; ++k) tb[2 * ((4 * half + k) * 4 + t) + h] = dig[k];  // lane 4k' + t, word h
      }
    }
  }
  wmaxE = __reduce_max_sync(0xffffffffu, wmaxE);
  if (lane == 0) ewp[cw] = wmaxE;
  if constexpr (TPS == 2) {  // the slice's two warps: named barrier 2 + ks (immediate ids)
    switch (ks) {
      case 0: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
      case 1: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
      case 2: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
      case 3: asm volatile("bar.sync 5, 64;" ::: "memory"); break;
      case 4: asm volatile("bar.sync 6, 64;" ::: "memory"); break;
      case 5: asm volatile("bar.sync 7, 64;" ::: "memory"); break;
      case 6: asm volatile("bar.sync 8, 64;" ::: "memory"); break;
      default: asm volatile("bar.sync 9, 64;" ::: "memory"); break;
    }
  } else {
    __syncwarp();
  }
  int Ew = ewp[ks * TPS];
  if constexpr (TPS == 2) Ew = max(Ew, ewp[ks * TPS + 1]);
  if (tl == 0 && lane == 0) ewt[ks] = Ew;  // read by the producer after the first release
  // The warp's block factors 2^(E_b - E_w) 2^(16t) (zero for blocks more than
  // 2^126 below the slice's largest), per block of its slice and digit pair t.
  float *fw = fwt + cw * (kMaxSliceBlocks * 4);
  for (int i = lane; i < 4 * (kb1 - kb0); i += 32) {
    const int eb = ebt[kb0 + (i >> 2)] - Ew;
    fw[i] = eb >= -126 ? __int_as_float((127 + eb) << 23) * __int_as_float((127 + 16 * (i & 3)) << 23) : 0.f;
  }
  __syncwarp();

  // MMA rows g and g + 8 of tile tl. Q8_0 (verbatim rows of 952 bytes): the
  // tile's rows 2g and 2g + 1; Q4_0 (grouped rows): rowmap[g], rowmap[g + 8],
  // chosen on the host so that each MMA half's eight rows start on distinct banks.
  const int ra = WT == QMM_Q8_0 ? tl * 16 + 2 * g : tl * 16 + p.rowmap[g];
  const int rb = WT == QMM_Q8_0 ? ra + 1 : tl * 16 + p.rowmap[g + 8];
  int s = 0;
  uint32_t ph = 0;
  for (int c = 0; c < nchunks; ++c) {
    if (!mbar_wait(&full[s], ph)) {
      if (lane == 0) atomicOr(&g_q8_gemv_status, kDevTimeoutFull);
      return;  // the producer times out on this warp's missing arrival and drains
    }
    const int64_t r0 = ch.r0;
    const int rows = ch.rows;
    const uint32_t base = smem_u32(stage_mem) + s * p.stage_bytes +
                          (p.padded ? 0u : static_cast<uint32_t>((r0 * p.row_bytes) & 15));
    // rows past the chunk read its last row and are never written out
    auto row_off = [&](int r) -> uint32_t {
      r = min(r, rows - 1);
      if constexpr (WT == QMM_Q8_0) return static_cast<uint32_t>(r * p.row_bytes);
      else return static_cast<uint32_t>((r >> p.lg_sub) * p.sub_pitch + (r & ((1 << p.lg_sub) - 1)) * p.row_bytes);
    };
    const uint32_t pa = base + row_off(ra), pb = base + row_off(rb);
    float2 acc = make_float2(0.f, 0.f);  // rows ra, rb
    // Block b of both rows: codes k = 4t..4t+3 (A0, A1) and 16+4t..16+4t+3
    // (A2, A3). FORM 0: codes word-aligned; 1: codes 2 bytes past a word
    // (byte permutes of aligned words); 2: alignment known at run time only.
    auto block = [&](auto form, int b) {
      constexpr int kForm = decltype(form)::value;
      const uint32_t ca = pa + kBB * b, cb = pb + kBB * b;  // block starts (scale d)
      uint32_t A0, A1, A2, A3;
      if constexpr (WT == QMM_Q4_0) {
        // bytes 4t..4t+3 of the packed codes: low nibbles are elements 4t..4t+3,
        // high nibbles 16+4t..16+4t+3; each becomes the int8 16 (q - 8)
        uint32_t wa, wb;
        if constexpr (kForm == 0) {
          wa = lds_u32(ca + 2u + 4u * t);
          wb = lds_u32(cb + 2u + 4u * t);
        } else if constexpr (kForm == 1) {
          wa = __byte_perm(lds_u32(ca + 4u * t), lds_u32(ca + 4u * t + 4u), 0x5432u);
          wb = __byte_perm(lds_u32(cb + 4u * t), lds_u32(cb + 4u * t + 4u), 0x5432u);
        } else {
          const uint32_t xa = ca + 2u + 4u * t, xb = cb + 2u + 4u * t;
          wa = __funnelshift_r(lds_u32(xa & ~3u), lds_u32((xa & ~3u) + 4u), (xa & 3u) << 3);
          wb = __funnelshift_r(lds_u32(xb & ~3u), lds_u32((xb & ~3u) + 4u), (xb & 3u) << 3);
        }
        A0 = ((wa << 4) & 0xF0F0F0F0u) ^ 0x80808080u;
        A2 = (wa & 0xF0F0F0F0u) ^ 0x80808080u;
        A1 = ((wb << 4) & 0xF0F0F0F0u) ^ 0x80808080u;
        A3 = (wb & 0xF0F0F0F0u) ^ 0x80808080u;
      } else if constexpr (kForm == 0) {
        A0 = lds_u32(ca + 2u + 4u * t);
        A2 = lds_u32(ca + 18u + 4u * t);
        A1 = lds_u32(cb + 2u + 4u * t);
        A3 = lds_u32(cb + 18u + 4u * t);
      } else if constexpr (kForm == 1) {
        const uint32_t ea = ca + 4u * t, eb = cb + 4u * t;
        A0 = __byte_perm(lds_u32(ea), lds_u32(ea + 4u), 0x5432u);
        A2 = __byte_perm(lds_u32(ea + 16u), lds_u32(ea + 20u), 0x5432u);
        A1 = __byte_perm(lds_u32(eb), lds_u32(eb + 4u), 0x5432u);
        A3 = __byte_perm(lds_u32(eb + 16u), lds_u32(eb + 20u), 0x5432u);
      } else {
        const uint32_t xa = ca + 2u + 4u * t, xb = cb + 2u + 4u * t;
        const uint32_t sa = (xa & 3u) << 3, sb = (xb & 3u) << 3, ya = xa & ~3u, yb = xb & ~3u;
        A0 = __funnelshift_r(lds_u32(ya), lds_u32(ya + 4u), sa);
        A2 = __funnelshift_r(lds_u32(ya + 16u), lds_u32(ya + 20u), sa);
        A1 = __funnelshift_r(lds_u32(yb), lds_u32(yb + 4u), sb);
        A3 = __funnelshift_r(lds_u32(yb + 16u), lds_u32(yb + 20u), sb);
      }
      const float2 dd = make_float2(half_bits_to_float(lds_u16(ca)), half_bits_to_float(lds_u16(cb)));
      const uint2 B = tab[b * kTabStride + lane];
      int cc[4];
      imma_16832(cc, A0, A1, A2, A3, B.x, B.y);
      // this lane's digits 2t, 2t+1 of both rows as one exact int32 (< 2^28)
      const float2 v = make_float2(__int2float_rn(cc[0] + cc[1] * 256), __int2float_rn(cc[2] + cc[3] * 256));
      const float f = fw[4 * (b - kb0) + t];
      acc = __ffma2_rn(v, __fmul2_rn(dd, make_float2(f, f)), acc);
    };
    if (p.rows_aligned) {  // rows are whole words: odd blocks aligned, even ones 2 bytes past
      int b = kb0;
      if (b < kb1 && (b & 1)) block(std::integral_constant<int, 0>{}, b++);
#pragma unroll 2
      for (; b + 1 < kb1; b += 2) {
        block(std::integral_constant<int, 1>{}, b);
        block(std::integral_constant<int, 0>{}, b + 1);
      }
      if (b < kb1) block(std::integral_constant<int, 1>{}, b);
    } else {
#pragma unroll 4
      for (int b = kb0; b < kb1; ++b) block(std::integral_constant<int, 2>{}, b);
    }
    // the four digit lanes of each row
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 1);
    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 1);
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 2);
    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 2);
    if (t == 0) {
      float *rbuf = red + (s * kSlices + ks) * kRows;
      rbuf[ra] = acc.x;
      rbuf[rb] = acc.y;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
    if (c + 1 < nchunks) ch = chunk(c + 1);
  }
}

int align_up(int64_t v, int a) { return static_cast<int>((v + a - 1) / a * a); }

template <int MODE, int MP, int RG>
cudaError_t launch(const cudaLaunchConfig_t &cfg, const Params &p) {
  static DeviceFlags configured;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!configured.done(dev)) {
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaError_t e = cudaFuncSetAttribute(q8_gemv_kernel<MODE, MP, RG>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    configured.set(dev);
  }
  return cudaLaunchKernelEx(&cfg, q8_gemv_kernel<MODE, MP, RG>, p);
}

}  // namespace

namespace {

template <int MODE>
qmm_status launch_stream(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X, const int8_t *QX,
                         const float *DX, float *Y, int32_t *isum, cudaStream_t stream, uint32_t flags,
                         const uint8_t *XB = nullptr, uint64_t wait_ns = kWaitLimitNs, int withhold = 0) {
  Params p{};
  p.wait_ns = wait_ns;
  p.withhold = withhold;
  p.W = static_cast<const uint8_t *>(W);
  p.X = X;
  p.QX = QX;
  p.DX = DX;
  p.XB = XB;
  p.Y = Y;
  p.isum = isum;
  p.N = N;
  p.M = M;
  p.K = K;
  p.KB = K / 32;
  p.row_bytes = 34ll * p.KB;
  p.total_bytes = N * p.row_bytes;
  p.cg = (p.KB + 31) / 32;
  // consumer warps: the K windows side by side, then rows
  // Small problems: few rows per CTA, so a lean CTA (more launches resident
  // per SM under programmatic dependent launch); large problems: two CTAs per SM.
  const int64_t rows_one_wave = (N + dev.sms - 1) / dev.sms;
  p.cs = std::min(p.cg, kMaxConsumerWarps);
  p.rs = p.cs > 1 ? std::max(1, 10 / p.cs) : (rows_one_wave <= 16 ? 4 : 8);
  const int nconsumer = p.cs * p.rs;
  const int threads = (nconsumer + 1) * 32;
  const int64_t ctas_per_sm = rows_one_wave >= 128 ? 2 : 1;
  p.grid = static_cast<int>(std::min<int64_t>(N, dev.sms * ctas_per_sm));
  const int64_t rows_max = (N + p.grid - 1) / p.grid;
  // rows per warp step: more rows amortise the cross-lane reduction, but every
  // row-slot warp should get work when a CTA owns only a few rows
  int rg = 1;
  if (M == 1) {
    if (rows_max >= 4ll * p.rs * 2) rg = 4;
    else if (rows_max >= 2ll * p.rs) rg = 2;
  }
  int64_t rc = std::max<int64_t>(1, kStageTarget / p.row_bytes);
  const int64_t quantum = static_cast<int64_t>(p.rs) * rg;
  rc = (rc >= quantum) ? rc / quantum * quantum : quantum;
  rc = std::min<int64_t>(rc, rows_max);
  p.rows_chunk = static_cast<int>(rc);
  // data + up to 15 bytes of alignment slack in front + over-read of the last block
  p.stage_bytes = align_up(rc * p.row_bytes + 32, 128);
  const int64_t nchunks_max = (rows_max + rc - 1) / rc;
  int S = std::max(1, kSmemBudget / p.stage_bytes);
  S = static_cast<int>(std::min<int64_t>({S, kMaxStages, nchunks_max}));
  p.stages = S;
  const int red_bytes = p.cg > 1 ? S * M * p.cg * p.rows_chunk * 4 : 0;
  const int64_t xs_bytes = static_cast<int64_t>(M) * K * (MODE == kModeF32 ? 4 : 1);
  const bool panel = xs_bytes <= kPanelBytes && XB == nullptr;  // block-form activations: read directly
  p.xs_off = panel ? align_up(kBarBytes + red_bytes, 1024) : 0;  // 128-byte swizzle needs 1024-byte alignment
  p.xs_rows = panel ? static_cast<int>(xs_bytes / 128) : 0;
  p.xs_bytes = panel ? static_cast<int>(xs_bytes) : 0;
  p.stage_off = panel ? align_up(p.xs_off + xs_bytes, 128) : kBarBytes + align_up(red_bytes, 128);
  if (panel && MODE == kModeF32) {
    const uint64_t dims[2] = {32, static_cast<uint64_t>(p.xs_rows)};
    const uint64_t strides[1] = {128};
    const uint32_t box[2] = {32, static_cast<uint32_t>(p.xs_rows)};
    qmm_status st = encode_tiled(&p.xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, X, dims, strides, box,
                                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != QMM_OK) return st;
  }
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
  if (M > 1) e = launch<MODE, 2, 1>(cfg, p);
  else if (rg == 4) e = launch<MODE, 1, 4>(cfg, p);
  else if (rg == 2) e = launch<MODE, 1, 2>(cfg, p);
  else e = launch<MODE, 1, 1>(cfg, p);
  return cuda_check(e, MODE == kModeF32 ? "q8_gemv launch" : "q8q8_gemv launch");
}


// Resident variant when every CTA's weight slice fits (returns false if not).
bool try_launch_resident(const DevInfo &dev, int64_t N, int K, const void *W, const float *X, float *Y,
                         cudaStream_t stream, uint32_t flags, qmm_status *out) {
  const int KB = K / 32;
  const int cg = (KB + 31) / 32;
  if (K * 4 > kPanelBytes) return false;
  const int grid = static_cast<int>(std::min<int64_t>(N, dev.sms));
  const int64_t rows = (N + grid - 1) / grid;
  const int64_t row_bytes = 34ll * KB;
  // U rows per warp; max warps per CTA for each U (register budget)
  const int maxw[3] = {16, 16, 11};
  int U = 0, wpw = 0;
  for (int ui = 0; ui < 3; ++ui) {
    const int u = 1 << ui;
    const int w = static_cast<int>((rows + u - 1) / u);
    if (cg * w <= maxw[ui]) {
      U = u;
      wpw = w;
      break;
    }
  }
  if (U == 0) return false;
  const int64_t slice = rows * row_bytes + 48;
  if (slice > 48 * 1024) return false;
  RParams p{};
  p.W = static_cast<const uint8_t *>(W);
  p.Y = Y;
  p.N = N;
  p.row_bytes = row_bytes;
  p.total_bytes = N * row_bytes;
  p.K = K;
  p.KB = KB;
  p.grid = grid;
  p.cg = cg;
  p.wpw = wpw;
  p.max_rows = static_cast<int>(rows);
  p.prefetch_before_wait = (flags & kPrefetchBeforeWait) ? 1 : 0;
  p.xs_off = 1024;
  p.red_off = align_up(p.xs_off + KB * 128, 128);
  p.w_off = align_up(p.red_off + cg * rows * 4, 128);
  const size_t smem = static_cast<size_t>(align_up(p.w_off + slice, 128)) + 1024;
  const uint64_t dims[2] = {32, static_cast<uint64_t>(KB)};
  const uint64_t strides[1] = {128};
  const uint32_t box[2] = {32, static_cast<uint32_t>(KB)};
  qmm_status st = encode_tiled(&p.xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, X, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QMM_OK) {
    *out = st;
    return true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(cg * wpw * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto go = [&](auto kern) -> cudaError_t {
    static DeviceFlags configured[3];
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    const int idx = U == 1 ? 0 : U == 2 ? 1 : 2;
    if (!configured[idx].done(dev_id)) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
      if (e != cudaSuccess) return e;
      configured[idx].set(dev_id);
    }
    return cudaLaunchKernelEx(&cfg, kern, p);
  };
  cudaError_t e = U == 1 ? go(q8_gemv_resident_kernel<1>) : U == 2 ? go(q8_gemv_resident_kernel<2>)
                                                                    : go(q8_gemv_resident_kernel<4>);
  *out = cuda_check(e, "q8_gemv launch");
  return true;
}

// Fused Q8xQ8 resident variant: false when the slice does not fit. Warps per
// CTA are capped so that two CTAs' registers fit one SM (the next launch in the
// stream can then start, and prefetch its weights, while this one runs).
bool try_launch_q8q8_resident(const DevInfo &dev, int64_t N, int K, const void *W, const float *X, int8_t *QX,
                              float *DX, float *Y, cudaStream_t stream, uint32_t flags, qmm_status *out,
                              int32_t *isum = nullptr) {
  constexpr int64_t kMaxSlice = 96 * 1024;
  const int KB = K / 32;
  const int cg = (KB + 31) / 32;
  if (K * 4 > kPanelBytes) return false;
  const int grid = static_cast<int>(std::min<int64_t>(N, dev.sms));
  const int64_t rows = (N + grid - 1) / grid;
  const int64_t row_bytes = 34ll * KB;
  // U rows per warp; at about 48 / 56 / 72 registers a thread for U = 1, 2, 4
  // these warp counts leave room for two CTAs per SM
  const int maxw[3] = {16, 16, 14};
  int U = 0, wpw = 0;
  for (int ui = 0; ui < 3; ++ui) {
    const int u = 1 << ui;
    const int w = static_cast<int>((rows + u - 1) / u);
    if (cg * w <= maxw[ui]) {
      U = u;
      wpw = w;
      break;
    }
  }
  if (U == 0) return false;
  const int64_t slice = rows * row_bytes + 48;
  if (slice > kMaxSlice) return false;
  RParams p{};
  p.W = static_cast<const uint8_t *>(W);
  p.Y = Y;
  p.N = N;
  p.row_bytes = row_bytes;
  p.total_bytes = N * row_bytes;
  p.K = K;
  p.KB = KB;
  p.grid = grid;
  p.cg = cg;
  p.wpw = wpw;
  p.max_rows = static_cast<int>(rows);
  p.prefetch_before_wait = (flags & kPrefetchBeforeWait) ? 1 : 0;
  p.QXo = QX;
  p.DXo = DX;
  p.isum = isum;
  p.xs_off = 1024;
  p.qx_off = align_up(p.xs_off + KB * 128, 128);
  p.dx_off = align_up(p.qx_off + KB * 32, 128);
  p.red_off = align_up(p.dx_off + KB * 4, 128);
  p.w_off = align_up(p.red_off + cg * rows * 4, 128);
  const size_t smem = static_cast<size_t>(align_up(p.w_off + slice, 128)) + 1024;
  constexpr size_t kSmemAttr = 160 * 1024;
  if (smem > kSmemAttr) return false;
  const uint64_t dims[2] = {32, static_cast<uint64_t>(KB)};
  const uint64_t strides[1] = {128};
  const uint32_t box[2] = {32, static_cast<uint32_t>(KB)};
  qmm_status st = encode_tiled(&p.xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, X, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QMM_OK) {
    *out = st;
    return true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(cg * wpw * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto go = [&](auto kern) -> cudaError_t {
    static DeviceFlags configured[2][3];
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    const int idx = U == 1 ? 0 : U == 2 ? 1 : 2;
    if (!configured[isum != nullptr][idx].done(dev_id)) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemAttr));
      if (e != cudaSuccess) return e;
      configured[isum != nullptr][idx].set(dev_id);
    }
    return cudaLaunchKernelEx(&cfg, kern, p);
  };
  cudaError_t e;
  if (isum)
    e = U == 1 ? go(q8q8_resident_kernel<1, true>) : U == 2 ? go(q8q8_resident_kernel<2, true>)
                                                            : go(q8q8_resident_kernel<4, true>);
  else
    e = U == 1 ? go(q8q8_resident_kernel<1, false>) : U == 2 ? go(q8q8_resident_kernel<2, false>)
                                                             : go(q8q8_resident_kernel<4, false>);
  *out = cuda_check(e, "q8q8_gemv_fused launch");
  return true;
}

// Tensor-core resident variant (returns false when the shape does not suit it).
bool try_launch_mma(const DevInfo &dev, int64_t N, int K, const void *W, const float *X, float *Y,
                    cudaStream_t stream, uint32_t flags, qmm_status *out) {
  constexpr int kMaxWarps = 8;
  constexpr int kSmemMax = 110 * 1024;  // two CTAs per SM
  const int KB = K / 32;
  const int KBp = (KB + 1) & ~1;
  const int P = KBp / 2;
  if (static_cast<int64_t>(KBp) * 128 > kPanelBytes) return false;
  const int64_t ngroups = (N + 7) / 8;
  const int grid = static_cast<int>(std::min<int64_t>(ngroups, dev.sms));
  const int gmax = static_cast<int>((ngroups + grid - 1) / grid);
  // instances: row groups per CTA (GM) x block pairs per warp (NPM)
  struct Inst {
    int gm, npm;
    void (*kern)(MParams);
  };
  static const Inst insts[] = {
      {1, 2, q8_gemv_mma_kernel<1, 2>}, {1, 4, q8_gemv_mma_kernel<1, 4>}, {2, 5, q8_gemv_mma_kernel<2, 5>},
      {3, 3, q8_gemv_mma_kernel<3, 3>}, {4, 2, q8_gemv_mma_kernel<4, 2>}, {5, 2, q8_gemv_mma_kernel<5, 2>},
      {8, 1, q8_gemv_mma_kernel<8, 1>},
  };
  constexpr int kInsts = static_cast<int>(sizeof(insts) / sizeof(insts[0]));
  int pick = -1, nw = 0;
  for (int i = 0; i < kInsts; ++i) {
    const int w = (P + insts[i].npm - 1) / insts[i].npm;
    if (insts[i].gm >= gmax && w <= kMaxWarps) {
      pick = i;
      nw = w;
      break;
    }
  }
  if (pick < 0) return false;
  const Inst &in = insts[pick];
  const int64_t row_bytes = 34ll * KB;
  MParams p{};
  p.W = static_cast<const uint8_t *>(W);
  p.X = X;
  p.Y = Y;
  p.N = N;
  p.row_bytes = row_bytes;
  p.total_bytes = N * row_bytes;
  p.ngroups = ngroups;
  p.K = K;
  p.KB = KB;
  p.KBp = KBp;
  p.grid = grid;
  p.np = (P + nw - 1) / nw;
  p.prefetch_before_wait = (flags & kPrefetchBeforeWait) ? 1 : 0;
  p.x_off = 128;
  p.d_off = align_up(p.x_off + 128ll * KBp, 16);
  p.e_off = align_up(p.d_off + 32ll * in.gm * KBp, 16);
  p.red_off = align_up(p.e_off + 4ll * KBp, 16);
  p.w_off = align_up(p.red_off + 32ll * nw * in.gm, 128);
  const int64_t slice = 8ll * gmax * row_bytes + 48;
  const size_t smem = static_cast<size_t>(align_up(p.w_off + slice, 128));
  if (smem > static_cast<size_t>(kSmemMax)) return false;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(32 * nw);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static DeviceFlags configured[kInsts];
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  if (!configured[pick].done(dev_id)) {
    cudaError_t e = cudaFuncSetAttribute(in.kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
    if (e != cudaSuccess) {
      *out = cuda_check(e, "q8_gemv attribute");
      return true;
    }
    configured[pick].set(dev_id);
  }
  *out = cuda_check(cudaLaunchKernelEx(&cfg, in.kern, p), "q8_gemv launch");
  return true;
}


// Integer tensor-core streaming variant for M = 1, K <= 2048 and enough rows
// for two CTAs per SM (returns false when the shape does not suit it).
// Row placement in shared memory and the MMA row order. Verbatim rows (Q8_0):
// one copy per chunk, MMA rows g, g + 8 = tile rows 2g, 2g + 1. Grouped rows
// (Q4_0, rows of 16-byte multiples): the tile's rows come in copies of 2^lg
// consecutive rows, copy i at i * sub_pitch; the largest groups (fewest
// copies: many small bulk copies are slow) and smallest gap for which the
// tile's rows split into two halves of eight whose start banks (4-word
// groups) are all distinct; rowmap lists half 0, then half 1. tile_span:
// shared-memory bytes a 16-row tile takes.
bool place_rows(DParams &p, int &tile_span) {
  if (!p.padded) {
    for (int g = 0; g < 8; ++g) {
      p.rowmap[g] = static_cast<uint8_t>(2 * g);
      p.rowmap[g + 8] = static_cast<uint8_t>(2 * g + 1);
    }
    tile_span = 16 * static_cast<int>(p.row_bytes);
    return true;
  }
  const int64_t rb = p.row_bytes;
  for (int lg = 4; lg >= 0; --lg) {
    const int gr = 1 << lg;
    for (int gap = 0; gap < 128; gap += 16) {
      const int64_t pitch = gr * rb + gap;
      int first[8], second[8], seen[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      bool ok = true;
      for (int r = 0; r < 16 && ok; ++r) {
        const int bank = static_cast<int>((((r >> lg) * pitch + (r & (gr - 1)) * rb) / 4) % 32) / 4;
        if (seen[bank] == 0) first[bank] = r;
        else if (seen[bank] == 1) second[bank] = r;
        else ok = false;
        ++seen[bank];
      }
      for (int b = 0; b < 8 && ok; ++b) ok = seen[b] == 2;
      if (!ok) continue;
      for (int b = 0; b < 8; ++b) {
        p.rowmap[b] = static_cast<uint8_t>(first[b]);
        p.rowmap[b + 8] = static_cast<uint8_t>(second[b]);
      }
      p.lg_sub = lg;
      p.sub_pitch = static_cast<int>(pitch);
      tile_span = static_cast<int>((16 >> lg) * pitch);
      return true;
    }
  }
  return false;
}

bool try_launch_digits(const DevInfo &dev, int nproj, const int64_t *N, const void *const *W, int K, const float *X,
                       float *const *Y, bool single, cudaStream_t stream, uint32_t flags, qmm_status *out,
                       int wtype = QMM_Q8_0) {
  const bool q4 = wtype == QMM_Q4_0;
  if (nproj < 1 || nproj > kMaxProj) return false;
  if (!q4 && K > 2048) return false;
  // Q4_0: one GEMV whose rows are 16-byte multiples (copied in groups of rows)
  if (q4 && (nproj != 1 || K % 256 != 0 || K > 8192)) return false;
  const int KB = K / 32;
  const int tps = K <= 1024 ? 2 : 1;
  if ((KB + 16 / tps - 1) / (16 / tps) > kMaxSliceBlocks) return false;  // checked again below for 8 warps
  DParams p{};
  int64_t chunks = 0;
  for (int i = 0; i < nproj; ++i) {
    p.Wp[i] = static_cast<const uint8_t *>(W[i]);
    p.Yp[i] = Y[i];
    p.Np[i] = N[i];
    p.chunk0[i] = chunks;
    chunks += (N[i] + 16 * tps - 1) / (16 * tps);
  }
  p.chunk0[nproj] = chunks;
  p.nproj = nproj;
  p.X = X;
  p.K = K;
  p.KB = KB;
  p.row_bytes = (q4 ? 18ll : 34ll) * KB;
  p.padded = q4 ? 1 : 0;
  int tile_span = 16 * static_cast<int>(p.row_bytes);  // bytes of a 16-row tile in shared memory
  if (!place_rows(p, tile_span)) return false;
  p.wexp = q4 ? -4 : 0;
  p.tps = tps;
  p.prefetch_before_wait = (flags & kPrefetchBeforeWait) ? 1 : 0;
  p.stage_bytes = align_up(static_cast<int64_t>(tps) * tile_span + 64, 128);
  p.rows_aligned = (p.row_bytes % 4) == 0 ? 1 : 0;
  auto layout = [&](int warps) {  // shared-memory offsets for `warps` consumer warps
    p.tab_off = 1024;
    p.ftab_off = p.tab_off + 8 * kTabStride * KB;
    p.eb_off = p.ftab_off + warps * kMaxSliceBlocks * 4 * 4;
    p.red_off = align_up(p.eb_off + 4ll * KB, 16);
    p.stage_off = align_up(p.red_off + 4ll * kMaxStages * 16 * warps, 128);  // K-slice partials
  };
  // two CTAs of eight consumer warps per SM when two stages fit in half the
  // shared memory; Q4_0 rows of long K may take one CTA of sixteen per SM
  constexpr int kHalfBudget = 113 * 1024;
  int per_sm = 2, budget = kHalfBudget, nw = kDigitWarps;
  layout(nw);
  if (p.stage_off + 2 * p.stage_bytes > kHalfBudget) {
    if (!q4) return false;
    per_sm = 1;
    budget = 2 * kHalfBudget;
    nw = 16;
    layout(nw);
  }
  if ((KB + nw / tps - 1) / (nw / tps) > kMaxSliceBlocks) return false;
  int grid = per_sm * dev.sms;
  if (single && !q4) {
    if (N[0] < static_cast<int64_t>(grid) * 32) return false;  // one GEMV takes this kernel only for many rows
  } else {
    grid = static_cast<int>(std::min<int64_t>(grid, chunks));  // every CTA at least one chunk
  }
  if (grid < 1) return false;
  p.grid = grid;
  p.stages = std::min(kMaxStages, (budget - p.stage_off) / p.stage_bytes);
  if (p.stages < 2) return false;
  const size_t smem = static_cast<size_t>(p.stage_off) + static_cast<size_t>(p.stages) * p.stage_bytes;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3((nw + 1) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // the projection table is a compile-time choice: one matrix keeps the plain loop
  const bool multi = nproj > 1;
  void (*kern)(DParams) =
      q4 ? (nw == 16 ? (tps == 2 ? q8_gemv_digits_kernel<2, false, QMM_Q4_0, 16> : q8_gemv_digits_kernel<1, false, QMM_Q4_0, 16>)
                     : (tps == 2 ? q8_gemv_digits_kernel<2, false, QMM_Q4_0, 8> : q8_gemv_digits_kernel<1, false, QMM_Q4_0, 8>))
         : (tps == 2 ? (multi ? q8_gemv_digits_kernel<2, true, QMM_Q8_0, 8> : q8_gemv_digits_kernel<2, false, QMM_Q8_0, 8>)
                     : (multi ? q8_gemv_digits_kernel<1, true, QMM_Q8_0, 8> : q8_gemv_digits_kernel<1, false, QMM_Q8_0, 8>));
  static DeviceFlags configured[2][2][2][2];
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  if (!configured[q4][nw == 16][tps - 1][multi].done(dev_id)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * kHalfBudget);
    if (e != cudaSuccess) {
      *out = cuda_check(e, "q8_gemv attribute");
      return true;
    }
    configured[q4][nw == 16][tps - 1][multi].set(dev_id);
  }
  *out = cuda_check(cudaLaunchKernelEx(&cfg, kern, p), "q8_gemv launch");
  return true;
}

}  // namespace

bool launch_q4_gemv_digits(const DevInfo &dev, int64_t N, int K, const void *W, const float *X, float *Y,
                           cudaStream_t stream, uint32_t flags, qmm_status *out) {
  const int64_t n1[1] = {N};
  const void *w1[1] = {W};
  float *y1[1] = {Y};
  return try_launch_digits(dev, 1, n1, w1, K, X, y1, true, stream, flags, out, QMM_Q4_0);
}

qmm_status launch_q8_gemv(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X, float *Y,
                          cudaStream_t stream, uint32_t flags) {
  qmm_status st;
  if (M == 1) {
    // Slices whose fp32 register form would fill the SM go to the tensor-core
    // variant (two launches per SM); smaller ones to the fp32 resident kernel.
    const int64_t rows_per_cta = (N + dev.sms - 1) / dev.sms;
    if (rows_per_cta * K >= kMmaMinSliceWeights && K <= kMmaMaxK && try_launch_mma(dev, N, K, W, X, Y, stream, flags, &st))
      return st;
    if (try_launch_resident(dev, N, K, W, X, Y, stream, flags, &st)) return st;
    const int64_t n1[1] = {N};
    const void *w1[1] = {W};
    float *y1[1] = {Y};
    if (try_launch_digits(dev, 1, n1, w1, K, X, y1, true, stream, flags, &st)) return st;
  }
  return launch_stream<kModeF32>(dev, M, N, K, W, X, nullptr, nullptr, Y, nullptr, stream, flags);
}

// Short rows (at most 64 blocks) at M = 1: the fused Q8xQ8 form when its
// weight slice fits on chip; everything else the fp32-activation GEMV.
constexpr int kAutoMaxKBlocks = 64;

qmm_status launch_q8_gemv_auto(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X, float *Y,
                               int8_t *QX, float *DX, cudaStream_t stream, uint32_t flags) {
  qmm_status st;
  if (M == 1 && K / 32 <= kAutoMaxKBlocks && try_launch_q8q8_resident(dev, N, K, W, X, QX, DX, Y, stream, flags, &st))
    return st;
  return launch_q8_gemv(dev, M, N, K, W, X, Y, stream, flags);
}

qmm_status launch_q8_gemv_multi(const DevInfo &dev, int M, int K, int nproj, const int64_t *N, const void *const *W,
                                const float *X, float *const *Y, cudaStream_t stream, uint32_t flags) {
  qmm_status st;
  // One launch over all projections: the integer streaming kernel (M = 1, K <= 2048).
  if (M == 1 && try_launch_digits(dev, nproj, N, W, K, X, Y, false, stream, flags, &st)) return st;
  // Otherwise one launch per projection.
  for (int i = 0; i < nproj; ++i) {
    st = launch_q8_gemv(dev, M, N[i], K, W[i], X, Y[i], stream, flags);
    if (st != QMM_OK) return st;
  }
  return QMM_OK;
}

qmm_status launch_q8q8_gemv(const DevInfo &dev, int M, int64_t N, int K, const void *W, const int8_t *QX,
                            const float *DX, float *Y, cudaStream_t stream, uint32_t flags) {
  return launch_stream<kModeQ8>(dev, M, N, K, W, nullptr, QX, DX, Y, nullptr, stream, flags);
}

qmm_status launch_q8q8_gemv_fused(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X,
                                  int8_t *QX, float *DX, float *Y, cudaStream_t stream, uint32_t flags) {
  qmm_status st;
  if (M == 1 && try_launch_q8q8_resident(dev, N, K, W, X, QX, DX, Y, stream, flags, &st)) return st;
  // Other shapes: the same quantisation as its own launch into the caller's
  // QX / DX, then the streaming Q8xQ8 kernel.
  st = launch_quantize_act_q8(dev, M, K, X, QX, DX, stream, kLaunchPdl);
  if (st != QMM_OK) return st;
  return launch_stream<kModeQ8>(dev, M, N, K, W, nullptr, QX, DX, Y, nullptr, stream, flags);
}

qmm_status launch_q8q8_gemv_q8_0(const DevInfo &dev, int M, int64_t N, int K, const void *W, const uint8_t *XB,
                                 float *Y, cudaStream_t stream, uint32_t flags) {
  return launch_stream<kModeQ8>(dev, M, N, K, W, nullptr, nullptr, nullptr, Y, nullptr, stream, flags, XB);
}

qmm_status launch_q8q8_block_dots(const DevInfo &dev, int M, int64_t N, int K, const void *W, const int8_t *QX,
                                  const uint8_t *XB, int32_t *isum, cudaStream_t stream) {
  return launch_stream<kModeQ8Dots>(dev, M, N, K, W, nullptr, QX, nullptr, nullptr, isum, stream, kLaunchPdl, XB);
}

qmm_status launch_q8q8_gemv_fused_dots(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X,
                                       int8_t *QX, float *DX, float *Y, int32_t *isum, cudaStream_t stream) {
  qmm_status st;
  // the kernel choice of launch_q8q8_gemv_fused; its resident kernel in the dump instance
  if (M == 1 && try_launch_q8q8_resident(dev, N, K, W, X, QX, DX, Y, stream, kLaunchPdl, &st, isum)) return st;
  st = launch_quantize_act_q8(dev, M, K, X, QX, DX, stream, kLaunchPdl);
  if (st != QMM_OK) return st;
  st = launch_stream<kModeQ8>(dev, M, N, K, W, nullptr, QX, DX, Y, nullptr, stream, kLaunchPdl);
  if (st != QMM_OK) return st;
  return launch_stream<kModeQ8Dots>(dev, M, N, K, W, nullptr, QX, nullptr, nullptr, isum, stream, kLaunchPdl);
}

qmm_status launch_q8_gemv_withheld(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X,
                                   float *Y, uint64_t wait_ns, cudaStream_t stream) {
  return launch_stream<kModeF32>(dev, M, N, K, W, X, nullptr, nullptr, Y, nullptr, stream, kLaunchPdl, nullptr,
                                 wait_ns, 1);
}

cudaError_t q8_gemv_status(uint32_t *bits) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(bits, g_q8_gemv_status, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_q8_gemv_status, &zero, sizeof(uint32_t));
  return e;
}

}  // namespace qmm
