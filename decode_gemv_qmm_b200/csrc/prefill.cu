// prefill.cu -- many-token matmul Y = X . W^T on the tcgen05 tensor cores, with
// W in Q8_0 or Q4_0 blocks decoded to bf16 in shared memory.
//
// Operation ("LSE v0.4.16", section "Retained optimizations and
// compatibility": the M1024 prefill panels): Y[m][n] = sum_k X[m][k] W[n][k]
// with bf16 activations X, block-quantized weights and fp32 output. Each weight
// is decoded once per tile as bf16_rne(q * d) (exact q * d in fp32, one
// round-to-nearest-even to bf16) and the products accumulate in fp32 in
// tensor memory.
//
// B200 design (one CTA per 128 x MT output tile, MT <= 256 tokens):
//  * MMA shape M = 128 weight rows, N = MT tokens, K = 16 (kind::f16, bf16
//    inputs, fp32 accumulator in TMEM, one thread issues, cta_group::1). The
//    accumulator D[n][m] lives in MT TMEM columns x 128 lanes.
//  * A (weights, 128 x 64 per stage) is written by four "dequant" warps in
//    the canonical K-major 128-byte-swizzled layout (8-row atoms of 1 KB,
//    16-byte chunk c of row r at c ^ (r % 8)); B (X, MT x 64 per stage) comes
//    straight from a 2-D TMA load with the same 128-byte swizzle.
//  * Raw weight blocks arrive in 8-block (256 k) chunks per 128-row tile:
//    by 2-D TMA (W viewed as uint16 rows; needs 16-byte row pitch, i.e.
//    K % 256 == 0) or, otherwise, by the dequant warps' own global loads.
//  * Pipelines: producer -> (X tile, raw chunk) -> dequant -> A tile -> MMA
//    -> tcgen05.commit frees the stage. After the last MMA a commit signals
//    the four dequant warps, which become the epilogue: tcgen05.ld 32 columns
//    at a time (lane = weight row) and coalesced stores of Y.
//  * Every mbarrier wait is bounded; on a timeout the kernel records a status
//    bit, finishes without waiting further and still frees its TMEM.
#include <algorithm>

#include "qmm_common.cuh"
#include "qmm_internal.h"
#include "qmm_tmap.h"

namespace qmm {
namespace {

static __device__ uint32_t g_prefill_status;

constexpr int kThreads = 192;          // warp 0 producer, warp 1 MMA, warps 2-5 dequant + epilogue
constexpr int kRawBlocks = 8;          // blocks per raw weight chunk
constexpr int kStageK = 64;            // k per MMA stage (one 128-byte swizzle row of bf16)
constexpr int kATileBytes = 128 * 128; // 128 rows x 64 bf16
constexpr int kRawStages = 2;

struct alignas(64) Params {
  CUtensorMap tm_x;    // X: dims {K, M} bf16, box {64, MT}, 128-byte swizzle
  CUtensorMap tm_w;    // W: dims {row_bytes / 2, N} uint16, box {raw_box_elems, 128}
  const uint8_t *W;
  float *Y;
  int M, K, KB;
  int64_t N;
  int64_t row_bytes;
  int MT;              // tokens per tile (multiple of 16, <= 256)
  int tmem_cols;
  int stages;          // MMA stages in flight
  int raw_pitch;       // bytes per row of a raw chunk in shared memory
  int x_stage_bytes;
  int off_x, off_a, off_raw;  // shared-memory offsets (1024-aligned)
  int tma_w;           // raw weights by TMA (1) or by the dequant warps' loads (0)
};

// ---------------------------------------------------------------- tcgen05 PTX

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major; accumulate when `acc`.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc ? 1u : 0u)
      : "memory");
}
// Arrive once on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Generic-proxy shared-memory writes -> visible to the async proxy (the MMA).
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// K-major, 128-byte swizzle, 8-row atoms 1024 bytes apart (SM100 descriptor).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}
// kind::f16 instruction descriptor: D f32, A = B = bf16, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// ------------------------------------------------------------- block decode

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}
// Four int8 codes (word w) times d -> two bf16x2 words (elements in order).
__device__ __forceinline__ void q8_word_bf16(uint32_t w, float d, uint32_t &o01, uint32_t &o23) {
  const uint32_t q = w ^ 0x80808080u;
  const float2 nb = make_float2(-8388736.0f, -8388736.0f), dd = make_float2(d, d);
  float2 f01 = make_float2(__uint_as_float(__byte_perm(q, 0x4B000000u, 0x7440u)),
                           __uint_as_float(__byte_perm(q, 0x4B000000u, 0x7441u)));
  float2 f23 = make_float2(__uint_as_float(__byte_perm(q, 0x4B000000u, 0x7442u)),
                           __uint_as_float(__byte_perm(q, 0x4B000000u, 0x7443u)));
  f01 = __fmul2_rn(__fadd2_rn(f01, nb), dd);  // q exact, then q * d exact in fp32
  f23 = __fmul2_rn(__fadd2_rn(f23, nb), dd);
  o01 = bf16x2(f01.x, f01.y);
  o23 = bf16x2(f23.x, f23.y);
}
// Four 4-bit codes in the low nibble of each byte of v: (n - 8) * d -> bf16.
__device__ __forceinline__ void q4_nib_bf16(uint32_t v, float d, uint32_t &o01, uint32_t &o23) {
  const float2 nb = make_float2(-8388616.0f, -8388616.0f), dd = make_float2(d, d);  // -(2^23 + 8)
  float2 f01 = make_float2(__uint_as_float(__byte_perm(v, 0x4B000000u, 0x7440u)),
                           __uint_as_float(__byte_perm(v, 0x4B000000u, 0x7441u)));
  float2 f23 = make_float2(__uint_as_float(__byte_perm(v, 0x4B000000u, 0x7442u)),
                           __uint_as_float(__byte_perm(v, 0x4B000000u, 0x7443u)));
  f01 = __fmul2_rn(__fadd2_rn(f01, nb), dd);
  f23 = __fmul2_rn(__fadd2_rn(f23, nb), dd);
  o01 = bf16x2(f01.x, f01.y);
  o23 = bf16x2(f23.x, f23.y);
}

// Store 16-byte chunk c (bf16 elements 8c..8c+7) of A-tile row r, swizzled.
__device__ __forceinline__ void st_a_chunk(uint32_t a_base, int r, int c, uint32_t w0, uint32_t w1, uint32_t w2,
                                           uint32_t w3) {
  const uint32_t addr = a_base + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4);
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1), "r"(w2), "r"(w3)
               : "memory");
}

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // barriers: x_full[8], a_full[8], st_empty[8], raw_full[2], raw_empty[2], acc_full, tmem slot
  uint64_t *x_full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *a_full = x_full + 8;
  uint64_t *st_empty = a_full + 8;
  uint64_t *raw_full = st_empty + 8;
  uint64_t *raw_empty = raw_full + 2;
  uint64_t *acc_full = raw_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
  volatile uint32_t *abort_flag = tmem_slot + 1;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.stages;
  const int nstages = (p.K + kStageK - 1) / kStageK;
  const int nraw = (p.KB + kRawBlocks - 1) / kRawBlocks;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 128;
  const int m0 = blockIdx.y * p.MT;
  constexpr int kBlockBytes = (WT == QMM_Q8_0) ? 34 : 18;

  pdl_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&a_full[s], 4);
      mbar_init(&st_empty[s], 1);
    }
    for (int r = 0; r < kRawStages; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], 4);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, static_cast<uint32_t>(p.tmem_cols));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Bounded wait shared by all roles: after any timeout every later wait
  // returns at once, so the CTA always reaches the TMEM release below.
  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    atomicOr(&g_prefill_status, kDevTimeoutFull);
    return false;
  };

  const uint32_t sbase = smem_u32(smem);
  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      pdl_wait();
      int raw_issued = 0;
      auto issue_raw = [&](int r) {
        const int slot = r % kRawStages;
        if (r >= kRawStages) wait(&raw_empty[slot], static_cast<uint32_t>(r / kRawStages - 1) & 1u);
        mbar_arrive_expect_tx(&raw_full[slot], static_cast<uint32_t>(128 * p.raw_pitch));
        tma_load_2d(smem + p.off_raw + slot * 128 * p.raw_pitch, &p.tm_w, r * kRawBlocks * kBlockBytes / 2,
                    static_cast<int>(n0), &raw_full[slot]);
      };
      for (int j = 0; j < nstages; ++j) {
        const int s = j % S;
        if (p.tma_w) {  // keep the raw chunk feeding this stage (and the next) in flight
          const int need = min(nraw, (j * kStageK) / (kRawBlocks * 32) + 2);
          while (raw_issued < need) issue_raw(raw_issued++);
        }
        if (j >= S) wait(&st_empty[s], static_cast<uint32_t>(j / S - 1) & 1u);
        mbar_arrive_expect_tx(&x_full[s], static_cast<uint32_t>(p.x_stage_bytes));
        tma_load_2d(smem + p.off_x + s * p.x_stage_bytes, &p.tm_x, j * kStageK, m0, &x_full[s]);
      }
    }
    __syncwarp();  // no early exit: every warp meets at the final barrier
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(p.MT);
      for (int j = 0; j < nstages; ++j) {
        const int s = j % S;
        const uint32_t ph = static_cast<uint32_t>(j / S) & 1u;
        wait(&x_full[s], ph);
        wait(&a_full[s], ph);
        tc_fence_after();
        if (!*abort_flag) {
          const uint32_t a_addr = sbase + p.off_a + s * kATileBytes;
          const uint32_t b_addr = sbase + p.off_x + s * p.x_stage_bytes;
#pragma unroll
          for (int kk = 0; kk < kStageK / 16; ++kk)
            umma_f16(tmem, sw128_kmajor_desc(a_addr + 32 * kk), sw128_kmajor_desc(b_addr + 32 * kk), idesc,
                     j > 0 || kk > 0);
        }
        umma_commit(&st_empty[s]);  // frees this stage's A and X buffers when the MMAs finish
      }
      umma_commit(acc_full);        // accumulator complete
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ dequant warps
    pdl_wait();
    const int r = tid - 64;  // A-tile row = weight row n0 + r
    const int64_t n = n0 + r;
    const bool row_ok = n < p.N;
    const uint32_t a_base0 = sbase + p.off_a;
    for (int j = 0; j < nstages; ++j) {
      const int s = j % S;
      const int kb0 = j * 2;  // first of this stage's two blocks
      const int raw = kb0 / kRawBlocks, q = (kb0 % kRawBlocks) / 2;
      if (p.tma_w && q == 0) wait(&raw_full[raw % kRawStages], static_cast<uint32_t>(raw / kRawStages) & 1u);
      if (j >= S) wait(&st_empty[s], static_cast<uint32_t>(j / S - 1) & 1u);
      const uint32_t a_base = a_base0 + s * kATileBytes;
      // the two blocks' bytes as aligned 32-bit words (Q8: 68 bytes = 17 words, Q4: 36 bytes = 9 words)
      constexpr int kWords = (2 * kBlockBytes + 3) / 4;
      uint32_t w[kWords];
      const bool have2 = kb0 + 1 < p.KB;
      if (p.tma_w) {
        const uint32_t ra = sbase + p.off_raw + (raw % kRawStages) * 128 * p.raw_pitch + r * p.raw_pitch +
                            q * 2 * kBlockBytes;  // 4-byte aligned: 68q / 36q
#pragma unroll
        for (int i = 0; i < kWords; ++i) w[i] = lds_u32(ra + 4 * i);
      } else if (row_ok) {
        const uint8_t *src = p.W + n * p.row_bytes + static_cast<int64_t>(kb0) * kBlockBytes;
        if (have2 && (reinterpret_cast<uintptr_t>(src) & 3) == 0) {
#pragma unroll
          for (int i = 0; i < kWords; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t *>(src) + i);
        } else {  // 2-byte aligned, or a lone final block: never read past the block
          const uint16_t *h = reinterpret_cast<const uint16_t *>(src);
#pragma unroll
          for (int i = 0; i < kWords; ++i) {
            const bool in0 = have2 || 4 * i + 2 <= kBlockBytes, in1 = have2 || 4 * i + 4 <= kBlockBytes;
            w[i] = (in0 ? static_cast<uint32_t>(__ldg(h + 2 * i)) : 0u) |
                   (in1 ? static_cast<uint32_t>(__ldg(h + 2 * i + 1)) << 16 : 0u);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < kWords; ++i) w[i] = 0u;
      }
      if constexpr (WT == QMM_Q8_0) {
        // block 0: d = bytes 0-1, qs at bytes 2..33; block 1: d = bytes 34-35, qs at 36..67
        float d0 = half_bits_to_float(w[0]), d1 = half_bits_to_float(w[8] >> 16);
        if (!row_ok) d0 = d1 = 0.f;
        if (!have2) d1 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // block 0 -> chunks 0..3 (qs words unaligned by 2 bytes)
          uint32_t o[4];
          q8_word_bf16(__funnelshift_r(w[2 * c], w[2 * c + 1], 16), d0, o[0], o[1]);
          q8_word_bf16(__funnelshift_r(w[2 * c + 1], w[2 * c + 2], 16), d0, o[2], o[3]);
          st_a_chunk(a_base, r, c, o[0], o[1], o[2], o[3]);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // block 1 -> chunks 4..7 (qs words aligned)
          uint32_t o[4];
          q8_word_bf16(w[9 + 2 * c], d1, o[0], o[1]);
          q8_word_bf16(w[10 + 2 * c], d1, o[2], o[3]);
          st_a_chunk(a_base, r, 4 + c, o[0], o[1], o[2], o[3]);
        }
      } else {
        // block 0: d = bytes 0-1, qs at 2..17; block 1: d = bytes 18-19, qs at 20..35
        float d0 = half_bits_to_float(w[0]), d1 = half_bits_to_float(w[4] >> 16);
        if (!row_ok) d0 = d1 = 0.f;
        if (!have2) d1 = 0.f;
        uint32_t qs0[4], qs1[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          qs0[i] = __funnelshift_r(w[i], w[i + 1], 16);
          qs1[i] = w[5 + i];
        }
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const uint32_t *qs = b ? qs1 : qs0;
          const float d = b ? d1 : d0;
#pragma unroll
          for (int half = 0; half < 2; ++half) {  // low nibbles: elements 0..15, high: 16..31
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint32_t v0 = half ? (qs[2 * c] >> 4) & 0x0F0F0F0Fu : qs[2 * c] & 0x0F0F0F0Fu;
              const uint32_t v1 = half ? (qs[2 * c + 1] >> 4) & 0x0F0F0F0Fu : qs[2 * c + 1] & 0x0F0F0F0Fu;
              uint32_t o[4];
              q4_nib_bf16(v0, d, o[0], o[1]);
              q4_nib_bf16(v1, d, o[2], o[3]);
              st_a_chunk(a_base, r, b * 4 + half * 2 + c, o[0], o[1], o[2], o[3]);
            }
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&a_full[s]);
        if (p.tma_w && (q == kRawBlocks / 2 - 1 || kb0 + 2 >= p.KB)) mbar_arrive(&raw_empty[raw % kRawStages]);
      }
    }

    // ------------------------------------------------------------ epilogue
    wait(acc_full, 0);
    tc_fence_after();
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 belong to this warp
    const int64_t row = n0 + 32 * quarter + lane;
    for (int c0 = 0; c0 < p.MT; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + static_cast<uint32_t>(c0), v);
      if (!*abort_flag && row < p.N) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int m = m0 + c0 + c;
          if (m < p.M) p.Y[static_cast<int64_t>(m) * p.N + row] = __uint_as_float(v[c]);
        }
      }
    }
  }

  // release the accumulator (all tcgen05.ld done before the barrier)
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}

template <int WT>
cudaError_t launch(const cudaLaunchConfig_t &cfg, const Params &p) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<WT>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return cudaLaunchKernelEx(&cfg, prefill_kernel<WT>, p);
}

int round_up(int v, int a) { return (v + a - 1) / a * a; }

}  // namespace

qmm_status launch_prefill(const DevInfo &dev, int wtype, int64_t M, int64_t N, int K, const void *W,
                          const uint16_t *X, float *Y, cudaStream_t stream, uint32_t flags) {
  Params p{};
  p.W = static_cast<const uint8_t *>(W);
  p.Y = Y;
  p.M = static_cast<int>(M);
  p.K = K;
  p.KB = K / 32;
  p.N = N;
  const int bb = wtype == QMM_Q8_0 ? 34 : 18;
  p.row_bytes = static_cast<int64_t>(bb) * p.KB;
  p.MT = static_cast<int>(std::min<int64_t>(256, round_up(static_cast<int>(std::min<int64_t>(M, 256)), 16)));
  p.tmem_cols = p.MT <= 32 ? 32 : p.MT <= 64 ? 64 : p.MT <= 128 ? 128 : 256;
  p.x_stage_bytes = p.MT * 128;
  p.tma_w = (p.row_bytes % 16 == 0) ? 1 : 0;
  p.raw_pitch = kRawBlocks * bb;  // 272 (Q8) or 144 (Q4): box rows are dense
  const int raw_bytes = p.tma_w ? kRawStages * 128 * p.raw_pitch : 0;
  const int per_stage = p.x_stage_bytes + kATileBytes;
  const int budget = dev.smem_optin - 1024 /*align*/ - 1024 /*barriers*/ - round_up(raw_bytes, 1024);
  p.stages = std::max(2, std::min(8, budget / per_stage));
  p.off_x = 1024;
  p.off_a = p.off_x + p.stages * p.x_stage_bytes;
  p.off_raw = p.off_a + p.stages * kATileBytes;
  const size_t smem = static_cast<size_t>(p.off_raw) + raw_bytes + 1024;
  if (smem > static_cast<size_t>(dev.smem_optin))
    return set_error(QMM_ERR_SHAPE, "prefill: tile needs %zu bytes of shared memory", smem);

  const uint64_t xd[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  const uint64_t xs[1] = {static_cast<uint64_t>(K) * 2};
  const uint32_t xb[2] = {64, static_cast<uint32_t>(p.MT)};
  qmm_status st = encode_tiled(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, xd, xs, xb, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QMM_OK) return st;
  if (p.tma_w) {
    const uint64_t wd[2] = {static_cast<uint64_t>(p.row_bytes / 2), static_cast<uint64_t>(N)};
    const uint64_t ws[1] = {static_cast<uint64_t>(p.row_bytes)};
    const uint32_t wb[2] = {static_cast<uint32_t>(p.raw_pitch / 2), 128};
    st = encode_tiled(&p.tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, W, wd, ws, wb, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != QMM_OK) return st;
  }

  const int64_t ntiles = (N + 127) / 128, mtiles = (M + p.MT - 1) / p.MT;
  if (ntiles > 0x7fffffff || mtiles > 65535) return set_error(QMM_ERR_SHAPE, "prefill: grid too large");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(ntiles), static_cast<unsigned>(mtiles));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(wtype == QMM_Q8_0 ? launch<QMM_Q8_0>(cfg, p) : launch<QMM_Q4_0>(cfg, p), "prefill launch");
}

cudaError_t prefill_status(uint32_t *bits) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(bits, g_prefill_status, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_prefill_status, &zero, sizeof(uint32_t));
  return e;
}

}  // namespace qmm
