// prefill.cu -- many-token matmul Y = X . W^T on Q8_0 or Q4_0 blocks: above 32
// tokens on the tcgen05 tensor cores, each block decoded to bf16 and written
// into tensor memory as the A operand; up to 32 tokens by a small-M mma.sync
// kernel on the exact integer codes held in shared memory.
//
// Operation ("LSE v0.4.16", section "Retained optimizations and
// compatibility": the M1024 prefill panels): Y[m][n] = sum_k X[m][k] W[n][k]
// with bf16 activations X, block-quantized weights and fp32 output. Each weight
// is decoded once per tile as bf16_rne(q * d) (exact q * d in fp32, one
// round-to-nearest-even to bf16) and the products accumulate in fp32 in
// tensor memory.
//
// B200 design (one CTA per 128 x MT output tile and K range, MT <= 384 tokens):
//  * MMA shape M = 128 weight rows, N = MT tokens, K = 16 (kind::f16, bf16
//    inputs, fp32 accumulator in TMEM, one thread issues, cta_group::1). The
//    accumulator D[n][m] lives in MT TMEM columns x 128 lanes. A tile wider
//    than 256 tokens (one MMA's limit) takes two MMAs per k step, tokens
//    0..255 and 256..MT-1 of the same A; the launcher picks such tiles when
//    they cut the number of waves (1024 tokens x 4864 rows: 114 tiles of 352
//    tokens in one wave instead of 152 of 256 in two).
//  * A (weights, 128 x 64 per stage) never touches shared memory: sixteen
//    "dequant" warps in two groups that take alternate stages (each warp has
//    two stages of MMA time per stage it converts) write each decoded row
//    into tensor memory (tcgen05.st,
//    lane = weight row, two bf16 per 32-bit column; a ring of 32-column stages
//    beside the accumulator) and the MMA takes A from there. Shared memory
//    then carries only X and the raw blocks, which is what let the pipeline
//    keep up: with A in shared memory the operand reads, TMA writes and
//    dequant stores of one stage exceeded the SM's shared-memory bandwidth.
//    B (X, MT x 64 per stage) comes from a 2-D TMA load with the 128-byte
//    swizzle.
//  * Raw weight blocks arrive in 8-block (256 k) chunks per 128-row tile by
//    2-D TMA. A Q8_0 row is 34 * K/32 bytes, in general not a multiple of 16
//    (a TMA row pitch must be), so W is viewed as super-rows of rs = 1, 2, 4
//    or 8 rows whose pitch is; one box per row position of a super-row, each
//    started at the 16-byte boundary below the chunk, and the dequant warps
//    index from the row's offset. The < rs rows at the end of W that do not
//    fill a super-row are read by the dequant warps directly.
//  * Split K: when the output tiles alone leave SMs idle, the K range is split
//    across the CTAs of a thread-block cluster (gridDim.z = cluster size).
//    After every CTA's accumulator is complete, each CTA scatters its partial
//    tile through distributed shared memory so that rank r receives all
//    partials of its 128/S weight rows, then sums them in rank order and
//    writes Y: deterministic, and no global scratch memory.
//  * Pipelines: producer -> (X tile, raw chunk) -> dequant -> A tile -> MMA
//    -> tcgen05.commit frees the stage. One barrier per stage tells the MMA
//    issuer that both its X tile and its A columns are ready; the issuer
//    keeps slots and ring passes incrementally and offsets precomputed
//    descriptors (it is a single thread: every cycle there shows up as an
//    idle tensor pipe). After the last MMA a commit signals the dequant
//    warps, which become the epilogue: tcgen05.ld 32 columns
//    at a time (lane = weight row) and coalesced stores of Y (or the scatter).
//  * Every mbarrier wait is bounded; on a timeout the kernel records a status
//    bit, finishes without waiting further (still meeting both cluster
//    barriers) and frees its TMEM.
//
// Panels of at most 32 tokens run a second kernel in this file, the small-M
// kernel (mma.sync on whole shares of W and X held in shared memory; see its
// description below): at that size the work is bound by streaming the weights
// and by latency, not by the tensor cores.
#include <algorithm>

#include "qmm_common.cuh"
#include "qmm_internal.h"
#include "qmm_tmap.h"

namespace qmm {
namespace {

static __device__ uint32_t g_prefill_status;

constexpr int kDqGroups = 2;           // dequant groups; group g converts the stages i = g (mod kDqGroups)
constexpr int kDqWarps = 8 * kDqGroups; // dequant (then epilogue) warps: thread = (weight row, block of the stage)
constexpr int kThreads = 64 + 32 * kDqWarps;  // warp 0 producer, warp 1 MMA, warps 2.. dequant + epilogue
constexpr int kRawBlocks = 8;          // blocks per raw weight chunk
constexpr int kStageK = 64;            // k per MMA stage (one 128-byte swizzle row of bf16)
constexpr int kMaxMT = 384;            // widest token tile (two MMAs per k step above 256)
constexpr int kACols = 32;             // TMEM columns per A stage: 128 rows x 64 bf16 (two per 32-bit cell)
// Raw chunks in flight. Q8 chunks are twice the size of Q4 ones; two in flight
// (eight stages of lead) leave room for four X stages instead of two, which
// measured 8-15% faster on the Q8 panels.
template <int WT>
constexpr int raw_stages() { return WT == QMM_Q8_0 ? 2 : 4; }
constexpr int kMaxSplit = 8;           // portable cluster size

struct alignas(64) Params {
  CUtensorMap tm_x;    // X: dims {K, M} bf16, box {64, min(MT, 256)}, 128-byte swizzle
  CUtensorMap tm_x2;   // MT > 256: the same X, box {64, MT - 256} (tokens 256.. of a tile)
  CUtensorMap tm_w;    // W as super-rows of rs rows: dims {rs * row_bytes / 2, N / rs} uint16, box {raw_pitch / 2, 128 / rs}
  const uint8_t *W;
  float *Y;
  int M, K, KB;
  int64_t N;
  int64_t row_bytes;
  int64_t tma_rows;    // rows loaded by TMA (whole super-rows); the rest by the dequant warps
  int rs;              // rows per super-row: the smallest of 1, 2, 4, 8 whose pitch is a multiple of 16
  int MT;              // tokens per tile (multiple of 16; above 256 a multiple of 32, <= kMaxMT)
  int acc_cols;        // TMEM columns of the accumulator (max(256, MT)); the A stages follow
  int tmem_cols;
  int stages;          // MMA stages in flight
  int raw_pitch;       // bytes per row of a raw chunk in shared memory (a chunk + up to 15 bytes in front)
  int x_stage_bytes;
  int off_x, off_raw;  // shared-memory offsets (1024-aligned)
  int split;           // K ranges per output tile (cluster size along z)
  int prefetch_before_wait;  // weights may be read before the preceding grid completes
  int red_pitch;       // floats per token column of the split-K exchange buffer (rows of one rank)
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

// D[tmem] (+)= A[tmem] * B[smem]^T: A is 128 lanes (rows) x K packed two
// bf16 per 32-bit column, B K-major in shared memory.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc ? 1u : 0u)
      : "memory");
}
// Each thread of the warp writes 16 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
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

// K-major, 128-byte swizzle, 8-row atoms 1024 bytes apart (SM100 descriptor).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}
// kind::f16 instruction descriptor: D f32, A = B = bf16, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// ---------------------------------------------------------------- cluster PTX

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of all CTAs of the cluster; orders shared-memory accesses across it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared-memory address of this CTA's `saddr` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void st_cluster_b32(uint32_t addr, uint32_t a) {
  asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
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

// WIDE: tiles of more than 256 tokens (two MMAs per k step); a template
// parameter so that the narrow form's single-thread issue loop carries no
// extra test.
template <int WT, bool WIDE>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kRawStages = raw_stages<WT>();
  // barriers: full[8], st_empty[8], raw_full[kRawStages], raw_empty[kRawStages], acc_full, tmem slot.
  // full[s]: the stage's X tile has landed (producer arrival + TMA bytes) and
  // all dequant warps have written its A columns -- one wait for the issuer.
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *st_empty = full + 8;
  uint64_t *raw_full = st_empty + 8;
  uint64_t *raw_empty = raw_full + kRawStages;
  uint64_t *acc_full = raw_empty + kRawStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
  volatile uint32_t *abort_flag = tmem_slot + 1;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.stages;
  const int nst_all = (p.KB + 1) / 2;  // stages of two blocks over the whole K
  const int split = p.split;
  const int zr = split > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int j_lo = zr * nst_all / split, j_hi = (zr + 1) * nst_all / split;
  const int nst = j_hi - j_lo;                              // this CTA's stages
  const int nraw = (nst + kRawBlocks / 2 - 1) / (kRawBlocks / 2);  // raw chunks (four stages each)
  // token tiles vary fastest, so the CTAs sharing a weight tile run together
  // and all but the first read its blocks from L2
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * 128;
  const int m0 = blockIdx.x * p.MT;
  constexpr int kBlockBytes = (WT == QMM_Q8_0) ? 34 : 18;

  pdl_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1 + 8);  // the producer, and the eight warps of the group that converts stage s
      mbar_init(&st_empty[s], 1);
    }
    for (int r = 0; r < kRawStages; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], kDqWarps);  // every dequant warp, after its last stage of the chunk
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
  // The preceding grid's writes (X, and any reader of Y) must be done before
  // X is loaded and Y written. With early weights only the X producer waits
  // here; the weight stream, the dequantisation and the MMAs start at once,
  // and every thread waits again before the epilogue writes Y.
  if (!p.prefetch_before_wait) pdl_wait();

  // Bounded wait shared by all roles: after any timeout every later wait
  // returns at once, so the CTA always reaches the cluster barriers and the
  // TMEM release below.
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
    // raw chunk c: blocks from kb of the tile's 128 rows; one TMA box per row
    // position j of a super-row, started at the 16-byte boundary below the
    // chunk (the dequant warps index from the offset); out-of-range bytes read 0
    auto issue_raw = [&](int c) {
      const int slot = c % kRawStages;
      if (c >= kRawStages) wait(&raw_empty[slot], static_cast<uint32_t>(c / kRawStages - 1) & 1u);
      if (*abort_flag) return;  // after a timeout nothing more is copied
      const int kb = 2 * (j_lo + c * (kRawBlocks / 2));
      if (n0 < p.tma_rows) {
        mbar_arrive_expect_tx(&raw_full[slot], static_cast<uint32_t>(128 * p.raw_pitch));
        const int sub = 128 / p.rs;
        for (int j = 0; j < p.rs; ++j) {
          const int64_t off = j * p.row_bytes + static_cast<int64_t>(kb) * kBlockBytes;
          tma_load_2d(smem + p.off_raw + (slot * 128 + j * sub) * p.raw_pitch, &p.tm_w,
                      static_cast<int>((off & ~int64_t(15)) / 2), static_cast<int>(n0 / p.rs), &raw_full[slot]);
        }
      } else {
        mbar_arrive(&raw_full[slot]);  // every row of this tile is read directly
      }
    };
    // Two independent streams, so that neither waits behind the other's ring:
    // lane 0 feeds the X stages, lane 1 the raw chunks.
    if (lane == 0) {
      if (p.prefetch_before_wait) pdl_wait();
      // stage slot and ring pass kept incrementally: a runtime division per
      // stage costs the serial issuers hundreds of cycles
      for (int i = 0, s = 0, pass = 0; i < nst; ++i) {
        if (pass > 0) wait(&st_empty[s], static_cast<uint32_t>(pass - 1) & 1u);
        if (!*abort_flag) {
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(p.x_stage_bytes));
          tma_load_2d(smem + p.off_x + s * p.x_stage_bytes, &p.tm_x, (j_lo + i) * kStageK, m0, &full[s]);
          if (WIDE)  // tokens 256.. of the tile: 8-row atoms continue 32 KB further on
            tma_load_2d(smem + p.off_x + s * p.x_stage_bytes + 256 * 128, &p.tm_x2, (j_lo + i) * kStageK, m0 + 256,
                        &full[s]);
        }
        if (++s == S) {
          s = 0;
          ++pass;
        }
      }
    } else if (lane == 1) {
      for (int c = 0; c < nraw; ++c) issue_raw(c);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(WIDE ? 256 : p.MT);
      const uint32_t idesc2 = idesc_bf16_f32(WIDE ? p.MT - 256 : 16);  // tokens 256..MT-1
      const uint32_t acc_cols = WIDE ? static_cast<uint32_t>(p.acc_cols) : 256u;
      // descriptors of stage 0; a stage / k step is an offset in 16-byte units
      // of the descriptor's address field (shared-memory addresses < 256 KB)
      const uint64_t bdesc0 = sw128_kmajor_desc(sbase + p.off_x);
      const uint32_t xs16 = static_cast<uint32_t>(p.x_stage_bytes) >> 4;
      for (int i = 0, s = 0, pass = 0; i < nst; ++i) {
        wait(&full[s], static_cast<uint32_t>(pass) & 1u);  // after a timeout: garbage in, discarded
        tc_fence_after();
        const uint64_t bd = bdesc0 + static_cast<uint64_t>(s * xs16);
        const uint32_t at = tmem + acc_cols + static_cast<uint32_t>(s * kACols);
        if (!WIDE) {
          umma_f16_ts(tmem, at, bd, idesc, i > 0);
          umma_f16_ts(tmem, at + 8, bd + 2, idesc, true);
          umma_f16_ts(tmem, at + 16, bd + 4, idesc, true);
          umma_f16_ts(tmem, at + 24, bd + 6, idesc, true);
        } else {
          // tokens 256.. start 256 rows (32 KB = 2048 descriptor units) into the stage
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            umma_f16_ts(tmem, at + 8 * kk, bd + 2 * kk, idesc, i > 0 || kk > 0);
            umma_f16_ts(tmem + 256, at + 8 * kk, bd + 2048 + 2 * kk, idesc2, i > 0 || kk > 0);
          }
        }
        umma_commit(&st_empty[s]);  // frees this stage's A and X buffers when the MMAs finish
        if (++s == S) {
          s = 0;
          ++pass;
        }
      }
      umma_commit(acc_full);        // accumulator complete
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ dequant warps
    // thread (r, h): weight row n0 + r, block h of each stage's two blocks. A
    // warp may only reach its own quarter of the TMEM lanes, so warp w takes
    // rows 32 (w % 4) .. +31; lane = row. Group dg takes every kDqGroups-th
    // stage, so each warp has kDqGroups stages of MMA time per stage it converts.
    const int quarter = warp & 3;
    const int dw = warp - 2, dg = dw >> 3;
    const int r = 32 * quarter + lane, h = (dw >> 2) & 1;
    const int64_t n = n0 + r;
    const bool row_ok = n < p.N;
    const uint32_t a_lane = tmem + (static_cast<uint32_t>(32 * quarter) << 16) +
                            static_cast<uint32_t>((WIDE ? p.acc_cols : 256) + 16 * h);
    constexpr int kWords = (kBlockBytes + 2 + 3) / 4;  // the block as words, plus the 16-bit shift (Q8: 9, Q4: 5)
    int s0 = dg, pass0 = 0;  // the slot and ring pass of stage dg (S >= kDqGroups)
    for (int i = dg, s = s0, pass = pass0; i < nst;
         i += kDqGroups, (s += kDqGroups) >= S ? (s -= S, ++pass) : 0) {
      const int c = i / (kRawBlocks / 2), q = i % (kRawBlocks / 2);
      const int kb = 2 * (j_lo + i) + h;  // this thread's block
      if (q < kDqGroups) wait(&raw_full[c % kRawStages], static_cast<uint32_t>(c / kRawStages) & 1u);
      if (pass > 0) wait(&st_empty[s], static_cast<uint32_t>(pass - 1) & 1u);
      tc_fence_after();  // the MMAs that read this stage's A columns are complete
      const bool have = row_ok && kb < p.KB;
      // w: the block's bytes from its fp16 scale on, as little-endian words
      uint32_t w[kWords];
      if (n < p.tma_rows) {
        // row r sits at position j = r % rs of super-row r / rs; its chunk starts
        // at the source offset modulo 16 inside the box
        const int j = r % p.rs, sub = 128 / p.rs;
        const int64_t off = j * p.row_bytes + static_cast<int64_t>(2 * (j_lo + c * (kRawBlocks / 2))) * kBlockBytes;
        const uint32_t ra = sbase + p.off_raw + ((c % kRawStages) * 128 + j * sub + r / p.rs) * p.raw_pitch +
                            static_cast<uint32_t>(off & 15) + (2 * q + h) * kBlockBytes;
        const uint32_t mis = ra & 3u, wa = ra - mis;  // 2-byte aligned
        if (mis == 0) {
#pragma unroll
          for (int k = 0; k < kWords; ++k) w[k] = lds_u32(wa + 4 * k);
        } else {
          uint32_t prev = lds_u32(wa);
#pragma unroll
          for (int k = 0; k < kWords; ++k) {
            const uint32_t next = lds_u32(wa + 4 * (k + 1));
            w[k] = __funnelshift_r(prev, next, 16);
            prev = next;
          }
        }
      } else if (have) {  // the last rows of W, short of a whole super-row: global loads
        const uint16_t *hp = reinterpret_cast<const uint16_t *>(p.W + n * p.row_bytes + static_cast<int64_t>(kb) * kBlockBytes);
#pragma unroll
        for (int k = 0; k < kWords; ++k) {
          const bool in0 = 4 * k + 2 <= kBlockBytes, in1 = 4 * k + 4 <= kBlockBytes;  // never past the block
          w[k] = (in0 ? static_cast<uint32_t>(__ldg(hp + 2 * k)) : 0u) |
                 (in1 ? static_cast<uint32_t>(__ldg(hp + 2 * k + 1)) << 16 : 0u);
        }
      } else {
#pragma unroll
        for (int k = 0; k < kWords; ++k) w[k] = 0u;
      }
      float d = half_bits_to_float(w[0]);
      if (!have || *abort_flag) d = 0.f;
      uint32_t o[16];  // bf16 pairs of the block's 32 weights, in k order
      if constexpr (WT == QMM_Q8_0) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)  // codes at bytes 2..33
          q8_word_bf16(__funnelshift_r(w[cc], w[cc + 1], 16), d, o[2 * cc], o[2 * cc + 1]);
      } else {
        // nibbles at bytes 2..17: low nibbles = elements 0..15, high = 16..31
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t qs = __funnelshift_r(w[k], w[k + 1], 16);
          q4_nib_bf16(qs & 0x0F0F0F0Fu, d, o[2 * k], o[2 * k + 1]);
          q4_nib_bf16((qs >> 4) & 0x0F0F0F0Fu, d, o[8 + 2 * k], o[9 + 2 * k]);
        }
      }
      tmem_st16(a_lane + static_cast<uint32_t>(s * kACols), o);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&full[s]);
        // this warp's last stage of the chunk (a chunk's slot is reused only after a whole chunk)
        if (q + kDqGroups >= kRawBlocks / 2 || i + kDqGroups >= nst) mbar_arrive(&raw_empty[c % kRawStages]);
      }
    }
    wait(acc_full, 0);  // accumulator complete: every MMA (and so every stage buffer) is done
  }

  // ------------------------------------------------------------ epilogue
  pdl_wait();  // (already passed without early weights)
  const bool epi = warp >= 2;
  const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 belong to this warp
  const int col0 = warp >= 2 ? 32 * ((warp - 2) >> 2) : 0;  // the warps of a quarter take turns at 32 columns
  if (split == 1) {
    if (epi) {
      tc_fence_after();
      const int64_t row = n0 + 32 * quarter + lane;
      // a 32-column load past MT happens only for a single tile (MT = M
      // rounded up to 16, M <= 256); tiles above 256 tokens are multiples of 32
      for (int c0 = col0; c0 < p.MT; c0 += 32 * (kDqWarps / 4)) {
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
  } else {
    // Split K: rank r owns weight rows [r*128/split, (r+1)*128/split) of the
    // tile and receives every rank's partial of them in its X stage and raw
    // chunk buffers (free once all ranks' accumulators are complete: first
    // cluster barrier). The buffer is [source rank][token column][row of the
    // owner], rows contiguous: a warp holds 32 consecutive rows of one column
    // after each TMEM load, so every remote store is one contiguous 128-byte
    // segment (storing each row's columns instead scattered a warp's store
    // over 32 rows and made the exchange several times slower).
    const uint32_t xbuf = sbase + p.off_x;
    cluster_sync_all();
    if (epi) {
      tc_fence_after();
      const int row = 32 * quarter + lane;
      const int dst = (row * split + split - 1) / 128;  // owner rank of this row
      const int lr = row - dst * 128 / split;
      const uint32_t laddr = xbuf + static_cast<uint32_t>((zr * p.MT * p.red_pitch + lr) * 4);
      const uint32_t raddr = map_rank(laddr, static_cast<uint32_t>(dst));
      const bool own = dst == zr;  // this rank's own rows: plain local stores
      const uint32_t cstride = static_cast<uint32_t>(p.red_pitch) * 4u;
      for (int c0 = col0; c0 < p.MT; c0 += 32 * (kDqWarps / 4)) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + static_cast<uint32_t>(c0), v);
        if (own) {
#pragma unroll
          for (int c = 0; c < 32; ++c)  // MT is a multiple of 16: the last load may hold 16 columns
            if (c0 + c < p.MT)
              asm volatile("st.shared.b32 [%0], %1;" ::"r"(laddr + static_cast<uint32_t>(c0 + c) * cstride), "r"(v[c])
                           : "memory");
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c0 + c < p.MT) st_cluster_b32(raddr + static_cast<uint32_t>(c0 + c) * cstride, v[c]);
        }
      }
    }
    cluster_sync_all();  // every partial has landed
    // sum in rank order: warp w takes token columns w, w + nwarps, ...; its
    // lanes 32 consecutive rows of the rank's share (contiguous in the buffer
    // and in Y); no division per element
    const int rbase = zr * 128 / split, rown = (zr + 1) * 128 / split - rbase;
    if (!*abort_flag) {
      const uint32_t srcstride = static_cast<uint32_t>(p.MT * p.red_pitch) * 4u;
      for (int lr0 = 0; lr0 < rown; lr0 += 32) {
        const int lr = lr0 + lane;
        const int64_t row = n0 + rbase + lr;
        const bool rok = lr < rown && row < p.N;
        for (int col = warp; col < p.MT; col += kThreads / 32) {
          const uint32_t a0 = xbuf + static_cast<uint32_t>((col * p.red_pitch + lr) * 4);
          float acc = 0.f;
#pragma unroll
          for (int src = 0; src < kMaxSplit; ++src)
            if (src < split) acc += lds_f32(a0 + static_cast<uint32_t>(src) * srcstride);
          const int m = m0 + col;
          if (rok && m < p.M) p.Y[static_cast<int64_t>(m) * p.N + row] = acc;
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

template <int WT, bool WIDE>
void *kernel_ptr() {
  return reinterpret_cast<void *>(prefill_kernel<WT, WIDE>);
}

int round_up(int v, int a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------------------
// Small-M panels (M <= 32 tokens). Two to four MFLOP per weight row are no
// work for the tensor cores; such a panel is bound by streaming its weights
// from HBM once, plus launch and dependency latency. So no tensor-memory
// pipeline: every CTA copies its whole share of W (rows [r0, r0 + R), K blocks
// [kb0, kb1)) and the matching X slice into shared memory and multiplies with
// mma.sync.m16n8k16 (bf16, fp32 accumulation), one block at a time:
//  * Few, large copies (many small ones made the launch latency-bound: 65 bulk
//    copies of 1-2 KB per CTA took 11.3 us where two take 6.9). Without split
//    K the CTA's rows are one contiguous byte range of W and X is one
//    contiguous range too: one bulk copy each. With split K the rows' segments
//    come as one 2-D TMA box (W viewed as rows of 4-byte words; rows a
//    multiple of 16 bytes long) and X as boxes of 256 k x 8 QM tokens (token
//    rows past M read as zero); other row lengths fall back to a bulk copy
//    per row segment.
//  * The compute loop reads shared memory with plain loads (after the
//    mbarrier waits, which order them) so that a warp's loads, conversions and
//    mma instructions of several tiles and blocks overlap.
//  * A = 16 weight rows x 16 k as bf16 holding the exact integer codes (Q8:
//    q, Q4: n - 8); B = 16 k x 8 tokens of X; C = the block's dot for 16 rows
//    x 8 tokens, exact products summed in fp32, then acc += d * C. The block
//    scale is applied in fp32, so no decoded weight is rounded (the tcgen05
//    path rounds q * d to bf16).
//  * Inside a block k is permuted (the same way in A and B) so that each lane
//    reads its codes as one run of bytes and its activations with one or two
//    vector loads.
//  * Consumer warp (kq, t) takes 16-row tile t and the kq-th quarter of the
//    CTA's K blocks, for every token group; the four quarters' sums are added
//    in order in shared memory. Rows too few for all SMs split K over a
//    thread-block cluster (cluster rank = K range): each rank sends its sums
//    for the rows another rank owns to that rank with remote shared-memory
//    stores, and every rank adds, for its own rows, all ranks' sums in rank
//    order. Deterministic, no global scratch.
//  * With early weights the W copies are issued before the dependency wait;
//    X is copied and Y written after it.

constexpr int kSmMaxTiles = 4;  // 16-row weight tiles per CTA (R <= 64)
constexpr int kSmKParts = 4;    // K ranges per tile inside a CTA
constexpr int kSmWarps = kSmMaxTiles * kSmKParts;  // consumer warps: warp = (K range, tile)
constexpr int kSmMaxM = 32;     // tokens

struct alignas(64) SParams {
  const uint8_t *W;
  const uint16_t *X;
  float *Y;
  int64_t N;
  int64_t row_bytes;
  int64_t total_bytes;
  int M, K, KB;
  int groups;     // row groups (clusters of `split` CTAs)
  int split;      // K ranges per row group
  CUtensorMap tm_x;  // split K: X dims {K, M} bf16, box {256, 8 QM}
  CUtensorMap tm_w;  // split K, rows a multiple of 16 bytes: W as {row_bytes / 4, N} words, box {seg_pitch / 4, rows}
  int w_tma;         // the weight segments come as one tm_w box
  int seg_pitch;     // split K: shared-memory bytes per weight-row segment (16-byte multiple)
  int xjpb;          // K blocks per X row in shared memory (a box of them per 8 QM tokens)
  int w_off, x_off, part_off;
  int prefetch_before_wait;
  // failure-path test only (defaults: kWaitLimitNs, 0): the limit of the
  // consumers' waits, and whether CTA 0 withholds its whole weight copy
  uint64_t wait_ns;
  int withhold;
};

// Not volatile: a pure function of its operands, so the compiler may overlap
// it with the loads of the next tiles (volatile shared loads and mma kept
// every load, conversion and mma of a warp in program order: 5 us of a 7 us
// launch).
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Codes c0..c3 (bytes of w, two's complement) -> bf16 pairs (c0, c1), (c2, c3),
// exact and without a conversion instruction (those issue slowly): c is exact
// in fp32 after the 2^23 trick, and with at most 8 significant bits its bf16
// is the upper half of that fp32.
__device__ __forceinline__ void q8_codes_bf16(uint32_t w, uint32_t &o01, uint32_t &o23) {
  const uint32_t q = w ^ 0x80808080u;
  const float2 nb = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
  float2 f01 = make_float2(__uint_as_float(__byte_perm(q, 0x4B000000u, 0x7440u)),
                           __uint_as_float(__byte_perm(q, 0x4B000000u, 0x7441u)));
  float2 f23 = make_float2(__uint_as_float(__byte_perm(q, 0x4B000000u, 0x7442u)),
                           __uint_as_float(__byte_perm(q, 0x4B000000u, 0x7443u)));
  f01 = __fadd2_rn(f01, nb);
  f23 = __fadd2_rn(f23, nb);
  o01 = __byte_perm(__float_as_uint(f01.x), __float_as_uint(f01.y), 0x7632u);
  o23 = __byte_perm(__float_as_uint(f23.x), __float_as_uint(f23.y), 0x7632u);
}
// fp16 bits -> fp32 without a conversion instruction, exact for normal and
// subnormal values: the exponent and fraction shifted into fp32 position read
// as x * 2^-112 (an fp32 subnormal for an fp16 subnormal), times 2^112.
__device__ __forceinline__ float half_bits_to_float_alu(uint32_t h) {
  return __fmul_rn(__uint_as_float(((h & 0x8000u) << 16) | ((h & 0x7fffu) << 13)), 0x1p112f);
}
// Two nibbles in bits 0..3 and 16..19 of v -> bf16 pair (n - 8), exact:
// 0x4300 | n is 128 + n, minus 136.
__device__ __forceinline__ uint32_t q4_pair_bf16(uint32_t v) {
  uint32_t t = (v & 0x000F000Fu) | 0x43004300u;
  const __nv_bfloat162 k136 = __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308));
  __nv_bfloat162 h = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&t), k136);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Shared-memory offset of weight row r's first block of the CTA's K range
// (2-byte aligned): without split K the rows follow each other at the row
// pitch from the range's offset modulo 16; with it each row segment has its
// own slot.
__device__ __forceinline__ uint32_t small_row_base(const SParams &p, int64_t r0, int kb0, int kbb, int r) {
  if (p.split == 1) return static_cast<uint32_t>((r0 * p.row_bytes) & 15) + static_cast<uint32_t>(r * p.row_bytes);
  return static_cast<uint32_t>(r * p.seg_pitch) +
         static_cast<uint32_t>(((r0 + r) * p.row_bytes + static_cast<int64_t>(kb0) * kbb) & 15);
}

// A fragments (both k steps) and the scale of the block at shared-memory
// offset blk; zero for a row past the last.
template <int WT>
__device__ __forceinline__ void small_row(const uint8_t *wbase, uint32_t blk, bool valid, int qd, uint32_t (&o)[4],
                                          float &d) {
  if (!valid) {
    o[0] = o[1] = o[2] = o[3] = 0u;
    d = 0.f;
    return;
  }
  auto w32 = [&](uint32_t off) { return *reinterpret_cast<const uint32_t *>(wbase + off); };
  d = half_bits_to_float_alu(*reinterpret_cast<const uint16_t *>(wbase + blk));
  if constexpr (WT == QMM_Q8_0) {
    // codes 8 qd .. 8 qd + 7 (2-byte aligned): k slots 2qd, 2qd+1 <- 0, 1 and
    // 2qd+8, 2qd+9 <- 2, 3 (step 0); the same with 4..7 (step 1)
    const uint32_t ca = blk + 2u + 8u * qd, mis = ca & 2u, wa = ca - mis;
    const uint32_t v0 = w32(wa), v1 = w32(wa + 4), v2 = w32(wa + 8);
    q8_codes_bf16(__funnelshift_r(v0, v1, mis << 3), o[0], o[1]);
    q8_codes_bf16(__funnelshift_r(v1, v2, mis << 3), o[2], o[3]);
  } else {
    // bytes 4 qd .. 4 qd + 3: low nibbles = elements 4qd + i, high = 16 + 4qd + i;
    // k slots 2qd, 2qd+1 <- elements (0, 2), 2qd+8, 2qd+9 <- (1, 3), low (step 0) then high (step 1)
    const uint32_t ca = blk + 2u + 4u * qd, mis = ca & 2u, wa = ca - mis;
    const uint32_t v = __funnelshift_r(w32(wa), w32(wa + 4), mis << 3);
    o[0] = q4_pair_bf16(v);
    o[1] = q4_pair_bf16(v >> 8);
    o[2] = q4_pair_bf16(v >> 4);
    o[3] = q4_pair_bf16(v >> 12);
  }
}

template <int WT, int QM>  // QM token groups of eight (M <= 8 QM)
__global__ void __launch_bounds__((kSmWarps + 1) * 32, 1) prefill_small_kernel(const __grid_constant__ SParams p) {
  extern __shared__ __align__(128) uint8_t smem_sm[];
  // 128-byte aligned base, derived by pointer arithmetic on the shared array so
  // that the compiler keeps plain loads through it in the shared address space
  // (a round trip through an integer made them generic loads)
  uint8_t *smem = smem_sm + ((128u - (smem_u32(smem_sm) & 127u)) & 127u);
  uint64_t *wbar = reinterpret_cast<uint64_t *>(smem);
  uint64_t *xbar = wbar + 1;
  constexpr int kBB = WT == QMM_Q8_0 ? 34 : 18;
  constexpr int kCols = 8 * QM;  // token columns of the partial sums
  const int xrow = 64 * p.xjpb;            // bytes per token row of an X box
  const int xbox = 8 * QM * xrow;           // bytes of one X box

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = p.split;
  const int zr = split > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int grp = static_cast<int>(blockIdx.x) / split;
  const int64_t r0 = static_cast<int64_t>(grp) * p.N / p.groups;
  const int R = static_cast<int>((static_cast<int64_t>(grp) + 1) * p.N / p.groups - r0);
  const int kb0 = zr * p.KB / split, kb1 = (zr + 1) * p.KB / split;
  const int nb = kb1 - kb0;
  const uint32_t sbase = smem_u32(smem);

  // abort flag (shared word after the two barriers): set when copies may still
  // be landing in W / X on an error path
  const uint32_t abort_sa = smem_u32(smem) + 16u;
  pdl_launch_dependents();
  if (tid == 0) {
    mbar_init(wbar, 1);
    mbar_init(xbar, 1);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(abort_sa), "r"(0u) : "memory");
    fence_mbar_init();
  }
  // without split K, token rows M .. 8 QM - 1 of X are not copied: zero
  if (split == 1)
    for (int i = tid; i < (kCols - p.M) * xrow / 4; i += blockDim.x)
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(smem_u32(smem) + static_cast<uint32_t>(p.x_off + p.M * xrow + 4 * i)),
                   "r"(0u)
                   : "memory");
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Weights: segment [s, e) of W widened to 16-byte boundaries [a, b); the
    // bytes of the last stretch of W past its last 16-byte boundary `lim` by
    // plain loads, before the arrival that counts the bulk bytes.
    const int64_t lim = p.total_bytes & ~int64_t(15);
    auto seg = [&](int i, int64_t &s0, int64_t &e0, int64_t &a, int64_t &b) {
      if (split == 1) {  // all rows of the CTA: one contiguous range
        s0 = r0 * p.row_bytes;
        e0 = (r0 + R) * p.row_bytes;
      } else {
        s0 = (r0 + i) * p.row_bytes + static_cast<int64_t>(kb0) * kBB;
        e0 = (r0 + i) * p.row_bytes + static_cast<int64_t>(kb1) * kBB;
      }
      a = s0 & ~int64_t(15);
      b = min((e0 + 15) & ~int64_t(15), max(lim, a));
    };
    const int nseg = split == 1 ? (R > 0 ? 1 : 0) : R;
    auto issue_w = [&]() {
      if (p.withhold && blockIdx.x == 0) return;  // failure-path test: W never lands in this CTA
      if (p.w_tma) {  // every row segment of the group in one box (rows past N read as zero)
        if (lane == 0 && R > 0) {
          mbar_arrive_expect_tx(wbar, static_cast<uint32_t>(p.seg_pitch * ((p.N + p.groups - 1) / p.groups)));
          tma_load_2d(smem + p.w_off, &p.tm_w, static_cast<int>(((static_cast<int64_t>(kb0) * kBB) & ~int64_t(15)) / 4),
                      static_cast<int>(r0), wbar);
        } else if (lane == 0) {
          mbar_arrive(wbar);
        }
        return;
      }
      if (lane == 0) {
        uint32_t bytes = 0;
        for (int i = 0; i < nseg; ++i) {
          int64_t s0, e0, a, b;
          seg(i, s0, e0, a, b);
          uint8_t *dst = smem + p.w_off + static_cast<int64_t>(i) * p.seg_pitch;
          for (int64_t t = b; t < e0; ++t) dst[t - a] = p.W[t];
          bytes += static_cast<uint32_t>(b - a);
        }
        mbar_arrive_expect_tx(wbar, bytes);
      }
      __syncwarp();
      const uint64_t pol = l2_evict_first_policy();
      for (int i = lane; i < nseg; i += 32) {
        int64_t s0, e0, a, b;
        seg(i, s0, e0, a, b);
        uint8_t *dst = smem + p.w_off + static_cast<int64_t>(i) * p.seg_pitch;
        for (int64_t o = 0; o < b - a; o += 65536)
          bulk_g2s(dst + o, p.W + a + o, static_cast<uint32_t>(b - a - o < 65536 ? b - a - o : 65536), wbar, pol);
      }
    };
    auto issue_x = [&]() {
      if (lane != 0) return;
      if (split == 1) {  // the whole of X: one range
        const uint32_t len = static_cast<uint32_t>(p.M) * static_cast<uint32_t>(p.K) * 2u;
        mbar_arrive_expect_tx(xbar, len);
        const uint64_t pol = l2_evict_last_policy();
        for (uint32_t o = 0; o < len; o += 65536)
          bulk_g2s(smem + p.x_off + o, p.X + o / 2, len - o < 65536u ? len - o : 65536u, xbar, pol);
      } else {  // boxes of xjpb blocks x 8 QM tokens
        const int nbox = (nb + p.xjpb - 1) / p.xjpb;
        mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(nbox * xbox));
        for (int bx = 0; bx < nbox; ++bx)
          tma_load_2d(smem + p.x_off + bx * xbox, &p.tm_x, 32 * (kb0 + p.xjpb * bx), 0, xbar);
      }
    };
    if (p.prefetch_before_wait) {
      issue_w();
      pdl_wait();
      issue_x();
    } else {
      pdl_wait();
      issue_w();
      issue_x();
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ consumers
    const int cw = warp - 1;
    const int t = cw % kSmMaxTiles, kq = cw / kSmMaxTiles;  // this warp's tile and K range
    const int g = lane >> 2, qd = lane & 3;
    float acc[QM][4];
#pragma unroll
    for (int q = 0; q < QM; ++q)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[q][i] = 0.f;
    bool ok = mbar_wait(wbar, 0, p.wait_ns);
    ok = mbar_wait(xbar, 0, p.wait_ns) && ok;
    ok = __all_sync(0xffffffffu, ok);  // the mma.sync loop below needs the whole warp
    if (!ok) {
      // record, then wait once more for copies still in flight before the
      // buffers are reused and the CTA exits
      if (lane == 0) atomicOr(&g_prefill_status, kDevTimeoutFull);
      const bool drained = mbar_wait(wbar, 0, p.wait_ns) && mbar_wait(xbar, 0, p.wait_ns);
      if (!__all_sync(0xffffffffu, drained) && lane == 0) {
        // a copy may still be writing W / X, whose space the reduction below
        // reuses: this CTA then stores no partial sums and no output
        atomicOr(&g_prefill_status, kDevTimeoutDrain);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(abort_sa), "r"(1u) : "memory");
      }
    }
    const int T = (R + 15) / 16;
    const uint8_t *wbase = smem + p.w_off;
    const int jb = kq * nb / kSmKParts, je = (kq + 1) * nb / kSmKParts;
    // loop-invariant addresses: rows 16t + g and + 8, token row g of block jb
    // (block j of token 8q + g: box j / xjpb, row 8q + g, 64 bytes at (j mod xjpb) * 64)
    const bool va = 16 * t + g < R, vb = 16 * t + g + 8 < R;
    uint32_t ba = va ? small_row_base(p, r0, kb0, kBB, 16 * t + g) + static_cast<uint32_t>(jb * kBB) : 0u;
    uint32_t bb = vb ? small_row_base(p, r0, kb0, kBB, 16 * t + g + 8) + static_cast<uint32_t>(jb * kBB) : 0u;
    int jx = jb % p.xjpb;
    const uint8_t *xg = smem + p.x_off + (jb / p.xjpb) * xbox + g * xrow + 64 * jx;
    if (ok && t < T) {
#pragma unroll 2
      for (int j = jb; j < je; ++j) {
        // B fragments of block j for every token group: b[q][2 s + h]
        uint32_t bq[QM][4];
#pragma unroll
        for (int q = 0; q < QM; ++q) {
          const uint8_t *xr = xg + 8 * q * xrow;
          if constexpr (WT == QMM_Q8_0) {
            const uint4 v = *reinterpret_cast<const uint4 *>(xr + 16 * qd);  // elements 8qd .. 8qd + 7
            bq[q][0] = v.x;
            bq[q][1] = v.y;
            bq[q][2] = v.z;
            bq[q][3] = v.w;
          } else {
            // elements 4qd .. 4qd + 3 and 16 + 4qd .. 16 + 4qd + 3
            const uint2 lo = *reinterpret_cast<const uint2 *>(xr + 8 * qd);
            const uint2 hi = *reinterpret_cast<const uint2 *>(xr + 32 + 8 * qd);
            bq[q][0] = __byte_perm(lo.x, lo.y, 0x5410u);
            bq[q][1] = __byte_perm(lo.x, lo.y, 0x7632u);
            bq[q][2] = __byte_perm(hi.x, hi.y, 0x5410u);
            bq[q][3] = __byte_perm(hi.x, hi.y, 0x7632u);
          }
        }
        uint32_t oa[4], ob[4];
        float da, db;
        small_row<WT>(wbase, ba, va, qd, oa, da);
        small_row<WT>(wbase, bb, vb, qd, ob, db);
        ba += kBB;
        bb += kBB;
        xg += 64;
        if (++jx == p.xjpb) {  // next box
          jx = 0;
          xg += xbox - 64 * p.xjpb;
        }
        const uint32_t a0[4] = {oa[0], ob[0], oa[1], ob[1]};  // k step 0
        const uint32_t a1[4] = {oa[2], ob[2], oa[3], ob[3]};  // k step 1
#pragma unroll
        for (int q = 0; q < QM; ++q) {
          float c[4] = {0.f, 0.f, 0.f, 0.f};
          mma_bf16_16816(c, a0, bq[q][0], bq[q][1]);
          mma_bf16_16816(c, a1, bq[q][2], bq[q][3]);
          acc[q][0] = __fmaf_rn(da, c[0], acc[q][0]);
          acc[q][1] = __fmaf_rn(da, c[1], acc[q][1]);
          acc[q][2] = __fmaf_rn(db, c[2], acc[q][2]);
          acc[q][3] = __fmaf_rn(db, c[3], acc[q][3]);
        }
      }
    }
    // every consumer is past its last read of W and X: their space takes the
    // warps' sums red[warp][group][lane] (float4)
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kSmWarps) : "memory");
    const bool aborted = lds_u32(abort_sa) != 0u;  // uniform: read after the barrier
    const uint32_t red = sbase + static_cast<uint32_t>(p.w_off);
    if (!aborted) {
#pragma unroll
      for (int q = 0; q < QM; ++q)
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                         red + static_cast<uint32_t>(((cw * QM + q) * 32 + lane) * 16)),
                     "f"(acc[q][0]), "f"(acc[q][1]), "f"(acc[q][2]), "f"(acc[q][3])
                     : "memory");
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kSmWarps) : "memory");
    // (r, m): the K ranges' sums in order; kept in part[r][m] without split K,
    // else stored into the owner rank's slot recv[source rank][row of the owner][m]
    const int ctid = tid - 32;
    const int rpr = (R + split - 1) / split;  // rows per rank share (at most)
    for (int o = aborted ? R * kCols : ctid; o < R * kCols; o += 32 * kSmWarps) {
      const int r = o / kCols, m = o % kCols;
      const int tt = r >> 4, rr = r & 15, q = m >> 3, mm = m & 7;
      const int ln = (rr & 7) * 4 + (mm >> 1), i = (rr >> 3) * 2 + (mm & 1);
      float v = 0.f;
#pragma unroll
      for (int k = 0; k < kSmKParts; ++k)
        v += lds_f32(red + static_cast<uint32_t>(((((k * kSmMaxTiles + tt) * QM + q) * 32 + ln) * 4 + i) * 4));
      if (split == 1) {
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(sbase + static_cast<uint32_t>(p.part_off + 4 * (r * (kCols + 1) + m))),
                     "f"(v)
                     : "memory");
      } else {
        const int own = r / rpr;  // owner rank of row r
        const uint32_t la =
            sbase + static_cast<uint32_t>(p.part_off + 4 * (((zr * rpr) + (r - own * rpr)) * (kCols + 1) + m));
        if (own == zr)
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(la), "f"(v) : "memory");
        else
          st_cluster_b32(map_rank(la, static_cast<uint32_t>(own)), __float_as_uint(v));
      }
    }
  }

  // ------------------------------------------------------------ output
  __syncthreads();
  pdl_wait();  // (Y is written only after the preceding grid; a no-op by now)
  const bool aborted = lds_u32(abort_sa) != 0u;
  if (split == 1) {
    for (int o = aborted ? R * p.M : tid; o < R * p.M; o += blockDim.x) {
      const int m = o / R, r = o % R;
      p.Y[static_cast<int64_t>(m) * p.N + r0 + r] =
          lds_f32(sbase + static_cast<uint32_t>(p.part_off + 4 * (r * (kCols + 1) + m)));
    }
  } else {
    cluster_sync_all();  // every rank's sums have landed in their owners' slots
    const int rpr = (R + split - 1) / split;
    const int rb = zr * rpr, re = min(R, rb + rpr);  // this rank's rows of the group
    const uint32_t pa = sbase + static_cast<uint32_t>(p.part_off);
    for (int o = aborted ? (re - rb) * p.M : tid; o < (re - rb) * p.M; o += blockDim.x) {
      const int m = o / (re - rb), lr = o % (re - rb);
      float v = 0.f;
      for (int src = 0; src < split; ++src)
        v += lds_f32(pa + static_cast<uint32_t>(4 * ((src * rpr + lr) * (kCols + 1) + m)));
      p.Y[static_cast<int64_t>(m) * p.N + r0 + rb + lr] = v;
    }
    // no remote access after the barrier above: a rank may leave
  }
}

template <int WT, int QM>
void *small_kernel_ptr() {
  return reinterpret_cast<void *>(prefill_small_kernel<WT, QM>);
}

// Small-M launch: one wave of clusters of `split` CTAs along K, each cluster a
// group of at most 64 rows; the split is the one that moves the fewest bytes
// into a CTA (its W share plus its X slice). False when M is too large or no
// split fits (the tcgen05 path takes over).
bool try_launch_small(const DevInfo &dev, int wtype, int64_t M, int64_t N, int K, const void *W, const uint16_t *X,
                      float *Y, cudaStream_t stream, uint32_t flags, PrefillPlan *plan, qmm_status *out,
                      uint64_t wait_ns = kWaitLimitNs, int withhold = 0) {
  if (M > kSmMaxM) return false;
  const int KB = K / 32, bb = wtype == QMM_Q8_0 ? 34 : 18;
  const int QM = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
  void *kerns[2][3] = {{small_kernel_ptr<QMM_Q8_0, 1>(), small_kernel_ptr<QMM_Q8_0, 2>(), small_kernel_ptr<QMM_Q8_0, 4>()},
                       {small_kernel_ptr<QMM_Q4_0, 1>(), small_kernel_ptr<QMM_Q4_0, 2>(), small_kernel_ptr<QMM_Q4_0, 4>()}};
  void *kern = kerns[wtype][QM == 1 ? 0 : (QM == 2 ? 1 : 2)];
  static DeviceFlags configured[2];
  if (!configured[wtype].done(dev.device)) {
    for (int i = 0; i < 3; ++i) {
      cudaError_t e = cudaFuncSetAttribute(kerns[wtype][i], cudaFuncAttributeMaxDynamicSharedMemorySize, dev.smem_optin);
      if (e != cudaSuccess) {
        *out = cuda_check(e, "prefill attribute");
        return true;
      }
    }
    configured[wtype].set(dev.device);
  }

  struct Layout {
    int split, groups, rmax, seg_pitch, xjpb, w_tma, w_off, x_off, part_off;
    size_t smem;
    int64_t cost;
  };
  const int64_t row_bytes = static_cast<int64_t>(bb) * KB;
  auto layout = [&](int split, int64_t groups) -> Layout {
    Layout l{};
    l.split = split;
    l.groups = static_cast<int>(groups);
    const int nbm = (KB + split - 1) / split;
    const int R = static_cast<int>((N + groups - 1) / groups);
    // split K: a slot per row segment, the segment plus up to 15 bytes of
    // alignment on either side; otherwise the rows' contiguous range plus 32
    l.rmax = R;
    l.seg_pitch = round_up(nbm * bb + 30, 16);
    l.w_tma = split > 1 && row_bytes % 16 == 0 && l.seg_pitch <= 1024;  // a TMA box row: at most 256 words
    const int64_t wbytes = split == 1 ? R * row_bytes + 32 : static_cast<int64_t>(R) * l.seg_pitch;
    // X rows: the whole K without split (one copy), else boxes of 8 blocks
    l.xjpb = split == 1 ? KB : 8;
    const int64_t xbytes = static_cast<int64_t>((nbm + l.xjpb - 1) / l.xjpb) * 8 * QM * 64 * l.xjpb;
    const int red = kSmWarps * QM * 32 * 16;
    l.w_off = 128;
    if (wbytes + xbytes > (1 << 20)) {
      l.smem = SIZE_MAX;
      return l;
    }
    l.x_off = round_up(l.w_off + static_cast<int>(wbytes), 128);
    l.part_off = round_up(std::max(l.x_off + static_cast<int>(xbytes), l.w_off + red), 16);
    // part: R rows x (8 QM + 1) floats; with split K the owner's slots, split x ceil(R / split) rows
    const int prow = split == 1 ? R : split * ((R + split - 1) / split);
    l.smem = static_cast<size_t>(l.part_off) + static_cast<size_t>(prow) * (8 * QM + 1) * 4 + 128;  // + base alignment
    l.cost = static_cast<int64_t>(R) * nbm * bb + M * nbm * 64;
    return l;
  };

  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3((kSmWarps + 1) * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  cfg.attrs = attr;

  // candidates by their cost with one wave of groups, then checked for
  // cluster residency (fewer groups, larger ones, when not all fit at once)
  const int64_t gmin = (N + kSmMaxTiles * 16 - 1) / (kSmMaxTiles * 16);
  Layout cand[kMaxSplit];
  int nc = 0;
  for (int s = 1; s <= kMaxSplit && s <= KB; ++s) {
    const int64_t gmax = std::min<int64_t>(dev.sms / s, N);
    if (gmax < gmin) continue;
    const Layout l = layout(s, gmax);
    if (l.smem <= static_cast<size_t>(dev.smem_optin)) cand[nc++] = l;
  }
  std::sort(cand, cand + nc, [](const Layout &a, const Layout &b) {
    return a.cost != b.cost ? a.cost < b.cost : a.split < b.split;
  });
  Layout best{};
  bool found = false;
  for (int i = 0; i < nc; ++i) {
    if (found && cand[i].cost >= best.cost) break;
    Layout l = cand[i];
    if (l.split > 1) {
      cfg.gridDim = dim3(static_cast<unsigned>(l.groups * l.split));
      cfg.dynamicSmemBytes = l.smem;
      attr[1].val.clusterDim.x = static_cast<unsigned>(l.split);
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      cfg.numAttrs = 2;
      int active = 0;
      if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();  // a refused query is not an error of this call
        continue;
      }
      if (active < l.groups) {
        if (active < gmin) continue;
        l = layout(l.split, active);
        if (l.smem > static_cast<size_t>(dev.smem_optin)) continue;
      }
    }
    if (!found || l.cost < best.cost) {
      best = l;
      found = true;
    }
  }
  if (!found) return false;

  if (plan) {
    *plan = PrefillPlan{8 * QM, best.split, 0, best.groups * best.split, 1};
    *out = QMM_OK;
    return true;
  }
  SParams p{};
  p.W = static_cast<const uint8_t *>(W);
  p.X = X;
  p.Y = Y;
  p.N = N;
  p.row_bytes = static_cast<int64_t>(bb) * KB;
  p.total_bytes = N * p.row_bytes;
  p.M = static_cast<int>(M);
  p.K = K;
  p.KB = KB;
  p.groups = best.groups;
  p.split = best.split;
  p.seg_pitch = best.seg_pitch;
  p.xjpb = best.xjpb;
  p.w_tma = best.w_tma;
  if (best.split > 1) {
    const uint64_t xd[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t xs[1] = {static_cast<uint64_t>(K) * 2};
    const uint32_t xb[2] = {256, static_cast<uint32_t>(8 * QM)};
    qmm_status st = encode_tiled(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, xd, xs, xb, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st == QMM_OK && best.w_tma) {
      const uint64_t wd[2] = {static_cast<uint64_t>(row_bytes / 4), static_cast<uint64_t>(N)};
      const uint64_t ws[1] = {static_cast<uint64_t>(row_bytes)};
      const uint32_t wb[2] = {static_cast<uint32_t>(best.seg_pitch / 4), static_cast<uint32_t>(best.rmax)};
      st = encode_tiled(&p.tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, W, wd, ws, wb, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (st != QMM_OK) {
      *out = st;
      return true;
    }
  }
  p.w_off = best.w_off;
  p.x_off = best.x_off;
  p.part_off = best.part_off;
  p.prefetch_before_wait = (flags & kPrefetchBeforeWait) ? 1 : 0;
  p.wait_ns = wait_ns;
  p.withhold = withhold;
  cfg.gridDim = dim3(static_cast<unsigned>(best.groups * best.split));
  cfg.dynamicSmemBytes = best.smem;
  attr[1].val.clusterDim.x = static_cast<unsigned>(best.split);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.numAttrs = best.split > 1 ? 2 : 1;
  void *args[] = {&p};
  *out = cuda_check(cudaLaunchKernelExC(&cfg, kern, args), "prefill launch");
  return true;
}

}  // namespace

qmm_status launch_prefill_small_withheld(const DevInfo &dev, int wtype, int64_t M, int64_t N, int K, const void *W,
                                         const uint16_t *X, float *Y, uint64_t wait_ns, cudaStream_t stream) {
  qmm_status st = QMM_OK;
  if (try_launch_small(dev, wtype, M, N, K, W, X, Y, stream, kLaunchPdl, nullptr, &st, wait_ns, 1)) return st;
  return set_error(QMM_ERR_SHAPE, "prefill: M=%lld N=%lld K=%d does not take the small-M kernel", (long long)M,
                   (long long)N, K);
}

qmm_status launch_prefill(const DevInfo &dev, int wtype, int64_t M, int64_t N, int K, const void *W,
                          const uint16_t *X, float *Y, cudaStream_t stream, uint32_t flags, PrefillPlan *plan) {
  {
    qmm_status st = QMM_OK;
    if (try_launch_small(dev, wtype, M, N, K, W, X, Y, stream, flags, plan, &st)) return st;
  }
  Params p{};
  p.prefetch_before_wait = (flags & kPrefetchBeforeWait) ? 1 : 0;
  p.W = static_cast<const uint8_t *>(W);
  p.Y = Y;
  p.M = static_cast<int>(M);
  p.K = K;
  p.KB = K / 32;
  p.N = N;
  const int bb = wtype == QMM_Q8_0 ? 34 : 18;
  p.row_bytes = static_cast<int64_t>(bb) * p.KB;
  p.rs = 1;
  while ((p.rs * p.row_bytes) % 16 != 0) p.rs *= 2;  // at most 8: 8 * 34 = 16 * 17, 8 * 18 = 16 * 9
  p.tma_rows = N / p.rs * p.rs;
  // a row's chunk plus up to 15 bytes of alignment in front, rounded to 16
  // and then to 16 mod 32 (rows spread over eight 4-byte bank groups)
  p.raw_pitch = wtype == QMM_Q8_0 ? 304 : 176;
  const int raw_bytes = (wtype == QMM_Q8_0 ? raw_stages<QMM_Q8_0>() : raw_stages<QMM_Q4_0>()) * 128 * p.raw_pitch;
  const int budget = dev.smem_optin - 1024 /*align*/ - 1024 /*barriers*/ - round_up(raw_bytes, 1024);
  // MMA stages of a tile MT tokens wide: X stages in shared memory (A lives in
  // tensor memory), A stages in the TMEM columns past the accumulator
  auto stages_for = [&](int mt) {
    return std::min({8, budget / (mt * 128), (512 - std::max(256, mt)) / kACols});
  };
  auto smem_for = [&](int mt) {
    // Every CTA allocates all 512 TMEM columns, so never two CTAs on one SM (a
    // second one would wait in tcgen05.alloc, and across clusters that wait
    // could close a cycle): ask for more than half of the shared memory.
    return std::max<size_t>(static_cast<size_t>(1024 + stages_for(mt) * mt * 128) + raw_bytes + 1024,
                            static_cast<size_t>(dev.smem_optin / 2 + 1024));
  };

  void *kerns[2][2] = {{kernel_ptr<QMM_Q8_0, false>(), kernel_ptr<QMM_Q8_0, true>()},
                       {kernel_ptr<QMM_Q4_0, false>(), kernel_ptr<QMM_Q4_0, true>()}};
  static DeviceFlags configured[2];
  if (!configured[wtype].done(dev.device)) {
    for (int w = 0; w < 2; ++w) {
      cudaError_t e = cudaFuncSetAttribute(kerns[wtype][w], cudaFuncAttributeMaxDynamicSharedMemorySize, dev.smem_optin);
      if (e != cudaSuccess) return cuda_check(e, "prefill attribute");
    }
    configured[wtype].set(dev.device);
  }
  void *kern = kerns[wtype][0];  // split-K occupancy queries: narrow tiles

  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  cfg.attrs = attr;

  const int64_t ntiles = (N + 127) / 128;
  const int nst_all = (p.KB + 1) / 2;
  // Split K over a cluster when the output tiles leave SMs idle: as many
  // ranks as fit one wave, each with at least one stage, the exchange buffer
  // inside the stage buffers, and every cluster resident at once.
  auto choose_split = [&](int mt) -> int {
    const int64_t base = ntiles * ((M + mt - 1) / mt);
    if (base >= dev.sms) return 1;
    const int xbytes = stages_for(mt) * mt * 128;
    int split = static_cast<int>(std::min<int64_t>({kMaxSplit, nst_all, dev.sms / base}));
    for (; split > 1; --split) {
      const int rmax = (128 + split - 1) / split;
      // the exchange buffer reuses the X stages and the raw chunks (all consumed by then)
      if (static_cast<int64_t>(split) * mt * rmax * 4 > xbytes + raw_bytes) continue;
      cfg.gridDim = dim3(static_cast<unsigned>((M + mt - 1) / mt), static_cast<unsigned>(ntiles),
                         static_cast<unsigned>(split));
      cfg.dynamicSmemBytes = smem_for(mt);
      attr[1].val.clusterDim.x = 1;
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = static_cast<unsigned>(split);
      cfg.numAttrs = 2;
      int active = 0;
      if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) == cudaSuccess && active >= base) break;
      cudaGetLastError();  // a refused query is not an error of this call
    }
    return split;
  };
  // Makespan in units of one 64-k stage of one token: waves x stages per CTA x MT.
  auto cost_of = [&](int mt, int split) -> int64_t {
    const int64_t ctas = ntiles * ((M + mt - 1) / mt) * split;
    return (ctas + dev.sms - 1) / dev.sms * ((nst_all + split - 1) / split) * mt;
  };

  // Token tile: up to 256 tokens (one MMA). When the tiles fill at least one
  // wave (no split K), wider tiles (two MMAs per k step, at least three
  // stages) are taken if they cut the makespan by 15% or more, i.e. when
  // 256-token tiles leave a nearly empty last wave.
  int mt = static_cast<int>(std::min<int64_t>(256, round_up(static_cast<int>(std::min<int64_t>(M, 256)), 16)));
  int split = choose_split(mt);
  if (M > 256 && split == 1) {
    int64_t cost = cost_of(mt, 1);
    for (int64_t c = (M + kMaxMT - 1) / kMaxMT; c < (M + 255) / 256; ++c) {
      const int w = round_up(static_cast<int>((M + c - 1) / c), 32);
      if (w <= 256 || w > kMaxMT || stages_for(w) < 3) continue;
      const int64_t wc = cost_of(w, 1);
      if (wc * 100 <= cost * 85) {
        mt = w;
        cost = wc;
      }
    }
  }
  p.MT = mt;
  p.acc_cols = std::max(256, mt);
  p.tmem_cols = 512;  // accumulator in columns 0..acc_cols-1, A stage s at acc_cols + 32 s
  p.x_stage_bytes = p.MT * 128;
  p.stages = stages_for(mt);
  if (p.stages < 2) return set_error(QMM_ERR_SHAPE, "prefill: no room for two stages of %d tokens", mt);
  p.off_x = 1024;
  p.off_raw = p.off_x + p.stages * p.x_stage_bytes;
  const size_t smem = smem_for(mt);
  if (smem > static_cast<size_t>(dev.smem_optin))
    return set_error(QMM_ERR_SHAPE, "prefill: tile needs %zu bytes of shared memory", smem);
  cfg.dynamicSmemBytes = smem;
  const int64_t mtiles = (M + p.MT - 1) / p.MT;
  if (ntiles > 65535 || mtiles > 0x7fffffff) return set_error(QMM_ERR_SHAPE, "prefill: grid too large");
  if (plan) {
    *plan = PrefillPlan{p.MT, split, p.stages, static_cast<int>(ntiles * mtiles * split), 0};
    return QMM_OK;
  }

  const uint64_t xd[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  const uint64_t xs[1] = {static_cast<uint64_t>(K) * 2};
  const uint32_t xb[2] = {64, static_cast<uint32_t>(std::min(p.MT, 256))};
  qmm_status st = encode_tiled(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, xd, xs, xb, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QMM_OK) return st;
  if (p.MT > 256) {
    const uint32_t xb2[2] = {64, static_cast<uint32_t>(p.MT - 256)};
    st = encode_tiled(&p.tm_x2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, xd, xs, xb2, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != QMM_OK) return st;
  }

  p.split = split;
  p.red_pitch = (128 + split - 1) / split;  // rows of the largest rank share
  if (p.rs == 1 && split == 1) p.raw_pitch = kRawBlocks * bb;  // chunks start on 16-byte boundaries: 272 / 144
  if (p.tma_rows > 0) {
    const uint64_t wd[2] = {static_cast<uint64_t>(p.rs * p.row_bytes / 2), static_cast<uint64_t>(N / p.rs)};
    const uint64_t ws[1] = {static_cast<uint64_t>(p.rs * p.row_bytes)};
    const uint32_t wb[2] = {static_cast<uint32_t>(p.raw_pitch / 2), static_cast<uint32_t>(128 / p.rs)};
    st = encode_tiled(&p.tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, W, wd, ws, wb, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != QMM_OK) return st;
  }
  cfg.gridDim = dim3(static_cast<unsigned>(mtiles), static_cast<unsigned>(ntiles), static_cast<unsigned>(split));
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = static_cast<unsigned>(split);
  cfg.numAttrs = split > 1 ? 2 : 1;
  void *args[] = {&p};
  return cuda_check(cudaLaunchKernelExC(&cfg, kerns[wtype][p.MT > 256 ? 1 : 0], args), "prefill launch");
}

cudaError_t prefill_status(uint32_t *bits) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(bits, g_prefill_status, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_prefill_status, &zero, sizeof(uint32_t));
  return e;
}

}  // namespace qmm
