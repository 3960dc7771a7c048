// q4_gateup.cu -- fused gate/up projection with SwiGLU on Q4_0 weights (M <= 8),
// and with one matrix the Q4_0 GEMV (qmm_q4_gemv).
//
// Operation ("LSE v0.4.16", section "Combined M8 Q4 gate/up execution"): one
// launch reads one shared activation panel X and accumulates the gate and up
// projections in independent fp32 accumulators; only
//     Y[m][n] = silu(g) * u,  g = X[m] . Wg[n],  u = X[m] . Wu[n],  silu(g) = g / (1 + e^-g)
// is written -- no gate (or up) temporary ever reaches memory.
//
// Why tensor cores: at M = 8 every weight meets 8 activations, so on fp32
// FMAs the kernel is ALU-bound (~40 us for the 8 x 5120 x 17408 shape against
// ~15 us of HBM time). It is a genuine small-M matrix product, so it runs on
// mma.sync m16n8k16 (fp16 inputs, fp32 accumulation) with
//  * A = 16 weight rows x 16 k: Q4 nibbles q - 8 in [-8, 7] are exact in fp16
//    (two nibbles -> a half pair with one mask/or and one packed half
//    subtraction; one shift per 32-bit word);
//  * B = 16 k x 8 tokens: each activation is split into two fp16 parts,
//    x * s = hi + lo (hi = fp16(x s), lo = fp16(x s - hi)), with s a power of
//    two per 32-block chosen so the block maximum lands in [2^14, 2^15): the
//    pair carries ~22 significant bits, and the products are exact in fp32;
//  * each 32-block gives C = A0 B0hi + A1 B1hi + A0 B0lo + A1 B1lo (four
//    mma), then acc += (d * 2^-s) * C in fp32 -- the per-block scale applied
//    in fp32 exactly as the method defines it.
// Within a block the order of k is permuted (the same permutation on A and B
// leaves the dot product unchanged) so that lane t of a quad takes qs bytes
// 4t..4t+3 (one 32-bit word) and activations 4t..4t+3 / 16+4t..16+4t+3 (two
// 16-byte loads).
//
// Data movement: a producer warp streams 8-block (256 k) stages with 2-D TMA
// loads -- one 16-row x 144-byte box per weight tile and matrix, one
// 8-token x 32-float box (128-byte swizzle) per block of X. Consumer warp w
// owns block w % 8 of every stage for half of the CTA's row tiles (tiles i
// with i % 2 == w / 8): sixteen consumer warps, four per scheduler, so the
// chains of dependent mma / conversion instructions overlap (with eight the
// kernel was latency-bound: ncu showed issue 46% active, tensor pipe 22%).
// The tile loop has no data-dependent exit (the matrix count is a template
// parameter; tiles past the CTA's count are computed and dropped), so the
// shared-memory loads of all its tiles are issued together; measured on B200
// this took the launch from 44.6 to 39.9 us. Its B fragments are built once
// and reused for its tiles. At the end the
// partial sums of the eight warps holding a tile are added in block order
// through shared memory and the SwiGLU epilogue writes Y. Rows of W must be 16-byte multiples for the
// tensor maps (K % 256 == 0); other K use the same code reading global memory
// directly.
//
// qmm_q4_gateup_unfused runs the same kernel with one matrix per launch
// (writing G, then U) and a third launch applying silu(G) * U with the same
// device function, so the fused output equals the unfused one bit for bit.
#include <algorithm>
#include <type_traits>

#include "qmm_common.cuh"
#include "qmm_internal.h"
#include "qmm_tmap.h"

namespace qmm {
namespace {

static __device__ uint32_t g_q4_status;

constexpr int kWarps = 16;           // consumer warps; warp w owns block w % 8 of each stage
constexpr int kHalves = kWarps / 8;  // ... and the row tiles i with i % kHalves == w / 8
constexpr int kBlocksPerStage = 8;   // 8 Q4_0 blocks = 256 k = 144 bytes per row
constexpr int kTilesMax = 8;         // 16-row tiles per CTA
constexpr int kStages = 4;
constexpr int kRowStageBytes = kBlocksPerStage * 18;             // 144
constexpr int kTileBytes = 16 * kRowStageBytes;                  // 2304
constexpr int kXStageBytes = kBlocksPerStage * 8 * 128;          // 8 blocks x 8 tokens x 32 floats
constexpr int kStageBytes = kXStageBytes + 2 * kTilesMax * kTileBytes;  // 45056 (multiple of 1024)
constexpr int kBarBytes = 1024;

enum : int { kOutFused = 0, kOutProj = 1 };

struct alignas(64) Params {
  CUtensorMap tm_x;      // X: dims {K, M} fp32, box {32, 8}, 128-byte swizzle
  CUtensorMap tm_w[2];   // Wg, Wu: dims {9 * KB (uint16), N}, box {72, 16}
  const uint8_t *W[2];   // Wg, Wu (direct path)
  const float *X;
  float *Y;              // fused output, or the projection output
  int M, K, KB;
  int64_t N;
  int tiles;             // 16-row tiles in total
  int grid;
  int nmat;              // 2 (fused) or 1 (projection)
  int prefetch_before_wait;
  int split;             // K ranges per tile group (cluster size along x; 1 = none)
};

// ------------------------------------------------------------ cluster PTX
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of all CTAs of the cluster; orders shared-memory accesses across it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Eight Q4 codes (bytes b0..b3 of v; low nibble of byte j = element j, high
// nibble = element j + 16) -> exact fp16 pairs of q - 8:
//   lo02 = (lownib(b0), lownib(b2)), lo13 = (lownib(b1), lownib(b3)),
//   hi02 = (hinib(b0), hinib(b2)),   hi13 = (hinib(b1), hinib(b3)).
// A masked or puts each nibble in the mantissa of 1024 (step 1) or 64 (step
// 1/16); one packed half subtraction of 1032 / 72 leaves q - 8 exactly.
struct Nib4 {
  uint32_t lo02, lo13, hi02, hi13;
};
__device__ __forceinline__ Nib4 q4_word_to_half2(uint32_t v) {
  const uint32_t v8 = v >> 8;
  const __half2 k1032 = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
  const __half2 k72 = __halves2half2(__ushort_as_half(0x5480), __ushort_as_half(0x5480));
  Nib4 r;
  uint32_t t;
  t = (v & 0x000F000Fu) | 0x64006400u;  // 1024 + n
  __half2 h = __hsub2(*reinterpret_cast<__half2 *>(&t), k1032);
  r.lo02 = *reinterpret_cast<uint32_t *>(&h);
  t = (v8 & 0x000F000Fu) | 0x64006400u;
  h = __hsub2(*reinterpret_cast<__half2 *>(&t), k1032);
  r.lo13 = *reinterpret_cast<uint32_t *>(&h);
  t = (v & 0x00F000F0u) | 0x54005400u;  // 64 + n
  h = __hsub2(*reinterpret_cast<__half2 *>(&t), k72);
  r.hi02 = *reinterpret_cast<uint32_t *>(&h);
  t = (v8 & 0x00F000F0u) | 0x54005400u;
  h = __hsub2(*reinterpret_cast<__half2 *>(&t), k72);
  r.hi13 = *reinterpret_cast<uint32_t *>(&h);
  return r;
}

// B fragments of one 32-block for this lane (token g = lane / 4, quad t = lane % 4):
// activations 4t..4t+3 (k-step 0) and 16+4t..16+4t+3 (k-step 1), scaled by the
// block's power of two and split into fp16 hi + lo parts.
struct BFrag {
  uint32_t hi0, hi1, hi2, hi3;  // k-step 0: (b0, b1); k-step 1: (b0, b1)
  uint32_t lo0, lo1, lo2, lo3;
  float inv_scale;
};
__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ BFrag make_bfrag(float4 x0, float4 x1) {
  // block maximum over all 8 tokens x 32 activations (warp-wide)
  float mx = fmaxf(fmaxf(fmaxf(fabsf(x0.x), fabsf(x0.y)), fmaxf(fabsf(x0.z), fabsf(x0.w))),
                   fmaxf(fmaxf(fabsf(x1.x), fabsf(x1.y)), fmaxf(fabsf(x1.z), fabsf(x1.w))));
  mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
  // s = 2^(14 - e) where 2^e <= mx < 2^(e+1); clamped to the normal range
  const int e = static_cast<int>((__float_as_uint(mx) >> 23) & 0xff) - 127;
  int sexp = 14 - e;
  sexp = max(-100, min(100, sexp));
  const float s = __uint_as_float(static_cast<uint32_t>(sexp + 127) << 23);
  BFrag f;
  f.inv_scale = __uint_as_float(static_cast<uint32_t>(127 - sexp) << 23);
  const float v[8] = {x0.x * s, x0.y * s, x0.z * s, x0.w * s, x1.x * s, x1.y * s, x1.z * s, x1.w * s};
  uint32_t hi[4], lo[4];
  // pairs (j, j + 2) of the lane's four activations, matching the nibble pairs
  const int pa[4] = {0, 1, 4, 5}, pb[4] = {2, 3, 6, 7};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    hi[i] = pack_half2(v[pa[i]], v[pb[i]]);
    const float2 hf = __half22float2(*reinterpret_cast<__half2 *>(&hi[i]));
    lo[i] = pack_half2(v[pa[i]] - hf.x, v[pb[i]] - hf.y);
  }
  f.hi0 = hi[0]; f.hi1 = hi[1]; f.hi2 = hi[2]; f.hi3 = hi[3];
  f.lo0 = lo[0]; f.lo1 = lo[1]; f.lo2 = lo[2]; f.lo3 = lo[3];
  return f;
}

// One 16-row x 32-k block tile: c = W_tile . (hi + lo), then acc += (d * 2^-s) c.
__device__ __forceinline__ void tile_block(float (&acc)[4], uint32_t vg, uint32_t vh, float dg, float dh,
                                           const BFrag &b) {
  const Nib4 ng = q4_word_to_half2(vg), nh = q4_word_to_half2(vh);
  // one chain: the hi parts of both k-steps first, then the lo parts
  float c[4] = {0.f, 0.f, 0.f, 0.f};
  mma_16816(c, ng.lo02, nh.lo02, ng.lo13, nh.lo13, b.hi0, b.hi1);  // k-step 0 (low nibbles)
  mma_16816(c, ng.hi02, nh.hi02, ng.hi13, nh.hi13, b.hi2, b.hi3);  // k-step 1 (high nibbles)
  mma_16816(c, ng.lo02, nh.lo02, ng.lo13, nh.lo13, b.lo0, b.lo1);
  mma_16816(c, ng.hi02, nh.hi02, ng.hi13, nh.hi13, b.lo2, b.lo3);
  const float sg = __fmul_rn(dg, b.inv_scale), sh = __fmul_rn(dh, b.inv_scale);
  acc[0] = __fmaf_rn(sg, c[0], acc[0]);
  acc[1] = __fmaf_rn(sg, c[1], acc[1]);
  acc[2] = __fmaf_rn(sh, c[2], acc[2]);
  acc[3] = __fmaf_rn(sh, c[3], acc[3]);
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
}

// Outputs o in [o_begin, o_end) (o = token * rows + row of the CTA's tiles) from
// the partial sums red[warp][tile of the warp][mat][lane] (float4) of `nsrc`
// CTAs of a cluster (nsrc = 1: this CTA's own): the eight block warps of a
// tile in block order, ranks in rank order; then the SwiGLU (NMAT = 2) or the
// projection itself.
template <int NMAT>
__device__ __forceinline__ void finish_outputs(const Params &p, uint32_t red_saddr, int nsrc, int tile0, int ntiles,
                                               int tid, int nthreads, int o_begin, int o_end) {
  const int rows = ntiles * 16;
  for (int o = o_begin + tid; o < o_end; o += nthreads) {
    const int tok = o / rows, rl = o - tok * rows;
    const int i = rl >> 4, r = rl & 15;
    const int src_lane = (r & 7) * 4 + (tok >> 1), idx = (r >> 3) * 2 + (tok & 1);
    float v[2] = {0.f, 0.f};
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat) {
      float sum = 0.f;
      // the eight block warps that hold tile i, in block order
      const int wbase = 8 * (i % kHalves), ii = i / kHalves;
      for (int src = 0; src < nsrc; ++src) {
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const uint32_t off =
              4u * static_cast<uint32_t>(((((wbase + b) * (kTilesMax / kHalves) + ii) * 2 + mat) * 32 + src_lane) * 4 + idx);
          const float x = nsrc == 1 ? *reinterpret_cast<const float *>(__cvta_shared_to_generic(red_saddr + off))
                                    : ld_cluster_f32(map_rank(red_saddr + off, static_cast<uint32_t>(src)));
          sum = __fadd_rn(sum, x);
        }
      }
      v[mat] = sum;
    }
    const int64_t n = 16ll * tile0 + rl;
    if (tok < p.M && n < p.N) p.Y[static_cast<int64_t>(tok) * p.N + n] = (NMAT == 2) ? silu_mul(v[0], v[1]) : v[0];
  }
}

// DIRECT = false: TMA-fed shared-memory stages; true: reads global memory.
// NMAT: 2 (fused gate/up) or 1 (one projection).
template <bool DIRECT, int NMAT>
__global__ void __launch_bounds__((kWarps + 1) * 32, 1) q4_gateup_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + kStages;
  uint8_t *stages = smem + kBarBytes;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // Split K (few row tiles, long rows): the `split` CTAs of a cluster share a
  // tile group and take consecutive stage ranges; their partial sums are added
  // in rank order through distributed shared memory at the end.
  const int split = DIRECT ? 1 : p.split;
  const int rank = split > 1 ? static_cast<int>(cluster_rank()) : 0;
  const int group = static_cast<int>(blockIdx.x) / split;
  const int tile0 = static_cast<int>(static_cast<int64_t>(group) * p.tiles / p.grid);
  const int tile1 = static_cast<int>(static_cast<int64_t>(group + 1) * p.tiles / p.grid);
  const int ntiles = tile1 - tile0;
  const int nstages_all = (p.KB + kBlocksPerStage - 1) / kBlocksPerStage;
  const int j_lo = rank * nstages_all / split;
  const int nstages = (rank + 1) * nstages_all / split - j_lo;  // this CTA's stages

  pdl_launch_dependents();
  if (!DIRECT) {
    if (tid == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], kWarps);
      }
      fence_mbar_init();
    }
    __syncthreads();
  }

  if (warp == kWarps) {
    // -------------------------------------------------------------- producer
    if (DIRECT) return;
    const uint32_t wbytes = static_cast<uint32_t>(NMAT * ntiles * kTileBytes);
    auto issue_w = [&](int j) {  // weights of stage j (arrive + expect all bytes of the stage)
      const int s = j % kStages;
      uint8_t *st = stages + s * kStageBytes;
      mbar_arrive_expect_tx(&full[s], wbytes + kXStageBytes);
      for (int mat = 0; mat < NMAT; ++mat)
        for (int t = 0; t < ntiles; ++t)
          tma_load_2d(st + kXStageBytes + (mat * kTilesMax + t) * kTileBytes, &p.tm_w[mat], 72 * (j_lo + j),
                      16 * (tile0 + t), &full[s]);
    };
    auto issue_x = [&](int j) {
      uint8_t *st = stages + (j % kStages) * kStageBytes;
      for (int b = 0; b < kBlocksPerStage; ++b)
        tma_load_2d(st + b * 1024, &p.tm_x, 32 * ((j_lo + j) * kBlocksPerStage + b), 0, &full[j % kStages]);
    };
    const int prologue = min(kStages, nstages);
    if (lane == 0) {
      if (p.prefetch_before_wait) {
        for (int j = 0; j < prologue; ++j) issue_w(j);
        pdl_wait();
        for (int j = 0; j < prologue; ++j) issue_x(j);
      } else {
        pdl_wait();
        for (int j = 0; j < prologue; ++j) {
          issue_w(j);
          issue_x(j);
        }
      }
      bool ok = true;
      int issued = prologue;
      for (int j = 0; j < nstages && issued < nstages; ++j) {
        ok = mbar_wait(&empty[j % kStages], static_cast<uint32_t>(j / kStages) & 1u);
        if (!ok) break;
        issue_w(issued);
        issue_x(issued);
        ++issued;
      }
      if (!ok) {  // error path: record, then drain the copies still in flight
        atomicOr(&g_q4_status, kDevTimeoutFull);
        for (int j = max(0, issued - kStages); j < issued; ++j)
          if (!mbar_wait(&full[j % kStages], static_cast<uint32_t>(j / kStages) & 1u))
            atomicOr(&g_q4_status, kDevTimeoutDrain);
      }
    }
    __syncwarp();
    if (split == 1) return;
  } else {
  // ---------------------------------------------------------------- consumers
  pdl_wait();
  const int g = lane >> 2, t = lane & 3;
  const int wb = warp & 7, th = warp >> 3;  // this warp's block of the stage and tile parity
  float acc[kTilesMax / kHalves][2][4];
#pragma unroll
  for (int i = 0; i < kTilesMax / kHalves; ++i)
#pragma unroll
    for (int mat = 0; mat < 2; ++mat)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[i][mat][k] = 0.f;

  const int64_t row_bytes = 18ll * p.KB;
  // The stage loop, compiled once per parity of this warp's block (fixed for
  // the whole kernel): odd blocks start 2 bytes past a 4-byte boundary, so
  // their code words are aligned; even ones need a funnel shift. Returns 0, or
  // on a timeout 1 (leave) / 2 (split K: go on to the cluster barriers).
  auto stage_loop = [&](auto parity) -> int {
    constexpr bool kOdd = decltype(parity)::value;
    for (int j = 0; j < nstages; ++j) {
      const int s = j % kStages;
      if (!DIRECT && !mbar_wait(&full[s], static_cast<uint32_t>(j / kStages) & 1u)) {
        if (lane == 0) atomicOr(&g_q4_status, kDevTimeoutFull);
        return split == 1 ? 1 : 2;  // 1: leave (the producer gives up on this warp's missing
                                    // arrival and drains); 2: split K, still meet the cluster barriers
      }
      const int kb = (j_lo + j) * kBlocksPerStage + wb;  // this warp's block
      if (kb < p.KB) {
        // activations of block kb for token g
        float4 x0, x1;
        if (!DIRECT) {
          const uint32_t xa = smem_u32(stages + s * kStageBytes + wb * 1024) + g * 128;
          x0 = lds_f4(xa + 16u * (t ^ g));
          x1 = lds_f4(xa + 16u * ((4 + t) ^ g));
        } else if (g < p.M) {
          const float4 *xp = reinterpret_cast<const float4 *>(p.X + static_cast<int64_t>(g) * p.K + 32 * kb);
          x0 = __ldg(xp + t);
          x1 = __ldg(xp + 4 + t);
        } else {
          x0 = x1 = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const BFrag bf = make_bfrag(x0, x1);
  #pragma unroll
        for (int mat = 0; mat < 2; ++mat) {
          if (mat >= NMAT) break;
  #pragma unroll
          for (int ii = 0; ii < kTilesMax / kHalves; ++ii) {
            const int i = ii * kHalves + th;  // this warp's share of the row tiles
            // Staged tiles: no exit, so the loads of all tiles can be issued
            // together; a tile past ntiles reads stale stage bytes and its
            // accumulators are never used.
            if (DIRECT && i >= ntiles) break;
            uint32_t vg, vh;
            float dg, dh;
            if (!DIRECT) {
              // row r of the tile at r * 144 bytes; block `wb` at 18 * wb
              const uint32_t tb = smem_u32(stages + s * kStageBytes + kXStageBytes + (mat * kTilesMax + i) * kTileBytes);
              const uint32_t ag = tb + g * kRowStageBytes + 18 * wb, ah = ag + 8 * kRowStageBytes;
              if constexpr (kOdd) {  // block starts 2 bytes past a 4-byte boundary: qs word aligned
                vg = lds_u32(ag + 2 + 4 * t);
                vh = lds_u32(ah + 2 + 4 * t);
              } else {
                vg = __funnelshift_r(lds_u32(ag + 4 * t), lds_u32(ag + 4 * t + 4), 16);
                vh = __funnelshift_r(lds_u32(ah + 4 * t), lds_u32(ah + 4 * t + 4), 16);
              }
              dg = half_bits_to_float(lds_u16(ag));
              dh = half_bits_to_float(lds_u16(ah));
            } else {
              const int64_t rg = 16ll * (tile0 + i) + g, rh = rg + 8;
              const uint8_t *Wm = p.W[mat];
              auto word = [&](int64_t r, float &d) -> uint32_t {
                if (r >= p.N) {
                  d = 0.f;
                  return 0x88888888u;  // nibbles 8 -> value 0
                }
                const uint16_t *bp = reinterpret_cast<const uint16_t *>(Wm + r * row_bytes + 18ll * kb);
                d = half_bits_to_float(__ldg(bp));
                return static_cast<uint32_t>(__ldg(bp + 1 + 2 * t)) | (static_cast<uint32_t>(__ldg(bp + 2 + 2 * t)) << 16);
              };
              vg = word(rg, dg);
              vh = word(rh, dh);
            }
            tile_block(acc[ii][mat], vg, vh, dg, dh, bf);
          }
        }
      }
      if (!DIRECT) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
    return 0;
  };
  int loop_rc;
  if constexpr (DIRECT) {  // reads global memory: the parity does not matter
    loop_rc = stage_loop(std::false_type{});
  } else {
    loop_rc = (wb & 1) ? stage_loop(std::true_type{}) : stage_loop(std::false_type{});
  }
  if (loop_rc == 1) return;

  // ------------------------------------------ cross-warp sum, SwiGLU epilogue
  // Every consumer has passed its last stage, so the stage memory is free.
  asm volatile("bar.sync 1, %0;" ::"r"(kWarps * 32) : "memory");
  float4 *red = reinterpret_cast<float4 *>(stages);  // [warp][tile of the warp][mat][lane]
#pragma unroll
  for (int ii = 0; ii < kTilesMax / kHalves; ++ii) {
    if (ii * kHalves + th >= ntiles) break;
#pragma unroll
    for (int mat = 0; mat < 2; ++mat) {
      if (mat >= NMAT) break;
      red[((warp * (kTilesMax / kHalves) + ii) * 2 + mat) * 32 + lane] =
          make_float4(acc[ii][mat][0], acc[ii][mat][1], acc[ii][mat][2], acc[ii][mat][3]);
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kWarps * 32) : "memory");
  if (split == 1) {
    finish_outputs<NMAT>(p, smem_u32(red), 1, tile0, ntiles, tid, kWarps * 32, 0, 8 * ntiles * 16);
    return;
  }
  }  // consumers

  // Split K: every rank's partials are in its own shared memory; rank r adds
  // all ranks' partials (rank order, then block order) for its share of the
  // outputs, then no rank leaves while another may still read its memory.
  cluster_sync();
  const int nout = 8 * ntiles * 16;
  finish_outputs<NMAT>(p, smem_u32(stages), split, tile0, ntiles, tid, (kWarps + 1) * 32, rank * nout / split,
                       (rank + 1) * nout / split);
  cluster_sync();
}

__global__ void silu_mul_kernel(const float *__restrict__ G, const float *__restrict__ U, float *__restrict__ Y,
                                int64_t count) {
  pdl_launch_dependents();
  pdl_wait();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    Y[i] = silu_mul(G[i], U[i]);
}

template <bool DIRECT, int NMAT>
cudaError_t launch(const cudaLaunchConfig_t &cfg, const Params &p) {
  static DeviceFlags configured;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!configured.done(dev)) {
    cudaError_t e = cudaFuncSetAttribute(q4_gateup_kernel<DIRECT, NMAT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kBarBytes + kStages * kStageBytes + 1024);
    if (e != cudaSuccess) return e;
    configured.set(dev);
  }
  return cudaLaunchKernelEx(&cfg, q4_gateup_kernel<DIRECT, NMAT>, p);
}

// One gate/up launch over nmat matrices (W[0], W[1]) writing Y.
qmm_status launch_proj(const DevInfo &dev, int M, int64_t N, int K, const void *const *W, int nmat, const float *X,
                       float *Y, cudaStream_t stream, uint32_t flags) {
  Params p{};
  p.M = M;
  p.K = K;
  p.KB = K / 32;
  p.N = N;
  p.X = X;
  p.Y = Y;
  p.nmat = nmat;
  p.W[0] = static_cast<const uint8_t *>(W[0]);
  p.W[1] = static_cast<const uint8_t *>(nmat > 1 ? W[1] : W[0]);
  p.prefetch_before_wait = (flags & kPrefetchBeforeWait) ? 1 : 0;
  const int64_t tiles = (N + 15) / 16;
  if (tiles > (int64_t(1) << 30)) return set_error(QMM_ERR_SHAPE, "q4_gateup: N too large");
  p.tiles = static_cast<int>(tiles);
  p.grid = static_cast<int>(std::max<int64_t>(std::min<int64_t>(tiles, dev.sms), (tiles + kTilesMax - 1) / kTilesMax));
  const bool direct = (p.KB % kBlocksPerStage) != 0;
  // Split K when full tile groups leave at least half of the SMs idle (few
  // rows, long K): groups of kTilesMax tiles, `split` CTAs per group.
  p.split = 1;
  const int64_t groups = (tiles + kTilesMax - 1) / kTilesMax;
  const int nstages_all = (p.KB + kBlocksPerStage - 1) / kBlocksPerStage;
  if (!direct && 2 * groups <= dev.sms) {
    p.split = static_cast<int>(std::min<int64_t>({8, dev.sms / groups, nstages_all}));
    if (p.split > 1) p.grid = static_cast<int>(groups);
    else p.split = 1;
  }
  if (!direct) {
    const uint64_t xd[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t xs[1] = {static_cast<uint64_t>(K) * 4};
    const uint32_t xb[2] = {32, 8};
    qmm_status st = encode_tiled(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, X, xd, xs, xb, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != QMM_OK) return st;
    for (int mat = 0; mat < 2; ++mat) {
      const uint64_t wd[2] = {static_cast<uint64_t>(9) * p.KB, static_cast<uint64_t>(N)};
      const uint64_t ws[1] = {static_cast<uint64_t>(18) * p.KB};
      const uint32_t wb[2] = {72, 16};
      st = encode_tiled(&p.tm_w[mat], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.W[mat], wd, ws, wb,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
      if (st != QMM_OK) return st;
    }
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.grid * p.split);
  cfg.blockDim = dim3((kWarps + 1) * 32);
  cfg.dynamicSmemBytes = direct ? static_cast<size_t>(kWarps * (kTilesMax / kHalves) * 2 * 32 * 16 + 2048)
                                : static_cast<size_t>(kBarBytes + kStages * kStageBytes + 1024);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (flags & kLaunchPdl) ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(p.split);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.split > 1 ? 2 : 1;
  const cudaError_t e = nmat == 2 ? (direct ? launch<true, 2>(cfg, p) : launch<false, 2>(cfg, p))
                                  : (direct ? launch<true, 1>(cfg, p) : launch<false, 1>(cfg, p));
  return cuda_check(e, "q4_gateup launch");
}

}  // namespace

qmm_status launch_q4_gateup(const DevInfo &dev, int M, int64_t N, int K, const void *Wg, const void *Wu,
                            const float *X, float *Y, cudaStream_t stream, uint32_t flags) {
  const void *W[2] = {Wg, Wu};
  return launch_proj(dev, M, N, K, W, 2, X, Y, stream, flags);
}

qmm_status launch_q4_gemv(const DevInfo &dev, int M, int64_t N, int K, const void *W, const float *X, float *Y,
                          cudaStream_t stream, uint32_t flags) {
  // one token: raw codes on the integer tensor cores (a fraction of this
  // kernel's per-weight work, which serves eight tokens)
  qmm_status st;
  if (M == 1 && launch_q4_gemv_digits(dev, N, K, W, X, Y, stream, flags, &st)) return st;
  const void *Wp[1] = {W};
  return launch_proj(dev, M, N, K, Wp, 1, X, Y, stream, flags);
}

qmm_status launch_q4_gateup_unfused(const DevInfo &dev, int M, int64_t N, int K, const void *Wg, const void *Wu,
                                    const float *X, float *G, float *U, float *Y, cudaStream_t stream) {
  const void *Wgp[1] = {Wg}, *Wup[1] = {Wu};
  qmm_status st = launch_proj(dev, M, N, K, Wgp, 1, X, G, stream, kLaunchPdl);
  if (st != QMM_OK) return st;
  st = launch_proj(dev, M, N, K, Wup, 1, X, U, stream, kLaunchPdl);
  if (st != QMM_OK) return st;
  const int64_t count = static_cast<int64_t>(M) * N;
  const int grid = static_cast<int>(std::min<int64_t>((count + 255) / 256, dev.sms * 8ll));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(std::max(grid, 1));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, silu_mul_kernel, static_cast<const float *>(G),
                                       static_cast<const float *>(U), Y, count),
                    "silu_mul launch");
}

cudaError_t q4_gateup_status(uint32_t *bits) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(bits, g_q4_status, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_q4_status, &zero, sizeof(uint32_t));
  return e;
}

}  // namespace qmm
