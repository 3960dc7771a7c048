/*
 * qmm_oracle.c -- plain, slow CPU oracle for block-quantized weight matmul.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this code. It shares no code, header, table or
 * helper with the CUDA library; it decodes the block bytes itself with its own
 * fp16 / bf16 decoders and accumulates in double precision, so every result is
 * the plain definition of the operation, rounded once at the end.
 *
 * Operations and where they are defined:
 *  - Q8_0 / Q4_0 block decode and the decode GEMV with a per-block scale:
 *    "Lumen v0.2.0 -- Q8-native decode" release notes, section
 *    "Phase 7.D -- Q8-native fused matmul" (weights kept in the native Q8_0
 *    ggml block layout; per-block fp16 scale d broadcast over the block).
 *    Q4_0 value (q - 8) * d with the ggml nibble order (low nibbles are
 *    elements 0..15, high nibbles 16..31).
 *  - Activation quantisation and the Q8xQ8 integer block dot:
 *    "Lumen v0.4.0 -- shape-aware VNNI/fp32 hybrid dispatch", section
 *    "Phase 7.M -- Q8xQ8 AVX2 int dot" (activations quantised to Q8 per
 *    32-block, per-block integer dot, then dequantised and accumulated).
 *    The Q8_0-block form of the quantised activations (fp16 scale, the
 *    ggml reference rule) is the ggml-interoperable variant of the same step.
 *  - Fused gate/up SwiGLU out = silu(x.Wg) * (x.Wu):
 *    "LSE v0.4.16", section "Combined M8 Q4 gate/up execution".
 *  - Prefill panels Y = X . W^T with bf16 activations:
 *    "LSE v0.4.16", section "Retained optimizations and compatibility"
 *    (M1024 prefill panels).
 *
 * Every output routine works on a window of outputs [m0, m1) x [n0, n1) so
 * that full-size workloads can be checked on sampled outputs. Output arrays of
 * a window are dense, row-major, (m1 - m0) x (n1 - n0).
 *
 * The "S" outputs are the per-output absolute norms sum_k |w_k * x_k| used
 * for the tolerances |gpu - oracle| <= tol * S.
 *
 * Build: gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -shared -fPIC
 * (no contraction: the activation quantiser below is defined by separate
 * IEEE binary32 operations).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORA_BLOCK 32
#define ORA_Q8_0 0
#define ORA_Q4_0 1

/* ---- scalar decoders ---------------------------------------------------- */

/* IEEE binary16 bits -> double (exact). */
double ora_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal: m * 2^(1-15-10) */
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(m | 0x400), e - 25); /* (1 + m/2^10) * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* bfloat16 bits -> double (exact). */
double ora_bf16_to_double(uint16_t b) {
  int sign = (b >> 15) & 1;
  int e = (b >> 7) & 0xff;
  int m = b & 0x7f;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -133); /* subnormal: m * 2^(1-127-7) */
  } else if (e == 255) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(m | 0x80), e - 134); /* (1 + m/2^7) * 2^(e-127) */
  }
  return sign ? -v : v;
}

static int ora_block_bytes(int wtype) { return wtype == ORA_Q8_0 ? 34 : 18; }

/* Decode one block (34 or 18 bytes) into 32 exact doubles. */
void ora_decode_block(int wtype, const uint8_t *blk, double w[ORA_BLOCK]) {
  uint16_t dbits = (uint16_t)(blk[0] | (blk[1] << 8));
  double d = ora_half_to_double(dbits);
  const uint8_t *qs = blk + 2;
  if (wtype == ORA_Q8_0) {
    for (int j = 0; j < ORA_BLOCK; ++j) w[j] = (double)(int8_t)qs[j] * d;
  } else {
    for (int j = 0; j < 16; ++j) {
      w[j] = (double)((int)(qs[j] & 0x0f) - 8) * d;
      w[j + 16] = (double)((int)(qs[j] >> 4) - 8) * d;
    }
  }
}

/* Decode a whole N x K matrix (row-major by output feature) to doubles. */
void ora_dequantize(int wtype, int64_t n_rows, int64_t k, const uint8_t *W, double *out) {
  int64_t kb = k / ORA_BLOCK, bb = ora_block_bytes(wtype);
  for (int64_t n = 0; n < n_rows; ++n)
    for (int64_t b = 0; b < kb; ++b)
      ora_decode_block(wtype, W + (n * kb + b) * bb, out + n * k + b * ORA_BLOCK);
}

/* ---- decode GEMV / small-M matmul: Y[m][n] = sum_k X[m][k] * W[n][k] ---- */

void ora_gemv(int wtype, int64_t M, int64_t N, int64_t K, const uint8_t *W, const float *X,
              int64_t m0, int64_t m1, int64_t n0, int64_t n1, double *Y, double *S) {
  int64_t kb = K / ORA_BLOCK, bb = ora_block_bytes(wtype), wn = n1 - n0;
  double w[ORA_BLOCK];
  (void)M;
  (void)N;
  for (int64_t m = m0; m < m1; ++m) {
    for (int64_t n = n0; n < n1; ++n) {
      double acc = 0.0, nrm = 0.0;
      for (int64_t b = 0; b < kb; ++b) {
        ora_decode_block(wtype, W + (n * kb + b) * bb, w);
        for (int j = 0; j < ORA_BLOCK; ++j) {
          double p = w[j] * (double)X[m * K + b * ORA_BLOCK + j];
          acc += p;
          nrm += fabs(p);
        }
      }
      Y[(m - m0) * wn + (n - n0)] = acc;
      if (S) S[(m - m0) * wn + (n - n0)] = nrm;
    }
  }
}

/* ---- activation quantisation to Q8 (per 32-block, binary32) -------------
 * amax = max_j |x_j|; d = amax / 127 (binary32 division, round to nearest);
 * q_j = round-half-away-from-zero(x_j / d) (binary32 division), clamped to
 * [-127, 127]; a block whose d is zero gets all-zero codes.                */
void ora_quantize_act_q8(int64_t M, int64_t K, const float *X, int8_t *QX, float *DX) {
  int64_t kb = K / ORA_BLOCK;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t b = 0; b < kb; ++b) {
      const float *x = X + m * K + b * ORA_BLOCK;
      float amax = 0.0f;
      for (int j = 0; j < ORA_BLOCK; ++j) {
        float a = fabsf(x[j]);
        if (a > amax) amax = a;
      }
      float d = amax / 127.0f;
      DX[m * kb + b] = d;
      for (int j = 0; j < ORA_BLOCK; ++j) {
        int q = 0;
        if (d != 0.0f) {
          float v = x[j] / d;
          float r = roundf(v); /* C99 roundf: halfway cases away from zero */
          if (r > 127.0f) r = 127.0f;
          if (r < -127.0f) r = -127.0f;
          q = (int)r;
        }
        QX[m * K + b * ORA_BLOCK + j] = (int8_t)q;
      }
    }
  }
}

/* ---- Q8_0 activation blocks with an fp16 scale (ggml-compatible form) ---- */

/* binary32 -> IEEE binary16 bits, round to nearest even (subnormals, overflow
 * to infinity). Written from the format definitions: sign, 5-bit exponent with
 * bias 15, 10-bit fraction; values below 2^-14 are multiples of 2^-24. */
uint16_t ora_float_to_half_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  const uint32_t mag = u & 0x7fffffffu;
  if (mag >= 0x7f800000u) return (uint16_t)(sign | (mag > 0x7f800000u ? 0x7e00u : 0x7c00u)); /* NaN / Inf */
  const double a = fabs((double)f); /* exact */
  if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u); /* rounds to infinity (65504 + half an ulp of 32) */
  /* the multiple of the binary16 spacing at a's binade, rounded to nearest even */
  int e;
  (void)frexp(a, &e);                /* a = m * 2^e, m in [0.5, 1) */
  int exp16 = e - 1;                  /* a in [2^exp16, 2^(exp16+1)) */
  if (exp16 < -14) exp16 = -14;       /* subnormal range: spacing 2^-24 */
  const double ulp = ldexp(1.0, exp16 - 10);
  double q = a / ulp;                 /* exact: a power-of-two division */
  double r = floor(q);
  const double rem = q - r;
  if (rem > 0.5 || (rem == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
  const double v = r * ulp;           /* the rounded magnitude */
  if (v == 0.0) return sign;
  int ev;
  (void)frexp(v, &ev);
  const int ex = ev - 1;
  if (ex < -14) return (uint16_t)(sign | (uint16_t)(v / ldexp(1.0, -24))); /* subnormal */
  const uint16_t frac = (uint16_t)(v / ldexp(1.0, ex - 10) - 1024.0);
  return (uint16_t)(sign | (uint16_t)((ex + 15) << 10) | frac);
}

/* Activations as ggml Q8_0 blocks (34 bytes: fp16 d, then 32 int8 codes),
 * with ggml's reference rule: amax = max |x_j|; d = amax / 127; id = 1 / d
 * (0 when d == 0); q_j = round-half-away(x_j * id); the block stores
 * binary16(d) rounded to nearest even and the codes (|x_j * id| < 127.5, so
 * the clamp to [-127, 127] never acts). XB: M x (K/32) blocks, row-major. */
void ora_quantize_act_q8_0(int64_t M, int64_t K, const float *X, uint8_t *XB) {
  int64_t kb = K / ORA_BLOCK;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t b = 0; b < kb; ++b) {
      const float *x = X + m * K + b * ORA_BLOCK;
      uint8_t *blk = XB + (m * kb + b) * 34;
      float amax = 0.0f;
      for (int j = 0; j < ORA_BLOCK; ++j) {
        float a = fabsf(x[j]);
        if (a > amax) amax = a;
      }
      const float d = amax / 127.0f;
      const float id = d != 0.0f ? 1.0f / d : 0.0f;
      const uint16_t h = ora_float_to_half_rne(d);
      blk[0] = (uint8_t)(h & 0xff);
      blk[1] = (uint8_t)(h >> 8);
      for (int j = 0; j < ORA_BLOCK; ++j) {
        const float v = x[j] * id;
        float r = roundf(v);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        blk[2 + j] = (uint8_t)(int8_t)(int)r;
      }
    }
  }
}

/* ---- Q8 x Q8: exact integer block dots, then scaled accumulation -------- */

/* isum[(m-m0)][(n-n0)][b] = sum_j qw[n][32b+j] * qx[m][32b+j]; returns the
 * number of block dots that did not fit in int32 (0 for valid codes). */
int64_t ora_q8q8_block_dots(int64_t M, int64_t N, int64_t K, const uint8_t *W, const int8_t *QX,
                            int64_t m0, int64_t m1, int64_t n0, int64_t n1, int32_t *isum) {
  int64_t kb = K / ORA_BLOCK, bad = 0, wn = n1 - n0;
  (void)M;
  (void)N;
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t n = n0; n < n1; ++n)
      for (int64_t b = 0; b < kb; ++b) {
        const uint8_t *blk = W + (n * kb + b) * 34;
        int64_t s = 0;
        for (int j = 0; j < ORA_BLOCK; ++j)
          s += (int64_t)(int8_t)blk[2 + j] * (int64_t)QX[m * K + b * ORA_BLOCK + j];
        if (s > INT32_MAX || s < INT32_MIN) ++bad;
        isum[((m - m0) * wn + (n - n0)) * kb + b] = (int32_t)s;
      }
  return bad;
}

/* Y = sum_b d_w[n][b] * d_x[m][b] * isum[m][n][b] (double);
 * S = sum_b |d_w * d_x| * sum_j |qw * qx| (norm against the quantised x). */
void ora_q8q8_gemv(int64_t M, int64_t N, int64_t K, const uint8_t *W, const int8_t *QX,
                   const float *DX, int64_t m0, int64_t m1, int64_t n0, int64_t n1, double *Y,
                   double *S) {
  int64_t kb = K / ORA_BLOCK, wn = n1 - n0;
  (void)M;
  (void)N;
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t n = n0; n < n1; ++n) {
      double acc = 0.0, nrm = 0.0;
      for (int64_t b = 0; b < kb; ++b) {
        const uint8_t *blk = W + (n * kb + b) * 34;
        double dw = ora_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
        double dx = (double)DX[m * kb + b];
        int64_t s = 0, sa = 0;
        for (int j = 0; j < ORA_BLOCK; ++j) {
          int64_t p = (int64_t)(int8_t)blk[2 + j] * (int64_t)QX[m * K + b * ORA_BLOCK + j];
          s += p;
          sa += p < 0 ? -p : p;
        }
        acc += dw * dx * (double)s;
        nrm += fabs(dw * dx) * (double)sa;
      }
      Y[(m - m0) * wn + (n - n0)] = acc;
      if (S) S[(m - m0) * wn + (n - n0)] = nrm;
    }
}

/* ---- fused gate/up SwiGLU: out = silu(x.Wg) * (x.Wu), silu(g) = g/(1+e^-g) */

void ora_swiglu(int wtype, int64_t M, int64_t N, int64_t K, const uint8_t *Wg, const uint8_t *Wu,
                const float *X, int64_t m0, int64_t m1, int64_t n0, int64_t n1, double *OUT,
                double *G, double *U, double *SG, double *SU) {
  int64_t cnt = (m1 - m0) * (n1 - n0);
  ora_gemv(wtype, M, N, K, Wg, X, m0, m1, n0, n1, G, SG);
  ora_gemv(wtype, M, N, K, Wu, X, m0, m1, n0, n1, U, SU);
  for (int64_t i = 0; i < cnt; ++i) {
    double g = G[i];
    OUT[i] = g / (1.0 + exp(-g)) * U[i];
  }
}

/* ---- prefill panel: Y[m][n] = sum_k bf16(X[m][k]) * W[n][k] --------------- */

void ora_prefill(int wtype, int64_t M, int64_t N, int64_t K, const uint8_t *W, const uint16_t *Xbf,
                 int64_t m0, int64_t m1, int64_t n0, int64_t n1, double *Y, double *S) {
  int64_t kb = K / ORA_BLOCK, bb = ora_block_bytes(wtype), wn = n1 - n0;
  double w[ORA_BLOCK];
  (void)M;
  (void)N;
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t n = n0; n < n1; ++n) {
      double acc = 0.0, nrm = 0.0;
      for (int64_t b = 0; b < kb; ++b) {
        ora_decode_block(wtype, W + (n * kb + b) * bb, w);
        for (int j = 0; j < ORA_BLOCK; ++j) {
          double p = w[j] * ora_bf16_to_double(Xbf[m * K + b * ORA_BLOCK + j]);
          acc += p;
          nrm += fabs(p);
        }
      }
      Y[(m - m0) * wn + (n - n0)] = acc;
      if (S) S[(m - m0) * wn + (n - n0)] = nrm;
    }
}
