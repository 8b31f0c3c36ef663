/*
 * oracle.c -- plain, slow CPU reference for the grouped 4-bit MoE matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  The
 * product path (grouped_bit_weight_b200) never calls it and shares no code,
 * header, table or helper with it.
 *
 * Every function states the passage of the source pages it follows.  Page
 * names used below:
 *   [pypi]    "grouped-nf4-gemm 0.43.0" project page, sections "Try the
 *             packers and byte checks on CPU" (examples 1 and 2) and
 *             "Which entry point?".
 *   [receipts] "Receipts-driven engineering", opening paragraph (grouped
 *             matmul on 4-bit packed weights, NF4 in the bitsandbytes packed
 *             format unchanged, MXFP4 = OCP e2m1 on released bytes, NF4 path
 *             differentiable).
 *   [mxfp4]   "native MXFP4 MoE inference" record, "summary" field (e2m1
 *             blocks with e8m0 scales).
 *
 * Arithmetic: packers work in fp32 (the pages' packers take fp32 torch
 * tensors); decoders form the fp32 product code*scale; matmuls accumulate
 * in fp64 and round once to bf16 (round to nearest, ties to even).
 *
 * Parity status: every exported function is pinned by a "not gpu" test in
 * tests/test_oracle_pins.py against values the pages print, the OCP / QLoRA
 * definitions, closed forms or brute force.  None is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_SHAPE (-1)
#define ORC_ERR_NONFINITE (-2)
#define ORC_ERR_OFFSETS (-3)

/* ------------------------------------------------------------------ */
/* bf16 rounding                                                       */
/* ------------------------------------------------------------------ */

/* fp32 -> bf16, round to nearest even on the 16 dropped bits. NaN stays a
 * quiet NaN with its sign. */
static uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
    return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

static float bf16_to_f32(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* fp64 -> bf16 with a single rounding (no detour through fp32, which would
 * round twice).  bf16: 1 sign, 8 exponent (bias 127), 7 fraction bits;
 * subnormals are multiples of 2^-133. */
static uint16_t f64_to_bf16(double v) {
  if (isnan(v)) return 0x7fc0u;
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  double a = fabs(v);
  if (isinf(a)) return sign | 0x7f80u;
  if (a == 0.0) return sign;
  if (a < ldexp(1.0, -126)) {
    /* subnormal range: integer count of 2^-133 units, ties to even */
    double k = nearbyint(ldexp(a, 133));
    return sign | (uint16_t)k; /* k == 128 encodes the smallest normal */
  }
  int e;
  double m = frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1) */
  double r = nearbyint(ldexp(m, 8));  /* 8 significant bits, ties to even */
  if (r == 256.0) { r = 128.0; e += 1; }
  int biased = e + 126;               /* a = (r/128) * 2^(e-1) */
  if (biased >= 255) return sign | 0x7f80u;
  return sign | (uint16_t)(biased << 7) | (uint16_t)((int)r - 128);
}

uint16_t orc_f32_to_bf16(float f) { return f32_to_bf16(f); }
uint16_t orc_f64_to_bf16(double v) { return f64_to_bf16(v); }

/* ------------------------------------------------------------------ */
/* NF4                                                                 */
/* ------------------------------------------------------------------ */

/* The 16-entry NF4 codebook of QLoRA (Dettmers et al. 2023), the
 * "standard QLoRA codebook" the bitsandbytes packed format uses.  [receipts]
 * names the bitsandbytes format; the table itself is the published one:
 * sorted, C[0] = -1, C[7] = 0 exactly, C[15] = +1. */
static const float NF4_CODE[16] = {
    -1.0f,
    -0.6961928009986877f,
    -0.5250730514526367f,
    -0.39491748809814453f,
    -0.28444138169288635f,
    -0.18477343022823334f,
    -0.09105003625154495f,
    0.0f,
    0.07958029955625534f,
    0.16093020141124725f,
    0.24611230194568634f,
    0.33791524171829224f,
    0.44070982933044434f,
    0.5626170039176941f,
    0.7229568362236023f,
    1.0f,
};

void orc_nf4_codebook(float out[16]) { memcpy(out, NF4_CODE, sizeof(NF4_CODE)); }

/* Nearest code to y: argmin_i |y - C[i]| with the distances formed in fp32;
 * the first (lowest) index wins a tie. */
static int nf4_nearest(float y) {
  int best = 0;
  float bd = fabsf(y - NF4_CODE[0]);
  for (int i = 1; i < 16; ++i) {
    float d = fabsf(y - NF4_CODE[i]);
    if (d < bd) { bd = d; best = i; }
  }
  return best;
}

/* [pypi] example 1: quantize_pack_nf4(w) for a per-expert weight w[N,K]
 * returns packed [N, K/2] uint8 and absmax [N, K/64] fp32.
 * Per row and per 64-element block along K:
 *   a = max |w|  (fp32),  y = w / a  (fp32),  q = nearest code,
 *   byte j of the block = (q[2j] << 4) | q[2j+1]   (high nibble = even k:
 *   the bitsandbytes byte layout, which [receipts] says is kept unchanged).
 * A block that is all zero stores a = 0 and code 7 (the exact zero).
 * Non-finite input is rejected. */
int orc_nf4_pack(const float* w, int64_t rows, int64_t K, uint8_t* packed,
                 float* absmax) {
  if (rows < 0 || K < 0 || K % 64 != 0) return ORC_ERR_SHAPE;
  for (int64_t i = 0; i < rows * K; ++i)
    if (!isfinite(w[i])) return ORC_ERR_NONFINITE;
  const int64_t nb = K / 64;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const float* blk = w + r * K + b * 64;
      float a = 0.0f;
      for (int i = 0; i < 64; ++i) {
        float m = fabsf(blk[i]);
        if (m > a) a = m;
      }
      absmax[r * nb + b] = a;
      uint8_t* out = packed + r * (K / 2) + b * 32;
      for (int j = 0; j < 32; ++j) {
        int q0 = 7, q1 = 7;
        if (a > 0.0f) {
          q0 = nf4_nearest(blk[2 * j] / a);
          q1 = nf4_nearest(blk[2 * j + 1] / a);
        }
        out[j] = (uint8_t)((q0 << 4) | q1);
      }
    }
  }
  return ORC_OK;
}

/* Code of element k of a packed NF4 row: even k sits in the high nibble. */
static int nf4_code_at(const uint8_t* row, int64_t k) {
  uint8_t byte = row[k >> 1];
  return (k & 1) ? (byte & 0x0f) : (byte >> 4);
}

/* [pypi] example 1: dequant_ref(packed, absmax, N, K) -> fp32 [N, K],
 * w[n,k] = C[q[n,k]] * absmax[n, k/64]   (one fp32 multiply). */
void orc_nf4_decode_f32(const uint8_t* packed, const float* absmax,
                        int64_t rows, int64_t K, float* w) {
  const int64_t nb = K / 64;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const uint8_t* row = packed + r * (K / 2);
    for (int64_t k = 0; k < K; ++k)
      w[r * K + k] = NF4_CODE[nf4_code_at(row, k)] * absmax[r * nb + k / 64];
  }
}

/* The bf16 weight the matmul multiplies: the fp32 product above rounded
 * once to bf16.  [receipts]: the codebook is decoded inside the matmul, so
 * the operand the matmul sees is this bf16 value. */
void orc_nf4_decode_bf16(const uint8_t* packed, const float* absmax,
                         int64_t rows, int64_t K, uint16_t* w) {
  const int64_t nb = K / 64;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const uint8_t* row = packed + r * (K / 2);
    for (int64_t k = 0; k < K; ++k)
      w[r * K + k] =
          f32_to_bf16(NF4_CODE[nf4_code_at(row, k)] * absmax[r * nb + k / 64]);
  }
}

/* ------------------------------------------------------------------ */
/* MXFP4 (OCP MX, e2m1 elements, e8m0 shared scale per 32)              */
/* ------------------------------------------------------------------ */

/* e2m1 code -> value, from the bit fields (OCP MX v1.0, FP4 E2M1:
 * 1 sign, 2 exponent bits with bias 1, 1 mantissa bit, subnormal when the
 * exponent field is 0). */
static float e2m1_value(int code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  float mag = (e == 0) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, e - 1);
  return s ? -mag : mag;
}

/* e8m0 scale byte -> 2^(s-127); 0xFF is NaN (OCP MX). */
static float e8m0_value(uint8_t s) {
  if (s == 0xff) return NAN;
  return ldexpf(1.0f, (int)s - 127);
}

/* Nearest e2m1 magnitude code (0..7) to v >= 0; a tie goes to the code
 * with an even last bit (round half to even on the mantissa); values past
 * 6 saturate to 6 (they are nearest to it). */
static int e2m1_nearest_mag(float v) {
  int best = 0;
  float bd = fabsf(v - e2m1_value(0));
  for (int c = 1; c < 8; ++c) {
    float d = fabsf(v - e2m1_value(c));
    if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1)) {
      bd = d;
      best = c;
    }
  }
  return best;
}

/* [pypi] example 2: quantize_pack_mxfp4(w) for w[.., K], K a multiple of
 * 32, returns blocks [.., K/32, 16] uint8 and scales [.., K/32] uint8
 * (e8m0).  Per 32-element block (OCP MX scale rule):
 *   amax = max |w|;  X = floor(log2 amax) - 2  (2 = largest e2m1 exponent),
 *   clamped to [-127, 127];  scale byte = X + 127;
 *   element code = nearest e2m1 to w / 2^X (ties to even, saturating),
 *   sign in bit 3 (kept for values that round to zero, as a cast does).
 * Two codes per byte, the even element in the LOW nibble (the byte order
 * of the released gpt-oss checkpoints that [mxfp4] runs on).
 * An all-zero block stores scale byte 0 and zero codes. */
int orc_mxfp4_pack(const float* w, int64_t rows, int64_t K, uint8_t* blocks,
                   uint8_t* scales) {
  if (rows < 0 || K < 0 || K % 32 != 0) return ORC_ERR_SHAPE;
  for (int64_t i = 0; i < rows * K; ++i)
    if (!isfinite(w[i])) return ORC_ERR_NONFINITE;
  const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const float* blk = w + r * K + b * 32;
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i) {
        float m = fabsf(blk[i]);
        if (m > amax) amax = m;
      }
      uint8_t* out = blocks + (r * nb + b) * 16;
      if (amax == 0.0f) {
        scales[r * nb + b] = 0;
        memset(out, 0, 16);
        continue;
      }
      int e2;
      (void)frexpf(amax, &e2); /* amax = f * 2^e2, f in [0.5,1) */
      int X = (e2 - 1) - 2;    /* floor(log2 amax) - emax(e2m1) */
      if (X < -127) X = -127;
      if (X > 127) X = 127;
      scales[r * nb + b] = (uint8_t)(X + 127);
      for (int j = 0; j < 16; ++j) {
        int c[2];
        for (int t = 0; t < 2; ++t) {
          float v = ldexpf(blk[2 * j + t], -X);
          int mag = e2m1_nearest_mag(fabsf(v));
          c[t] = signbit(v) ? (mag | 8) : mag; /* sign kept, as in a cast */
        }
        out[j] = (uint8_t)(c[0] | (c[1] << 4));
      }
    }
  }
  return ORC_OK;
}

static int mxfp4_code_at(const uint8_t* row, int64_t k) {
  uint8_t byte = row[k >> 1];
  return (k & 1) ? (byte >> 4) : (byte & 0x0f);
}

/* [pypi] example 2: dequant_mxfp4(blocks, scales) -> [.., K],
 * w = e2m1(code) * 2^(scale-127)  (exact in fp32 and in bf16 when the
 * result is in range). */
void orc_mxfp4_decode_f32(const uint8_t* blocks, const uint8_t* scales,
                          int64_t rows, int64_t K, float* w) {
  const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const uint8_t* row = blocks + r * (K / 2);
    for (int64_t k = 0; k < K; ++k)
      w[r * K + k] =
          e2m1_value(mxfp4_code_at(row, k)) * e8m0_value(scales[r * nb + k / 32]);
  }
}

void orc_mxfp4_decode_bf16(const uint8_t* blocks, const uint8_t* scales,
                           int64_t rows, int64_t K, uint16_t* w) {
  const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const uint8_t* row = blocks + r * (K / 2);
    for (int64_t k = 0; k < K; ++k)
      w[r * K + k] = f32_to_bf16(e2m1_value(mxfp4_code_at(row, k)) *
                                 e8m0_value(scales[r * nb + k / 32]));
  }
}

/* ------------------------------------------------------------------ */
/* Grouped matmuls                                                      */
/* ------------------------------------------------------------------ */

/* Routed rows are sorted by expert: rows off[e] .. off[e+1]-1 belong to
 * expert e.  Checks 0 = off[0] <= off[1] <= ... <= off[E] = P. */
static int check_offsets(const int32_t* off, int32_t E, int64_t P) {
  if (E < 0 || P < 0) return ORC_ERR_SHAPE;
  if (off[0] != 0 || off[E] != P) return ORC_ERR_OFFSETS;
  for (int32_t e = 0; e < E; ++e)
    if (off[e + 1] < off[e]) return ORC_ERR_OFFSETS;
  return ORC_OK;
}

/* [pypi] "Which entry point?": gemm_4bit_grouped -- one call over all
 * active experts; [receipts]: the experts' matmuls run on the packed
 * weights with the codebook decoded inside.  The plain definition:
 *   out[p, n] = bf16( sum_k x[tok(p), k] * W_e(p)[n, k] )
 * with W the bf16 decoded weight [E, N, K] (orc_*_decode_bf16 of each
 * expert), tok(p) = row_to_token[p] (identity when NULL), e(p) the expert
 * whose row range holds p, the sum in fp64, one final rounding.
 * out_f64 (optional) receives the unrounded sums. */
int orc_grouped_forward(const uint16_t* x, int64_t T, int64_t K,
                        const uint16_t* wdec, int32_t E, int64_t N,
                        const int32_t* off, const int32_t* row_to_token,
                        int64_t P, uint16_t* out, double* out_f64) {
  int rc = check_offsets(off, E, P);
  if (rc) return rc;
  for (int64_t p = 0; p < P; ++p) {
    int64_t t = row_to_token ? row_to_token[p] : p;
    if (t < 0 || t >= T) return ORC_ERR_OFFSETS;
  }
  for (int32_t e = 0; e < E; ++e) {
    const uint16_t* W = wdec + (int64_t)e * N * K;
    const int64_t p0 = off[e], p1 = off[e + 1];
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t p = p0; p < p1; ++p) {
      for (int64_t n = 0; n < N; ++n) {
        const uint16_t* xr = x + (row_to_token ? (int64_t)row_to_token[p] : p) * K;
        const uint16_t* wr = W + n * K;
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k)
          s += (double)bf16_to_f32(xr[k]) * (double)bf16_to_f32(wr[k]);
        if (out) out[p * N + n] = f64_to_bf16(s);
        if (out_f64) out_f64[p * N + n] = s;
      }
    }
  }
  return ORC_OK;
}

/* The same definition evaluated only at the listed (p, n) pairs, for
 * checking full-size launches on a sample of outputs. */
int orc_grouped_forward_sampled(const uint16_t* x, int64_t T, int64_t K,
                                const uint16_t* wdec, int32_t E, int64_t N,
                                const int32_t* off, const int32_t* row_to_token,
                                int64_t P, const int64_t* sp, const int64_t* sn,
                                int64_t ns, double* out_f64) {
  int rc = check_offsets(off, E, P);
  if (rc) return rc;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < ns; ++i) {
    int64_t p = sp[i], n = sn[i];
    int32_t e = 0;
    while (e < E && !(p >= off[e] && p < off[e + 1])) ++e;
    const uint16_t* xr = x + (row_to_token ? (int64_t)row_to_token[p] : p) * K;
    const uint16_t* wr = wdec + ((int64_t)e * N + n) * K;
    double s = 0.0;
    for (int64_t k = 0; k < K; ++k)
      s += (double)bf16_to_f32(xr[k]) * (double)bf16_to_f32(wr[k]);
    out_f64[i] = s;
  }
  return ORC_OK;
}

/* [pypi] "Which entry point?": dgrad_4bit_grouped -- the backward of the
 * grouped matmul with respect to its activations ([receipts]: the NF4
 * path is differentiable and never leaves the packed format).  For
 * out = x W^T per expert, the activation gradient is
 *   dx[p, k] = bf16( sum_n dy[p, n] * W_e(p)[n, k] ),
 * fp64 sum, rows in the same expert-sorted order as dy. */
int orc_grouped_dgrad(const uint16_t* dy, int64_t P, int64_t N,
                      const uint16_t* wdec, int32_t E, int64_t K,
                      const int32_t* off, uint16_t* dx, double* dx_f64) {
  int rc = check_offsets(off, E, P);
  if (rc) return rc;
  for (int32_t e = 0; e < E; ++e) {
    const uint16_t* W = wdec + (int64_t)e * N * K;
#pragma omp parallel for schedule(static)
    for (int64_t p = off[e]; p < off[e + 1]; ++p) {
      double* acc = (double*)calloc((size_t)K, sizeof(double));
      const uint16_t* g = dy + p * N;
      for (int64_t n = 0; n < N; ++n) {
        double gv = (double)bf16_to_f32(g[n]);
        const uint16_t* wr = W + n * K;
        for (int64_t k = 0; k < K; ++k) acc[k] += gv * (double)bf16_to_f32(wr[k]);
      }
      for (int64_t k = 0; k < K; ++k) {
        if (dx) dx[p * K + k] = f64_to_bf16(acc[k]);
        if (dx_f64) dx_f64[p * K + k] = acc[k];
      }
      free(acc);
    }
  }
  return ORC_OK;
}

int orc_grouped_dgrad_sampled(const uint16_t* dy, int64_t P, int64_t N,
                              const uint16_t* wdec, int32_t E, int64_t K,
                              const int32_t* off, const int64_t* sp,
                              const int64_t* sk, int64_t ns, double* out_f64) {
  int rc = check_offsets(off, E, P);
  if (rc) return rc;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < ns; ++i) {
    int64_t p = sp[i], k = sk[i];
    int32_t e = 0;
    while (e < E && !(p >= off[e] && p < off[e + 1])) ++e;
    const uint16_t* g = dy + p * N;
    const uint16_t* W = wdec + (int64_t)e * N * K;
    double s = 0.0;
    for (int64_t n = 0; n < N; ++n)
      s += (double)bf16_to_f32(g[n]) * (double)bf16_to_f32(W[n * K + k]);
    out_f64[i] = s;
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* SwiGLU combine (the step between the two grouped matmuls of a fused  */
/* expert pass)                                                          */
/* ------------------------------------------------------------------ */

/* The fused gate_up -> SwiGLU -> down expert pass ("Receipts-driven
 * engineering", opening paragraph: the fused MoE path; the pages name the
 * activation but print neither its formula nor the gate/up layout).
 * Reading: the standard SwiGLU h = silu(gate) * up, silu(v) = v / (1 +
 * exp(-v)), with gate = columns [0, I) and up = columns [I, 2I) of the bf16
 * gate_up output, i.e. the gate_up weight stacks the gate rows above the up
 * rows.  gu [P, 2I] bf16 -> h [P, I] bf16, evaluated in fp64 from the bf16
 * inputs and rounded once to bf16 (the intermediate the down matmul reads). */
int orc_swiglu(const uint16_t* gu, int64_t P, int64_t I, uint16_t* h) {
  if (P < 0 || I <= 0) return ORC_ERR_SHAPE;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < P; ++p) {
    const uint16_t* g = gu + p * 2 * I;
    for (int64_t i = 0; i < I; ++i) {
      const double gv = (double)bf16_to_f32(g[i]);
      const double uv = (double)bf16_to_f32(g[I + i]);
      h[p * I + i] = f64_to_bf16(gv / (1.0 + exp(-gv)) * uv);
    }
  }
  return ORC_OK;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
