/*
 * CPU oracle for the NVFP4 W4A4 + Residual Activation Compensation (RAC) path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file;
 * only the tests, the package smoke check and the CPU-baseline leg of the
 * benchmark load it.  It shares no code, header, table or helper with the CUDA
 * library: every routine below is written from the definitions it cites.
 *
 * Sources (page title - section):
 *  [ABS]  "QUADS: Stabilizing NVFP4 Reinforcement Learning for MoE via QUantization-error
 *          Alignment across Dual Sides" (mlsanity.com) - Abstract (arXiv): NVFP4 pairs
 *          fine-grained scaling with native W4A4 FP4 GEMMs; weights are aligned through a
 *          shared quantize-dequantize path; activations are recomputed online.
 *  [FAIL] "Why 4-bit RL rollout collapses - and it isn't the weights" - The failure mode:
 *          the E2M1 grid has 8 magnitude levels per sign (E4M3 has 256 codes).
 *  [FIX]  same post - Two fixes, on two different sides: Asymmetric QAT fake-quantizes
 *          weights only; RAC picks roughly the top 50% of activation channels by
 *          quantization error and runs a second, residual FP4 pass over just those
 *          channels, leaving the W4A4 GEMM intact.
 *  The pages give no formulas.  The numeric format (E2M1 payload, one E4M3 scale per
 *  16 elements along K, FP32 per-tensor scale amax/(6*448)), the FP32 operation order and
 *  the residual / calibration readings are the ones listed in the design notes; each
 *  function below states the reading it implements.
 *
 * Precision: quantisation decisions are taken in IEEE binary32 with round-to-nearest-even
 * (this file must be compiled without -ffast-math and with -ffp-contract=off); GEMM dot
 * products are exact in 64-bit integers; calibration sums are binary64.
 *
 * Parity pins: every function here is pinned by the CPU tests (closed forms, brute force,
 * hand-worked fixtures, invariants).  No function is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------------------------ */
/* storage conversions                                                                        */
/* ------------------------------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* round a binary64 value to the nearest bf16 (ties to even), done on the exact value */
uint16_t orc_f64_to_bf16(double d) {
  if (isnan(d)) return 0x7FC0;
  int neg = signbit(d) ? 1 : 0;
  double a = fabs(d);
  if (a == 0.0) return (uint16_t)(neg << 15);
  /* bf16: 8 significant bits, exponent range like binary32 (normal min 2^-126) */
  int e;
  frexp(a, &e);              /* a = m * 2^e, m in [0.5, 1) */
  int exp2 = e - 1;          /* a in [2^exp2, 2^(exp2+1)) */
  if (exp2 < -126) exp2 = -126; /* subnormal spacing */
  double ulp = ldexp(1.0, exp2 - 7);
  double q = a / ulp;        /* exact: scaling by a power of two */
  double fl = floor(q);
  double rem = q - fl;
  double n;
  if (rem > 0.5) n = fl + 1.0;
  else if (rem < 0.5) n = fl;
  else n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  double r = n * ulp;
  if (r > 3.3895313892515355e38) return (uint16_t)((neg << 15) | 0x7F80); /* overflow -> inf */
  float f = (float)r;        /* exact: r has <= 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)((u >> 16) | (neg << 15));
}

uint16_t orc_f32_to_bf16(float f) { return orc_f64_to_bf16((double)f); }

/* ------------------------------------------------------------------------------------------ */
/* E2M1 element format [FAIL]: 1 sign bit, magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}            */
/* code = sign<<3 | index, index 0..7 in increasing magnitude; an odd index has mantissa 1.   */
/* ------------------------------------------------------------------------------------------ */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_decode(int code) {
  double m = E2M1_MAG[code & 7];
  return (code & 8) ? -m : m;
}

/* nearest representable magnitude, ties to the even index (mantissa 0), anything >= 6 -> 6;
 * the sign bit of the input is kept, so a negative value that rounds to zero gives 0x8. */
int orc_e2m1_encode(float v) {
  double m = fabs((double)v);
  int idx;
  if (!(m < 6.0)) {
    idx = 7;
  } else {
    int i = 0;
    while (E2M1_MAG[i + 1] <= m) ++i; /* E2M1_MAG[i] <= m < E2M1_MAG[i+1] */
    double dlo = m - E2M1_MAG[i], dhi = E2M1_MAG[i + 1] - m;
    if (dlo < dhi) idx = i;
    else if (dhi < dlo) idx = i + 1;
    else idx = (i % 2 == 0) ? i : i + 1;
  }
  return idx | (signbit(v) ? 8 : 0);
}

/* ------------------------------------------------------------------------------------------ */
/* E4M3 scale format (bias 7, no infinities, 0x7F/0xFF = NaN, max 448)                        */
/* ------------------------------------------------------------------------------------------ */
double orc_e4m3_decode(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
  return s ? -v : v;
}

/* non-negative input: nearest finite E4M3 value, ties to the even code, >= 448 -> 448 */
int orc_e4m3_encode(float raw) {
  double r = (double)raw;
  if (!(r >= 0.0)) return 0;
  if (r >= 448.0) return 0x7E;
  int c = 0;
  while (c < 0x7E && orc_e4m3_decode(c + 1) <= r) ++c; /* val(c) <= r < val(c+1) */
  double lo = orc_e4m3_decode(c), hi = orc_e4m3_decode(c + 1);
  double dlo = r - lo, dhi = hi - r;
  if (dlo < dhi) return c;
  if (dhi < dlo) return c + 1;
  return (c % 2 == 0) ? c : c + 1;
}

/* ------------------------------------------------------------------------------------------ */
/* per-tensor scale: amax exact in FP32, s_g = RN(amax / (6*448))                             */
/* ------------------------------------------------------------------------------------------ */
float orc_amax_bf16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld) {
  float amax = 0.0f;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      float a = fabsf(orc_bf16_to_f32(x[r * ld + c]));
      if (a > amax) amax = a;
    }
  return amax;
}

float orc_amax_f32(const float* t, int64_t n) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    float a = fabsf(t[i]);
    if (a > amax) amax = a;
  }
  return amax;
}

float orc_global_scale(float amax) {
  const float denom = 2688.0f; /* 6 (E2M1 max) * 448 (E4M3 max) */
  return amax / denom;
}

/* ------------------------------------------------------------------------------------------ */
/* quantisation of one 16-element block with per-tensor scale s_g (FP32, in this order):      */
/*   b = max|t_i|; raw = RN(b / RN(6*s_g)); S = E4M3(raw)                                     */
/*   d = RN(S*s_g); S == 0 -> all codes +0; else inv = RN(1/d), q_i = E2M1(RN(t_i*inv))       */
/*   DQ_i = RN(val(q_i)*d)                                                                    */
/* s_g == 0 (all-zero tensor) gives S = 0 and +0 codes.                                       */
/* ------------------------------------------------------------------------------------------ */
static void quant_block16(const float* t, float s_g, uint8_t* codes, uint8_t* S_out, float* dq) {
  float b = 0.0f;
  for (int i = 0; i < 16; ++i) {
    float a = fabsf(t[i]);
    if (a > b) b = a;
  }
  int S = 0;
  if (s_g > 0.0f) {
    float t6 = 6.0f * s_g;
    float raw = b / t6;
    S = orc_e4m3_encode(raw);
  }
  *S_out = (uint8_t)S;
  if (S == 0) {
    for (int i = 0; i < 16; ++i) {
      codes[i] = 0;
      if (dq) dq[i] = 0.0f;
    }
    return;
  }
  float d = (float)orc_e4m3_decode(S) * s_g;
  float inv = 1.0f / d;
  for (int i = 0; i < 16; ++i) {
    float v = t[i] * inv;
    int q = orc_e2m1_encode(v);
    codes[i] = (uint8_t)q;
    if (dq) dq[i] = (float)orc_e2m1_decode(q) * d;
  }
}

/* rows x L float values (L % 16 == 0), blocks along L.  codes: one code per byte [rows*L];
 * S: one E4M3 code per block [rows*L/16]; dq: dequantised values [rows*L] (nullable). */
void orc_quantize_f32(const float* t, int64_t rows, int64_t L, float s_g, uint8_t* codes, uint8_t* S,
                      float* dq) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < L / 16; ++b)
      quant_block16(t + r * L + b * 16, s_g, codes + r * L + b * 16, S + r * (L / 16) + b,
                    dq ? dq + r * L + b * 16 : NULL);
}

/* ------------------------------------------------------------------------------------------ */
/* online activation quantisation with the residual pass on the selected channels [FIX]       */
/*   Q(X) with s_g; r = RN(x - DQ(Q(X))) on channels sel[0..Kp) (ascending, compact order);   */
/*   Q(R_sel) with the same s_g (shared-scale reading), blocks of 16 along the compact axis.  */
/* x: bf16 [rows x K] with leading dimension ldx.                                             */
/* ------------------------------------------------------------------------------------------ */
void orc_act_quant_rac(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, float s_g,
                       const int32_t* sel, int32_t Kp, uint8_t* codes, uint8_t* S, uint8_t* rcodes,
                       uint8_t* rS, float* resid) {
#pragma omp parallel
  {
    float* t = (float*)malloc(sizeof(float) * (size_t)K);
    float* dq = (float*)malloc(sizeof(float) * (size_t)K);
    float* rr = (float*)malloc(sizeof(float) * (size_t)(Kp > 0 ? Kp : 1));
#pragma omp for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
      for (int64_t k = 0; k < K; ++k) t[k] = orc_bf16_to_f32(x[r * ldx + k]);
      for (int64_t b = 0; b < K / 16; ++b)
        quant_block16(t + b * 16, s_g, codes + r * K + b * 16, S + r * (K / 16) + b, dq + b * 16);
      for (int32_t j = 0; j < Kp; ++j) rr[j] = t[sel[j]] - dq[sel[j]];
      for (int32_t b = 0; b < Kp / 16; ++b)
        quant_block16(rr + b * 16, s_g, rcodes + r * Kp + b * 16, rS + r * (Kp / 16) + b, NULL);
      if (resid)
        for (int32_t j = 0; j < Kp; ++j) resid[r * Kp + j] = rr[j];
    }
    free(t);
    free(dq);
    free(rr);
  }
}

/* ------------------------------------------------------------------------------------------ */
/* RAC variant "masked full-K residual" (the selection is the same as above; only the layout   */
/* of the residual pass differs, so it is a flag of its own, not the method's default):         */
/*   m = RN(x - DQ(Q(X))) on the channels in sel and 0 on the others, kept at its channel (no   */
/*   compaction) and quantised with the same s_g in blocks of 16 along K.  The residual pass of  */
/*   the GEMM then multiplies Q(M) by the main packed weight Q(W): no W_sel is stored.           */
/* x: bf16 [rows x K] (leading dimension ldx); mcodes [rows x K], mS [rows x K/16].             */
/* ------------------------------------------------------------------------------------------ */
void orc_act_quant_masked(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, float s_g, const int32_t* sel,
                          int32_t Kp, uint8_t* codes, uint8_t* S, uint8_t* mcodes, uint8_t* mS) {
#pragma omp parallel
  {
    float* t = (float*)malloc(sizeof(float) * (size_t)K);
    float* dq = (float*)malloc(sizeof(float) * (size_t)K);
    float* m = (float*)malloc(sizeof(float) * (size_t)K);
#pragma omp for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
      for (int64_t k = 0; k < K; ++k) t[k] = orc_bf16_to_f32(x[r * ldx + k]);
      for (int64_t b = 0; b < K / 16; ++b)
        quant_block16(t + b * 16, s_g, codes + r * K + b * 16, S + r * (K / 16) + b, dq + b * 16);
      for (int64_t k = 0; k < K; ++k) m[k] = 0.0f;
      for (int32_t j = 0; j < Kp; ++j) m[sel[j]] = t[sel[j]] - dq[sel[j]];
      for (int64_t b = 0; b < K / 16; ++b)
        quant_block16(m + b * 16, s_g, mcodes + r * K + b * 16, mS + r * (K / 16) + b, NULL);
    }
    free(t);
    free(dq);
    free(m);
  }
}

/* ------------------------------------------------------------------------------------------ */
/* weight side of the shared QDQ path [ABS]: Q(W) with its own s_gw, and W_sel = W[:, sel]    */
/* (raw bf16 columns, ascending) quantised with the same s_gw.                                */
/* ------------------------------------------------------------------------------------------ */
void orc_weight_pack(const uint16_t* w, int64_t N, int64_t K, float s_gw, const int32_t* sel, int32_t Kp,
                     uint8_t* codes, uint8_t* S, uint8_t* scodes, uint8_t* sS) {
#pragma omp parallel
  {
    float* t = (float*)malloc(sizeof(float) * (size_t)K);
    float* ts = (float*)malloc(sizeof(float) * (size_t)(Kp > 0 ? Kp : 1));
#pragma omp for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
      for (int64_t k = 0; k < K; ++k) t[k] = orc_bf16_to_f32(w[n * K + k]);
      for (int64_t b = 0; b < K / 16; ++b)
        quant_block16(t + b * 16, s_gw, codes + n * K + b * 16, S + n * (K / 16) + b, NULL);
      for (int32_t j = 0; j < Kp; ++j) ts[j] = t[sel[j]];
      for (int32_t b = 0; b < Kp / 16; ++b)
        quant_block16(ts + b * 16, s_gw, scodes + n * Kp + b * 16, sS + n * (Kp / 16) + b, NULL);
    }
    free(t);
    free(ts);
  }
}

/* trainer-side fake quantisation [FIX, Asymmetric QAT]: out = bf16(DQ(Q(w))), one s_g per tensor */
void orc_weight_qdq(const uint16_t* w, int64_t n, float s_g, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < n / 16; ++b) {
    float t[16], dq[16];
    uint8_t c[16], S;
    for (int i = 0; i < 16; ++i) t[i] = orc_bf16_to_f32(w[b * 16 + i]);
    quant_block16(t, s_g, c, &S, dq);
    for (int i = 0; i < 16; ++i) out[b * 16 + i] = orc_f32_to_bf16(dq[i]);
  }
}

/* ------------------------------------------------------------------------------------------ */
/* W4A4 + RAC GEMM, exact [ABS, FIX]:                                                         */
/*   y[i,j] = s_a * s_w * ( sum_k DQ'(a[i,k]) DQ'(w[j,k]) + sum_k' DQ'(r[i,k']) DQ'(ws[j,k']) ) */
/* with DQ'(q) = e(q) * S(block) (the block-scaled value without the per-tensor scale).       */
/* Computed as integers: E = 2e in [-12, 12], S^ = S*2^9 in [0, 229376];                      */
/* acc = sum E_a S^_a E_w S^_w (int64, exact), y = acc * 2^-20 * s_a * s_w (binary64).        */
/* absdot[i,j] is the same sum over |terms| (for the tolerance).                              */
/* Codes are one per byte; S arrays are [rows x L/16] E4M3 codes.                             */
/* rows: indices of the A rows to evaluate (n_rows of them); y/absdot are [n_rows x N].       */
/* ------------------------------------------------------------------------------------------ */
static inline int64_t e2m1_times2(uint8_t q) { return (int64_t)(2.0 * orc_e2m1_decode(q)); }
static inline int64_t e4m3_times512(uint8_t s) { return (int64_t)ldexp(orc_e4m3_decode(s), 9); }

void orc_gemm_rac(const uint8_t* ac, const uint8_t* aS, const uint8_t* rc, const uint8_t* rS, int64_t K,
                  int32_t Kp, const uint8_t* wc, const uint8_t* wS, const uint8_t* wsc, const uint8_t* wsS,
                  int64_t N, double s_a, double s_w, const int64_t* rows, int64_t n_rows, double* y,
                  double* absdot) {
  const double unit = ldexp(1.0, -20) * s_a * s_w;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t ii = 0; ii < n_rows; ++ii) {
    int64_t i = rows[ii];
    for (int64_t j = 0; j < N; ++j) {
      int64_t acc = 0, aacc = 0;
      for (int64_t b = 0; b < K / 16; ++b) {
        int64_t sblk = e4m3_times512(aS[i * (K / 16) + b]) * e4m3_times512(wS[j * (K / 16) + b]);
        int64_t dot = 0, adot = 0;
        for (int64_t k = b * 16; k < b * 16 + 16; ++k) {
          int64_t p = e2m1_times2(ac[i * K + k]) * e2m1_times2(wc[j * K + k]);
          dot += p;
          adot += p < 0 ? -p : p;
        }
        acc += dot * sblk;
        aacc += adot * sblk;
      }
      for (int64_t b = 0; b < Kp / 16; ++b) {
        int64_t sblk = e4m3_times512(rS[i * (Kp / 16) + b]) * e4m3_times512(wsS[j * (Kp / 16) + b]);
        int64_t dot = 0, adot = 0;
        for (int64_t k = b * 16; k < b * 16 + 16; ++k) {
          int64_t p = e2m1_times2(rc[i * Kp + k]) * e2m1_times2(wsc[j * Kp + k]);
          dot += p;
          adot += p < 0 ? -p : p;
        }
        acc += dot * sblk;
        aacc += adot * sblk;
      }
      y[ii * N + j] = (double)acc * unit;
      if (absdot) absdot[ii * N + j] = (double)aacc * fabs(unit);
    }
  }
}

/* ------------------------------------------------------------------------------------------ */
/* RAC channel selection [FIX]: quantise the calibration batch with its own s_g; per channel  */
/* e_k = sum_t r_{t,k}^2 in binary64 (t ascending; r is FP32 so r^2 is exact in binary64);   */
/* keep the Kp channels with the largest e_k (ties -> lower k); return them ascending.        */
/* ------------------------------------------------------------------------------------------ */
static const double* g_sort_err;
static int cmp_err_desc(const void* a, const void* b) {
  int32_t i = *(const int32_t*)a, j = *(const int32_t*)b;
  double ei = g_sort_err[i], ej = g_sort_err[j];
  if (ei > ej) return -1;
  if (ei < ej) return 1;
  return (i < j) ? -1 : (i > j) ? 1 : 0;
}
static int cmp_int_asc(const void* a, const void* b) {
  int32_t i = *(const int32_t*)a, j = *(const int32_t*)b;
  return (i < j) ? -1 : (i > j) ? 1 : 0;
}

/* residuals r = x - DQ(Q(x)) of the calibration batch, quantised with its own s_g (FP32) */
static float* calib_residuals(const uint16_t* x, int64_t T, int64_t K) {
  float amax = orc_amax_bf16(x, T, K, K);
  float s_g = orc_global_scale(amax);
  float* resid = (float*)malloc(sizeof(float) * (size_t)(T * K));
#pragma omp parallel
  {
    float* t = (float*)malloc(sizeof(float) * (size_t)K);
    float* dq = (float*)malloc(sizeof(float) * (size_t)K);
    uint8_t* c = (uint8_t*)malloc((size_t)K);
    uint8_t* S = (uint8_t*)malloc((size_t)(K / 16));
#pragma omp for schedule(static)
    for (int64_t r = 0; r < T; ++r) {
      for (int64_t k = 0; k < K; ++k) t[k] = orc_bf16_to_f32(x[r * K + k]);
      for (int64_t b = 0; b < K / 16; ++b) quant_block16(t + b * 16, s_g, c + b * 16, S + b, dq + b * 16);
      for (int64_t k = 0; k < K; ++k) resid[r * K + k] = t[k] - dq[k];
    }
    free(t);
    free(dq);
    free(c);
    free(S);
  }
  return resid;
}

/* e_k = sum over rows [r0, r1) of r_{t,k}^2, t ascending, binary64 */
static void calib_errors(const float* resid, int64_t r0, int64_t r1, int64_t K, double* err) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < K; ++k) {
    double e = 0.0;
    for (int64_t r = r0; r < r1; ++r) {
      double v = (double)resid[r * K + k];
      e += v * v;
    }
    err[k] = e;
  }
}

/* the Kp channels with the largest e_k (ties -> lower k), ascending */
static void calib_select(const double* err, int64_t K, int32_t Kp, int32_t* sel) {
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
  for (int32_t k = 0; k < K; ++k) idx[k] = k;
  g_sort_err = err;
  qsort(idx, (size_t)K, sizeof(int32_t), cmp_err_desc);
  for (int32_t j = 0; j < Kp; ++j) sel[j] = idx[j];
  qsort(sel, (size_t)Kp, sizeof(int32_t), cmp_int_asc);
  free(idx);
}

void orc_calibrate(const uint16_t* x, int64_t T, int64_t K, int32_t Kp, int32_t* sel, double* err_out) {
  float* resid = calib_residuals(x, T, K);
  double* err = (double*)malloc(sizeof(double) * (size_t)K);
  calib_errors(resid, 0, T, K, err);
  calib_select(err, K, Kp, sel);
  if (err_out) memcpy(err_out, err, sizeof(double) * (size_t)K);
  free(err);
  free(resid);
}

/* Per-expert selection (a variant the pages leave open: one channel list per expert of the    */
/* down projection).  Reading: the pooled calibration batch (rows grouped by expert, group g =  */
/* rows [off[g], off[g+1])) is quantised once with its own s_g, as for the shared list; e_k of  */
/* group g sums only that group's rows, t ascending; each group keeps its own Kp channels.      */
/* sel: [G x Kp]; err_out (nullable): [G x K].                                                  */
void orc_calibrate_grouped(const uint16_t* x, int64_t T, int64_t K, const int64_t* off, int32_t G, int32_t Kp,
                           int32_t* sel, double* err_out) {
  float* resid = calib_residuals(x, T, K);
  double* err = (double*)malloc(sizeof(double) * (size_t)K);
  for (int32_t g = 0; g < G; ++g) {
    calib_errors(resid, off[g], off[g + 1], K, err);
    calib_select(err, K, Kp, sel + (int64_t)g * Kp);
    if (err_out) memcpy(err_out + (int64_t)g * K, err, sizeof(double) * (size_t)K);
  }
  free(err);
  free(resid);
}

/* ------------------------------------------------------------------------------------------ */
/* SwiGLU of the MoE expert (gate rows first, then up rows): h = bf16(silu(g) * u), computed  */
/* in binary64 from the bf16 gate_up output; silu(g) = g / (1 + exp(-g)).                     */
/* gu: bf16 [rows x 2I]; h: bf16 [rows x I]; h_exact (nullable): the unrounded binary64 value. */
/* ------------------------------------------------------------------------------------------ */
void orc_swiglu(const uint16_t* gu, int64_t rows, int64_t I, uint16_t* h, double* h_exact) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t j = 0; j < I; ++j) {
      double g = (double)orc_bf16_to_f32(gu[r * 2 * I + j]);
      double u = (double)orc_bf16_to_f32(gu[r * 2 * I + I + j]);
      double v = g / (1.0 + exp(-g)) * u;
      h[r * I + j] = orc_f64_to_bf16(v);
      if (h_exact) h_exact[r * I + j] = v;
    }
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* array forms of the element and scale encoders (used by the codec sweeps in the tests) */
void orc_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)orc_e2m1_encode(v[i]);
}

void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)orc_e4m3_encode(v[i]);
}

void orc_f64_to_bf16_array(const double* v, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_f64_to_bf16(v[i]);
}

/* ------------------------------------------------------------------------------------------ */
/* The MoE block around the expert GEMMs: routing, dispatch layout, combine.                  */
/* The pages fix none of this; the readings are:                                              */
/*  - routing: the top-k of softmax(logits) are the top-k logits (softmax is monotone), ties   */
/*    to the lower expert index; the combine weight of a chosen expert is its probability     */
/*    renormalised over the k chosen, w_j = exp(l_j - l_max) / sum_i exp(l_i - l_max),        */
/*    evaluated in binary64 and stored as binary32;                                            */
/*  - dispatch: (token, expert) pairs grouped by expert, tokens ascending inside an expert;    */
/*    expert e's segment starts at offsets[e] and is padded to a multiple of `pad` rows;       */
/*  - combine: out[t] = sum_j w_tj * y[row(t, j)] in binary64 over the expert outputs.         */
/* ------------------------------------------------------------------------------------------ */
void orc_route_topk(const float* logits, int64_t T, int32_t E, int32_t k, int32_t* ids, float* w) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * E;
    unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
    double* p = (double*)malloc(sizeof(double) * (size_t)k);
    for (int32_t j = 0; j < k; ++j) {
      int32_t best = -1;
      for (int32_t e = 0; e < E; ++e) /* strictly greater: the lower index keeps a tie */
        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
      taken[best] = 1;
      ids[t * k + j] = best;
    }
    const double lmax = (double)l[ids[t * k]];
    double s = 0.0;
    for (int32_t j = 0; j < k; ++j) {
      p[j] = exp((double)l[ids[t * k + j]] - lmax);
      s += p[j];
    }
    for (int32_t j = 0; j < k; ++j) w[t * k + j] = (float)(p[j] / s);
    free(p);
    free(taken);
  }
}

/* offsets [E+1] (padded segment starts), row_of [T*k] (row of pair (t, j)) */
void orc_dispatch_plan(const int32_t* ids, int64_t T, int32_t k, int32_t E, int32_t pad, int64_t* offsets,
                       int64_t* row_of) {
  int64_t* count = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  for (int64_t i = 0; i < T * k; ++i) count[ids[i]] += 1;
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + (count[e] + pad - 1) / pad * pad;
  memset(count, 0, sizeof(int64_t) * (size_t)E);
  for (int64_t t = 0; t < T; ++t) /* tokens in increasing order fill each segment */
    for (int32_t j = 0; j < k; ++j) {
      const int32_t e = ids[t * k + j];
      row_of[t * k + j] = offsets[e] + count[e];
      count[e] += 1;
    }
  free(count);
}

/* y: bf16 [.. x ldy]; out: binary64 [T x H] */
void orc_combine(const uint16_t* y, int64_t ldy, const int64_t* row_of, const float* w, int64_t T, int32_t k,
                 int64_t H, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int64_t h = 0; h < H; ++h) {
      double s = 0.0;
      for (int32_t j = 0; j < k; ++j)
        s += (double)w[t * k + j] * (double)orc_bf16_to_f32(y[row_of[t * k + j] * ldy + h]);
      out[t * H + h] = s;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* FP8 comparison format (the pages set their FP4 path against FP8 without fixing an FP8       */
/* recipe; reading): E4M3 elements with one power-of-two scale 2^X per 32 consecutive elements */
/* along K (stored as the E8M0 code X + 127), no tensor scale.  X is the smallest integer with */
/* 448 * 2^X >= b, b = max|x| of the block, clamped to [-127, 127] (b = 0 gives X = -127), so  */
/* no element saturates.  q = E4M3_RNE_satfinite(RN(x * 2^-X)) with the sign kept; the value  */
/* of a code pair is val(q) * 2^X.                                                             */
/* ------------------------------------------------------------------------------------------ */
int orc_mx8_exponent(float b) {
  int X = -127;
  while (X < 127 && ldexp(448.0, X) < (double)b) ++X;
  return X;
}

/* signed E4M3: sign bit 0x80 from the sign of v (so -0 gives 0x80), magnitude by orc_e4m3_encode */
int orc_e4m3_encode_signed(float v) {
  int c = orc_e4m3_encode(fabsf(v));
  return signbit(v) ? (c | 0x80) : c;
}

double orc_e4m3_decode_signed(int code) {
  double m = orc_e4m3_decode(code & 0x7F);
  return (code & 0x80) ? -m : m;
}

/* x: bf16 [rows x K] (pitch ldx), K % 32 == 0 -> codes u8 [rows x K], S (E8M0) u8 [rows x K/32] */
void orc_mx8_quantize(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* S) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < K / 32; ++b) {
      float t[32], m = 0.0f;
      for (int i = 0; i < 32; ++i) {
        t[i] = orc_bf16_to_f32(x[r * ldx + b * 32 + i]);
        if (fabsf(t[i]) > m) m = fabsf(t[i]);
      }
      const int X = orc_mx8_exponent(m);
      const float inv = (float)ldexp(1.0, -X); /* exact: 2^-X is a normal binary32 number */
      S[r * (K / 32) + b] = (uint8_t)(X + 127);
      for (int i = 0; i < 32; ++i) codes[r * K + b * 32 + i] = (uint8_t)orc_e4m3_encode_signed(t[i] * inv);
    }
}

/* y[m, n] = sum over 32-blocks of (sum_i qa_i qw_i) 2^(Xa + Xw): each block's sum is exact in    */
/* int64 (values times 2^9 are integers below 2^18), scaled by a power of two and added in     */
/* binary64 in block order.  absdot = sum |a_k w_k| (for the tolerance).  [rows x K] x [N x K]. */
void orc_mx8_gemm(const uint8_t* ac, const uint8_t* aS, const uint8_t* wc, const uint8_t* wS, int64_t rows,
                  int64_t N, int64_t K, double* y, double* absdot) {
  int64_t* qa = (int64_t*)malloc(sizeof(int64_t) * (size_t)(rows * K));
  int64_t* qw = (int64_t*)malloc(sizeof(int64_t) * (size_t)(N * K));
  for (int64_t i = 0; i < rows * K; ++i) qa[i] = (int64_t)ldexp(orc_e4m3_decode_signed(ac[i]), 9);
  for (int64_t i = 0; i < N * K; ++i) qw[i] = (int64_t)ldexp(orc_e4m3_decode_signed(wc[i]), 9);
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < rows; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double s = 0.0, sa = 0.0;
      for (int64_t b = 0; b < K / 32; ++b) {
        int64_t acc = 0, aacc = 0;
        for (int64_t i = b * 32; i < b * 32 + 32; ++i) {
          const int64_t p = qa[m * K + i] * qw[n * K + i];
          acc += p;
          aacc += p < 0 ? -p : p;
        }
        const int e = (int)aS[m * (K / 32) + b] + (int)wS[n * (K / 32) + b] - 254 - 18;
        s += ldexp((double)acc, e);
        sa += ldexp((double)aacc, e);
      }
      y[m * N + n] = s;
      absdot[m * N + n] = sa;
    }
  free(qa);
  free(qw);
}
