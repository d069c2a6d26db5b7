/*
 * sage_oracle.c -- plain, slow CPU oracle for the SageAttention-family
 * quantized attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The CUDA
 * product path never calls it, links it, or shares a line of code with it.
 *
 * What it follows (all on the pages about SageAttention2 / SageAttention2++ /
 * SageAttention3):
 *   - SageAttention2 Technical Report, abstract: smooth the inputs, quantize
 *     (Q,K) at a warp-level granularity and (P~,V) to FP8.
 *   - SageAttention2++ summary, Sec. 2.1: Q, K and P~ carry per-block scale
 *     factors, V a per-channel scale; the quantized products are rescaled.
 *   - SageAttention2++ summary, Sec. 2 ("FlashAttention-based quantization
 *     method"): the attention is computed tile by tile with an online softmax.
 *   - SageAttention2++ summary, Sec. 3.1: P and V quantization ranges are
 *     narrowed so that an FP16 accumulator cannot overflow; the chosen pair is
 *     Pr = 224, Vr = 4.5.
 *   - SageAttention2++ summary, Sec. 3.2: two consecutive MMA results are
 *     accumulated in FP16 before the FP32 conversion.
 *   - SageAttention3 abstract: microscaling FP4 attention (NVFP4 mode).
 * Where the pages are silent the readings are written next to each function.
 *
 * Arithmetic: IEEE binary32 round-to-nearest-even, one rounding per written
 * operation (compiled with -ffp-contract=off, no fast-math; an FMA only where
 * fmaf is written).  The pages fix the formats of the quantized operands (INT8,
 * FP8, FP4, the FP16 accumulator) but no precision for the statistics and the
 * softmax; those steps are taken in fp32, the precision in which every
 * quantized code is decided, in the order the method states them.  Sums the
 * pages leave unspecified are exact (double holds them exactly, see each
 * comment).
 *
 * Layouts (all row-major, contiguous):
 *   x        [BH, N, d]        input (already converted to float)
 *   codes    [BH, Npad, d]     int8 Q/K codes, pad rows 0
 *   vt       [BH, d, Npad]     e4m3 V codes, transposed, pad columns 0
 *   scales   [BH, Npad/G]      fp32, G = granule (Q 32, K 64)
 *   stats    [BH, d]           fp32 means / absmax
 *   bias     [BH, Npad]        fp32, pad 0
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_EXPORT __attribute__((visibility("default")))

/* Number of host threads the parallel loops below use. */
ORC_EXPORT int orc_num_threads(void)
{
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Set the number of host threads of the parallel loops (1: single-threaded
 * timing). */
ORC_EXPORT void orc_set_num_threads(int n)
{
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* Small-float formats.                                                      */
/* ------------------------------------------------------------------------ */

/* FP8 E4M3 ("fn" variant: no infinities, 0x7F/0xFF are NaN, max 448).
 * Magnitude code c = eeee mmm: exponent field 0 is subnormal m * 2^-9,
 * otherwise (8 + m) * 2^(e - 10).  Used for V and P~ (SageAttention2 abstract,
 * SageAttention2++ Sec. 2.1). */
ORC_EXPORT double orc_e4m3_decode(int code)
{
  int sign = (code >> 7) & 1;
  int e = (code >> 3) & 0xF, m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);
  else v = ldexp((double)(8 + m), e - 10);
  return sign ? -v : v;
}

/* Table of the 127 finite non-negative magnitudes, ascending with the code. */
static double g_e4m3_mag[127];
/* e2m1 magnitudes (FP4, SageAttention3 abstract: microscaling FP4). */
static const double g_e2m1_mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
static int g_tables_ready = 0;

static void init_tables(void)
{
  if (g_tables_ready) return;
  for (int c = 0; c < 127; ++c) g_e4m3_mag[c] = orc_e4m3_decode(c);
  g_tables_ready = 1;
}

/* Nearest entry of an ascending table of magnitudes; ties go to the even
 * code; values beyond the last entry saturate to it. */
static int nearest_code(const double* tab, int n, double a)
{
  if (!(a > 0.0)) return 0;
  if (a >= tab[n - 1]) return n - 1;
  int lo = 0, hi = n - 1;            /* invariant: tab[lo] <= a < tab[hi] */
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (tab[mid] <= a) lo = mid; else hi = mid;
  }
  double dlo = a - tab[lo], dhi = tab[hi] - a;
  if (dlo < dhi) return lo;
  if (dhi < dlo) return hi;
  return (lo % 2 == 0) ? lo : hi;
}

/* e4m3 encode, round to nearest even, saturate to +-448 (satfinite).
 * The sign bit is kept for negative inputs, so -0 and tiny negatives give 0x80. */
ORC_EXPORT int orc_e4m3_encode(double x)
{
  init_tables();
  if (isnan(x)) return 0x7F;
  int sign = signbit(x) ? 0x80 : 0;
  return sign | nearest_code(g_e4m3_mag, 127, fabs(x));
}

/* ue4m3: unsigned e4m3, the block-scale format of the NVFP4 mode. */
ORC_EXPORT int orc_ue4m3_encode(double x)
{
  init_tables();
  if (!(x > 0.0)) return 0;
  return nearest_code(g_e4m3_mag, 127, x);
}
ORC_EXPORT double orc_ue4m3_decode(int code) { return orc_e4m3_decode(code & 0x7F); }

/* e2m1 (FP4) encode: nearest of {0,.5,1,1.5,2,3,4,6}, ties to even code,
 * saturating; sign in bit 3. */
ORC_EXPORT int orc_e2m1_encode(double x)
{
  int sign = signbit(x) ? 8 : 0;
  return sign | nearest_code(g_e2m1_mag, 8, fabs(x));
}
ORC_EXPORT double orc_e2m1_decode(int code)
{
  double v = g_e2m1_mag[code & 7];
  return (code & 8) ? -v : v;
}

/* Round to IEEE binary16, nearest even; overflow gives +-inf (no saturation:
 * the point of the narrowed ranges of SageAttention2++ Sec. 3.1 is that this
 * never happens).  Used to emulate the FP16 accumulator. */
ORC_EXPORT double orc_f16_round(double x)
{
  if (x == 0.0 || isnan(x) || isinf(x)) return x;
  double a = fabs(x);
  int e;
  frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) */
  int exp2 = e - 1;             /* a in [2^exp2, 2^(exp2+1)) */
  if (exp2 < -14) exp2 = -14;   /* subnormal spacing 2^-24 */
  double ulp = ldexp(1.0, exp2 - 10);
  double r = nearbyint(a / ulp) * ulp;   /* default rounding mode: nearest even */
  if (r > 65504.0) r = INFINITY;
  return x < 0 ? -r : r;
}

/* exp2 of the softmax: the library exp2 in double, rounded once to fp32
 * (the pages fix no accuracy for the exponential).  -inf gives +0. */
ORC_EXPORT float orc_exp2(float d)
{
  return (float)exp2((double)d);
}

/* ------------------------------------------------------------------------ */
/* Smoothing statistics (SageAttention2 abstract: smoothing; the mean is over */
/* tokens, per channel).                                                      */
/* ------------------------------------------------------------------------ */

/* Mean over tokens of one channel, in a fixed fp32 order: per 64-token chunk
 * a sequential sum from 0, then the chunk sums added sequentially, then one
 * IEEE division by N.  (The pages do not fix an order; the chunk of 64 is the
 * K granule.) */
ORC_EXPORT void orc_channel_mean(const float* x, int BH, int N, int d, float* mean)
{
  for (int bh = 0; bh < BH; ++bh) {
    const float* xb = x + (size_t)bh * N * d;
    for (int c = 0; c < d; ++c) {
      float total = 0.0f;
      for (int t0 = 0; t0 < N; t0 += 64) {
        float s = 0.0f;
        int t1 = t0 + 64 < N ? t0 + 64 : N;
        for (int t = t0; t < t1; ++t) s = s + xb[(size_t)t * d + c];
        total = total + s;
      }
      mean[(size_t)bh * d + c] = total / (float)N;
    }
  }
}

/* Per-channel max |x| over tokens (exact, order-free). */
ORC_EXPORT void orc_channel_absmax(const float* x, int BH, int N, int d, float* amax)
{
  for (int bh = 0; bh < BH; ++bh)
    for (int c = 0; c < d; ++c) {
      float a = 0.0f;
      for (int t = 0; t < N; ++t) {
        float v = fabsf(x[((size_t)bh * N + t) * d + c]);
        if (v > a) a = v;
      }
      amax[(size_t)bh * d + c] = a;
    }
}

/* ------------------------------------------------------------------------ */
/* INT8 quantization of Q and K (SageAttention2++ Sec. 2.1: per-block scale   */
/* factors; granules read as Q 32 tokens, K 64 tokens).                      */
/* ------------------------------------------------------------------------ */

/* x~ = x - mean (mean may be NULL: no smoothing).  Per granule of G tokens
 * (valid tokens only): a = max|x~|; a == 0 gives scale 0 and codes 0; else
 * inv = 127/a, scale = a/127, code = clamp(rint_even(x~ * inv), -127, 127).
 * Pad rows (t >= N) get code 0; fully padded granules get scale 0. */
ORC_EXPORT void orc_quant_int8(const float* x, const float* mean, int BH, int N, int Npad,
                               int d, int G, int8_t* codes, float* scale)
{
  float* xs = (float*)malloc(sizeof(float) * (size_t)G * d);
  for (int bh = 0; bh < BH; ++bh) {
    for (int g0 = 0; g0 < Npad; g0 += G) {
      float a = 0.0f;
      int nv = 0;
      for (int t = g0; t < g0 + G; ++t) {
        if (t >= N) break;
        ++nv;
        for (int c = 0; c < d; ++c) {
          float v = x[((size_t)bh * N + t) * d + c];
          if (mean) v = v - mean[(size_t)bh * d + c];
          xs[(size_t)(t - g0) * d + c] = v;
          if (fabsf(v) > a) a = fabsf(v);
        }
      }
      float inv = 0.0f, sc = 0.0f;
      if (a > 0.0f) { inv = 127.0f / a; sc = a / 127.0f; }
      scale[(size_t)bh * (Npad / G) + g0 / G] = sc;
      for (int t = g0; t < g0 + G; ++t) {
        int8_t* row = codes + ((size_t)bh * Npad + t) * d;
        for (int c = 0; c < d; ++c) {
          int q = 0;
          if (t - g0 < nv && a > 0.0f) {
            float y = xs[(size_t)(t - g0) * d + c] * inv;
            float r = nearbyintf(y);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            q = (int)r;
          }
          row[c] = (int8_t)q;
        }
      }
    }
  }
  free(xs);
}

/* Q-smoothing bias: bias[n] = sum_c mean_q[c] * k~[n,c], an fmaf chain over c
 * from 0 in channel order, on the unquantized fp32 k~ = k - mean_k.  Adding
 * it back to the logits undoes the subtraction of mean_q from Q up to a
 * per-row constant (the q_i . mean_k term), which softmax ignores. */
ORC_EXPORT void orc_q_bias(const float* k, const float* mean_k, const float* mean_q,
                           int BH, int N, int Npad, int d, float* bias)
{
  for (int bh = 0; bh < BH; ++bh)
    for (int t = 0; t < Npad; ++t) {
      float acc = 0.0f;
      if (t < N)
        for (int c = 0; c < d; ++c) {
          float kt = k[((size_t)bh * N + t) * d + c] - mean_k[(size_t)bh * d + c];
          acc = fmaf(mean_q[(size_t)bh * d + c], kt, acc);
        }
      bias[(size_t)bh * Npad + t] = acc;
    }
}

/* ------------------------------------------------------------------------ */
/* FP8 quantization of V, per channel (SageAttention2++ Sec. 2.1; range Vr of */
/* Sec. 3.1: 4.5 for the FP16-accumulator mode, the full 448 otherwise).      */
/* ------------------------------------------------------------------------ */

/* scale_v[c] = a_c / Vr, code = e4m3(v * (Vr / a_c)); a_c == 0 gives scale 0
 * and codes 0.  Codes are stored transposed, vt[c][t], pad columns 0. */
ORC_EXPORT void orc_quant_v_fp8(const float* v, const float* amax, int BH, int N, int Npad,
                                int d, float Vr, uint8_t* vt, float* scale_v)
{
  for (int bh = 0; bh < BH; ++bh)
    for (int c = 0; c < d; ++c) {
      float a = amax[(size_t)bh * d + c];
      float mul = 0.0f;
      scale_v[(size_t)bh * d + c] = 0.0f;
      if (a > 0.0f) { mul = Vr / a; scale_v[(size_t)bh * d + c] = a / Vr; }
      uint8_t* row = vt + ((size_t)bh * d + c) * Npad;
      for (int t = 0; t < Npad; ++t) {
        int code = 0;
        if (t < N && a > 0.0f) {
          float y = v[((size_t)bh * N + t) * d + c] * mul;
          code = orc_e4m3_encode((double)y);
        }
        row[t] = (uint8_t)code;
      }
    }
}

/* ------------------------------------------------------------------------ */
/* Exact integer QK^T (the INT8 Matmul of SageAttention2).                    */
/* ------------------------------------------------------------------------ */

/* s[i][j] = sum_c q[i][c] * k[j][c] in int32 (|s| <= d * 127^2 < 2^21). */
ORC_EXPORT void orc_qk_s32(const int8_t* q, const int8_t* k, int nq, int nk, int d, int32_t* s)
{
  for (int i = 0; i < nq; ++i)
    for (int j = 0; j < nk; ++j) {
      int32_t acc = 0;
      for (int c = 0; c < d; ++c) acc += (int32_t)q[(size_t)i * d + c] * (int32_t)k[(size_t)j * d + c];
      s[(size_t)i * nk + j] = acc;
    }
}

/* ------------------------------------------------------------------------ */
/* Tiled attention with online softmax, INT8 QK / FP8 PV                      */
/* (SageAttention2 abstract and SageAttention2++ Sec. 2-3).                   */
/* ------------------------------------------------------------------------ */

enum { ORC_MODE_FP32ACC = 0, ORC_MODE_F16ACC = 1 };

/* Distance from e4m3 magnitude code cm to its farther neighbour: the most a
 * P~ value moves when its code lands one step away. */
static double e4m3_step(int cm)
{
  double v = g_e4m3_mag[cm];
  double up = cm < 126 ? g_e4m3_mag[cm + 1] - v : 0.0;
  double dn = cm > 0 ? v - g_e4m3_mag[cm - 1] : 0.0;
  return up > dn ? up : dn;
}

/* One query row, FlashAttention order: key tiles of 128 in ascending order.
 * Per tile (only tiles holding at least one key the row may see), in fp32:
 *   t_j   = ((float(S_ij) * (sq_i * sk_g(j))) + bias_j) * (log2(e) / sqrt(d))
 *           (the dequantized score plus the Q-smoothing bias, in base-2 units;
 *           without Q smoothing there is no bias term)
 *   m_new = max(m, max_j t_j);  alpha = exp2(m - m_new)
 *   p_j   = exp2(t_j - m_new)                  (p <= 1)
 *   l     = alpha * l + sum_j p_j              (sequential fp32 sum)
 *   P~_j  = e4m3(p_j * Pr)                     (static P~ scale 1/Pr)
 *   FP32 accumulator: acc_c = alpha * acc_c + fl32(exact sum_j P~_j v^_jc)
 *   FP16 accumulator (SageAttention2++ Sec. 3.2): per 64-key chunk,
 *        h = f16(exact sum of its first 32 products), h = f16(h + exact sum of
 *        the next 32); acc_c = (alpha * acc_c + h_chunk0) + h_chunk1.  With
 *        chunk = 32 (the accuracy sweep's other depth: no delayed buffering)
 *        each 32-key sum is rounded to f16 and added to the fp32 value alone.
 *   O_ic  = acc_c * scale_v[c] / (Pr * l)
 * exp2 is orc_exp2 above.  Masked keys (j >= N, or j > i when causal) take no
 * part.  The exact sums of e4m3 products fit a double: each product has 8
 * significant bits within 2^-18..2^18 and at most 128 are added.
 * out_row receives fp32 results (the caller rounds to the output dtype).
 * flip_row (may be NULL) receives, per channel, the largest change of O_ic
 * that moving one P~ code of the row to a neighbouring code would cause:
 * max over keys of step(P~_j) * |v^_jc| carried through the later rescales,
 * times scale_v[c] / (Pr * l).  It is a sensitivity figure for comparisons
 * with implementations whose exponential differs in the last bits. */
static void attn_row(int i, const int8_t* qc, const int8_t* kc, const uint8_t* vt,
                     float sq, const float* sk, const float* bias, const float* scale_v,
                     int N, int Npad, int d, int causal, int koff, int mode, int chunk, float Pr,
                     float* acc, double* fl, float* tvals, int* pcode, float* out_row,
                     float* flip_row)
{
  const float c_log2 = (float)(1.4426950408889634 / sqrt((double)d));
  float m = -INFINITY, l = 0.0f;
  for (int c = 0; c < d; ++c) { acc[c] = 0.0f; fl[c] = 0.0; }
  /* last visible key: all N keys, or (causal) keys j <= i + koff */
  int jmax = causal ? (i + koff < N - 1 ? i + koff : N - 1) : N - 1;
  for (int j0 = 0; j0 <= jmax; j0 += 128) {
    float mt = -INFINITY;
    for (int j = j0; j < j0 + 128; ++j) {
      if (j > jmax) { tvals[j - j0] = -INFINITY; continue; }
      int32_t s = 0;
      for (int c = 0; c < d; ++c) s += (int32_t)qc[(size_t)i * d + c] * (int32_t)kc[(size_t)j * d + c];
      float deq = (float)s * (sq * sk[j / 64]);
      if (bias) deq = deq + bias[j];
      const float t = deq * c_log2;
      tvals[j - j0] = t;
      if (t > mt) mt = t;
    }
    const float m_new = m > mt ? m : mt;
    const float alpha = orc_exp2(m - m_new);   /* first tile: exp2(-inf) = 0 */
    float ps = 0.0f;
    for (int j = 0; j < 128; ++j) {
      float p = 0.0f;
      if (j0 + j <= jmax) p = orc_exp2(tvals[j] - m_new);
      ps = ps + p;
      pcode[j] = (j0 + j <= jmax) ? orc_e4m3_encode((double)(p * Pr)) : -1;
    }
    l = alpha * l + ps;
    for (int c = 0; c < d; ++c) {
      const uint8_t* vrow = vt + (size_t)c * Npad + j0;
      double fmx = fl[c] * alpha;
      for (int j = 0; j < 128; ++j) {
        if (pcode[j] < 0) continue;
        double e = e4m3_step(pcode[j] & 0x7F) * fabs(orc_e4m3_decode(vrow[j]));
        if (e > fmx) fmx = e;
      }
      fl[c] = fmx;
      if (mode == ORC_MODE_FP32ACC) {
        double sum = 0.0;
        for (int j = 0; j < 128; ++j)
          if (pcode[j] >= 0) sum += orc_e4m3_decode(pcode[j]) * orc_e4m3_decode(vrow[j]);
        acc[c] = alpha * acc[c] + (float)sum;
      } else {
        float a = alpha * acc[c];
        for (int ch = 0; ch < 128; ch += chunk) {
          double s0 = 0.0, s1 = 0.0;
          for (int j = ch; j < ch + 32; ++j)
            if (pcode[j] >= 0) s0 += orc_e4m3_decode(pcode[j]) * orc_e4m3_decode(vrow[j]);
          for (int j = ch + 32; j < ch + chunk; ++j)
            if (pcode[j] >= 0) s1 += orc_e4m3_decode(pcode[j]) * orc_e4m3_decode(vrow[j]);
          double h = orc_f16_round(s0);
          if (chunk == 64) h = orc_f16_round(h + s1);
          a = a + (float)h;
        }
        acc[c] = a;
      }
    }
    m = m_new;
  }
  const float den = Pr * l;
  for (int c = 0; c < d; ++c) {
    out_row[c] = acc[c] * scale_v[c] / den;
    if (flip_row) flip_row[c] = (float)(fl[c] * scale_v[c] / den);
  }
}

/* Attention with grouped key/value heads and separate query and key lengths.
 * Query head hq of batch b reads key/value head hq / G, G = Hq / Hkv (G = 1:
 * every head its own; Hkv = 1: one shared head).  Nq query rows, Nk keys;
 * a causal mask lets row i see keys j <= i + (Nk - Nq) (the last query row
 * sees every key; Nq == Nk is the usual j <= i).  Layouts:
 *   qc [B*Hq, Npq, d], sq [B*Hq, Npq/32], bias [B*Hq, Npk] (or NULL)
 *   kc [B*Hkv, Npk, d], sk [B*Hkv, Npk/64], vt [B*Hkv, d, Npk], scale_v [B*Hkv, d]
 * rows == NULL means all Nq rows.  out, flip: [B*Hq, nrows, d] (flip may be
 * NULL).  chunk: keys per FP16 partial in the FP16-accumulator mode. */
ORC_EXPORT void orc_attn_int8_fp8_gqa(const int8_t* qc, const float* sq, const int8_t* kc,
                                      const float* sk, const uint8_t* vt, const float* scale_v,
                                      const float* bias, int B, int Hq, int Hkv, int Nq, int Nk,
                                      int Npq, int Npk, int d, int causal, int mode, int chunk,
                                      float Pr, const int* rows, int nrows, float* out, float* flip)
{
  if (chunk != 32) chunk = 64;
  init_tables();
  const int BH = B * Hq, G = Hq / Hkv, koff = Nk - Nq;
#pragma omp parallel
  {
    float* acc = (float*)malloc(sizeof(float) * d);
    double* fl = (double*)malloc(sizeof(double) * d);
    float* tv = (float*)malloc(sizeof(float) * 128);
    int* pc = (int*)malloc(sizeof(int) * 128);
#pragma omp for schedule(dynamic, 4) collapse(2)
    for (int bh = 0; bh < BH; ++bh)
      for (int r = 0; r < nrows; ++r) {
        int i = rows ? rows[r] : r;
        const int bkv = (bh / Hq) * Hkv + (bh % Hq) / G;
        const size_t o = ((size_t)bh * nrows + r) * d;
        attn_row(i, qc + (size_t)bh * Npq * d, kc + (size_t)bkv * Npk * d,
                 vt + (size_t)bkv * d * Npk, sq[(size_t)bh * (Npq / 32) + i / 32],
                 sk + (size_t)bkv * (Npk / 64), bias ? bias + (size_t)bh * Npk : NULL,
                 scale_v + (size_t)bkv * d, Nk, Npk, d, causal, koff, mode, chunk, Pr, acc, fl, tv,
                 pc, out + o, flip ? flip + o : NULL);
      }
    free(acc); free(fl); free(tv); free(pc);
  }
}

/* Attention output for the listed query rows of every (b,h) slice.
 * rows == NULL means all N rows (then nrows must be N).  out: [BH, nrows, d].
 * chunk: keys per FP16 partial in the FP16-accumulator mode (64, or 32).
 * flip (may be NULL): [BH, nrows, d] single-code sensitivity (see attn_row). */
ORC_EXPORT void orc_attn_int8_fp8(const int8_t* qc, const float* sq, const int8_t* kc,
                                  const float* sk, const uint8_t* vt, const float* scale_v,
                                  const float* bias, int BH, int N, int Npad, int d,
                                  int causal, int mode, int chunk, float Pr, const int* rows,
                                  int nrows, float* out, float* flip)
{
  if (chunk != 32) chunk = 64;
  init_tables();
#pragma omp parallel
  {
    float* acc = (float*)malloc(sizeof(float) * d);
    double* fl = (double*)malloc(sizeof(double) * d);
    float* tv = (float*)malloc(sizeof(float) * 128);
    int* pc = (int*)malloc(sizeof(int) * 128);
#pragma omp for schedule(dynamic, 4) collapse(2)
    for (int bh = 0; bh < BH; ++bh)
      for (int r = 0; r < nrows; ++r) {
        int i = rows ? rows[r] : r;
        const size_t o = ((size_t)bh * nrows + r) * d;
        attn_row(i, qc + (size_t)bh * Npad * d, kc + (size_t)bh * Npad * d,
                 vt + (size_t)bh * d * Npad, sq[(size_t)bh * (Npad / 32) + i / 32],
                 sk + (size_t)bh * (Npad / 64), bias ? bias + (size_t)bh * Npad : NULL,
                 scale_v + (size_t)bh * d, N, Npad, d, causal, 0, mode, chunk, Pr, acc, fl, tv, pc,
                 out + o, flip ? flip + o : NULL);
      }
    free(acc); free(fl); free(tv); free(pc);
  }
}

/* ------------------------------------------------------------------------ */
/* NVFP4 mode (SageAttention3 abstract: microscaling FP4 attention).          */
/* Two-level scaling: an fp32 global scale per (b,h) slice and a ue4m3 scale  */
/* per block of 16 values along the contraction axis of each matmul.         */
/* ------------------------------------------------------------------------ */

/* One block of 16 values x[0..15] (stride st) with global scale g:
 * bs = ue4m3(a_blk / (6 g)); each value is scaled by the reciprocal of the
 * block's decode factor, r = 1 / (g * dec(bs)) rounded once, and encoded:
 * code = e2m1(x * r).  dec(bs) == 0 gives codes 0.  Codes go to out[k] (one
 * per byte, unpacked). */
static int fp4_block(const float* x, int st, float g, uint8_t* out)
{
  float a = 0.0f;
  for (int k = 0; k < 16; ++k) if (fabsf(x[k * st]) > a) a = fabsf(x[k * st]);
  int bs = 0;
  if (g > 0.0f) bs = orc_ue4m3_encode((double)(a / (6.0f * g)));
  float sd = (float)orc_ue4m3_decode(bs);
  float den = g * sd;
  float r = (sd > 0.0f) ? 1.0f / den : 0.0f;
  for (int k = 0; k < 16; ++k)
    out[k] = (uint8_t)((sd > 0.0f) ? orc_e2m1_encode((double)(x[k * st] * r)) : 0);
  return bs;
}

/* The block quantizer above for one block of 16 contiguous values: returns
 * the ue4m3 scale code, writes the 16 e2m1 codes (one per byte). */
ORC_EXPORT int orc_nvfp4_block(const float* x, float g, uint8_t* codes)
{
  init_tables();
  return fp4_block(x, 1, g, codes);
}

/* Q or K in NVFP4: x~ = x - mean (mean may be NULL); g = A / (6 * 448) with A
 * the slice's max |x~| over valid tokens; blocks of 16 along d.
 * codes: [BH, Npad, d] unpacked e2m1 codes (one per byte), pad rows 0;
 * bscale: [BH, Npad, d/16] ue4m3; gscale: [BH]. */
ORC_EXPORT void orc_quant_nvfp4_rows(const float* x, const float* mean, int BH, int N, int Npad,
                                     int d, uint8_t* codes, uint8_t* bscale, float* gscale)
{
  float* row = (float*)malloc(sizeof(float) * d);
  for (int bh = 0; bh < BH; ++bh) {
    float A = 0.0f;
    for (int t = 0; t < N; ++t)
      for (int c = 0; c < d; ++c) {
        float v = x[((size_t)bh * N + t) * d + c];
        if (mean) v = v - mean[(size_t)bh * d + c];
        if (fabsf(v) > A) A = fabsf(v);
      }
    float g = A / (6.0f * 448.0f);
    gscale[bh] = g;
    for (int t = 0; t < Npad; ++t) {
      uint8_t* cr = codes + ((size_t)bh * Npad + t) * d;
      uint8_t* br = bscale + ((size_t)bh * Npad + t) * (d / 16);
      if (t >= N) { memset(cr, 0, d); memset(br, 0, d / 16); continue; }
      for (int c = 0; c < d; ++c) {
        float v = x[((size_t)bh * N + t) * d + c];
        if (mean) v = v - mean[(size_t)bh * d + c];
        row[c] = v;
      }
      for (int b = 0; b < d / 16; ++b) br[b] = (uint8_t)fp4_block(row + b * 16, 1, g, cr + b * 16);
    }
  }
  free(row);
}

/* V in NVFP4, transposed: blocks of 16 tokens per channel (the contraction
 * axis of PV).  g = A / (6 * 448), A = slice max |v|.
 * codes: [BH, d, Npad] unpacked; bscale: [BH, d, Npad/16]; gscale: [BH]. */
ORC_EXPORT void orc_quant_nvfp4_vt(const float* v, int BH, int N, int Npad, int d,
                                   uint8_t* codes, uint8_t* bscale, float* gscale)
{
  float col[16];
  for (int bh = 0; bh < BH; ++bh) {
    float A = 0.0f;
    for (size_t e = 0; e < (size_t)N * d; ++e) {
      float a = fabsf(v[(size_t)bh * N * d + e]);
      if (a > A) A = a;
    }
    float g = A / (6.0f * 448.0f);
    gscale[bh] = g;
    for (int c = 0; c < d; ++c)
      for (int t0 = 0; t0 < Npad; t0 += 16) {
        for (int k = 0; k < 16; ++k) {
          int t = t0 + k;
          col[k] = (t < N) ? v[((size_t)bh * N + t) * d + c] : 0.0f;
        }
        bscale[((size_t)bh * d + c) * (Npad / 16) + t0 / 16] =
            (uint8_t)fp4_block(col, 1, g, codes + ((size_t)bh * d + c) * Npad + t0);
      }
  }
}

/* e2m1 step at magnitude code cm: distance to the farther neighbour. */
static double e2m1_step(int cm)
{
  double v = g_e2m1_mag[cm];
  double up = cm < 7 ? g_e2m1_mag[cm + 1] - v : 0.0;
  double dn = cm > 0 ? v - g_e2m1_mag[cm - 1] : 0.0;
  return up > dn ? up : dn;
}

/* NVFP4 attention for one row.  x_ij = sum_c dq_ic dk_jc where the
 * dequantized values are code * dec(block scale) (exact products, summed in
 * double, rounded once to fp32); then the steps of the INT8 mode with the
 * slice global scales in place of the per-granule scales:
 *   t_j = ((x_ij * (g_q * g_k)) + bias_j) * (log2(e) / sqrt(d)),
 *   m_new, alpha, p_j = exp2(t_j - m_new), l = alpha * l + sum_j p_j;
 * P~ in NVFP4 along keys: blocks of 16 keys, the block quantizer of Q/K/V
 * with the constant global scale g_p = 1 / (6 * 448) (p <= 1); PV summed
 * exactly per tile and added in fp32; O = acc * (g_p * g_v) / l.
 * flip_row (may be NULL): per channel, the largest change of O_ic that moving
 * every code of one P~ block by one e2m1 step, its scale by one ue4m3 step
 * (1/8), would cause -- the same sensitivity figure as in attn_row. */
static void attn_row_nvfp4(int i, const uint8_t* qc, const uint8_t* qs, float gq,
                           const uint8_t* kc, const uint8_t* ks, float gk,
                           const uint8_t* vc, const uint8_t* vs, float gv, const float* bias,
                           int N, int Npad, int d, int causal, double* qd, float* acc, double* fl,
                           float* tvals, float* pvals, uint8_t* pcodes, uint8_t* pbs,
                           float* out_row, float* flip_row)
{
  const float c_log2 = (float)(1.4426950408889634 / sqrt((double)d));
  const float gp = 1.0f / (6.0f * 448.0f);
  const float gqk = gq * gk;
  float m = -INFINITY, l = 0.0f;
  for (int c = 0; c < d; ++c) {
    acc[c] = 0.0f;
    fl[c] = 0.0;
    qd[c] = orc_e2m1_decode(qc[(size_t)i * d + c]) * orc_ue4m3_decode(qs[(size_t)i * (d / 16) + c / 16]);
  }
  int jmax = causal ? (i < N - 1 ? i : N - 1) : N - 1;
  for (int j0 = 0; j0 <= jmax; j0 += 128) {
    float mt = -INFINITY;
    for (int j = j0; j < j0 + 128; ++j) {
      if (j > jmax) { tvals[j - j0] = -INFINITY; continue; }
      double s = 0.0;
      for (int c = 0; c < d; ++c)
        s += qd[c] * orc_e2m1_decode(kc[(size_t)j * d + c]) * orc_ue4m3_decode(ks[(size_t)j * (d / 16) + c / 16]);
      float deq = (float)s * gqk;
      if (bias) deq = deq + bias[j];
      const float t = deq * c_log2;
      tvals[j - j0] = t;
      if (t > mt) mt = t;
    }
    const float m_new = m > mt ? m : mt;
    const float alpha = orc_exp2(m - m_new);
    float ps = 0.0f;
    for (int j = 0; j < 128; ++j) {
      float p = 0.0f;
      if (j0 + j <= jmax) p = orc_exp2(tvals[j] - m_new);
      pvals[j] = p;
      ps = ps + p;
    }
    l = alpha * l + ps;
    for (int b = 0; b < 8; ++b) pbs[b] = (uint8_t)fp4_block(pvals + b * 16, 1, gp, pcodes + b * 16);
    for (int c = 0; c < d; ++c) {
      double sum = 0.0, fmx = fl[c] * alpha;
      for (int b = 0; b < 8; ++b) {
        double fb = 0.0;
        for (int j = 16 * b; j < 16 * b + 16; ++j) {
          int t = j0 + j;
          if (t > jmax) continue;
          double vj = orc_e2m1_decode(vc[(size_t)c * Npad + t]) * orc_ue4m3_decode(vs[(size_t)c * (Npad / 16) + t / 16]);
          sum += orc_e2m1_decode(pcodes[j]) * orc_ue4m3_decode(pbs[b]) * vj;
          fb += (e2m1_step(pcodes[j] & 7) + 0.125 * orc_e2m1_decode(pcodes[j] & 7)) * orc_ue4m3_decode(pbs[b]) *
                fabs(vj);
        }
        if (fb > fmx) fmx = fb;
      }
      fl[c] = fmx;
      acc[c] = alpha * acc[c] + (float)sum;
    }
    m = m_new;
  }
  const float gpv = gp * gv;
  for (int c = 0; c < d; ++c) {
    out_row[c] = acc[c] * gpv / l;
    if (flip_row) flip_row[c] = (float)(fl[c] * gpv / l);
  }
}

ORC_EXPORT void orc_attn_nvfp4(const uint8_t* qc, const uint8_t* qs, const float* gq,
                               const uint8_t* kc, const uint8_t* ks, const float* gk,
                               const uint8_t* vc, const uint8_t* vs, const float* gv,
                               const float* bias, int BH, int N, int Npad, int d, int causal,
                               const int* rows, int nrows, float* out, float* flip)
{
  init_tables();
#pragma omp parallel
  {
    double* qd = (double*)malloc(sizeof(double) * d);
    float* acc = (float*)malloc(sizeof(float) * d);
    double* fl = (double*)malloc(sizeof(double) * d);
    float* tv = (float*)malloc(sizeof(float) * 128);
    float* pv = (float*)malloc(sizeof(float) * 128);
    uint8_t* pc = (uint8_t*)malloc(128);
    uint8_t pbs[8];
#pragma omp for schedule(dynamic, 4) collapse(2)
    for (int bh = 0; bh < BH; ++bh)
      for (int r = 0; r < nrows; ++r) {
        int i = rows ? rows[r] : r;
        const size_t o = ((size_t)bh * nrows + r) * d;
        attn_row_nvfp4(i, qc + (size_t)bh * Npad * d, qs + (size_t)bh * Npad * (d / 16), gq[bh],
                       kc + (size_t)bh * Npad * d, ks + (size_t)bh * Npad * (d / 16), gk[bh],
                       vc + (size_t)bh * d * Npad, vs + (size_t)bh * d * (Npad / 16), gv[bh],
                       bias ? bias + (size_t)bh * Npad : NULL, N, Npad, d, causal, qd, acc, fl, tv,
                       pv, pc, pbs, out + o, flip ? flip + o : NULL);
      }
    free(qd); free(acc); free(fl); free(tv); free(pv); free(pc);
  }
}
