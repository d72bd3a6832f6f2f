/*
 * mxref.c -- CPU oracle for MXAttention's MXFP4 forward attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * restatement of what the MXFP4 attention path computes.  It is used by the
 * tests, by the smoke check and by the bench's CPU-baseline leg, never by the
 * product path.  It shares no code, header, table or constant with the CUDA
 * library; the two only meet on seeded inputs.
 *
 * Sources (cited by page title and the paper's own section/figure numbers):
 *  - "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
 *    Quantization for MXFP4 Attention" (Pith review page, pith.science):
 *      axioms ledger: MXFP4 = 32-element blocks of E2M1 codes sharing one E8M0
 *        power-of-two scale, E2M1 grid {0,+-0.5,...,+-6}, round-to-nearest
 *        with saturation;
 *      Fig. 3: OCP floor rule maps the block maximum to [4,8), TFS (Qmax=6)
 *        to (3,6], UOS to (3.625,7.25];
 *      Fig. 1: fixed Hadamard rotation on Q/K; UOS applied to all
 *        MXFP4-quantized attention tensors;
 *      Fig. 4 and axioms (FlashAttention-2): online softmax with running max,
 *        row sum l and unnormalized accumulator; PNQ feeds one quantized
 *        exponential tile to both the l update and the output update, direct
 *        placement uses the unquantized tile for l;
 *      Fig. 9 / Eq. (96): ceiling form e_q = e_6 + ceil(log2(x_6 / q)).
 *  - 10100.com article on MXAttention: 32-element groups, E8M0 scale,
 *    OCP maps the block max to [4,8) and values above 7 round toward the
 *    unrepresentable 8 and saturate to 6; PNQ quantizes the unnormalized
 *    exponentials once and uses that one copy for the normalizer and output.
 *
 * Readings where the pages are silent are listed at each function.
 * Build: gcc -O2 -ffp-contract=off -fopenmp -fPIC -shared (float arithmetic is
 * IEEE single with one rounding per operation; no fused multiply-add).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define MXREF_RULE_UOS 0    /* ceiling rule, boundary q = 29/4            */
#define MXREF_RULE_QMAX6 1  /* ceiling rule, boundary q = 6 (TFS)         */
#define MXREF_RULE_OCP 2    /* OCP floor rule: floor(log2 amax) - 2       */
#define MXREF_RULE_CUSTOM 3 /* ceiling rule, caller's boundary q          */

/* Non-negative E2M1 magnitudes, indexed by the 3 low bits of a code
 * (2 exponent bits, 1 mantissa bit).  Index parity = mantissa bit. */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Value of a 4-bit E2M1 code (bit 3 = sign). */
double mxref_e2m1_decode(int code) {
  double m = kE2M1[code & 7];
  return (code & 8) ? -m : m;
}

/*
 * Round v to an E2M1 code: nearest grid magnitude, ties to the code whose
 * mantissa bit is 0, magnitudes at or above 6 saturate to 6.
 * Reading: the sign bit is kept even when the magnitude rounds to 0, so a
 * negative value (or -0.0) that rounds to zero gives code 0x8.
 */
int mxref_e2m1_encode(double v) {
  int sign = signbit(v) ? 8 : 0;
  double a = fabs(v);
  int best = 0;
  if (a >= 6.0) {
    best = 7;
  } else {
    double best_d = a; /* distance to grid[0] = 0 */
    for (int i = 1; i < 8; i++) {
      double dist = fabs(a - kE2M1[i]);
      if (dist < best_d) {
        best = i;
        best_d = dist;
      } else if (dist == best_d && (i & 1) == 0) {
        best = i; /* tie: prefer the even-mantissa code */
      }
    }
  }
  return sign | best;
}

static double rule_boundary(int rule, double qmax) {
  switch (rule) {
    case MXREF_RULE_UOS: return 7.25;
    case MXREF_RULE_QMAX6: return 6.0;
    case MXREF_RULE_CUSTOM: return qmax;
    default: return 0.0;
  }
}

/*
 * Shared E8M0 exponent e for a block whose largest magnitude is amax.
 *  ceiling rules (UOS, Qmax6, custom q): the smallest integer e with
 *    amax <= q * 2^e, found by stepping e one at a time (every comparison
 *    is exact in double);
 *  OCP floor rule: e = floor(log2 amax) - 2.
 * Reading: e is clamped to [-127, 127]; amax == 0 gives e = -127 (the E8M0
 * byte 0x00); the byte 0xFF (NaN) is never produced.
 */
int mxref_scale_exponent(double amax, int rule, double qmax) {
  if (!(amax > 0.0)) return -127;
  int E;
  frexp(amax, &E); /* amax = f * 2^E, f in [0.5, 1)  => floor(log2 amax) = E-1 */
  int e;
  if (rule == MXREF_RULE_OCP) {
    e = (E - 1) - 2;
  } else {
    double q = rule_boundary(rule, qmax);
    e = E - 200; /* far below the answer; step up until the boundary covers amax */
    if (e < -1100) e = -1100;
    while (ldexp(q, e) < amax) e++;
    while (ldexp(q, e - 1) >= amax) e--;
  }
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/*
 * Quantize one group of n (<= 32) values read with a stride; missing members
 * of a partial group count as zeros.  codes[i] gets the 4-bit code of x[i].
 * Returns the E8M0 byte (e + 127).
 */
static int quantize_group(const float* x, int64_t n, int64_t stride, int rule, double qmax,
                          uint8_t* codes) {
  double amax = 0.0;
  for (int64_t i = 0; i < n; i++) {
    double a = fabs((double)x[i * stride]);
    if (a > amax) amax = a;
  }
  int e = mxref_scale_exponent(amax, rule, qmax);
  for (int64_t i = 0; i < n; i++) codes[i] = (uint8_t)mxref_e2m1_encode(ldexp((double)x[i * stride], -e));
  return e + 127;
}

/*
 * NVFP4 comparison format (the pages compare MXAttention against NVFP4-based
 * baselines without defining the format; this is the public NVFP4 layout as
 * read for that comparison): blocks of 16 E2M1 codes sharing one scale that is
 * an FP8 E4M3 number (sign 0, 4 exponent bits with bias 7, 3 mantissa bits,
 * subnormals down to 2^-9, largest finite 448; the two NaN bytes 0x7F/0xFF are
 * never produced).
 */

/* Value of an E4M3 byte (bit 7 = sign; 0x7F/0xFF = NaN). */
double mxref_e4m3_decode(int byte) {
  int mag = byte & 0x7F;
  if (mag == 0x7F) return NAN;
  int e = mag >> 3, m = mag & 7;
  double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return (byte & 0x80) ? -v : v;
}

/*
 * Round v to the nearest E4M3 value, ties to the even byte (mantissa bit 0
 * clear), magnitudes above 448 saturating to 448 (the "satfinite" mode).
 * Searched over all 127 finite magnitudes.
 */
int mxref_e4m3_encode(double v) {
  int sign = signbit(v) ? 0x80 : 0;
  double a = fabs(v);
  int best = 0;
  double best_d = a;
  for (int b = 1; b < 0x7F; b++) {
    double dist = fabs(a - mxref_e4m3_decode(b));
    if (dist < best_d || (dist == best_d && (b & 1) == 0)) {
      best = b;
      best_d = dist;
    }
  }
  if (a >= 448.0) best = 0x7E;
  return sign | best;
}

/*
 * One NVFP4 block of n (<= 16) values read with a stride (missing members are
 * zeros).  Readings: the scale is the E4M3 rounding of fl32(amax / 6) (the block
 * maximum lands on the largest code, 6, up to the scale's rounding); each value
 * is divided by the scale in fp32 (one IEEE rounding) and rounded to E2M1 with
 * saturation; a scale that rounds to 0 gives all-zero codes.  Returns the scale
 * byte.
 */
static int quantize_block16(const float* x, int64_t n, int64_t stride, uint8_t* codes) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; i++) {
    float a = fabsf(x[i * stride]);
    if (a > amax) amax = a;
  }
  int sb = mxref_e4m3_encode((double)(amax / 6.0f));
  float s = (float)mxref_e4m3_decode(sb);
  for (int64_t i = 0; i < n; i++) codes[i] = s > 0.0f ? (uint8_t)mxref_e2m1_encode((double)(x[i * stride] / s)) : 0;
  return sb;
}

/*
 * NVFP4 quantization of a row-major [rows][cols] fp32 matrix, the layout of
 * mxref_quantize with blocks of 16: axis 0 along a row (codes [rows][ceil(cols/16)*16],
 * scales [rows][ceil(cols/16)]), axis 1 along a column (output transposed).
 */
void mxref_quantize_nvfp4(const float* x, int64_t rows, int64_t cols, int axis, uint8_t* codes, uint8_t* scales) {
  int64_t outer = axis == 0 ? rows : cols;
  int64_t inner = axis == 0 ? cols : rows;
  int64_t nb = (inner + 15) / 16;
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < outer; o++) {
    for (int64_t b = 0; b < nb; b++) {
      int64_t i0 = b * 16;
      int64_t n = inner - i0 < 16 ? inner - i0 : 16;
      const float* base = axis == 0 ? x + o * cols + i0 : x + i0 * cols + o;
      uint8_t* c = codes + o * nb * 16 + i0;
      memset(c, 0, 16);
      scales[o * nb + b] = (uint8_t)quantize_block16(base, n, axis == 0 ? 1 : cols, c);
    }
  }
}

/* Dequantize unpacked NVFP4 codes: out[i] = decode(code) * e4m3(scale of its block of 16). */
void mxref_dequantize_nvfp4(const uint8_t* codes, const uint8_t* scales, int64_t nblocks, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nblocks; b++) {
    double s = mxref_e4m3_decode(scales[b]);
    for (int i = 0; i < 16; i++) out[b * 16 + i] = mxref_e2m1_decode(codes[b * 16 + i]) * s;
  }
}

/*
 * Generic MXFP4 quantization of a row-major [rows][cols] fp32 matrix.
 *  axis 0: groups of 32 consecutive columns within a row.
 *     codes  [rows][ceil(cols/32)*32] one code per byte (unpacked)
 *     scales [rows][ceil(cols/32)]
 *  axis 1: groups of 32 consecutive rows within a column (output transposed).
 *     codes  [cols][ceil(rows/32)*32]
 *     scales [cols][ceil(rows/32)]
 * Groups start at index 0; the tail group is zero-padded (padding codes 0).
 */
void mxref_quantize(const float* x, int64_t rows, int64_t cols, int axis, int rule, double qmax,
                    uint8_t* codes, uint8_t* scales) {
  int64_t outer = axis == 0 ? rows : cols;
  int64_t inner = axis == 0 ? cols : rows;
  int64_t ng = (inner + 31) / 32;
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < outer; o++) {
    for (int64_t g = 0; g < ng; g++) {
      int64_t i0 = g * 32;
      int64_t n = inner - i0 < 32 ? inner - i0 : 32;
      const float* base = axis == 0 ? x + o * cols + i0 : x + i0 * cols + o;
      int64_t stride = axis == 0 ? 1 : cols;
      uint8_t* c = codes + o * ng * 32 + i0;
      memset(c, 0, 32);
      scales[o * ng + g] = (uint8_t)quantize_group(base, n, stride, rule, qmax, c);
    }
  }
}

/*
 * In-place fast Walsh-Hadamard transform of one row of length d (a power of
 * two), in fp32, normalized by c_d = fl32(1/sqrt(d)).
 * Stages h = 1, 2, 4, ..., d/2; within a stage every pair (i, i+h) with
 * (i & h) == 0 becomes (a+b, a-b); each operation rounds to fp32.  The result
 * is x * H_d / sqrt(d) for the Sylvester (natural order) Hadamard matrix H_d.
 * Readings: full-d rotation, natural order, no random sign flips, the fp32
 * operation order above, scale applied after the butterflies.
 */
void mxref_fwht_row(float* x, int d) {
  for (int h = 1; h < d; h *= 2) {
    for (int i = 0; i < d; i++) {
      if ((i & h) == 0) {
        float a = x[i];
        float b = x[i + h];
        x[i] = a + b;
        x[i + h] = a - b;
      }
    }
  }
  float c = (float)(1.0 / sqrt((double)d));
  for (int i = 0; i < d; i++) x[i] = x[i] * c;
}

/*
 * Q/K operand preparation: optional Hadamard rotation of each row of length d,
 * then MXFP4 quantization in groups of 32 along d.
 * x: [rows][d] fp32.  codes [rows][d] unpacked, scales [rows][d/32].
 * Reading: quantization reads the fp32 rotated values (no bf16 rounding
 * in between).
 */
void mxref_rotate_quantize_rows(const float* x, int64_t rows, int d, int rotate, int rule,
                                double qmax, uint8_t* codes, uint8_t* scales) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; r++) {
    float buf[1024];
    memcpy(buf, x + r * d, sizeof(float) * (size_t)d);
    if (rotate) mxref_fwht_row(buf, d);
    for (int g = 0; g < d / 32; g++)
      scales[r * (d / 32) + g] =
          (uint8_t)quantize_group(buf + g * 32, 32, 1, rule, qmax, codes + r * d + g * 32);
  }
}

/* The same with NVFP4 blocks of 16 along d: codes [rows][d], scales [rows][d/16]. */
void mxref_rotate_quantize_rows_nvfp4(const float* x, int64_t rows, int d, int rotate, uint8_t* codes,
                                      uint8_t* scales) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; r++) {
    float buf[1024];
    memcpy(buf, x + r * d, sizeof(float) * (size_t)d);
    if (rotate) mxref_fwht_row(buf, d);
    for (int b = 0; b < d / 16; b++)
      scales[r * (d / 16) + b] = (uint8_t)quantize_block16(buf + b * 16, 16, 1, codes + r * d + b * 16);
  }
}

/* Rotation alone (for the rotation-only and quantization-off checks). */
void mxref_rotate_rows(float* x, int64_t rows, int d) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; r++) mxref_fwht_row(x + r * d, d);
}

/* Dequantize unpacked codes of groups of 32: out[i] = decode(code) * 2^(byte-127). */
void mxref_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t ngroups, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t g = 0; g < ngroups; g++) {
    int e = (int)scales[g] - 127;
    for (int i = 0; i < 32; i++) out[g * 32 + i] = ldexp(mxref_e2m1_decode(codes[g * 32 + i]), e);
  }
}

typedef struct {
  int key_tile;   /* keys per online-softmax step (multiple of 32)           */
  int pnq;        /* 1: l from the quantized tile (PNQ); 0: direct placement */
  int quant_p;    /* 1: quantize the exponential tile; 0: keep it exact      */
  int rule;       /* scale rule for the exponential tile                    */
  double qmax;    /* boundary for MXREF_RULE_CUSTOM                           */
  double tau;     /* lazy max update threshold in log2 units; 0 = eager      */
  const int64_t* qpos; /* causal masking: key k is seen by row r only if k <= qpos[r]
                          (the row's position in the sequence); NULL: every key     */
  int fmt;        /* 0: MXFP4 (groups of 32, E8M0 scale by `rule`);
                     1: NVFP4 (blocks of 16, E4M3 scale), see below              */
} mxref_attn_cfg;

/* NVFP4 exponential tiles: P~ <= 1 is first multiplied by this tensor-level factor, 448 * 6, so
   that the block holding the running max (P~ = 1) gets the largest E4M3 scale, 448, and its
   maximum the largest code, 6; smaller blocks keep the E4M3 scale's full range.  P^ is divided
   by it again (it cancels in O = O~ / l either way). */
#define MXREF_NVFP4_P_GLOBAL 2688.0f

/*
 * Online-softmax attention for a set of query rows of one head, following the
 * FlashAttention-2 recurrence with PNQ (Fig. 4 of the paper as described on
 * the Pith review page; 10100.com article).
 *
 *  q     [nrows][d]  dequantized query rows (fp64, exact MXFP4 values)
 *  k, v  [N][d]      dequantized keys / values (V quantized along keys)
 *  scale softmax scale s (fp32 value)
 * Per row, for key tiles t of width T:
 *   S_k   = fl32(sum_c q_c k_kc)           (sum in fp64, then one rounding)
 *   x_k   = fl32(S_k * s)
 *   m'    = max_k x_k;  the running max m moves to m' when m is unset or
 *           (m' - m) * log2(e) > tau, else it stays (tau = 0: eager max)
 *   alpha = exp(m_old - m_new)             (unquantized)
 *   P~_k  = fl32(exp(x_k - m_new))  for keys < N, 0 beyond N
 *   P^    = MXFP4(P~) in groups of 32 keys from the tile start, same rule as
 *           Q/K/V (Fig. 1: UOS applies to all quantized attention tensors);
 *           with fmt = 1, NVFP4 blocks of 16 keys of fl32(P~ * 2688), divided
 *           by 2688 again
 *   l     = alpha*l + sum P^   (PNQ)   or   alpha*l + sum P~   (direct)
 *   O~    = alpha*O~ + sum_k P^_k v_k
 * O = O~ / l.
 * Outputs (any may be NULL except out): out [nrows][d] (fp64), m (natural-log
 * units, fp32 value), l, and wsum = sum over keys of the induced weights
 * w_k = P^_k * prod(alpha of the later tiles) / l, accumulated key by key
 * independently of the l recurrence, and ocheck [nrows][d] = sum_k w_k v_k,
 * the output rebuilt from those weights (both need wsum and ocheck non-NULL).
 * pcodes [nrows][ntiles*T] and pscales [nrows][ntiles*T/32], when non-NULL,
 * receive the E2M1 codes (one per byte, keys in order, padded keys 0) and the
 * E8M0 scale bytes of every quantized P~ group (quant_p only; NVFP4: the E4M3
 * bytes of the blocks of 16, [nrows][ntiles*T/16]).
 */
void mxref_attention_rows(const double* q, int64_t nrows, const double* k, const double* v, int N,
                          int d, float scale, const mxref_attn_cfg* cfg, double* out, double* m_out,
                          double* l_out, double* wsum_out, double* ocheck_out, uint8_t* pcodes_out,
                          uint8_t* pscales_out) {
  const int T = cfg->key_tile;
  const int ntiles = (N + T - 1) / T;
#pragma omp parallel
  {
    float* x = (float*)malloc(sizeof(float) * (size_t)T);
    float* pt = (float*)malloc(sizeof(float) * (size_t)T);
    double* ph = (double*)malloc(sizeof(double) * (size_t)T);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    double* pall = wsum_out ? (double*)malloc(sizeof(double) * (size_t)N) : NULL;
    double* alphas = wsum_out ? (double*)malloc(sizeof(double) * (size_t)ntiles) : NULL;
    uint8_t codes[32];
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; r++) {
      const double* qr = q + r * d;
      /* keys this row sees: the first `lim` (all N, or up to its position under causal masking);
         tiles past them hold only masked keys: no max move, P~ = 0 */
      const int64_t lim = cfg->qpos ? (cfg->qpos[r] + 1 < N ? cfg->qpos[r] + 1 : N) : N;
      double l = 0.0;
      float m = -INFINITY;
      for (int c = 0; c < d; c++) acc[c] = 0.0;
      for (int t = 0; t < ntiles; t++) {
        int k0 = t * T;
        int nk = lim - k0 < T ? (int)(lim - k0) : T;
        if (nk < 0) nk = 0;
        float mt = -INFINITY;
        for (int j = 0; j < nk; j++) {
          const double* kr = k + (int64_t)(k0 + j) * d;
          double s = 0.0;
          for (int c = 0; c < d; c++) s += qr[c] * kr[c];
          float sf = (float)s;
          x[j] = sf * scale;
          if (x[j] > mt) mt = x[j];
        }
        float mnew = m;
        if (m == -INFINITY || ((double)mt - (double)m) * M_LOG2E > cfg->tau) mnew = mt;
        double alpha = (m == -INFINITY) ? 0.0 : exp((double)m - (double)mnew);
        m = mnew;
        for (int j = 0; j < T; j++) pt[j] = j < nk ? (float)exp((double)x[j] - (double)m) : 0.0f;
        if (cfg->quant_p && cfg->fmt == 1) {
          for (int b = 0; b < T / 16; b++) {
            float y[16];
            for (int i = 0; i < 16; i++) y[i] = pt[b * 16 + i] * MXREF_NVFP4_P_GLOBAL;
            int sb = quantize_block16(y, 16, 1, codes);
            double sv = mxref_e4m3_decode(sb);
            for (int i = 0; i < 16; i++)
              ph[b * 16 + i] = mxref_e2m1_decode(codes[i]) * sv / (double)MXREF_NVFP4_P_GLOBAL;
            if (pcodes_out) memcpy(pcodes_out + ((size_t)r * ntiles + t) * T + b * 16, codes, 16);
            if (pscales_out) pscales_out[((size_t)r * ntiles + t) * (T / 16) + b] = (uint8_t)sb;
          }
        } else if (cfg->quant_p) {
          for (int g = 0; g < T / 32; g++) {
            int sb = quantize_group(pt + g * 32, 32, 1, cfg->rule, cfg->qmax, codes);
            for (int i = 0; i < 32; i++) ph[g * 32 + i] = ldexp(mxref_e2m1_decode(codes[i]), sb - 127);
            if (pcodes_out) memcpy(pcodes_out + ((size_t)r * ntiles + t) * T + g * 32, codes, 32);
            if (pscales_out) pscales_out[((size_t)r * ntiles + t) * (T / 32) + g] = (uint8_t)sb;
          }
        } else {
          for (int j = 0; j < T; j++) ph[j] = (double)pt[j];
        }
        double ls = 0.0;
        for (int j = 0; j < nk; j++) ls += cfg->pnq ? ph[j] : (double)pt[j];
        l = alpha * l + ls;
        for (int c = 0; c < d; c++) acc[c] *= alpha;
        for (int j = 0; j < nk; j++) {
          if (ph[j] == 0.0) continue;
          const double* vr = v + (int64_t)(k0 + j) * d;
          for (int c = 0; c < d; c++) acc[c] += ph[j] * vr[c];
        }
        if (wsum_out) {
          alphas[t] = alpha;
          for (int j = 0; j < nk; j++) pall[k0 + j] = ph[j];
        }
      }
      for (int c = 0; c < d; c++) out[r * d + c] = acc[c] / l;
      if (m_out) m_out[r] = (double)m;
      if (l_out) l_out[r] = l;
      if (wsum_out) {
        /* suffix products of alpha: weight of tile t is prod_{t' > t} alpha_t' */
        double w = 0.0, suffix = 1.0;
        double* oc = ocheck_out ? ocheck_out + r * d : NULL;
        if (oc)
          for (int c = 0; c < d; c++) oc[c] = 0.0;
        for (int t = ntiles - 1; t >= 0; t--) {
          int k0 = t * T;
          int nk = lim - k0 < T ? (int)(lim - k0) : T;
          if (nk < 0) nk = 0;
          for (int j = 0; j < nk; j++) {
            double wk = pall[k0 + j] * suffix / l;
            w += wk;
            if (oc && wk != 0.0) {
              const double* vr = v + (int64_t)(k0 + j) * d;
              for (int c = 0; c < d; c++) oc[c] += wk * vr[c];
            }
          }
          suffix *= alphas[t];
        }
        wsum_out[r] = w;
      }
    }
    free(x);
    free(pt);
    free(ph);
    free(acc);
    free(pall);
    free(alphas);
  }
}

/*
 * Per-block Qmax sweep (scale-rule diagnostic; the pages' per-block MSE-optimal boundary study of
 * Table 4, Pith review page, and the 7.25 argument of Fig. 2 / Theorem 1, applied to synthetic
 * tensors).
 *
 *  x      [rows][cols] fp32, groups of 32 consecutive elements along each row from index 0, the
 *         tail of the last group zero-padded; rotate: each row (cols = d) is Hadamard-rotated first
 *         exactly as the Q/K quantizer does.
 *  qs     nq boundaries q_k (fp32 values, each in [4, 8]).
 * For each group and each q_k: e_k = the ceiling-rule exponent with boundary q_k (smallest e with
 * amax <= q_k 2^e, clamped as everywhere); SSE_k = sum_i (x_i - xhat_i)^2 with
 * xhat_i = E2M1(x_i 2^-e_k) 2^e_k, each difference and square rounded in fp64 and the sum taken in
 * index order.  counts[k] += 1 for every k whose SSE_k equals the group's smallest (a group counts
 * for every optimal boundary); sse_sums[k] += SSE_k.  Both outputs are accumulated (the caller
 * zeroes them); the group count is rows * ceil(cols / 32).
 */
void mxref_qmax_sweep(const float* x, int64_t rows, int64_t cols, int rotate, const float* qs, int nq,
                      uint64_t* counts, double* sse_sums) {
  const int64_t ng = (cols + 31) / 32;
  const int nt = omp_get_max_threads();
  double* part = (double*)calloc((size_t)nt * (size_t)nq, sizeof(double));  /* per-thread sums */
#pragma omp parallel num_threads(nt)
  {
    uint64_t* my_counts = (uint64_t*)calloc((size_t)nq, sizeof(uint64_t));
    double* my_sums = part + (size_t)omp_get_thread_num() * (size_t)nq;
    double* sse = (double*)malloc(sizeof(double) * (size_t)nq);
    float* row = (float*)malloc(sizeof(float) * (size_t)(ng * 32));
    uint8_t code;
#pragma omp for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
      for (int64_t c = 0; c < ng * 32; c++) row[c] = c < cols ? x[r * cols + c] : 0.0f;
      if (rotate) mxref_fwht_row(row, (int)cols);
      for (int64_t g = 0; g < ng; g++) {
        const float* b = row + g * 32;
        double amax = 0.0;
        for (int i = 0; i < 32; i++)
          if (fabs((double)b[i]) > amax) amax = fabs((double)b[i]);
        double best = INFINITY;
        int prev_e = 1000;
        double prev_sse = 0.0;
        for (int k = 0; k < nq; k++) {
          const int e = mxref_scale_exponent(amax, MXREF_RULE_CUSTOM, (double)qs[k]);
          if (e != prev_e) {
            double s = 0.0;
            for (int i = 0; i < 32; i++) {
              code = (uint8_t)mxref_e2m1_encode(ldexp((double)b[i], -e));
              const double d = (double)b[i] - ldexp(mxref_e2m1_decode(code), e);
              s += d * d;
            }
            prev_e = e;
            prev_sse = s;
          }
          sse[k] = prev_sse;
          if (prev_sse < best) best = prev_sse;
        }
        for (int k = 0; k < nq; k++) {
          my_sums[k] += sse[k];
          if (sse[k] == best) my_counts[k]++;
        }
      }
    }
#pragma omp critical
    for (int k = 0; k < nq; k++) counts[k] += my_counts[k];
    free(my_counts);
    free(sse);
    free(row);
  }
  /* the partial sums are added in thread order, so the result does not depend on timing */
  for (int t = 0; t < nt; t++)
    for (int k = 0; k < nq; k++) sse_sums[k] += part[(size_t)t * (size_t)nq + k];
  free(part);
}

/* Number of OpenMP threads the oracle runs with. */
int mxref_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    n = omp_get_num_threads();
  }
  return n;
}
