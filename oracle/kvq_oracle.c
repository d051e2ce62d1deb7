/*
 * kvq_oracle.c -- plain, slow CPU oracle for quantized-KV decode attention
 * with a certified per-query error bound.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline leg use it.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * What it follows ("Runtime-Certified Bounded-Error Quantized Attention"):
 *   - Methodology 1, Tier 1: keys stored as INT8 codes, values as per-group
 *     INT4 codes with scale/offset metadata and a per-block error annotation
 *     eta_b; Tier 2: unquantized originals kept for exact recomputation.
 *   - Methodology 1, fallback: exact dense attention (scaled-dot-product
 *     semantics) on the originals for a query whose bound is exceeded.
 *   - Methodology 2: the error splits into a key term E_key (total-variation
 *     distance between exact and approximate softmax, bounded through the
 *     per-token score perturbation Delta) and a value term E_val (block
 *     errors eta_b weighted by attention mass), both computed from the
 *     quantization scales, the query norms and the value range.
 * and ("Statistical Inference and Quality Measures of KV Cache Quantisations
 * Inspired by TurboQuant", Quantisation schemes, KQV): a Walsh-Hadamard
 * rotation applied to K before scalar quantization, and the KQV codec (oq_*);
 * and ("Hurwitz Quaternion Multiplicative Quantization for KV Cache
 * Compression", Method 1-3): the HQMQ codec (oh_*) and Med3x extraction.
 *
 * Readings taken where the pages are silent (all listed in the design notes):
 *   keys per token and group, symmetric, codes in [-Q, Q] with Q = 127 (8 bit)
 *   or 7 (4 bit); values per token and 32-channel group, asymmetric, codes in
 *   [0, 15]; scale rounded UP to fp16 and zero rounded DOWN to fp16 so codes
 *   never clip; rounding half-to-even after an IEEE fp32 division; block =
 *   one 16-token page of one kv head, eta = max |v - v_hat| rounded up by one
 *   fp32 ulp; softmax scale 1/sqrt(d); GQA head h reads kv head h/(Hq/Hkv);
 *   error norm = max-abs over the d output channels; flag = bound > tau.
 *
 * Codec arithmetic is fp32 in the exact operation order below (the decision
 * of every integer code is taken in fp32, as the CUDA path takes it);
 * attention, softmax and the bound are fp64.  Compile without FMA
 * contraction (-ffp-contract=off) and without fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OC_PAGE 16
#define OC_OK 0
#define OC_ERR_ARG (-1)
#define OC_ERR_RANGE (-3)

/* Slack factor applied to the bound: absorbs fp32 rounding of the quantizer
 * (x/s rounded before rint), of the value dequantization and of the
 * fixed-order Hadamard rotation. */
#define OC_KAPPA (1.0 + 1.0 / 1024.0)
/* Relative size of the fp32 rotation error term added to Delta for rotated
 * keys (the fp32 FWHT of q and k deviates from an exact orthogonal map by far
 * less than this fraction of |q|*|k|). */
#define OC_ROT_SLACK (1.0 / 65536.0)

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16, from its definition.                                   */
/* ------------------------------------------------------------------------ */

/* value of a binary16 bit pattern: sign, 5-bit exponent (bias 15),
 * 10-bit fraction; exponent 0 = subnormal, 31 = inf/nan */
double oc_f16_value(uint16_t h) {
  int sign = (h >> 15) & 1, e = (h >> 10) & 31, f = h & 1023;
  double v;
  if (e == 31) v = f ? NAN : INFINITY;
  else if (e == 0) v = ldexp((double)f, -24);            /* f/1024 * 2^-14 */
  else v = ldexp(1.0 + f / 1024.0, e - 15);
  return sign ? -v : v;
}

typedef struct { double v; uint16_t h; } oc_f16_entry;
static oc_f16_entry oc_tab[63490];  /* all finite binary16 values, sorted */
static int oc_tab_n = 0;

static int oc_cmp(const void* a, const void* b) {
  double x = ((const oc_f16_entry*)a)->v, y = ((const oc_f16_entry*)b)->v;
  return (x > y) - (x < y);
}

static void oc_tab_init(void) {
  if (oc_tab_n) return;
  int n = 0;
  for (uint32_t h = 0; h < 65536u; ++h) {
    if (((h >> 10) & 31) == 31) continue;       /* skip inf / nan */
    if (h == 0x8000u) continue;                  /* -0 handled by sign rule */
    oc_tab[n].v = oc_f16_value((uint16_t)h);
    oc_tab[n].h = (uint16_t)h;
    ++n;
  }
  qsort(oc_tab, n, sizeof(oc_tab[0]), oc_cmp);
  oc_tab_n = n;
}

/* Directed rounding of a finite fp32 to binary16:
 *   up   -> smallest binary16 >= x (or +inf),
 *   down -> largest  binary16 <= x (or -inf).
 * A zero result keeps the sign of x (IEEE rule for directed rounding). */
uint16_t oc_f16_round(float xf, int up) {
  oc_tab_init();
  double x = (double)xf;
  if (isnan(x)) return 0x7E00u;
  int lo = 0, hi = oc_tab_n - 1;
  uint16_t r;
  if (up) {
    if (x > oc_tab[hi].v) return 0x7C00u;           /* +inf */
    /* first entry with v >= x */
    while (lo < hi) { int mid = (lo + hi) / 2; if (oc_tab[mid].v >= x) hi = mid; else lo = mid + 1; }
    r = oc_tab[lo].h;
  } else {
    if (x < oc_tab[0].v) return 0xFC00u;            /* -inf */
    /* last entry with v <= x */
    while (lo < hi) { int mid = (lo + hi + 1) / 2; if (oc_tab[mid].v <= x) lo = mid; else hi = mid - 1; }
    r = oc_tab[lo].h;
  }
  if ((r & 0x7FFFu) == 0) r = signbit(xf) ? 0x8000u : 0x0000u;
  return r;
}

int oc_f16_round_n(const float* x, int64_t n, int up, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oc_f16_round(x[i], up);
  return OC_OK;
}

void oc_f16_value_n(const uint16_t* h, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oc_f16_value(h[i]);
}

static float oc_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ------------------------------------------------------------------------ */
/* Randomized Walsh-Hadamard rotation (KQV scheme: WHT before quantization). */
/* y = c * H_d * (sigma o x), H_d the Sylvester Hadamard matrix,             */
/* c = fp32(1/sqrt(d)).  Butterflies in a fixed order: stride 1, 2, ...,     */
/* d/2; each pair (a, b) at (j, j + stride) becomes (a + b, a - b).  Then    */
/* every element is multiplied by c.  All in fp32.                           */
/* ------------------------------------------------------------------------ */
void oc_rotate(const float* x, const int8_t* sigma, int d, float* y) {
  float c = (float)(1.0 / sqrt((double)d));
  for (int i = 0; i < d; ++i) y[i] = sigma[i] < 0 ? -x[i] : x[i];
  for (int h = 1; h < d; h *= 2)
    for (int i = 0; i < d; i += 2 * h)
      for (int j = i; j < i + h; ++j) {
        float a = y[j], b = y[j + h];
        y[j] = a + b;
        y[j + h] = a - b;
      }
  for (int i = 0; i < d; ++i) y[i] = y[i] * c;
}

void oc_rotate_n(const float* x, int64_t n, int d, const int8_t* sigma, float* y) {
  for (int64_t i = 0; i < n; ++i) oc_rotate(x + i * d, sigma, d, y + i * d);
}

/* ------------------------------------------------------------------------ */
/* Scalar codecs (Tier 1: INT8/INT4 keys, INT4 values with scale/offset).     */
/* ------------------------------------------------------------------------ */

/* Symmetric group quantizer for keys.
 * a = max|x|; s = fp16_up(a / Q); code = clamp(rint(x / s), -Q, Q); s = 0 -> 0.
 * Returns OC_ERR_RANGE (and zero codes/scale) on a non-finite input or an
 * fp16-overflowing scale. */
int oc_quantize_sym(const float* x, int n, int Q, uint16_t* scale_bits, int8_t* codes) {
  float a = 0.0f;
  for (int c = 0; c < n; ++c) {
    if (!isfinite(x[c])) { *scale_bits = 0; memset(codes, 0, n); return OC_ERR_RANGE; }
    float m = fabsf(x[c]);
    if (m > a) a = m;
  }
  float t = a / (float)Q;
  uint16_t sb = oc_f16_round(t, 1);
  if ((sb & 0x7C00u) == 0x7C00u) { *scale_bits = 0; memset(codes, 0, n); return OC_ERR_RANGE; }
  float s = (float)oc_f16_value(sb);
  *scale_bits = sb;
  for (int c = 0; c < n; ++c) {
    if (s == 0.0f) { codes[c] = 0; continue; }
    float r = rintf(x[c] / s);
    if (r > (float)Q) r = (float)Q;
    if (r < (float)-Q) r = (float)-Q;
    codes[c] = (int8_t)r;
  }
  return OC_OK;
}

/* The same two quantizers with the channels [skip0, skip1) of the group left
 * out (an extracted outlier chunk): they take no part in the scale, the zero
 * or the error, and get code 0.  skip0 = skip1 is the plain quantizer. */
static int oc_quantize_sym_skip(const float* x, int n, int Q, int skip0, int skip1,
                                uint16_t* scale_bits, int8_t* codes) {
  float y[128];
  for (int c = 0; c < n; ++c) y[c] = (c >= skip0 && c < skip1) ? 0.0f : x[c];
  return oc_quantize_sym(y, n, Q, scale_bits, codes);   /* 0 leaves max|x| unchanged */
}

int oc_quantize_asym(const float* x, int n, uint16_t* scale_bits, uint16_t* zero_bits,
                     uint8_t* codes, float* max_err);

static int oc_quantize_asym_skip(const float* x, int n, int skip0, int skip1,
                                 uint16_t* scale_bits, uint16_t* zero_bits, uint8_t* codes,
                                 float* max_err) {
  if (skip0 >= skip1) return oc_quantize_asym(x, n, scale_bits, zero_bits, codes, max_err);
  float y[128];
  int first = skip0 > 0 ? 0 : skip1;   /* a channel of the group that is kept */
  for (int c = 0; c < n; ++c) y[c] = (c >= skip0 && c < skip1) ? x[first] : x[c];
  int rc = oc_quantize_asym(y, n, scale_bits, zero_bits, codes, max_err);
  for (int c = skip0; c < skip1; ++c) codes[c] = 0;
  return rc;   /* max_err: the kept channels' (the copies add no new error) */
}

/* Asymmetric 4-bit group quantizer for values.
 * z = fp16_down(min x); s = fp16_up((max x - z) / 15);
 * code = clamp(rint((x - z) / s), 0, 15) (s = 0 -> 0);
 * v_hat = fmaf(code, s, z); max_err = max |x - v_hat| (fp32). */
int oc_quantize_asym(const float* x, int n, uint16_t* scale_bits, uint16_t* zero_bits,
                     uint8_t* codes, float* max_err) {
  float lo = x[0], hi = x[0];
  for (int c = 0; c < n; ++c) {
    if (!isfinite(x[c])) goto range;
    if (x[c] < lo) lo = x[c];
    if (x[c] > hi) hi = x[c];
  }
  {
    uint16_t zb = oc_f16_round(lo, 0);
    if ((zb & 0x7C00u) == 0x7C00u) goto range;
    float z = (float)oc_f16_value(zb);
    float t = (hi - z) / 15.0f;
    uint16_t sb = oc_f16_round(t, 1);
    if ((sb & 0x7C00u) == 0x7C00u) goto range;
    float s = (float)oc_f16_value(sb);
    float e = 0.0f;
    for (int c = 0; c < n; ++c) {
      float r = 0.0f;
      if (s != 0.0f) {
        r = rintf((x[c] - z) / s);
        if (r > 15.0f) r = 15.0f;
        if (r < 0.0f) r = 0.0f;
      }
      codes[c] = (uint8_t)r;
      float vh = fmaf(r, s, z);
      float err = fabsf(x[c] - vh);
      if (err > e) e = err;
    }
    *scale_bits = sb;
    *zero_bits = zb;
    *max_err = e;
    return OC_OK;
  }
range:
  *scale_bits = 0;
  *zero_bits = 0;
  memset(codes, 0, n);
  *max_err = 0.0f;
  return OC_ERR_RANGE;
}

/* ------------------------------------------------------------------------ */
/* Paged Tier-1 layout.  One block per (physical page, kv head), 16 tokens:  */
/*   [K codes][V codes][K scales fp16 [16][d/gk]][V scale,zero fp16 [16][d/32][2]] */
/* K codes, per token d*bits/8 bytes in 4 stripes; channel c (block          */
/*   b = c/32, w = c%32, stripe s = w/8, i = w%8) sits in                     */
/*   8 bit: byte s*(8*nb) + 8*b + i, int8 two's complement (the library's    */
/*          device layout also permutes the 16-byte chunks of 128-byte rows  */
/*          by the token's slot; that is a byte permutation the tests apply  */
/*          to this logical order before comparing pools);                   */
/*   4 bit: byte s*(4*nb) + 4*b + i/2, low nibble for even c, 4-bit two's    */
/*          complement;  nb = d/32.                                           */
/* V codes: per token d/2 bytes; channel c (group g = c/32, w = c%32) sits in */
/*   byte (w/4)*(2*nb) + 2*g + (w%4)/2, low nibble for even c, unsigned.     */
/* eta is a separate fp32 array [num_pages][Hkv].                             */
/* With outlier extraction (outliers = 1) the block ends in an outlier       */
/* section: [K chunk index u8 [16]][V chunk index u8 [16]]                   */
/* [K chunk values fp16 [16][4]][V chunk values fp16 [16][4]]; index 0xFF =  */
/* no outlier in that token.                                                  */
/* ------------------------------------------------------------------------ */
typedef struct {
  int32_t d, hkv, kbits, kgroup, krotate, vbits, vgroup, num_pages, outliers;
} oc_cfg;

#define OC_NO_OUTLIER 0xFFu
#define OC_OUT_BYTES (2 * OC_PAGE + 2 * OC_PAGE * 4 * 2)

static int oc_cfg_ok(const oc_cfg* c) {
  if (!c || (c->d != 64 && c->d != 128) || c->hkv <= 0 || c->num_pages < 0) return 0;
  if (c->kbits != 8 && c->kbits != 4) return 0;
  if (c->kgroup <= 0 || c->kgroup % 32 || c->d % c->kgroup) return 0;
  if (c->vbits != 4 || c->vgroup != 32) return 0;
  if (c->outliers != 0 && c->outliers != 1) return 0;
  return 1;
}

static int64_t oc_kcode_bytes(const oc_cfg* c) { return (int64_t)OC_PAGE * c->d * c->kbits / 8; }
static int64_t oc_vcode_bytes(const oc_cfg* c) { return (int64_t)OC_PAGE * c->d / 2; }
static int64_t oc_kscale_bytes(const oc_cfg* c) { return (int64_t)OC_PAGE * (c->d / c->kgroup) * 2; }
static int64_t oc_vmeta_bytes(const oc_cfg* c) { return (int64_t)OC_PAGE * (c->d / 32) * 4; }

static int64_t oc_out_off(const oc_cfg* c) {
  return oc_kcode_bytes(c) + oc_vcode_bytes(c) + oc_kscale_bytes(c) + oc_vmeta_bytes(c);
}

int64_t oc_block_bytes(const oc_cfg* c) {
  if (!oc_cfg_ok(c)) return -1;
  return oc_out_off(c) + (c->outliers ? OC_OUT_BYTES : 0);
}

/* ------------------------------------------------------------------------ */
/* Median-multiplier outlier extraction (Med3x; "Hurwitz Quaternion          */
/* Multiplicative Quantization for KV Cache Compression", Method 3): a      */
/* vector is cut into 4-element chunks; a chunk whose norm exceeds 3x the    */
/* median chunk norm is an outlier, kept in fp16 with a flag, and the bulk   */
/* codec quantizes the rest.  Readings: the median is taken over the chunks */
/* of one token's vector (K after rotation, or V); chunk norm =              */
/* sqrt((x0*x0 + x1*x1) + (x2*x2 + x3*x3)) in fp32, each product rounded;    */
/* the median of the even count of norms is the mean of the two middle       */
/* ones, 0.5f * (a + b); at most one chunk per vector is extracted: the      */
/* largest norm above 3.0f * median (ties: the lower chunk index).           */
/* Returns the chunk index, or -1.                                            */
/* ------------------------------------------------------------------------ */
int oc_med3_chunk(const float* x, int d) {
  int nc = d / 4;
  float r[32], srt[32];
  for (int i = 0; i < nc; ++i) {
    float a = x[4 * i] * x[4 * i], b = x[4 * i + 1] * x[4 * i + 1];
    float e = x[4 * i + 2] * x[4 * i + 2], f = x[4 * i + 3] * x[4 * i + 3];
    r[i] = sqrtf((a + b) + (e + f));
    if (isnan(r[i])) return -1;   /* a NaN input: no extraction (the bulk codec flags it) */
    srt[i] = r[i];
  }
  for (int i = 1; i < nc; ++i)   /* insertion sort, ascending */
    for (int j = i; j > 0 && srt[j - 1] > srt[j]; --j) {
      float t = srt[j]; srt[j] = srt[j - 1]; srt[j - 1] = t;
    }
  float med = 0.5f * (srt[nc / 2 - 1] + srt[nc / 2]);
  float thr = 3.0f * med;
  int best = -1;
  for (int i = 0; i < nc; ++i)
    if (r[i] > thr && (best < 0 || r[i] > r[best])) best = i;
  return best;
}

/* binary16 round-to-nearest, ties to the even pattern (the directed
 * neighbours from oc_f16_round, then the nearer one). */
uint16_t oc_f16_rn(float xf) {
  uint16_t dn = oc_f16_round(xf, 0), up = oc_f16_round(xf, 1);
  if (dn == up) return dn;
  double x = (double)xf, vd = oc_f16_value(dn), vu = oc_f16_value(up);
  if (isinf(vu) || isinf(vd)) return isinf(vu) ? dn : up;
  double ed = x - vd, eu = vu - x;
  if (ed < eu) return dn;
  if (eu < ed) return up;
  return (dn & 1u) == 0 ? dn : up;
}

static int64_t oc_k8_byte(int d, int ch) {
  int nb = d / 32, b = ch / 32, w = ch % 32;
  return (int64_t)(w / 8) * (8 * nb) + 8 * b + w % 8;
}
static int64_t oc_k4_byte(int d, int ch) {
  int nb = d / 32, b = ch / 32, w = ch % 32;
  return (int64_t)(w / 8) * (4 * nb) + 4 * b + (w % 8) / 2;
}
static int64_t oc_v4_byte(int d, int ch) {
  int nb = d / 32, g = ch / 32, w = ch % 32;
  return (int64_t)(w / 4) * (2 * nb) + 2 * g + (w % 4) / 2;
}

static void oc_put_nibble(uint8_t* row, int64_t byte, int ch, unsigned v) {
  if (ch % 2 == 0) row[byte] = (uint8_t)((row[byte] & 0xF0u) | (v & 0xFu));
  else row[byte] = (uint8_t)((row[byte] & 0x0Fu) | ((v & 0xFu) << 4));
}
static unsigned oc_get_nibble(const uint8_t* row, int64_t byte, int ch) {
  return ch % 2 == 0 ? (row[byte] & 0xFu) : (row[byte] >> 4);
}

static uint16_t oc_rd16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static void oc_wr16(uint8_t* p, uint16_t v) { p[0] = (uint8_t)(v & 0xFF); p[1] = (uint8_t)(v >> 8); }

/* Quantize one token of one kv head into slot `slot` of block `blk`.
 * x_k, x_v: fp32 [d]; returns the token's fp32 max value error through *verr. */
/* Channels [skip0, skip1) of the group [g0, g0 + n) that lie in the chunk
 * [4*chunk, 4*chunk + 4) (an empty range when chunk < 0 or no overlap). */
static void oc_chunk_in_group(int chunk, int g0, int n, int* skip0, int* skip1) {
  *skip0 = *skip1 = 0;
  if (chunk < 0) return;
  int a = 4 * chunk - g0, b = a + 4;
  if (a < 0) a = 0;
  if (b > n) b = n;
  if (a < b) { *skip0 = a; *skip1 = b; }
}

static int oc_quantize_token(const oc_cfg* c, uint8_t* blk, int slot, const float* xk_in,
                             const float* xv, const int8_t* sigma, float* verr) {
  int d = c->d, rc = OC_OK;
  float xk_rot[128];
  const float* xk = xk_in;
  if (c->krotate) { oc_rotate(xk_in, sigma, d, xk_rot); xk = xk_rot; }
  /* outlier chunks (Med3x), at most one per vector, kept in fp16 */
  int ck = -1, cv = -1;
  float out_err = 0.0f;
  if (c->outliers) {
    ck = oc_med3_chunk(xk, d);
    cv = oc_med3_chunk(xv, d);
    uint8_t* os = blk + oc_out_off(c);
    os[slot] = ck < 0 ? OC_NO_OUTLIER : (uint8_t)ck;
    os[OC_PAGE + slot] = cv < 0 ? OC_NO_OUTLIER : (uint8_t)cv;
    for (int i = 0; i < 4; ++i) {
      uint16_t hk = 0, hv = 0;
      if (ck >= 0) {
        float x = xk[4 * ck + i];
        if (!isfinite(x) || fabsf(x) > 65504.0f) rc = OC_ERR_RANGE;
        else hk = oc_f16_rn(x);
      }
      if (cv >= 0) {
        float x = xv[4 * cv + i];
        if (!isfinite(x) || fabsf(x) > 65504.0f) {
          rc = OC_ERR_RANGE;
        } else {
          hv = oc_f16_rn(x);
          float err = fabsf(x - (float)oc_f16_value(hv));
          if (err > out_err) out_err = err;
        }
      }
      oc_wr16(os + 2 * OC_PAGE + (slot * 4 + i) * 2, hk);
      oc_wr16(os + 2 * OC_PAGE + OC_PAGE * 8 + (slot * 4 + i) * 2, hv);
    }
  }
  /* keys */
  int Q = c->kbits == 8 ? 127 : 7;
  uint8_t* kcodes = blk;
  uint8_t* kscales = blk + oc_kcode_bytes(c) + oc_vcode_bytes(c);
  for (int g = 0; g < d / c->kgroup; ++g) {
    int8_t codes[128];
    uint16_t sb;
    int s0, s1;
    oc_chunk_in_group(ck, g * c->kgroup, c->kgroup, &s0, &s1);
    int r = oc_quantize_sym_skip(xk + g * c->kgroup, c->kgroup, Q, s0, s1, &sb, codes);
    if (r != OC_OK) rc = r;
    oc_wr16(kscales + ((int64_t)slot * (d / c->kgroup) + g) * 2, sb);
    for (int i = 0; i < c->kgroup; ++i) {
      int ch = g * c->kgroup + i;
      if (c->kbits == 8) {
        kcodes[(int64_t)slot * d + oc_k8_byte(d, ch)] = (uint8_t)codes[i];
      } else {
        uint8_t* row = kcodes + (int64_t)slot * (d / 2);
        oc_put_nibble(row, oc_k4_byte(d, ch), ch, (unsigned)(codes[i] & 0xF));
      }
    }
  }
  /* values */
  uint8_t* vrow = blk + oc_kcode_bytes(c) + (int64_t)slot * (d / 2);
  uint8_t* vmeta = blk + oc_kcode_bytes(c) + oc_vcode_bytes(c) + oc_kscale_bytes(c);
  float e = out_err;
  for (int g = 0; g < d / 32; ++g) {
    uint8_t codes[32];
    uint16_t sb, zb;
    float ge;
    int s0, s1;
    oc_chunk_in_group(cv, g * 32, 32, &s0, &s1);
    int r = oc_quantize_asym_skip(xv + g * 32, 32, s0, s1, &sb, &zb, codes, &ge);
    if (r != OC_OK) rc = r;
    oc_wr16(vmeta + ((int64_t)slot * (d / 32) + g) * 4, sb);
    oc_wr16(vmeta + ((int64_t)slot * (d / 32) + g) * 4 + 2, zb);
    for (int i = 0; i < 32; ++i) {
      int ch = g * 32 + i;
      oc_put_nibble(vrow, oc_v4_byte(d, ch), ch, codes[i]);
    }
    if (ge > e) e = ge;
  }
  *verr = e;
  return rc;
}

static void oc_load_vec(const void* base, int is_f32, int64_t off, int d, float* out) {
  if (is_f32) memcpy(out, (const float*)base + off, sizeof(float) * d);
  else for (int i = 0; i < d; ++i) out[i] = oc_bf16_to_f32(((const uint16_t*)base)[off + i]);
}

/* Quantize-on-append.  Token t (< valid[b], or < num_tokens if valid is NULL)
 * of sequence b goes to logical position start_pos[b] + t, i.e. physical page
 * page_table[b][pos/16], slot pos%16.  Element (b, h, t, ch) of k and v is at
 * b*seq_stride + h*head_stride + t*tok_stride + ch.
 * eta[page][h] = max(eta, nextafter(token max error, +inf)). */
int oc_append(const oc_cfg* c, uint8_t* pool, float* eta, const void* k, const void* v,
              int in_is_f32, int64_t seq_stride, int64_t head_stride, int64_t tok_stride,
              int num_seqs, int num_tokens, const int32_t* valid, const int32_t* page_table,
              int max_pages, const int32_t* start_pos, const int8_t* sigma) {
  if (!oc_cfg_ok(c) || (c->krotate && !sigma)) return OC_ERR_ARG;
  int64_t bb = oc_block_bytes(c);
  int rc = OC_OK;
  float xk[128], xv[128];
  for (int b = 0; b < num_seqs; ++b) {
    int nt = valid ? valid[b] : num_tokens;
    for (int t = 0; t < nt; ++t) {
      int pos = start_pos[b] + t;
      int lp = pos / OC_PAGE;
      if (lp >= max_pages) return OC_ERR_ARG;
      int page = page_table[(int64_t)b * max_pages + lp];
      if (page < 0 || page >= c->num_pages) return OC_ERR_ARG;
      for (int h = 0; h < c->hkv; ++h) {
        int64_t off = b * seq_stride + h * head_stride + t * tok_stride;
        oc_load_vec(k, in_is_f32, off, c->d, xk);
        oc_load_vec(v, in_is_f32, off, c->d, xv);
        uint8_t* blk = pool + ((int64_t)page * c->hkv + h) * bb;
        float e;
        int r = oc_quantize_token(c, blk, pos % OC_PAGE, xk, xv, sigma, &e);
        if (r != OC_OK) rc = r;
        float eu = nextafterf(e, INFINITY);
        float* ep = eta + (int64_t)page * c->hkv + h;
        if (eu > *ep) *ep = eu;
      }
    }
  }
  return rc;
}

/* Dequantized view of one token of one kv head, read back from the layout. */
static void oc_read_token(const oc_cfg* c, const uint8_t* blk, int slot, double* khat,
                          double* kscale, double* vhat, double* vs, double* vz,
                          double* vtop, int* kchunk, int* vchunk) {
  int d = c->d, ngk = d / c->kgroup;
  const uint8_t* kcodes = blk;
  const uint8_t* vrow = blk + oc_kcode_bytes(c) + (int64_t)slot * (d / 2);
  const uint8_t* kscales = blk + oc_kcode_bytes(c) + oc_vcode_bytes(c);
  const uint8_t* vmeta = kscales + oc_kscale_bytes(c);
  for (int g = 0; g < ngk; ++g)
    kscale[g] = oc_f16_value(oc_rd16(kscales + ((int64_t)slot * ngk + g) * 2));
  for (int ch = 0; ch < d; ++ch) {
    int code;
    if (c->kbits == 8) code = (int8_t)kcodes[(int64_t)slot * d + oc_k8_byte(d, ch)];
    else {
      unsigned nib = oc_get_nibble(kcodes + (int64_t)slot * (d / 2), oc_k4_byte(d, ch), ch);
      code = nib >= 8 ? (int)nib - 16 : (int)nib;
    }
    khat[ch] = kscale[ch / c->kgroup] * code;
  }
  for (int g = 0; g < d / 32; ++g) {
    uint16_t sb = oc_rd16(vmeta + ((int64_t)slot * (d / 32) + g) * 4);
    uint16_t zb = oc_rd16(vmeta + ((int64_t)slot * (d / 32) + g) * 4 + 2);
    vs[g] = oc_f16_value(sb);
    vz[g] = oc_f16_value(zb);
    /* top of the representable range of this group: fmaf(15, s, z) in fp32 */
    vtop[g] = (double)fmaf(15.0f, (float)vs[g], (float)vz[g]);
  }
  for (int ch = 0; ch < d; ++ch) {
    unsigned code = oc_get_nibble(vrow, oc_v4_byte(d, ch), ch);
    vhat[ch] = vs[ch / 32] * (double)code + vz[ch / 32];   /* exact in fp64 */
  }
  *kchunk = *vchunk = -1;
  if (c->outliers) {   /* the fp16 outlier chunks, in place of their codes */
    const uint8_t* os = blk + oc_out_off(c);
    if (os[slot] != OC_NO_OUTLIER) {
      *kchunk = os[slot];
      for (int i = 0; i < 4; ++i)
        khat[4 * *kchunk + i] = oc_f16_value(oc_rd16(os + 2 * OC_PAGE + (slot * 4 + i) * 2));
    }
    if (os[OC_PAGE + slot] != OC_NO_OUTLIER) {
      *vchunk = os[OC_PAGE + slot];
      for (int i = 0; i < 4; ++i)
        vhat[4 * *vchunk + i] =
            oc_f16_value(oc_rd16(os + 2 * OC_PAGE + OC_PAGE * 8 + (slot * 4 + i) * 2));
    }
  }
}

/* Quantized decode attention and its certified bound, for every query row
 * (sequence b, query i, q head h), kv head h / (Hq/Hkv):
 *   q'   = rotated q if keys are rotated (same fp32 rotation as the keys)
 *   z^_j = scale * q' . k^_j                          (fp64)
 *   p^   = softmax(z^),  o^ = sum_j p^_j v^_j
 *   Delta_j = kappa*scale*( sum_g |q'_g|_1 * sK_{j,g} / 2
 *                           + [rotated] 2^-16*sqrt(d)*Q*|q'|_2*max_g sK_{j,g} )
 *   A = sum_j p^_j (exp(Delta_j) - 1),  B = sum_j p^_j exp(-Delta_j)
 *   TV = min(tanh(max_j Delta_j / 2), A / B)
 *   range = max_g ( max_j fmaf(15, sV_{j,g}, zV_{j,g}) - min_j zV_{j,g} )
 *   E_key = TV * (range + 2 * max_b eta_b)
 *   E_val = sum_j p^_j eta_{block(j)}
 *   bound = kappa * (E_key + E_val);  flag = bound > tau.
 * An empty context gives o^ = 0, bound = 0, flag = 0.
 * diag (optional) gets per row: TV, E_key, E_val, max Delta, A, B, range, eta_max.
 * row_mask (optional): only rows with a nonzero entry are computed. */
/* Per-token terms of one query row over its context of n tokens:
 * z[j] = z^_j, dl[j] = Delta_j, et[j] = eta of token j's block; also the
 * value range and the largest eta of the context. */
static void oc_row_terms(const oc_cfg* c, const uint8_t* pool, const float* eta,
                         const float* qp, int b, int kv, int n, const int32_t* page_table,
                         int max_pages, double sc, double* z, double* dl, double* et,
                         double* range_out, double* eta_max_out) {
  int d = c->d, ngk = d / c->kgroup, ngv = d / 32;
  int Q = c->kbits == 8 ? 127 : 7;
  int64_t bb = oc_block_bytes(c);
  double qn1[4] = {0, 0, 0, 0}, qn2 = 0.0;
  for (int ch = 0; ch < d; ++ch) {
    qn1[ch / c->kgroup] += fabs((double)qp[ch]);
    qn2 += (double)qp[ch] * (double)qp[ch];
  }
  qn2 = sqrt(qn2);
  double rot = c->krotate ? OC_ROT_SLACK * sqrt((double)d) * Q * qn2 : 0.0;
  double vtop_max[4], vz_min[4], eta_max = 0.0;
  for (int g = 0; g < ngv; ++g) { vtop_max[g] = -INFINITY; vz_min[g] = INFINITY; }
  double khat[128], ks[4], vhat[128], vs[4], vz[4], vtop[4];
  int kc, vc;
  for (int j = 0; j < n; ++j) {
    int page = page_table[(int64_t)b * max_pages + j / OC_PAGE];
    const uint8_t* blk = pool + ((int64_t)page * c->hkv + kv) * bb;
    oc_read_token(c, blk, j % OC_PAGE, khat, ks, vhat, vs, vz, vtop, &kc, &vc);
    double dot = 0.0, smax = 0.0, qs = 0.0;
    for (int ch = 0; ch < d; ++ch) dot += (double)qp[ch] * khat[ch];
    for (int g = 0; g < ngk; ++g) {
      qs += qn1[g] * ks[g] / 2.0;
      if (ks[g] > smax) smax = ks[g];
    }
    /* an fp16 outlier chunk: |k - k^| <= 2^-11 |k^| + 2^-25 per channel (half an
     * fp16 ulp), and, for rotated keys, its norm joins the rotation allowance */
    double qo = 0.0, kon = 0.0;
    if (kc >= 0)
      for (int i = 0; i < 4; ++i) {
        double kx = khat[4 * kc + i];
        qo += fabs((double)qp[4 * kc + i]) * (ldexp(fabs(kx), -11) + ldexp(1.0, -25));
        kon += kx * kx;
      }
    z[j] = sc * dot;
    dl[j] = OC_KAPPA * sc * (qs + rot * smax + qo +
                             (c->krotate ? OC_ROT_SLACK * qn2 * sqrt(kon) : 0.0));
    et[j] = (double)eta[(int64_t)page * c->hkv + kv];
    if (et[j] > eta_max) eta_max = et[j];
    for (int g = 0; g < ngv; ++g) {
      if (vtop[g] > vtop_max[g]) vtop_max[g] = vtop[g];
      if (vz[g] < vz_min[g]) vz_min[g] = vz[g];
    }
    if (vc >= 0)   /* the stored outlier values lie outside [z, z + 15 s] */
      for (int i = 0; i < 4; ++i) {
        int g = (4 * vc + i) / 32;
        if (vhat[4 * vc + i] > vtop_max[g]) vtop_max[g] = vhat[4 * vc + i];
        if (vhat[4 * vc + i] < vz_min[g]) vz_min[g] = vhat[4 * vc + i];
      }
  }
  double range = 0.0;
  for (int g = 0; g < ngv; ++g)
    if (vtop_max[g] - vz_min[g] > range) range = vtop_max[g] - vz_min[g];
  *range_out = range;
  *eta_max_out = eta_max;
}

static const float* oc_row_query(const oc_cfg* c, const void* q, int q_is_f32, int64_t row,
                                 const int8_t* sigma, float* qf, float* qr) {
  oc_load_vec(q, q_is_f32, row * c->d, c->d, qf);
  if (!c->krotate) return qf;
  oc_rotate(qf, sigma, c->d, qr);
  return qr;
}

/* Quantized decode attention and its certified bound, for every query row
 * (sequence b, query i, q head h), kv head h / (Hq/Hkv):
 *   q'   = rotated q if keys are rotated (same fp32 rotation as the keys)
 *   z^_j = scale * q' . k^_j                          (fp64)
 *   p^   = softmax(z^),  o^ = sum_j p^_j v^_j
 *   Delta_j = kappa*scale*( sum_g |q'_g|_1 * sK_{j,g} / 2
 *                           + [rotated] 2^-16*sqrt(d)*Q*|q'|_2*max_g sK_{j,g} )
 *   A = sum_j p^_j (exp(Delta_j) - 1),  B = sum_j p^_j exp(-Delta_j)
 *   TV = min(tanh(max_j Delta_j / 2), A / B)
 *   range = max_g ( max_j fmaf(15, sV_{j,g}, zV_{j,g}) - min_j zV_{j,g} )
 *   E_key = TV * (range + 2 * max_b eta_b)
 *   E_val = sum_j p^_j eta_{block(j)}
 *   bound = kappa * (E_key + E_val);  flag = bound > tau.
 * An empty context gives o^ = 0, bound = 0, flag = 0.
 * diag (optional) gets per row: TV, E_key, E_val, max Delta, A, B, range, eta_max.
 * row_mask (optional): only rows with a nonzero entry are computed. */
int oc_decode(const oc_cfg* c, const uint8_t* pool, const float* eta, const void* q,
              int q_is_f32, int num_seqs, int nq, int hq, const int32_t* page_table,
              int max_pages, const int32_t* seq_lens, float scale, float tau,
              const int8_t* sigma, double* out, double* bound, uint8_t* flags, double* diag,
              const uint8_t* row_mask) {
  if (!oc_cfg_ok(c) || hq % c->hkv || (c->krotate && !sigma)) return OC_ERR_ARG;
  int d = c->d, G = hq / c->hkv;
  int64_t bb = oc_block_bytes(c);
  double sc = (double)scale;
  for (int b = 0; b < num_seqs; ++b) {
    int n = seq_lens[b];
    double* z = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* dl = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* et = n ? (double*)malloc(sizeof(double) * n) : NULL;
    for (int i = 0; i < nq; ++i)
      for (int h = 0; h < hq; ++h) {
        int64_t row = ((int64_t)b * nq + i) * hq + h;
        if (row_mask && !row_mask[row]) continue;
        int kv = h / G;
        double* o = out + row * d;
        for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
        if (n == 0) {
          bound[row] = 0.0;
          flags[row] = 0;
          if (diag) for (int t = 0; t < 8; ++t) diag[row * 8 + t] = 0.0;
          continue;
        }
        float qf[128], qr[128];
        const float* qp = oc_row_query(c, q, q_is_f32, row, sigma, qf, qr);
        double range, eta_max;
        oc_row_terms(c, pool, eta, qp, b, kv, n, page_table, max_pages, sc, z, dl, et, &range,
                     &eta_max);
        double m = -INFINITY;
        for (int j = 0; j < n; ++j) if (z[j] > m) m = z[j];
        double l = 0.0;
        for (int j = 0; j < n; ++j) l += exp(z[j] - m);
        double A = 0.0, B = 0.0, Ev = 0.0, dmax = 0.0;
        double khat[128], ks[4], vhat[128], vs[4], vz[4], vtop[4];
        int kc, vc;
        for (int j = 0; j < n; ++j) {
          double p = exp(z[j] - m) / l;
          int page = page_table[(int64_t)b * max_pages + j / OC_PAGE];
          const uint8_t* blk = pool + ((int64_t)page * c->hkv + kv) * bb;
          oc_read_token(c, blk, j % OC_PAGE, khat, ks, vhat, vs, vz, vtop, &kc, &vc);
          for (int ch = 0; ch < d; ++ch) o[ch] += p * vhat[ch];
          A += p * expm1(dl[j]);
          B += p * exp(-dl[j]);
          Ev += p * et[j];
          if (dl[j] > dmax) dmax = dl[j];
        }
        double tv = tanh(dmax / 2.0);
        if (A / B < tv) tv = A / B;
        double ekey = tv * (range + 2.0 * eta_max);
        double bd = OC_KAPPA * (ekey + Ev);
        bound[row] = bd;
        flags[row] = bd > (double)tau ? 1 : 0;
        if (diag) {
          double* dg = diag + row * 8;
          dg[0] = tv; dg[1] = ekey; dg[2] = Ev; dg[3] = dmax;
          dg[4] = A; dg[5] = B; dg[6] = range; dg[7] = eta_max;
        }
      }
    free(z);
    free(dl);
    free(et);
  }
  return OC_OK;
}

/* Per-token scores z^_j and perturbation bounds Delta_j of one query row
 * (for tests of the bound's ingredients). */
int oc_decode_terms(const oc_cfg* c, const uint8_t* pool, const float* eta, const void* q,
                    int q_is_f32, int nq, int hq, int b, int i, int h,
                    const int32_t* page_table, int max_pages, int n, float scale,
                    const int8_t* sigma, double* z, double* dl) {
  if (!oc_cfg_ok(c) || hq % c->hkv || (c->krotate && !sigma) || n <= 0) return OC_ERR_ARG;
  int64_t row = ((int64_t)b * nq + i) * hq + h;
  float qf[128], qr[128];
  const float* qp = oc_row_query(c, q, q_is_f32, row, sigma, qf, qr);
  double* et = (double*)malloc(sizeof(double) * n);
  double range, eta_max;
  oc_row_terms(c, pool, eta, qp, b, h / (hq / c->hkv), n, page_table, max_pages,
               (double)scale, z, dl, et, &range, &eta_max);
  free(et);
  return OC_OK;
}

/* Value promotion: rung 2 of the fallback ladder ("Runtime-Certified
 * Bounded-Error Quantized Attention", Methodology 3: page in full-precision
 * values for the blocks whose estimated value-error contribution exceeds a
 * threshold).  A block is one page of one kv head.  Per query row, with z^,
 * p^, Delta, E_key as in oc_decode:
 *   M_b    = sum_{j in b} p^_j          (the block's estimated attention mass)
 *   c_b    = M_b * eta_b                (its share of E_val)
 *   promoted blocks: c_b > v_tol
 *   o'     = sum_j p^_j v~_j,  v~_j = the original v_j in a promoted block,
 *                              else v^_j
 *   E_val' = sum of c_b over the blocks not promoted
 *   bound' = kappa * (E_key + E_val');  flag' = bound' > tau.
 * E_key is unchanged: a promoted value lies within eta_b of its code's value,
 * which the 2 * max eta of E_key's range term already covers.
 * v_orig element (b, h, t, ch) at b*seq_stride + h*head_stride + t*tok_stride
 * + ch (fp32, or bf16 bits when v_is_f32 is 0).  promoted (optional) gets per
 * row the number of promoted blocks; diag as in oc_decode, with E_val'. */
int oc_decode_promote_values(const oc_cfg* c, const uint8_t* pool, const float* eta,
                             const void* q, int q_is_f32, int num_seqs, int nq, int hq,
                             const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                             float scale, float tau, const int8_t* sigma, const void* v_orig,
                             int v_is_f32, int64_t seq_stride, int64_t head_stride,
                             int64_t tok_stride, double v_tol, double* out, double* bound,
                             uint8_t* flags, int32_t* promoted, double* diag,
                             const uint8_t* row_mask) {
  if (!oc_cfg_ok(c) || hq % c->hkv || (c->krotate && !sigma) || !v_orig) return OC_ERR_ARG;
  int d = c->d, G = hq / c->hkv;
  int64_t bb = oc_block_bytes(c);
  double sc = (double)scale;
  for (int b = 0; b < num_seqs; ++b) {
    int n = seq_lens[b];
    int npg = (n + OC_PAGE - 1) / OC_PAGE;
    double* z = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* dl = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* et = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* mass = npg ? (double*)malloc(sizeof(double) * npg) : NULL;
    uint8_t* prom = npg ? (uint8_t*)malloc(npg) : NULL;
    for (int i = 0; i < nq; ++i)
      for (int h = 0; h < hq; ++h) {
        int64_t row = ((int64_t)b * nq + i) * hq + h;
        if (row_mask && !row_mask[row]) continue;
        int kv = h / G;
        double* o = out + row * d;
        for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
        if (n == 0) {
          bound[row] = 0.0;
          flags[row] = 0;
          if (promoted) promoted[row] = 0;
          if (diag) for (int t = 0; t < 8; ++t) diag[row * 8 + t] = 0.0;
          continue;
        }
        float qf[128], qr[128], vf[128];
        const float* qp = oc_row_query(c, q, q_is_f32, row, sigma, qf, qr);
        double range, eta_max;
        oc_row_terms(c, pool, eta, qp, b, kv, n, page_table, max_pages, sc, z, dl, et, &range,
                     &eta_max);
        double m = -INFINITY;
        for (int j = 0; j < n; ++j) if (z[j] > m) m = z[j];
        double l = 0.0;
        for (int j = 0; j < n; ++j) l += exp(z[j] - m);
        for (int lp = 0; lp < npg; ++lp) mass[lp] = 0.0;
        for (int j = 0; j < n; ++j) mass[j / OC_PAGE] += exp(z[j] - m) / l;
        int np_ = 0;
        for (int lp = 0; lp < npg; ++lp) {
          prom[lp] = mass[lp] * et[lp * OC_PAGE] > v_tol ? 1 : 0;
          np_ += prom[lp];
        }
        double A = 0.0, B = 0.0, Ev = 0.0, dmax = 0.0;
        double khat[128], ks[4], vhat[128], vs[4], vz[4], vtop[4];
        int kc, vc;
        for (int j = 0; j < n; ++j) {
          double p = exp(z[j] - m) / l;
          if (prom[j / OC_PAGE]) {
            oc_load_vec(v_orig, v_is_f32, b * seq_stride + kv * head_stride + j * tok_stride, d,
                        vf);
            for (int ch = 0; ch < d; ++ch) o[ch] += p * (double)vf[ch];
          } else {
            int page = page_table[(int64_t)b * max_pages + j / OC_PAGE];
            const uint8_t* blk = pool + ((int64_t)page * c->hkv + kv) * bb;
            oc_read_token(c, blk, j % OC_PAGE, khat, ks, vhat, vs, vz, vtop, &kc, &vc);
            for (int ch = 0; ch < d; ++ch) o[ch] += p * vhat[ch];
            Ev += p * et[j];
          }
          A += p * expm1(dl[j]);
          B += p * exp(-dl[j]);
          if (dl[j] > dmax) dmax = dl[j];
        }
        double tv = tanh(dmax / 2.0);
        if (A / B < tv) tv = A / B;
        double ekey = tv * (range + 2.0 * eta_max);
        double bd = OC_KAPPA * (ekey + Ev);
        bound[row] = bd;
        flags[row] = bd > (double)tau ? 1 : 0;
        if (promoted) promoted[row] = np_;
        if (diag) {
          double* dg = diag + row * 8;
          dg[0] = tv; dg[1] = ekey; dg[2] = Ev; dg[3] = dmax;
          dg[4] = A; dg[5] = B; dg[6] = range; dg[7] = eta_max;
        }
      }
    free(z);
    free(dl);
    free(et);
    free(mass);
    free(prom);
  }
  return OC_OK;
}

/* Exact dense attention on the originals (the fallback's ground truth):
 * o = softmax(scale * q . k_j) v, fp64, no quantization, no rotation.
 * k, v element (b, h, t, ch) at b*seq_stride + h*head_stride + t*tok_stride + ch. */
int oc_dense(const void* q, int q_is_f32, const void* k, const void* v, int kv_is_f32,
             int64_t seq_stride, int64_t head_stride, int64_t tok_stride, int num_seqs,
             int nq, int hq, int hkv, int d, const int32_t* seq_lens, float scale, double* out,
             const uint8_t* row_mask) {
  if (d <= 0 || d > 128 || hkv <= 0 || hq % hkv) return OC_ERR_ARG;
  int G = hq / hkv;
  double sc = (double)scale;
  float qf[128], kf[128], vf[128];
  for (int b = 0; b < num_seqs; ++b) {
    int n = seq_lens[b];
    double* z = n ? (double*)malloc(sizeof(double) * n) : NULL;
    for (int i = 0; i < nq; ++i)
      for (int h = 0; h < hq; ++h) {
        int64_t row = ((int64_t)b * nq + i) * hq + h;
        if (row_mask && !row_mask[row]) continue;
        int kv = h / G;
        double* o = out + row * d;
        for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
        if (n == 0) continue;
        oc_load_vec(q, q_is_f32, row * d, d, qf);
        double m = -INFINITY;
        for (int j = 0; j < n; ++j) {
          oc_load_vec(k, kv_is_f32, b * seq_stride + kv * head_stride + j * tok_stride, d, kf);
          double dot = 0.0;
          for (int ch = 0; ch < d; ++ch) dot += (double)qf[ch] * (double)kf[ch];
          z[j] = sc * dot;
          if (z[j] > m) m = z[j];
        }
        double l = 0.0;
        for (int j = 0; j < n; ++j) l += exp(z[j] - m);
        for (int j = 0; j < n; ++j) {
          double p = exp(z[j] - m) / l;
          oc_load_vec(v, kv_is_f32, b * seq_stride + kv * head_stride + j * tok_stride, d, vf);
          for (int ch = 0; ch < d; ++ch) o[ch] += p * (double)vf[ch];
        }
      }
    free(z);
  }
  return OC_OK;
}

/* Certified output: o = exact dense attention where flag is set, else o^. */
void oc_certified_output(const double* ohat, const double* odense, const uint8_t* flags,
                         int64_t rows, int d, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int ch = 0; ch < d; ++ch)
      out[r * d + ch] = flags[r] ? odense[r * d + ch] : ohat[r * d + ch];
}

/* ------------------------------------------------------------------------ */
/* Adaptive precision and the first rungs of the fallback ladder             */
/* ("Runtime-Certified Bounded-Error Quantized Attention", Methodology 3:    */
/* adaptive top-K* block selection from a light scoring pass with the       */
/* quantized keys, promotion of those blocks to full-precision keys, the    */
/* ranking-consistency check, and value promotion).  A block is one page of */
/* one kv head.  Per query row (sequence b, query i, q head h; kv head      */
/* h / (Hq/Hkv)), with z^, p^, Delta as in oc_decode:                       */
/*   M^_b   = sum_{j in b} p^_j     (estimated mass of the block)             */
/*   order  = blocks by M^_b descending, ties by lower block index            */
/*   K*     = the smallest k whose first k blocks in that order have mass     */
/*            >= tau_cov (every block if none does); they are key-promoted    */
/*   z~_j   = scale * q . k_j from the originals (q unrotated) in a          */
/*            key-promoted block, else z^_j                                   */
/*   Delta~ = kappa * scale * 2^-16 * |q|_2 * |k_j|_2 in a key-promoted block */
/*            (allowance for an fp32 dot product of the originals), else      */
/*            Delta_j                                                         */
/*   p~     = softmax(z~)                                                     */
/*   value-promoted blocks: M^_b * eta_b > v_tol (rung 2: the block's         */
/*            estimated share of E_val, from the same scoring pass)            */
/*   o~     = sum_j p~_j v~_j, v~_j = the original v_j in a value-promoted    */
/*            block, else v^_j                                                */
/*   A = sum p~ (e^Delta~ - 1), B = sum p~ e^-Delta~, TV = min(tanh(max      */
/*   Delta~ / 2), A/B); E_key = TV (range + 2 max eta) with range and eta as */
/*   in oc_decode; E_val = sum of p~_j eta_{block(j)} over the blocks whose   */
/*   values are not promoted; bound = kappa (E_key + E_val)                   */
/*   ranking check: L_b = log sum_{j in b} e^{z~_j} over the key-promoted     */
/*   blocks in their selection order; the ranking is inconsistent when a     */
/*   later block's L exceeds an earlier block's L by more than rank_tol       */
/*   flag   = inconsistent || bound > tau.                                    */
/* kprom, vprom (optional): [rows][max_pages] 1 for a promoted block;        */
/* nkey, nval, rank_fail (optional): per row.  row_mask as in oc_decode.     */
/* k_orig / v_orig element (b, h, t, ch) at b*seq_stride + h*head_stride +   */
/* t*tok_stride + ch (fp32, or bf16 bits when kv_is_f32 is 0).               */
/* ------------------------------------------------------------------------ */
typedef struct { double m; int b; } oc_blk;

static int oc_blk_cmp(const void* x, const void* y) {
  const oc_blk* a = (const oc_blk*)x;
  const oc_blk* b = (const oc_blk*)y;
  if (a->m > b->m) return -1;
  if (a->m < b->m) return 1;
  return (a->b > b->b) - (a->b < b->b);
}

int oc_decode_adaptive(const oc_cfg* c, const uint8_t* pool, const float* eta, const void* q,
                       int q_is_f32, int num_seqs, int nq, int hq, const int32_t* page_table,
                       int max_pages, const int32_t* seq_lens, float scale, float tau,
                       const int8_t* sigma, const void* k_orig, const void* v_orig,
                       int kv_is_f32, int64_t seq_stride, int64_t head_stride,
                       int64_t tok_stride, double tau_cov, double v_tol, double rank_tol,
                       double* out, double* bound, uint8_t* flags, uint8_t* kprom,
                       uint8_t* vprom, int32_t* nkey, int32_t* nval, uint8_t* rank_fail,
                       double* diag, const uint8_t* row_mask) {
  if (!oc_cfg_ok(c) || hq % c->hkv || (c->krotate && !sigma) || !k_orig || !v_orig)
    return OC_ERR_ARG;
  int d = c->d, G = hq / c->hkv;
  int64_t bb = oc_block_bytes(c);
  double sc = (double)scale;
  for (int b = 0; b < num_seqs; ++b) {
    int n = seq_lens[b];
    int npg = (n + OC_PAGE - 1) / OC_PAGE;
    double* z = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* dl = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* et = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* p = n ? (double*)malloc(sizeof(double) * n) : NULL;
    oc_blk* ord = npg ? (oc_blk*)malloc(sizeof(oc_blk) * npg) : NULL;
    uint8_t* kp = npg ? (uint8_t*)malloc(npg) : NULL;
    uint8_t* vp = npg ? (uint8_t*)malloc(npg) : NULL;
    for (int i = 0; i < nq; ++i)
      for (int h = 0; h < hq; ++h) {
        int64_t row = ((int64_t)b * nq + i) * hq + h;
        if (row_mask && !row_mask[row]) continue;
        int kv = h / G;
        double* o = out + row * d;
        for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
        if (kprom) memset(kprom + row * max_pages, 0, max_pages);
        if (vprom) memset(vprom + row * max_pages, 0, max_pages);
        if (nkey) nkey[row] = 0;
        if (nval) nval[row] = 0;
        if (rank_fail) rank_fail[row] = 0;
        if (n == 0) {
          bound[row] = 0.0;
          flags[row] = 0;
          if (diag) for (int t = 0; t < 8; ++t) diag[row * 8 + t] = 0.0;
          continue;
        }
        float qf[128], qr[128], kf[128], vf[128];
        const float* qp = oc_row_query(c, q, q_is_f32, row, sigma, qf, qr);
        double range, eta_max;
        oc_row_terms(c, pool, eta, qp, b, kv, n, page_table, max_pages, sc, z, dl, et, &range,
                     &eta_max);
        /* scoring pass: estimated block masses under the quantized softmax */
        double m = -INFINITY;
        for (int j = 0; j < n; ++j) if (z[j] > m) m = z[j];
        double l = 0.0;
        for (int j = 0; j < n; ++j) l += exp(z[j] - m);
        for (int lp = 0; lp < npg; ++lp) { ord[lp].m = 0.0; ord[lp].b = lp; }
        for (int j = 0; j < n; ++j) ord[j / OC_PAGE].m += exp(z[j] - m) / l;
        /* value promotion on the estimated masses (before the sort reorders them) */
        int nv = 0;
        for (int lp = 0; lp < npg; ++lp) {
          vp[lp] = ord[lp].m * et[lp * OC_PAGE] > v_tol ? 1 : 0;
          nv += vp[lp];
        }
        /* top-K* blocks covering tau_cov of the estimated mass */
        qsort(ord, npg, sizeof(oc_blk), oc_blk_cmp);
        int kstar = 0;
        double cum = 0.0;
        while (kstar < npg && cum < tau_cov) cum += ord[kstar++].m;
        for (int lp = 0; lp < npg; ++lp) kp[lp] = 0;
        for (int k = 0; k < kstar; ++k) kp[ord[k].b] = 1;
        /* mixed scores: originals in the key-promoted blocks */
        double qn2 = 0.0;
        for (int ch = 0; ch < d; ++ch) qn2 += (double)qf[ch] * (double)qf[ch];
        qn2 = sqrt(qn2);
        for (int j = 0; j < n; ++j) {
          if (!kp[j / OC_PAGE]) continue;
          oc_load_vec(k_orig, kv_is_f32, b * seq_stride + kv * head_stride + j * tok_stride, d,
                      kf);
          double dot = 0.0, kn2 = 0.0;
          for (int ch = 0; ch < d; ++ch) {
            dot += (double)qf[ch] * (double)kf[ch];
            kn2 += (double)kf[ch] * (double)kf[ch];
          }
          z[j] = sc * dot;
          dl[j] = OC_KAPPA * sc * OC_ROT_SLACK * qn2 * sqrt(kn2);
        }
        m = -INFINITY;
        for (int j = 0; j < n; ++j) if (z[j] > m) m = z[j];
        l = 0.0;
        for (int j = 0; j < n; ++j) l += exp(z[j] - m);
        for (int j = 0; j < n; ++j) p[j] = exp(z[j] - m) / l;
        /* output and bound */
        double A = 0.0, B = 0.0, Ev = 0.0, dmax = 0.0;
        double khat[128], ks[4], vhat[128], vs[4], vz[4], vtop[4];
        int kc, vc;
        for (int j = 0; j < n; ++j) {
          if (vp[j / OC_PAGE]) {
            oc_load_vec(v_orig, kv_is_f32, b * seq_stride + kv * head_stride + j * tok_stride,
                        d, vf);
            for (int ch = 0; ch < d; ++ch) o[ch] += p[j] * (double)vf[ch];
          } else {
            int page = page_table[(int64_t)b * max_pages + j / OC_PAGE];
            const uint8_t* blk = pool + ((int64_t)page * c->hkv + kv) * bb;
            oc_read_token(c, blk, j % OC_PAGE, khat, ks, vhat, vs, vz, vtop, &kc, &vc);
            for (int ch = 0; ch < d; ++ch) o[ch] += p[j] * vhat[ch];
            Ev += p[j] * et[j];
          }
          A += p[j] * expm1(dl[j]);
          B += p[j] * exp(-dl[j]);
          if (dl[j] > dmax) dmax = dl[j];
        }
        double tv = tanh(dmax / 2.0);
        if (A / B < tv) tv = A / B;
        double ekey = tv * (range + 2.0 * eta_max);
        double bd = OC_KAPPA * (ekey + Ev);
        /* ranking check over the key-promoted blocks, in selection order */
        int fail = 0;
        double lmin = INFINITY;
        for (int k = 0; k < kstar; ++k) {
          int lp = ord[k].b;
          int j0 = lp * OC_PAGE, j1 = j0 + OC_PAGE < n ? j0 + OC_PAGE : n;
          double s = 0.0;
          for (int j = j0; j < j1; ++j) s += exp(z[j] - m);
          double L = log(s) + m;
          if (L - lmin > rank_tol) fail = 1;
          if (L < lmin) lmin = L;
        }
        bound[row] = bd;
        flags[row] = (fail || bd > (double)tau) ? 1 : 0;
        if (kprom) for (int lp = 0; lp < npg; ++lp) kprom[row * max_pages + lp] = kp[lp];
        if (vprom) for (int lp = 0; lp < npg; ++lp) vprom[row * max_pages + lp] = vp[lp];
        if (nkey) nkey[row] = kstar;
        if (nval) nval[row] = nv;
        if (rank_fail) rank_fail[row] = (uint8_t)fail;
        if (diag) {
          double* dg = diag + row * 8;
          dg[0] = tv; dg[1] = ekey; dg[2] = Ev; dg[3] = dmax;
          dg[4] = A; dg[5] = B; dg[6] = range; dg[7] = eta_max;
        }
      }
    free(z); free(dl); free(et); free(p); free(ord); free(kp); free(vp);
  }
  return OC_OK;
}

/* ======================================================================== */
/* KQV codec ("Statistical Inference and Quality Measures of KV Cache       */
/* Quantisations Inspired by TurboQuant", Quantisation schemes: KQV).       */
/* K and V both get the randomized Walsh-Hadamard rotation (oc_rotate, one  */
/* sign vector sigma).  K takes the n-bit scalar MSE (Lloyd-Max) quantizer  */
/* of the rotated unit vector's coordinates; V takes the (n-1)-bit one plus */
/* the 1-bit QJL sketch of its residual.  Here n = 4.                       */
/* Readings (the pages give the scheme, not its arithmetic):                */
/*  - the coordinates of a rotated unit vector follow the page's             */
/*    Beta((d-1)/2, (d-1)/2) marginal on [-1, 1], which tends to N(0, 1/d);  */
/*    the codebook is the Lloyd-Max quantizer of N(0, 1) scaled by 1/sqrt(d) */
/*    (centroids c_i / sqrt(d), thresholds (c_i + c_{i+1}) / (2 sqrt(d)),    */
/*    computed in fp64 and rounded once to fp32);                            */
/*  - a vector's Euclidean norm |x'| is kept in fp32, u = x' / |x'| (u = 0   */
/*    for a zero vector); code = the number of thresholds strictly below u; */
/*  - QJL: S is a d x d matrix of N(0, 1) entries (an input, drawn from the  */
/*    seed); r = u - c_code; bit i = [sum_c S_ic r_c >= 0] (1 = +1, 0 = -1); */
/*    r~ = sqrt(pi/2)/d * |r| * S^T b, so v^' = |v'| (c_code + r~);          */
/*  - every dot product and squared norm is a sequential fmaf chain over     */
/*    c = 0 .. d-1 (the decisions of codes and bits depend on its rounding); */
/*  - the certified bound keeps the structure of oc_decode: Delta_j =        */
/*    kappa*s*(|q'|_1 eps_j + 2^-16 |q'|_2 |k_j|) with eps_j the token's     */
/*    largest |k' - k^'| (fp32, one ulp up); eta_b = the block's largest      */
/*    |v - v^| in the unrotated domain plus 2^-16 |v| (fp32 reconstruction   */
/*    allowance), one ulp up; the value range per 32-channel group from a   */
/*    per-block max / min of v^ that starts at 0 (a zeroed block).           */
/* Block of one (page, kv head), 16 tokens:                                   */
/*   [K codes u4 [16][d/2]][V codes u4 (3-bit) [16][d/2]][V sketch [16][d/8]] */
/*   [|k'| f32 [16]][eps f32 [16]][|v'| f32 [16]][|r| f32 [16]]              */
/*   [v^ max, min f32 [d/32][2]]                                             */
/* nibble of channel c in byte c/2, low nibble for even c; sketch bit i in   */
/* byte i/8, bit i%8 (least significant first).                              */
/* ======================================================================== */
typedef struct {
  int32_t d, hkv, num_pages;
} oq_cfg;

#define OQ_KBITS 4
#define OQ_VBITS 3
#define OQ_PI 3.14159265358979323846

static int oq_ok(const oq_cfg* c) {
  return c && (c->d == 64 || c->d == 128) && c->hkv > 0 && c->num_pages >= 0;
}
static int64_t oq_off_vc(const oq_cfg* c) { return (int64_t)OC_PAGE * c->d / 2; }
static int64_t oq_off_vs(const oq_cfg* c) { return (int64_t)OC_PAGE * c->d; }
static int64_t oq_off_kn(const oq_cfg* c) { return (int64_t)OC_PAGE * c->d + OC_PAGE * c->d / 8; }
static int64_t oq_off_ke(const oq_cfg* c) { return oq_off_kn(c) + 4 * OC_PAGE; }
static int64_t oq_off_vn(const oq_cfg* c) { return oq_off_kn(c) + 8 * OC_PAGE; }
static int64_t oq_off_vr(const oq_cfg* c) { return oq_off_kn(c) + 12 * OC_PAGE; }
static int64_t oq_off_rg(const oq_cfg* c) { return oq_off_kn(c) + 16 * OC_PAGE; }

int64_t oq_block_bytes(const oq_cfg* c) {
  if (!oq_ok(c)) return -1;
  return oq_off_rg(c) + (int64_t)(c->d / 32) * 2 * 4;
}

/* Lloyd-Max quantizer of N(0, 1) with 2^bits levels (ascending centroids
 * into c): Lloyd's iteration from evenly spaced positive centroids, using
 * the symmetric half.  A cell [a, b] (a >= 0) has centroid
 * (phi(a) - phi(b)) / (Q(a) - Q(b)), phi the density and Q(x) = P(X > x) =
 * erfc(x / sqrt 2) / 2; thresholds are midpoints, 0 in the middle.  Stops
 * when no centroid moves by more than 2^-52 of the largest.  Returns the
 * iterations taken. */
static double oq_phi(double x) { return isinf(x) ? 0.0 : exp(-0.5 * x * x) / sqrt(2.0 * OQ_PI); }
static double oq_tail(double x) { return isinf(x) ? 0.0 : 0.5 * erfc(x / sqrt(2.0)); }

int oq_lloyd_max(int bits, double* c) {
  if (bits < 1 || bits > 6) return OC_ERR_ARG;
  int n = (1 << bits) / 2;
  double p[32], t[33];
  for (int i = 0; i < n; ++i) p[i] = 3.0 * (i + 0.5) / n;
  int it;
  for (it = 1; it <= 1000000; ++it) {
    t[0] = 0.0;
    for (int i = 1; i < n; ++i) t[i] = 0.5 * (p[i - 1] + p[i]);
    t[n] = INFINITY;
    double move = 0.0;
    for (int i = 0; i < n; ++i) {
      double np = (oq_phi(t[i]) - oq_phi(t[i + 1])) / (oq_tail(t[i]) - oq_tail(t[i + 1]));
      if (fabs(np - p[i]) > move) move = fabs(np - p[i]);
      p[i] = np;
    }
    if (move <= ldexp(p[n - 1], -52)) break;
  }
  for (int i = 0; i < n; ++i) {
    c[n + i] = p[i];
    c[n - 1 - i] = -p[i];
  }
  return it;
}

/* fp32 tables for unit vectors in dimension d: cent[i] = c_i / sqrt(d),
 * thr[i] = (c_i + c_{i+1}) / (2 sqrt(d)) (i < 2^bits - 1). */
int oq_tables(int bits, int d, float* cent, float* thr) {
  double c[64];
  int r = oq_lloyd_max(bits, c);
  if (r < 0) return r;
  int L = 1 << bits;
  double sd = sqrt((double)d);
  for (int i = 0; i < L; ++i) cent[i] = (float)(c[i] / sd);
  for (int i = 0; i + 1 < L; ++i) thr[i] = (float)((c[i] + c[i + 1]) / (2.0 * sd));
  return OC_OK;
}

static float oq_dot(const float* a, const float* b, int n) {
  float s = 0.0f;
  for (int i = 0; i < n; ++i) s = fmaf(a[i], b[i], s);
  return s;
}

static int oq_code(float u, const float* thr, int L) {
  int k = 0;
  for (int i = 0; i + 1 < L; ++i) k += thr[i] < u;
  return k;
}

/* The QJL sketch of r (bits, d/8 bytes) and its estimate r~ (without the
 * |r| * sqrt(pi/2)/d factor when unit_scale is 0: sum_i S_ic b_i). */
void oq_qjl(const float* r, const float* S, int d, uint8_t* bits, float* rsum) {
  memset(bits, 0, (size_t)d / 8);
  for (int i = 0; i < d; ++i)
    if (oq_dot(S + (int64_t)i * d, r, d) >= 0.0f) bits[i / 8] |= (uint8_t)(1u << (i % 8));
  for (int ch = 0; ch < d; ++ch) {
    float acc = 0.0f;
    for (int i = 0; i < d; ++i) {
      float b = (bits[i / 8] >> (i % 8)) & 1u ? 1.0f : -1.0f;
      acc = fmaf(S[(int64_t)i * d + ch], b, acc);
    }
    rsum[ch] = acc;
  }
}

static void oq_wrf(uint8_t* p, float x) { memcpy(p, &x, 4); }
static float oq_rdf(const uint8_t* p) { float x; memcpy(&x, p, 4); return x; }

/* Quantize one token of one kv head into slot `slot`; returns its eta
 * contribution (one ulp up) and raises the block's v^ range. */
static int oq_quantize_token(const oq_cfg* c, uint8_t* blk, int slot, const float* k,
                             const float* v, const int8_t* sigma, const float* S,
                             const float* kcent, const float* kthr, const float* vcent,
                             const float* vthr, float* eta_out) {
  int d = c->d, rc = OC_OK;
  int LK = 1 << OQ_KBITS, LV = 1 << OQ_VBITS;
  float kr[128], vr[128], u[128], r[128], rs[128], vh[128], tmp[128];
  int8_t ones[128];
  for (int i = 0; i < d; ++i) ones[i] = 1;
  /* keys */
  oc_rotate(k, sigma, d, kr);
  float nk = sqrtf(oq_dot(kr, kr, d));
  if (!isfinite(nk)) { rc = OC_ERR_RANGE; nk = 0.0f; }
  float eps = 0.0f;
  uint8_t* kc = blk + (int64_t)slot * (d / 2);
  for (int ch = 0; ch < d; ++ch) {
    float uu = nk > 0.0f ? kr[ch] / nk : 0.0f;
    int code = oq_code(uu, kthr, LK);
    oc_put_nibble(kc, ch / 2, ch, (unsigned)code);
    float kh = nk * kcent[code];
    float e = fabsf(kr[ch] - kh);
    if (nk > 0.0f && e > eps) eps = e;
  }
  oq_wrf(blk + oq_off_kn(c) + 4 * slot, nk);
  oq_wrf(blk + oq_off_ke(c) + 4 * slot, nextafterf(eps, INFINITY));
  /* values */
  oc_rotate(v, sigma, d, vr);
  float nv = sqrtf(oq_dot(vr, vr, d));
  if (!isfinite(nv)) { rc = OC_ERR_RANGE; nv = 0.0f; }
  uint8_t* vc = blk + oq_off_vc(c) + (int64_t)slot * (d / 2);
  int code[128];
  for (int ch = 0; ch < d; ++ch) {
    u[ch] = nv > 0.0f ? vr[ch] / nv : 0.0f;
    code[ch] = oq_code(u[ch], vthr, LV);
    oc_put_nibble(vc, ch / 2, ch, (unsigned)code[ch]);
    r[ch] = u[ch] - vcent[code[ch]];
  }
  float rn = sqrtf(oq_dot(r, r, d));
  uint8_t* bits = blk + oq_off_vs(c) + (int64_t)slot * (d / 8);
  oq_qjl(r, S, d, bits, rs);
  oq_wrf(blk + oq_off_vn(c) + 4 * slot, nv);
  oq_wrf(blk + oq_off_vr(c) + 4 * slot, rn);
  /* reconstruction in the unrotated domain: v^ = sigma o (c H v^') */
  float rho = (float)(sqrt(OQ_PI / 2.0) / d) * rn;
  for (int ch = 0; ch < d; ++ch) tmp[ch] = nv * (vcent[code[ch]] + rho * rs[ch]);
  oc_rotate(tmp, ones, d, vh);
  float err = 0.0f;
  for (int ch = 0; ch < d; ++ch) {
    if (sigma[ch] < 0) vh[ch] = -vh[ch];
    float e = fabsf(v[ch] - vh[ch]);
    if (e > err) err = e;
  }
  if (rc != OC_OK) err = 0.0f;
  *eta_out = nextafterf(fmaf(1.0f / 65536.0f, nv, err), INFINITY);
  uint8_t* rg = blk + oq_off_rg(c);
  for (int g = 0; g < d / 32; ++g) {
    float hi = oq_rdf(rg + 8 * g), lo = oq_rdf(rg + 8 * g + 4);
    for (int ch = 32 * g; ch < 32 * g + 32; ++ch) {
      if (vh[ch] > hi) hi = vh[ch];
      if (vh[ch] < lo) lo = vh[ch];
    }
    oq_wrf(rg + 8 * g, hi);
    oq_wrf(rg + 8 * g + 4, lo);
  }
  return rc;
}

/* Quantize-on-append for the KQV codec; arguments as oc_append, plus the
 * QJL matrix S (fp32 [d][d], row i = projection i). */
int oq_append(const oq_cfg* c, uint8_t* pool, float* eta, const void* k, const void* v,
              int in_is_f32, int64_t seq_stride, int64_t head_stride, int64_t tok_stride,
              int num_seqs, int num_tokens, const int32_t* valid, const int32_t* page_table,
              int max_pages, const int32_t* start_pos, const int8_t* sigma, const float* S) {
  if (!oq_ok(c) || !sigma || !S) return OC_ERR_ARG;
  float kcent[16], kthr[15], vcent[8], vthr[7];
  oq_tables(OQ_KBITS, c->d, kcent, kthr);
  oq_tables(OQ_VBITS, c->d, vcent, vthr);
  int64_t bb = oq_block_bytes(c);
  int rc = OC_OK;
  float xk[128], xv[128];
  for (int b = 0; b < num_seqs; ++b) {
    int nt = valid ? valid[b] : num_tokens;
    for (int t = 0; t < nt; ++t) {
      int pos = start_pos[b] + t;
      int lp = pos / OC_PAGE;
      if (lp >= max_pages) return OC_ERR_ARG;
      int page = page_table[(int64_t)b * max_pages + lp];
      if (page < 0 || page >= c->num_pages) return OC_ERR_ARG;
      for (int h = 0; h < c->hkv; ++h) {
        int64_t off = b * seq_stride + h * head_stride + t * tok_stride;
        oc_load_vec(k, in_is_f32, off, c->d, xk);
        oc_load_vec(v, in_is_f32, off, c->d, xv);
        int bad = 0;
        for (int i = 0; i < c->d; ++i) bad |= !isfinite(xk[i]) || !isfinite(xv[i]);
        uint8_t* blk = pool + ((int64_t)page * c->hkv + h) * bb;
        float e;
        int r = oq_quantize_token(c, blk, pos % OC_PAGE, xk, xv, sigma, S, kcent, kthr, vcent,
                                  vthr, &e);
        if (r != OC_OK || bad) rc = OC_ERR_RANGE;
        float* ep = eta + (int64_t)page * c->hkv + h;
        if (e > *ep) *ep = e;
      }
    }
  }
  return rc;
}

/* Decode attention and its certified bound over a KQV cache, for every query
 * row (sequence b, query i, q head h; kv head h / (Hq/Hkv)), in fp64:
 *   q' = rotated q;  k^'_jc = |k_j| * cent4[code] (the fp32 product the
 *   append used);  z^_j = scale * q' . k^'_j
 *   v^'_jc = |v_j| (cent3[code] + sqrt(pi/2)/d |r_j| sum_i S_ic b_ji)
 *   o^ = sigma o (H sum_j p^_j v^'_j) / sqrt(d)      (unrotated)
 *   Delta_j = kappa*scale*(|q'|_1 eps_j + 2^-16 |q'|_2 |k_j|)
 *   A, B, TV as in oc_decode; range = max_g (max_b hi_{b,g} - min_b lo_{b,g})
 *   over the context's blocks; E_key = TV (range + 2 max eta); E_val =
 *   sum_j p^_j eta_{block(j)}; bound = kappa (E_key + E_val).
 * diag (optional) as in oc_decode. */
int oq_decode(const oq_cfg* c, const uint8_t* pool, const float* eta, const void* q,
              int q_is_f32, int num_seqs, int nq, int hq, const int32_t* page_table,
              int max_pages, const int32_t* seq_lens, float scale, float tau,
              const int8_t* sigma, const float* S, double* out, double* bound, uint8_t* flags,
              double* diag, const uint8_t* row_mask) {
  if (!oq_ok(c) || hq % c->hkv || !sigma || !S) return OC_ERR_ARG;
  int d = c->d, G = hq / c->hkv, NG = d / 32;
  float kcent[16], kthr[15], vcent[8], vthr[7];
  oq_tables(OQ_KBITS, d, kcent, kthr);
  oq_tables(OQ_VBITS, d, vcent, vthr);
  int64_t bb = oq_block_bytes(c);
  double sc = (double)scale, sd = sqrt((double)d);
  for (int b = 0; b < num_seqs; ++b) {
    int n = seq_lens[b];
    double* z = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* dl = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* vh = n ? (double*)malloc(sizeof(double) * n * d) : NULL;
    int vh_kv = -1;
    for (int h = 0; h < hq; ++h)     /* q heads outermost: the rows of one kv head together */
      for (int i = 0; i < nq; ++i) {
        int64_t row = ((int64_t)b * nq + i) * hq + h;
        if (row_mask && !row_mask[row]) continue;
        int kv = h / G;
        double* o = out + row * d;
        for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
        if (n == 0) {
          bound[row] = 0.0;
          flags[row] = 0;
          if (diag) for (int t = 0; t < 8; ++t) diag[row * 8 + t] = 0.0;
          continue;
        }
        float qf[128], qr[128];
        oc_load_vec(q, q_is_f32, row * d, d, qf);
        oc_rotate(qf, sigma, d, qr);
        double qn1 = 0.0, qn2 = 0.0;
        for (int ch = 0; ch < d; ++ch) {
          qn1 += fabs((double)qr[ch]);
          qn2 += (double)qr[ch] * (double)qr[ch];
        }
        qn2 = sqrt(qn2);
        double hi[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        double lo[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
        double eta_max = 0.0, m = -INFINITY;
        for (int j = 0; j < n; ++j) {
          int page = page_table[(int64_t)b * max_pages + j / OC_PAGE], slot = j % OC_PAGE;
          const uint8_t* blk = pool + ((int64_t)page * c->hkv + kv) * bb;
          float nk = oq_rdf(blk + oq_off_kn(c) + 4 * slot);
          double dot = 0.0;
          for (int ch = 0; ch < d; ++ch) {
            unsigned code = oc_get_nibble(blk + (int64_t)slot * (d / 2), ch / 2, ch);
            dot += (double)qr[ch] * (double)(nk * kcent[code]);
          }
          z[j] = sc * dot;
          dl[j] = OC_KAPPA * sc * (qn1 * (double)oq_rdf(blk + oq_off_ke(c) + 4 * slot) +
                                   OC_ROT_SLACK * qn2 * (double)nk);
          if (z[j] > m) m = z[j];
          if (slot == 0 || j == 0) {   /* each block of the context once */
            const uint8_t* rg = blk + oq_off_rg(c);
            for (int g = 0; g < NG; ++g) {
              if (oq_rdf(rg + 8 * g) > hi[g]) hi[g] = oq_rdf(rg + 8 * g);
              if (oq_rdf(rg + 8 * g + 4) < lo[g]) lo[g] = oq_rdf(rg + 8 * g + 4);
            }
            double e = (double)eta[(int64_t)page * c->hkv + kv];
            if (e > eta_max) eta_max = e;
          }
        }
        double l = 0.0;
        for (int j = 0; j < n; ++j) l += exp(z[j] - m);
        /* the rotated reconstructions v^'_j of this (sequence, kv head), once for
         * the rows that share them */
        if (kv != vh_kv) {
          for (int j = 0; j < n; ++j) {
            int page = page_table[(int64_t)b * max_pages + j / OC_PAGE], slot = j % OC_PAGE;
            const uint8_t* blk = pool + ((int64_t)page * c->hkv + kv) * bb;
            double nv = oq_rdf(blk + oq_off_vn(c) + 4 * slot);
            double rho = sqrt(OQ_PI / 2.0) / d * (double)oq_rdf(blk + oq_off_vr(c) + 4 * slot);
            const uint8_t* bits = blk + oq_off_vs(c) + (int64_t)slot * (d / 8);
            for (int ch = 0; ch < d; ++ch) {
              unsigned code = oc_get_nibble(blk + oq_off_vc(c) + (int64_t)slot * (d / 2), ch / 2, ch);
              double s = 0.0;
              for (int ii = 0; ii < d; ++ii)
                s += ((bits[ii / 8] >> (ii % 8)) & 1u ? 1.0 : -1.0) * (double)S[(int64_t)ii * d + ch];
              vh[(int64_t)j * d + ch] = nv * ((double)vcent[code] + rho * s);
            }
          }
          vh_kv = kv;
        }
        double A = 0.0, B = 0.0, Ev = 0.0, dmax = 0.0, op[128];
        for (int ch = 0; ch < d; ++ch) op[ch] = 0.0;
        for (int j = 0; j < n; ++j) {
          double p = exp(z[j] - m) / l;
          int page = page_table[(int64_t)b * max_pages + j / OC_PAGE];
          for (int ch = 0; ch < d; ++ch) op[ch] += p * vh[(int64_t)j * d + ch];
          A += p * expm1(dl[j]);
          B += p * exp(-dl[j]);
          Ev += p * (double)eta[(int64_t)page * c->hkv + kv];
          if (dl[j] > dmax) dmax = dl[j];
        }
        /* o = sigma o (H op) / sqrt(d), fp64 butterflies */
        for (int hh = 1; hh < d; hh *= 2)
          for (int i0 = 0; i0 < d; i0 += 2 * hh)
            for (int jj = i0; jj < i0 + hh; ++jj) {
              double a = op[jj], bq = op[jj + hh];
              op[jj] = a + bq;
              op[jj + hh] = a - bq;
            }
        for (int ch = 0; ch < d; ++ch) o[ch] = (sigma[ch] < 0 ? -op[ch] : op[ch]) / sd;
        double range = 0.0;
        for (int g = 0; g < NG; ++g)
          if (hi[g] - lo[g] > range) range = hi[g] - lo[g];
        double tv = tanh(dmax / 2.0);
        if (A / B < tv) tv = A / B;
        double ekey = tv * (range + 2.0 * eta_max);
        double bd = OC_KAPPA * (ekey + Ev);
        bound[row] = bd;
        flags[row] = bd > (double)tau ? 1 : 0;
        if (diag) {
          double* dg = diag + row * 8;
          dg[0] = tv; dg[1] = ekey; dg[2] = Ev; dg[3] = dmax;
          dg[4] = A; dg[5] = B; dg[6] = range; dg[7] = eta_max;
        }
      }
    free(z);
    free(dl);
    free(vh);
  }
  return OC_OK;
}

/* ======================================================================== */
/* HQMQ codec ("Hurwitz Quaternion Multiplicative Quantization for KV Cache */
/* Compression", Method 1-2).  Every 4-channel chunk x of a K or V vector   */
/* is a quaternion (x0 + x1 i + x2 j + x3 k) split into its radius r = |x|  */
/* and its direction on S^3; the direction is coded by the product         */
/* codebook C = { q_p q_s : q_p in 2T, q_s in the secondary set } (24 S    */
/* codewords), the radius is stored in 8 bits.                              */
/* Readings (the page gives the structure, not the arithmetic):            */
/*  - 2T, the 24 Hurwitz units, in the order p = 0..7: +-1, +-i, +-j, +-k   */
/*    (p = 2n + [negative], n the axis), p = 8..23: (+-1 +-i +-j +-k)/2     */
/*    with component n negative when bit n of p - 8 is set;                 */
/*  - the secondary set: S unit quaternions per (kv head, role), an input   */
/*    (drawn from the seed), fp32 [hkv][2][S][4], role 0 = K, 1 = V;        */
/*  - codeword i = 24 s + p is the Hamilton product q_p q_s in fp32: each   */
/*    component is the 4-term signed sum of the products (exact: q_p's      */
/*    entries are 0, +-1, +-1/2) added left to right, each add rounded;     */
/*  - the direction's code maximizes <x, c> (equivalently <x/r, c>, r > 0). */
/*    The inner products are taken through the group: <x, q_p q_s> =        */
/*    <x conj(q_s), q_p>; y = x conj(q_s) has each component a sequential  */
/*    fmaf chain over x0..x3; over the 8 axis units the best is max_n |y_n| */
/*    (the first n on ties, sign of y_n), over the 16 half units it is      */
/*    0.5 (((|y0| + |y1|) + |y2|) + |y3|) with the signs of y (-0 as +);    */
/*    the half unit wins over the axis one only when strictly larger, and a */
/*    later s only when strictly larger than every earlier candidate;       */
/*  - r = sqrt((x0^2 + x1^2) + (x2^2 + x3^2)) in fp32 (the Med3x chunk      */
/*    norm); stored as fp8 E4M3 (round to nearest, ties to even; above 448  */
/*    it saturates to 448); a chunk with a non-finite norm gets code 0 and  */
/*    radius 0; a token with a non-finite K or V value sets the range error */
/*    and gets eps = eta = +inf (K) or eta = +inf (V), so every query over  */
/*    its block is flagged;                                                  */
/*  - the reconstruction takes the codeword rounded to fp16 (nearest, ties  */
/*    to even), c16: x^ = r^ * c16, exact in fp32 (4 and 11 significant    */
/*    bits);                                                                 */
/*  - per token: |k|_2 (sequential fmaf chain) and eps = |k - k^|_2 (the    */
/*    same chain over the channels' differences) raised by 2^-16 of itself, */
/*    one ulp up; the bound's Delta_j = kappa*s*|q|_2 (eps_j + 2^-16 |k_j|);*/
/*  - eta_b = the block's largest max_c |v - v^| + 2^-16 |v|_2, one ulp up; */
/*    the value range per 32-channel group starts at [0, 0] (a zeroed      */
/*    block) and widens to every v^ appended;                                */
/*  - with Med3x extraction (Method 3, the page's combination for           */
/*    outlier-heavy models; outliers = 1): the chunk oc_med3_chunk picks in */
/*    K and in V is kept in fp16 (R32's rules) in the Tier-1 outlier        */
/*    section appended to the block, takes code 0 and radius 0, and         */
/*    reconstructs to its fp16 values; eps, eta and the range are measured  */
/*    on that reconstruction.                                                */
/* Block of one (page, kv head), 16 tokens, d/4 chunks per vector, chunk-   */
/* major (the 16 tokens of one chunk side by side):                         */
/*   [K codes u16 [d/4][16]][V codes u16 [d/4][16]][K radii e4m3 [d/4][16]]  */
/*   [V radii e4m3 [d/4][16]][|k| f32 [16]][eps f32 [16]]                    */
/*   [v^ max, min f32 [d/32][2]]                                             */
/*   (outliers = 1) [chunk K u8 [16]][chunk V u8 [16]][k16 f16 [16][4]]      */
/*   [v16 f16 [16][4]] (0xFF: none; the values zero then)                    */
/* u16 little-endian.                                                        */
/* ======================================================================== */
typedef struct {
  int32_t d, hkv, num_pages, S, outliers;
} oh_cfg;

#define OH_MAX_S 2730   /* 24 S codewords index in 16 bits */

static int oh_ok(const oh_cfg* c) {
  return c && (c->d == 64 || c->d == 128) && c->hkv > 0 && c->num_pages >= 0 && c->S >= 1 &&
         c->S <= OH_MAX_S && (c->outliers == 0 || c->outliers == 1);
}
static int64_t oh_off_vi(const oh_cfg* c) { return (int64_t)OC_PAGE * (c->d / 4) * 2; }
static int64_t oh_off_kr(const oh_cfg* c) { return (int64_t)OC_PAGE * (c->d / 4) * 4; }
static int64_t oh_off_vr(const oh_cfg* c) { return oh_off_kr(c) + (int64_t)OC_PAGE * (c->d / 4); }
static int64_t oh_off_kn(const oh_cfg* c) { return oh_off_vr(c) + (int64_t)OC_PAGE * (c->d / 4); }
static int64_t oh_off_ke(const oh_cfg* c) { return oh_off_kn(c) + 4 * OC_PAGE; }
static int64_t oh_off_rg(const oh_cfg* c) { return oh_off_kn(c) + 8 * OC_PAGE; }

static int64_t oh_off_out(const oh_cfg* c) { return oh_off_rg(c) + (int64_t)(c->d / 32) * 2 * 4; }

int64_t oh_block_bytes(const oh_cfg* c) {
  if (!oh_ok(c)) return -1;
  return oh_off_out(c) + (c->outliers ? OC_OUT_BYTES : 0);
}

/* Unit p of 2T (Method 1: the 24 vertices of the 24-cell). */
void oh_primary(int p, float* q) {
  for (int n = 0; n < 4; ++n) q[n] = 0.0f;
  if (p < 8) {
    q[p / 2] = (p & 1) ? -1.0f : 1.0f;
  } else {
    for (int n = 0; n < 4; ++n) q[n] = ((p - 8) >> n) & 1 ? -0.5f : 0.5f;
  }
}

/* Hamilton product a b with exact term products (a from 2T), each component
 * summed left to right in fp32. */
static void oh_mul(const float* a, const float* b, float* c) {
  float t[4][4] = {
      {a[0] * b[0], -(a[1] * b[1]), -(a[2] * b[2]), -(a[3] * b[3])},
      {a[0] * b[1], a[1] * b[0], a[2] * b[3], -(a[3] * b[2])},
      {a[0] * b[2], -(a[1] * b[3]), a[2] * b[0], a[3] * b[1]},
      {a[0] * b[3], a[1] * b[2], -(a[2] * b[1]), a[3] * b[0]},
  };
  for (int n = 0; n < 4; ++n) c[n] = ((t[n][0] + t[n][1]) + t[n][2]) + t[n][3];
}

/* Codeword i = 24 s + p of one secondary set (sec: [S][4]). */
void oh_codeword(const float* sec, int i, float* c) {
  float qp[4];
  oh_primary(i % 24, qp);
  oh_mul(qp, sec + 4 * (i / 24), c);
}

/* Codeword i with every component rounded to fp16 (the reconstruction's). */
void oh_codeword16(const float* sec, int i, float* c) {
  oh_codeword(sec, i, c);
  for (int n = 0; n < 4; ++n) c[n] = (float)oc_f16_value(oc_f16_rn(c[n]));
}

/* The direction code of chunk x (Method 1: the codeword of largest inner
 * product), through y = x conj(q_s) as the readings above fix. */
int oh_direction(const float* x, const float* sec, int S) {
  int best = 0;
  float bv = -INFINITY;
  for (int s = 0; s < S; ++s) {
    const float* b = sec + 4 * s;
    float y[4];
    y[0] = fmaf(x[3], b[3], fmaf(x[2], b[2], fmaf(x[1], b[1], x[0] * b[0])));
    y[1] = fmaf(x[3], b[2], fmaf(-x[2], b[3], fmaf(x[1], b[0], -x[0] * b[1])));
    y[2] = fmaf(-x[3], b[1], fmaf(x[2], b[0], fmaf(x[1], b[3], -x[0] * b[2])));
    y[3] = fmaf(x[3], b[0], fmaf(x[2], b[1], fmaf(-x[1], b[2], -x[0] * b[3])));
    float a[4];
    for (int n = 0; n < 4; ++n) a[n] = fabsf(y[n]);
    int n0 = 0;
    for (int n = 1; n < 4; ++n)
      if (a[n] > a[n0]) n0 = n;
    float v = a[n0];
    int p = 2 * n0 + (y[n0] < 0.0f);
    float h = 0.5f * (((a[0] + a[1]) + a[2]) + a[3]);
    if (h > v) {
      v = h;
      p = 8;
      for (int n = 0; n < 4; ++n) p += (y[n] < 0.0f) << n;
    }
    if (v > bv) {
      bv = v;
      best = 24 * s + p;
    }
  }
  return best;
}

/* fp8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 * infinities, 0x7F NaN): the value of a non-negative code, and the code of a
 * non-negative finite x rounded to nearest, ties to the even code, saturating
 * at 448 (0x7E). */
double oh_e4m3_value(uint8_t code) {
  int e = (code >> 3) & 15, m = code & 7;
  double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return (code & 0x80) ? -v : v;
}

uint8_t oh_e4m3_rn(float x) {
  double xv = (double)x;
  if (!(xv > 0.0)) return 0;
  if (xv >= 448.0) return 0x7E;
  int lo = 0;
  while (lo + 1 <= 0x7E && oh_e4m3_value((uint8_t)(lo + 1)) <= xv) ++lo;
  if (oh_e4m3_value((uint8_t)lo) == xv) return (uint8_t)lo;
  double dl = xv - oh_e4m3_value((uint8_t)lo), du = oh_e4m3_value((uint8_t)(lo + 1)) - xv;
  if (dl < du) return (uint8_t)lo;
  if (du < dl) return (uint8_t)(lo + 1);
  return (uint8_t)((lo & 1) ? lo + 1 : lo);
}

static float oh_chunk_radius(const float* x) {
  float a = x[0] * x[0], b = x[1] * x[1], e = x[2] * x[2], f = x[3] * x[3];
  return sqrtf((a + b) + (e + f));
}

/* Code one d-vector x: chunk codes (u16, chunk ch at idx + 2 * 16 ch) and
 * radii (at rad + 16 ch), and the fp32 reconstruction; chunk `skip` (an
 * extracted one, or -1) takes code 0 and radius 0. */
static int oh_code_vector(const float* x, int d, const float* sec, int S, uint8_t* idx,
                          uint8_t* rad, float* xh, int skip) {
  int rc = OC_OK;
  for (int ch = 0; ch < d / 4; ++ch) {
    const float* xc = x + 4 * ch;
    float r = oh_chunk_radius(xc);
    int i = 0;
    uint8_t rq = 0;
    if (ch == skip) {
      /* kept in fp16 by the caller */
    } else if (!isfinite(r)) {
      rc = OC_ERR_RANGE;
    } else {
      i = oh_direction(xc, sec, S);
      rq = oh_e4m3_rn(r);
    }
    oc_wr16(idx + 2 * OC_PAGE * ch, (uint16_t)i);
    rad[OC_PAGE * ch] = rq;
    float cw[4];
    oh_codeword16(sec, i, cw);
    float rv = (float)oh_e4m3_value(rq);
    for (int n = 0; n < 4; ++n) xh[4 * ch + n] = rv * cw[n];
  }
  return rc;
}

static float oh_chain_norm2(const float* a, int d) {
  float s = 0.0f;
  for (int i = 0; i < d; ++i) s = fmaf(a[i], a[i], s);
  return s;
}

/* Quantize one token of one kv head into slot `slot` (secs: this kv head's
 * [2][S][4]); returns its eta contribution and raises the block's range. */
static int oh_quantize_token(const oh_cfg* c, uint8_t* blk, int slot, const float* k,
                             const float* v, const float* secs, float* eta_out) {
  int d = c->d, S = c->S;
  float kh[128], vh[128], e[128];
  int ck = c->outliers ? oc_med3_chunk(k, d) : -1;
  int cv = c->outliers ? oc_med3_chunk(v, d) : -1;
  int rc = oh_code_vector(k, d, secs, S, blk + 2 * slot, blk + oh_off_kr(c) + slot, kh, ck);
  int rv = oh_code_vector(v, d, secs + 4 * S, S, blk + oh_off_vi(c) + 2 * slot,
                          blk + oh_off_vr(c) + slot, vh, cv);
  if (rv != OC_OK) rc = rv;
  if (c->outliers) {   /* the extracted chunks in fp16 (R32), their reconstruction */
    uint8_t* os = blk + oh_off_out(c);
    os[slot] = ck < 0 ? OC_NO_OUTLIER : (uint8_t)ck;
    os[OC_PAGE + slot] = cv < 0 ? OC_NO_OUTLIER : (uint8_t)cv;
    for (int role = 0; role < 2; ++role) {
      int cx = role ? cv : ck;
      const float* x = role ? v : k;
      float* xh = role ? vh : kh;
      for (int i = 0; i < 4; ++i) {
        uint16_t h = 0;
        if (cx >= 0) {
          float xi = x[4 * cx + i];
          if (!isfinite(xi) || fabsf(xi) > 65504.0f) rc = OC_ERR_RANGE;
          else h = oc_f16_rn(xi);
          xh[4 * cx + i] = (float)oc_f16_value(h);
        }
        oc_wr16(os + 2 * OC_PAGE + role * OC_PAGE * 8 + (slot * 4 + i) * 2, h);
      }
    }
  }
  int bad_k = 0, bad_v = 0;
  for (int i = 0; i < d; ++i) {
    bad_k |= !isfinite(k[i]);
    bad_v |= !isfinite(v[i]);
  }
  float nk = sqrtf(oh_chain_norm2(k, d));
  for (int i = 0; i < d; ++i) e[i] = k[i] - kh[i];
  float en = sqrtf(oh_chain_norm2(e, d));
  float eps = bad_k ? INFINITY : nextafterf(fmaf(en, 1.0f / 65536.0f, en), INFINITY);
  oq_wrf(blk + oh_off_kn(c) + 4 * slot, nk);
  oq_wrf(blk + oh_off_ke(c) + 4 * slot, eps);
  float err = 0.0f;
  for (int i = 0; i < d; ++i) {
    float ev = fabsf(v[i] - vh[i]);
    if (ev > err) err = ev;
  }
  float nv = sqrtf(oh_chain_norm2(v, d));
  *eta_out = bad_k || bad_v ? INFINITY : nextafterf(fmaf(1.0f / 65536.0f, nv, err), INFINITY);
  uint8_t* rg = blk + oh_off_rg(c);
  for (int g = 0; g < d / 32; ++g) {
    float hi = oq_rdf(rg + 8 * g), lo = oq_rdf(rg + 8 * g + 4);
    for (int ch = 32 * g; ch < 32 * g + 32; ++ch) {
      if (vh[ch] > hi) hi = vh[ch];
      if (vh[ch] < lo) lo = vh[ch];
    }
    oq_wrf(rg + 8 * g, hi);
    oq_wrf(rg + 8 * g + 4, lo);
  }
  return rc;
}

/* Quantize-on-append for the HQMQ codec; arguments as oc_append, plus the
 * secondary sets sec (fp32 [hkv][2][S][4]). */
int oh_append(const oh_cfg* c, uint8_t* pool, float* eta, const void* k, const void* v,
              int in_is_f32, int64_t seq_stride, int64_t head_stride, int64_t tok_stride,
              int num_seqs, int num_tokens, const int32_t* valid, const int32_t* page_table,
              int max_pages, const int32_t* start_pos, const float* sec) {
  if (!oh_ok(c) || !sec) return OC_ERR_ARG;
  int64_t bb = oh_block_bytes(c);
  int rc = OC_OK;
  float xk[128], xv[128];
  for (int b = 0; b < num_seqs; ++b) {
    int nt = valid ? valid[b] : num_tokens;
    for (int t = 0; t < nt; ++t) {
      int pos = start_pos[b] + t;
      int lp = pos / OC_PAGE;
      if (lp >= max_pages) return OC_ERR_ARG;
      int page = page_table[(int64_t)b * max_pages + lp];
      if (page < 0 || page >= c->num_pages) return OC_ERR_ARG;
      for (int h = 0; h < c->hkv; ++h) {
        int64_t off = b * seq_stride + h * head_stride + t * tok_stride;
        oc_load_vec(k, in_is_f32, off, c->d, xk);
        oc_load_vec(v, in_is_f32, off, c->d, xv);
        int bad = 0;
        for (int i = 0; i < c->d; ++i) bad |= !isfinite(xk[i]) || !isfinite(xv[i]);
        uint8_t* blk = pool + ((int64_t)page * c->hkv + h) * bb;
        float e;
        int r = oh_quantize_token(c, blk, pos % OC_PAGE, xk, xv, sec + (int64_t)h * 8 * c->S, &e);
        if (r != OC_OK || bad) rc = OC_ERR_RANGE;
        float* ep = eta + (int64_t)page * c->hkv + h;
        if (e > *ep) *ep = e;
      }
    }
  }
  return rc;
}

/* Read back token `slot` of a block: k^ and v^ as the append reconstructed
 * them (r^ * c16). */
void oh_read_token(const oh_cfg* c, const uint8_t* blk, int slot, const float* secs, float* kh,
                   float* vh) {
  int nc = c->d / 4;
  for (int role = 0; role < 2; ++role) {
    const uint8_t* idx = blk + (role ? oh_off_vi(c) : 0) + 2 * slot;
    const uint8_t* rad = blk + (role ? oh_off_vr(c) : oh_off_kr(c)) + slot;
    float* out = role ? vh : kh;
    for (int ch = 0; ch < nc; ++ch) {
      float cw[4];
      oh_codeword16(secs + role * 4 * c->S, oc_rd16(idx + 2 * OC_PAGE * ch), cw);
      float rv = (float)oh_e4m3_value(rad[OC_PAGE * ch]);
      for (int n = 0; n < 4; ++n) out[4 * ch + n] = rv * cw[n];
    }
    if (c->outliers) {   /* an extracted chunk reads back its fp16 values */
      const uint8_t* os = blk + oh_off_out(c);
      int cx = os[role * OC_PAGE + slot];
      if (cx != OC_NO_OUTLIER && cx < nc)
        for (int n = 0; n < 4; ++n)
          out[4 * cx + n] =
              (float)oc_f16_value(oc_rd16(os + 2 * OC_PAGE + role * OC_PAGE * 8 + (slot * 4 + n) * 2));
    }
  }
}

/* Decode attention and its certified bound over an HQMQ cache, for every
 * query row (sequence b, query i, q head h; kv head h / (Hq/Hkv)), in fp64
 * over the fp32 reconstructions:
 *   z^_j = scale * q . k^_j;  o^ = sum_j p^_j v^_j
 *   Delta_j = kappa*scale*|q|_2 (eps_j + 2^-16 |k_j|)
 *   A, B, TV, range, E_key, E_val, bound and flag as in oq_decode.
 * diag (optional) as in oc_decode. */
int oh_decode(const oh_cfg* c, const uint8_t* pool, const float* eta, const void* q,
              int q_is_f32, int num_seqs, int nq, int hq, const int32_t* page_table,
              int max_pages, const int32_t* seq_lens, float scale, float tau, const float* sec,
              double* out, double* bound, uint8_t* flags, double* diag,
              const uint8_t* row_mask) {
  if (!oh_ok(c) || hq % c->hkv || !sec) return OC_ERR_ARG;
  int d = c->d, G = hq / c->hkv, NG = d / 32;
  int64_t bb = oh_block_bytes(c);
  double sc = (double)scale;
  for (int b = 0; b < num_seqs; ++b) {
    int n = seq_lens[b];
    double* z = n ? (double*)malloc(sizeof(double) * n) : NULL;
    double* dl = n ? (double*)malloc(sizeof(double) * n) : NULL;
    float* kh = n ? (float*)malloc(sizeof(float) * n * d) : NULL;
    float* vh = n ? (float*)malloc(sizeof(float) * n * d) : NULL;
    int cur_kv = -1;
    for (int h = 0; h < hq; ++h)
      for (int i = 0; i < nq; ++i) {
        int64_t row = ((int64_t)b * nq + i) * hq + h;
        if (row_mask && !row_mask[row]) continue;
        int kv = h / G;
        double* o = out + row * d;
        for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
        if (n == 0) {
          bound[row] = 0.0;
          flags[row] = 0;
          if (diag) for (int t = 0; t < 8; ++t) diag[row * 8 + t] = 0.0;
          continue;
        }
        if (kv != cur_kv) {   /* the reconstructions of this (sequence, kv head) */
          for (int j = 0; j < n; ++j) {
            int page = page_table[(int64_t)b * max_pages + j / OC_PAGE];
            const uint8_t* blk = pool + ((int64_t)page * c->hkv + kv) * bb;
            oh_read_token(c, blk, j % OC_PAGE, sec + (int64_t)kv * 8 * c->S,
                          kh + (int64_t)j * d, vh + (int64_t)j * d);
          }
          cur_kv = kv;
        }
        float qf[128];
        oc_load_vec(q, q_is_f32, row * d, d, qf);
        double qn2 = 0.0;
        for (int ch = 0; ch < d; ++ch) qn2 += (double)qf[ch] * (double)qf[ch];
        qn2 = sqrt(qn2);
        double hi[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        double lo[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
        double eta_max = 0.0, m = -INFINITY;
        for (int j = 0; j < n; ++j) {
          int page = page_table[(int64_t)b * max_pages + j / OC_PAGE], slot = j % OC_PAGE;
          const uint8_t* blk = pool + ((int64_t)page * c->hkv + kv) * bb;
          double dot = 0.0;
          for (int ch = 0; ch < d; ++ch) dot += (double)qf[ch] * (double)kh[(int64_t)j * d + ch];
          z[j] = sc * dot;
          dl[j] = OC_KAPPA * sc * qn2 *
                  ((double)oq_rdf(blk + oh_off_ke(c) + 4 * slot) +
                   OC_ROT_SLACK * (double)oq_rdf(blk + oh_off_kn(c) + 4 * slot));
          if (z[j] > m) m = z[j];
          if (slot == 0 || j == 0) {   /* each block of the context once */
            const uint8_t* rg = blk + oh_off_rg(c);
            for (int g = 0; g < NG; ++g) {
              if (oq_rdf(rg + 8 * g) > hi[g]) hi[g] = oq_rdf(rg + 8 * g);
              if (oq_rdf(rg + 8 * g + 4) < lo[g]) lo[g] = oq_rdf(rg + 8 * g + 4);
            }
            double e = (double)eta[(int64_t)page * c->hkv + kv];
            if (e > eta_max) eta_max = e;
          }
        }
        double l = 0.0;
        for (int j = 0; j < n; ++j) l += exp(z[j] - m);
        double A = 0.0, B = 0.0, Ev = 0.0, dmax = 0.0;
        for (int j = 0; j < n; ++j) {
          double p = exp(z[j] - m) / l;
          int page = page_table[(int64_t)b * max_pages + j / OC_PAGE];
          for (int ch = 0; ch < d; ++ch) o[ch] += p * (double)vh[(int64_t)j * d + ch];
          A += p * expm1(dl[j]);
          B += p * exp(-dl[j]);
          Ev += p * (double)eta[(int64_t)page * c->hkv + kv];
          if (dl[j] > dmax) dmax = dl[j];
        }
        double range = 0.0;
        for (int g = 0; g < NG; ++g)
          if (hi[g] - lo[g] > range) range = hi[g] - lo[g];
        double tv = tanh(dmax / 2.0);
        if (A / B < tv) tv = A / B;
        double ekey = tv * (range + 2.0 * eta_max);
        double bd = OC_KAPPA * (ekey + Ev);
        bound[row] = bd;
        flags[row] = bd > (double)tau ? 1 : 0;
        if (diag) {
          double* dg = diag + row * 8;
          dg[0] = tv; dg[1] = ekey; dg[2] = Ev; dg[3] = dmax;
          dg[4] = A; dg[5] = B; dg[6] = range; dg[7] = eta_max;
        }
      }
    free(z);
    free(dl);
    free(kh);
    free(vh);
  }
  return OC_OK;
}
