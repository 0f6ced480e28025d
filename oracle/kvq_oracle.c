/*
 * kvq_oracle.c -- plain, slow CPU oracle for KV-cache rotation + low-bit
 * quantization (encode), its inverse (decode) and the decode-step q.K^T score.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference legs load this library. It shares no
 * code, header, table or constant generator with the CUDA library, and it
 * includes nothing from it.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no FMA contraction: every fused multiply-add below is an explicit fmaf()).
 *
 * Pages cited (title, then section / equation / code block):
 *   [RoPE-KV]  "RoPE启发的KV缓存压缩技术解析"
 *   [EliteKV]  "EliteKV - RoPE频率选择与低秩投影"
 *   [IsoQuant] "KV缓存压缩技术：IsoQuant在大语言模型中的应用"
 *   [RotateKV] "RotateKV: Accurate and Robust 2-Bit KV Cache Quantization for
 *               LLMs via Outlier-Aware Adaptive Rotations"
 *
 * Precision. The encode path decides integer codes, so it runs in fp32 -- the
 * precision of the kernels -- with one fixed operation order (stated at each
 * function); that is what lets codes and fp16 scale/zero be compared bit for
 * bit. Decode and score are computed in fp64 from the stored codes and are
 * compared against the kernels with a tolerance.
 *
 * Every function here is pinned by tests/test_oracle_*.py against closed
 * forms, brute force, textbook constants and invariants (see the pins named
 * at each function). The Lloyd-Max codebook uses numbers printed in Max's
 * 1960 table; no other constant is taken from anywhere but the pages.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_ROT_NONE 0
#define ORC_ROT_FWHT_HEAD 1
#define ORC_ROT_FWHT_GROUP 2
#define ORC_ROT_ISO 3
#define ORC_ROT_ISO3 4
#define ORC_Q_MINMAX 0
#define ORC_Q_CODEBOOK 1

/* ------------------------------------------------------------------------
 * IEEE binary16 <-> binary32.  Pins: exhaustive round trip of all 65536
 * half patterns, numpy float16 for round-to-nearest, brute-force neighbour
 * search for the directed roundings.
 * ---------------------------------------------------------------------- */
float orc_half_to_float(uint16_t h) {
  int sign = (h >> 15) & 1, ex = (h >> 10) & 0x1f, man = h & 0x3ff;
  float v;
  if (ex == 0)
    v = ldexpf((float)man, -24); /* zero and subnormals: man * 2^-24 */
  else if (ex == 31)
    v = man ? NAN : INFINITY;
  else
    v = ldexpf((float)(man | 0x400), ex - 25); /* 1.man * 2^(ex-15) */
  return sign ? -v : v;
}

/* encode a non-negative value that is exactly representable as a half */
static uint16_t exact_half_bits(double r) {
  if (r == 0.0) return 0;
  if (r < ldexp(1.0, -14)) return (uint16_t)(r / ldexp(1.0, -24)); /* subnormal */
  int e;
  frexp(r, &e); /* r = f * 2^e, f in [0.5, 1) -> r in [2^(e-1), 2^e) */
  int E = e - 1;
  uint16_t man = (uint16_t)((r / ldexp(1.0, E) - 1.0) * 1024.0);
  return (uint16_t)(((E + 15) << 10) | man);
}

uint16_t orc_float_to_half_rn(float f) {
  if (isnan(f)) return 0x7e00;
  uint16_t sign = signbit(f) ? 0x8000 : 0;
  double a = fabs((double)f);
  /* 65520 is the midpoint between 65504 (odd mantissa) and 2^16: ties go to
     the even neighbour, which is infinity. */
  if (a >= 65520.0) return sign | 0x7c00;
  double quantum;
  if (a < ldexp(1.0, -14)) {
    quantum = ldexp(1.0, -24);
  } else {
    int e;
    frexp(a, &e);
    quantum = ldexp(1.0, e - 1 - 10); /* 10 fraction bits */
  }
  double n = nearbyint(a / quantum); /* a/quantum is exact; ties to even */
  return sign | exact_half_bits(n * quantum);
}

static uint16_t half_next_up(uint16_t h) {
  if ((h & 0x7fff) == 0) return 0x0001;          /* +-0 -> smallest subnormal */
  if (h & 0x8000) return (uint16_t)(h - 1);       /* negative: towards zero */
  if (h == 0x7c00) return h;                      /* +inf stays */
  return (uint16_t)(h + 1);
}
static uint16_t half_next_down(uint16_t h) {
  if ((h & 0x7fff) == 0) return 0x8001;
  if (h & 0x8000) return h == 0xfc00 ? h : (uint16_t)(h + 1);
  return (uint16_t)(h - 1);
}

/* largest half <= f */
uint16_t orc_float_to_half_rd(float f) {
  if (isnan(f)) return 0x7e00;
  uint16_t h = orc_float_to_half_rn(f);
  if (orc_half_to_float(h) > f) h = half_next_down(h);
  return h;
}

/* smallest half >= f */
uint16_t orc_float_to_half_ru(float f) {
  if (isnan(f)) return 0x7e00;
  uint16_t h = orc_float_to_half_rn(f);
  if (orc_half_to_float(h) < f) h = half_next_up(h);
  return h;
}

/* ------------------------------------------------------------------------
 * RoPE.  [EliteKV §2.1]: R_m is block diagonal with 2x2 rotations of angle
 * m*theta_i acting on the channel pairs (2i, 2i+1); theta_i = theta0 *
 * alpha^(-2i/d) with alpha = 10000, and [RoPE-KV §1] gives the angle as
 * m / 10000^(2i/d), i.e. theta0 = 1.
 * The angle is formed in fp64 and cos/sin are rounded once to fp32.
 * Forward rotation in fp32, one fixed order:
 *   y0 = fmaf(x0, c, -(x1*s))     y1 = fmaf(x0, s, x1*c)
 * Pins: R(a)R(b) = R(a+b) ([RoPE-KV §7.1]); the score depends only on m-n
 * ([EliteKV §2.2]).
 * ---------------------------------------------------------------------- */
/* Frequency of pair i (0-based; the pages' j = i + 1). mode (the rope flag),
 * low two bits:
 * 1: the standard table theta_i = base^(-2i/d) ([EliteKV §2.1]);
 * 2: frequency-aware RoPE ([KV-Latent], frequency-aware RoPE): the first half
 *    of the pairs (i < d/4) take base^(-2(i + d/8)/d), the second half
 *    base^(-(i + 3d/4)/d): the highest frequencies are skipped and the low
 *    ones sampled twice as densely.
 * Bit 4 of the flag chooses the channel pairs: clear, pair i is the
 * interleaved (2i, 2i+1) of the rotation matrix ([EliteKV §2.1]); set, it is
 * the half-split (i, i + d/2) of the page's apply_rope code ([EliteKV §7.1]).
 * Pins: both pairings rotate by the same angles, the half-split one is the
 * interleaved one with the channels reordered, R(a)R(b) = R(a+b). */
#define ORC_ROPE_HALF 4
static void rope_pair(int i, int d, int mode, int* j0, int* j1) {
  if (mode & ORC_ROPE_HALF) {
    *j0 = i;
    *j1 = i + d / 2;
  } else {
    *j0 = 2 * i;
    *j1 = 2 * i + 1;
  }
}

double orc_rope_theta(int i, int d, double base, int mode) {
  if ((mode & 3) == 2)
    return i < d / 4 ? pow(base, -2.0 * (i + d / 8) / d) : pow(base, -(double)(i + 3 * d / 4) / d);
  return pow(base, -(2.0 * i) / d);
}

void orc_rope_cs(int64_t m, int d, double base, int mode, float* c, float* s) {
  for (int i = 0; i < d / 2; ++i) {
    double ang = (double)m * orc_rope_theta(i, d, base, mode);
    c[i] = (float)cos(ang);
    s[i] = (float)sin(ang);
  }
}

/* the fp32 rotation on the pairs chosen by mode (see above) */
void orc_rope_apply_f32_mode(float* y, const float* x, const float* c, const float* s, int d, int mode) {
  for (int i = 0; i < d / 2; ++i) {
    int j0, j1;
    rope_pair(i, d, mode, &j0, &j1);
    float x0 = x[j0], x1 = x[j1];
    float t1 = x1 * s[i];
    float t2 = x1 * c[i];
    y[j0] = fmaf(x0, c[i], -t1);
    y[j1] = fmaf(x0, s[i], t2);
  }
}

void orc_rope_apply_f32(float* y, const float* x, const float* c, const float* s, int d) {
  orc_rope_apply_f32_mode(y, x, c, s, d, 1);
}

/* exact-angle rotation in fp64; inverse != 0 rotates by -m*theta */
void orc_rope_apply_f64(double* y, const double* x, int64_t m, int d, double base, int mode, int inverse) {
  for (int i = 0; i < d / 2; ++i) {
    int j0, j1;
    rope_pair(i, d, mode, &j0, &j1);
    double ang = (double)m * orc_rope_theta(i, d, base, mode);
    double c = cos(ang), s = inverse ? -sin(ang) : sin(ang);
    double x0 = x[j0], x1 = x[j1];
    y[j0] = x0 * c - x1 * s;
    y[j1] = x0 * s + x1 * c;
  }
}

/* ------------------------------------------------------------------------
 * Fast Walsh-Hadamard transform, Sylvester (natural) order
 * ([RotateKV] abstract and 关键设计: channel reordering followed by the FWHT).
 * Unnormalised butterflies, strides h = 1, 2, 4, ..., n/2 in that order;
 * each pair (i, i+h) with (i & h) == 0 becomes (a+b, a-b).
 * Pins: equals the dense matrix H_ij = (-1)^popcount(i&j) by brute force;
 * H H^T = n I; H_1024 = H_8 (x) H_128.
 * ---------------------------------------------------------------------- */
void orc_fwht_f32(float* p, int n) {
  for (int h = 1; h < n; h <<= 1)
    for (int i = 0; i < n; ++i)
      if ((i & h) == 0) {
        float a = p[i], b = p[i + h];
        p[i] = a + b;
        p[i + h] = a - b;
      }
}

void orc_fwht_f64(double* p, int n) {
  for (int h = 1; h < n; h <<= 1)
    for (int i = 0; i < n; ++i)
      if ((i & h) == 0) {
        double a = p[i], b = p[i + h];
        p[i] = a + b;
        p[i + h] = a - b;
      }
}

/* the normalisation factor 1/sqrt(n) rounded once to fp32 */
float orc_fwht_scale_f32(int n) { return (float)(1.0 / sqrt((double)n)); }

/* ------------------------------------------------------------------------
 * Per-token per-group asymmetric min-max quantization with fp16 scale and
 * zero ([RotateKV] 2-bit KV quantization; the quantizer form is the reading
 * stated in the design notes).
 *   mn, mx   group minimum / maximum (fp32; -0 is folded to +0 by adding 0.0f)
 *   Z        = largest half <= mn                (zero, rounded down)
 *   S        = smallest half >= fp32((mx - Z) / L)  (scale, rounded up)
 *   R        = S > 0 ? fp32(1 / S) : 0
 *   code     = round-half-even of the exact product fp32(p - Z) * R
 * Rounding Z down and S up keeps the whole group range inside the grid
 * Z + k S, k = 0..L, so every code lies in [0, L] without a clamp.
 * Pins: codes in range; brute-force nearest grid point on small groups;
 * Q(D(c)) = c for fixed (S, Z); |p - D(Q(p))| <= S/2; constant group -> 0.
 * ---------------------------------------------------------------------- */
void orc_minmax_group(const float* p, int g, int bits, uint8_t* codes, uint16_t* s16, uint16_t* z16) {
  int L = (1 << bits) - 1;
  float mn = p[0], mx = p[0];
  for (int j = 1; j < g; ++j) {
    if (p[j] < mn) mn = p[j];
    if (p[j] > mx) mx = p[j];
  }
  mn = mn + 0.0f; /* -0 -> +0: the stored zero and scale never depend on zero signs */
  mx = mx + 0.0f;
  uint16_t zh = orc_float_to_half_rd(mn);
  float Z = orc_half_to_float(zh);
  float w = mx - Z;
  float q = w / (float)L;
  uint16_t sh = orc_float_to_half_ru(q);
  float S = orc_half_to_float(sh);
  float R = S > 0.0f ? 1.0f / S : 0.0f;
  for (int j = 0; j < g; ++j) {
    float dlt = p[j] - Z;
    double u = (double)dlt * (double)R; /* exact: 24 x 24 bits */
    codes[j] = (uint8_t)(int)nearbyint(u);
  }
  *s16 = sh;
  *z16 = zh;
}

/* ------------------------------------------------------------------------
 * Bit packing: code j of a record occupies bits [b*j, b*j + b) of the
 * record's little-endian byte stream (least significant bit first).
 * Pins: hand-fixed bytes for 2/3/4-bit ramps; unpack(pack(c)) = c.
 * ---------------------------------------------------------------------- */
void orc_pack(const uint8_t* codes, int n, int bits, uint8_t* out) {
  memset(out, 0, (size_t)(n * bits + 7) / 8);
  for (int j = 0; j < n; ++j)
    for (int k = 0; k < bits; ++k)
      if ((codes[j] >> k) & 1) {
        int pos = j * bits + k;
        out[pos >> 3] |= (uint8_t)(1u << (pos & 7));
      }
}

void orc_unpack(const uint8_t* in, int n, int bits, uint8_t* codes) {
  for (int j = 0; j < n; ++j) {
    int c = 0;
    for (int k = 0; k < bits; ++k) {
      int pos = j * bits + k;
      c |= ((in[pos >> 3] >> (pos & 7)) & 1) << k;
    }
    codes[j] = (uint8_t)c;
  }
}

/* ------------------------------------------------------------------------
 * Quaternions, stored (real, i, j, k).  Hamilton product with the term order
 * of the IsoQuant-Full listing ([IsoQuant §3.2]); fp32 products are rounded
 * and summed left to right.
 * Pins: equals the 4x4 left/right multiplication matrices; unit quaternions
 * preserve norms; i^2 = j^2 = k^2 = ijk = -1.
 * ---------------------------------------------------------------------- */
void orc_quat_mul_f32(const float* a, const float* b, float* o) {
  float r0 = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
  float r1 = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
  float r2 = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
  float r3 = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
  o[0] = r0; o[1] = r1; o[2] = r2; o[3] = r3;
}

void orc_quat_mul_f64(const double* a, const double* b, double* o) {
  double r0 = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
  double r1 = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
  double r2 = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
  double r3 = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
  o[0] = r0; o[1] = r1; o[2] = r2; o[3] = r3;
}

/* ------------------------------------------------------------------------
 * Lloyd-Max scalar quantizer for N(0,1) ([IsoQuant §3.1]: "scalar Lloyd-Max
 * quantization"). Lloyd's iteration: boundaries are midpoints of adjacent
 * levels, levels are the conditional means of their cells,
 *   l_k = (phi(b_{k-1}) - phi(b_k)) / (Phi(b_k) - Phi(b_{k-1})).
 * Iterates from a uniform start until no level moves by more than 1e-15.
 * Pins: Max (1960) table values for 2/3/4 bits; centroid and midpoint
 * conditions; symmetry.
 * ---------------------------------------------------------------------- */
static double npdf(double x) { return isinf(x) ? 0.0 : exp(-0.5 * x * x) / sqrt(2.0 * M_PI); }
/* P(a < X <= b) for X ~ N(0,1), computed from the side that keeps precision */
static double nprob(double a, double b) {
  if (a >= 0.0) return 0.5 * (erfc(a / M_SQRT2) - erfc(b / M_SQRT2));
  if (b <= 0.0) return 0.5 * (erfc(-b / M_SQRT2) - erfc(-a / M_SQRT2));
  return 1.0 - 0.5 * erfc(-a / M_SQRT2) - 0.5 * erfc(b / M_SQRT2);
}

int orc_lloyd_max_normal(int bits, double* levels, double* mse_out) {
  int n = 1 << bits;
  double* b = (double*)malloc(sizeof(double) * (n + 1));
  for (int k = 0; k < n; ++k) levels[k] = -3.0 + 6.0 * (k + 0.5) / n;
  int it;
  for (it = 0; it < 200000; ++it) {
    b[0] = -INFINITY;
    b[n] = INFINITY;
    for (int k = 1; k < n; ++k) b[k] = 0.5 * (levels[k - 1] + levels[k]);
    double delta = 0.0;
    for (int k = 0; k < n; ++k) {
      double nl = (npdf(b[k]) - npdf(b[k + 1])) / nprob(b[k], b[k + 1]);
      double dd = fabs(nl - levels[k]);
      if (dd > delta) delta = dd;
      levels[k] = nl;
    }
    if (delta < 1e-15) break;
  }
  if (mse_out) {
    /* E[(X - l_k)^2 ; cell k] = (1 + l^2) P + (a - 2l) phi(a) - (b - 2l) phi(b) */
    for (int k = 1; k < n; ++k) b[k] = 0.5 * (levels[k - 1] + levels[k]);
    double mse = 0.0;
    for (int k = 0; k < n; ++k) {
      double lo = b[k], hi = b[k + 1], l = levels[k];
      double tlo = isinf(lo) ? 0.0 : (lo - 2.0 * l) * npdf(lo);
      double thi = isinf(hi) ? 0.0 : (hi - 2.0 * l) * npdf(hi);
      mse += (1.0 + l * l) * nprob(lo, hi) + tlo - thi;
    }
    *mse_out = mse;
  }
  free(b);
  return it;
}

/* Codebook for the unit-norm direction of a d-dimensional vector: the
   N(0,1) levels scaled by sigma = 1/sqrt(d) (each coordinate of a random unit
   vector has variance 1/d), rounded once to fp32. */
void orc_codebook(int bits, int d, float* out) {
  double lv[32];
  orc_lloyd_max_normal(bits, lv, NULL);
  for (int k = 0; k < (1 << bits); ++k) out[k] = (float)(lv[k] / sqrt((double)d));
}

/* code = number of fp32 midpoints beta_k = 0.5f*(l_k + l_{k+1}) strictly
   below w (a tie goes to the lower code) */
static int codebook_code(float w, const float* cb, int bits) {
  int c = 0;
  for (int k = 0; k + 1 < (1 << bits); ++k) {
    float beta = 0.5f * (cb[k] + cb[k + 1]);
    if (w > beta) ++c;
  }
  return c;
}

/* ------------------------------------------------------------------------
 * Encode.  Tensor layouts (all dense, row-major):
 *   x     half  [B][H][T][D]      pos[T] = RoPE position m of each token
 *   codes u8    [B][H][T][D*bits/8]
 *   sz    half  [B][H][T][D/G][2]  (scale, zero)
 *   sink  half  [B][H][n_sink][D]  indexed by sink slot (= position without a list)
 *   norm  f32   [B][H][T]
 * Tokens with pos < n_sink are kept verbatim in sink ([RotateKV]: attention
 * sinks protected at high precision); their codes and sz entries are zero.
 *   pre   f32   [B][H][T][D] or NULL: the rotated values that were quantized
 *         (used by the tests to tell boundary ties from real mismatches)
 * ---------------------------------------------------------------------- */
typedef struct {
  int B, H, T, D, rot, quant, bits, group, group_heads, rope, n_sink;
  double base;
  const int32_t* sink_pos; /* [B][n_sink] positions of the sinks, or NULL: positions 0 .. n_sink-1 */
} orc_shape;

/* Sink slot of position m of sequence b: its index in the sequence's sink
 * list (the stored fp16 row), or -1 when m is not a sink. */
static int sink_slot(const int32_t* sink_pos, int n_sink, int b, int64_t m) {
  if (!sink_pos) return m < n_sink ? (int)m : -1;
  for (int k = 0; k < n_sink; ++k)
    if (sink_pos[(size_t)b * n_sink + k] == m) return k;
  return -1;
}

static size_t rec_bytes(const orc_shape* s) { return (size_t)s->D * s->bits / 8; }

static void quantize_head(const orc_shape* s, const float* p, uint8_t* rec, uint16_t* szrow) {
  uint8_t codes[1024];
  int ng = s->D / s->group;
  for (int g = 0; g < ng; ++g)
    orc_minmax_group(p + g * s->group, s->group, s->bits, codes + g * s->group, &szrow[2 * g],
                     &szrow[2 * g + 1]);
  orc_pack(codes, s->D, s->bits, rec);
}

static int check_shape(const orc_shape* s) {
  if (s->D <= 0 || s->D > 256 || (s->D & (s->D - 1))) return 1;
  if (s->bits < 2 || s->bits > 4) return 1;
  if (s->rot == ORC_ROT_ISO) {
    if (s->quant != ORC_Q_CODEBOOK || s->D % 4) return 1;
  } else if (s->rot == ORC_ROT_ISO3) {
    if (s->quant != ORC_Q_CODEBOOK) return 1;
  } else {
    if (s->quant != ORC_Q_MINMAX || s->group <= 0 || s->D % s->group) return 1;
  }
  if (s->rot == ORC_ROT_FWHT_GROUP) {
    int hg = s->group_heads;
    if (hg <= 0 || (hg & (hg - 1)) || s->H % hg || hg * s->D > 2048) return 1;
  }
  return 0;
}

/* ------------------------------------------------------------------------
 * 3-D sandwich ([IsoQuant §2.1]: a unit quaternion q rotates a vector v,
 * taken as the pure quaternion (0, v), by T(v) = q v q*; [IsoQuant §1]: with
 * 3-channel blocks, d = 128 gives 42 whole blocks and a 2-D tail).
 * Block k < D/3 is channels 3k .. 3k+2: w = q_k (x) ((0, u) (x) q_k*), the
 * same association as the 4-D sandwich's listing, and the block's output is
 * the vector part (w_i, w_j, w_k). A 2-channel tail (D mod 3 = 2) is the
 * pure quaternion (0, u_{D-2}, u_{D-1}, 0) rotated by the next table entry,
 * whose i and j parts are zero, so the sandwich turns the tail in its own
 * plane; its output is (w_i, w_j). A 1-channel tail is left as it is. q holds
 * ceil(D/3) unit quaternions (real, i, j, k).
 * Pins: scipy's rotation of each block, the planar rotation of the tail,
 * norm preservation, the block counts printed on the page.
 * ---------------------------------------------------------------------- */
static void iso3_rotate_f32(const float* u, const float* q, int D, float* w) {
  int nb = D / 3;
  for (int k = 0; k <= nb; ++k) {
    int c = 3 * k, n = D - c < 3 ? D - c : 3;
    if (n == 1) {
      w[c] = u[c];
      break;
    }
    if (n <= 0) break;
    float v4[4] = {0.0f, u[c], u[c + 1], n == 3 ? u[c + 2] : 0.0f};
    float qc[4] = {q[4 * k], -q[4 * k + 1], -q[4 * k + 2], -q[4 * k + 3]};
    float t4[4], w4[4];
    orc_quat_mul_f32(v4, qc, t4);
    orc_quat_mul_f32(q + 4 * k, t4, w4);
    for (int e = 0; e < n; ++e) w[c + e] = w4[1 + e];
  }
}

/* inverse in fp64: v = q* (x) (w (x) q) on each block (q unit) */
static void iso3_unrotate_f64(const double* w, const float* q, int D, double* v) {
  int nb = D / 3;
  for (int k = 0; k <= nb; ++k) {
    int c = 3 * k, n = D - c < 3 ? D - c : 3;
    if (n == 1) {
      v[c] = w[c];
      break;
    }
    if (n <= 0) break;
    double w4[4] = {0.0, w[c], w[c + 1], n == 3 ? w[c + 2] : 0.0};
    double qd[4] = {q[4 * k], q[4 * k + 1], q[4 * k + 2], q[4 * k + 3]};
    double qc[4] = {qd[0], -qd[1], -qd[2], -qd[3]};
    double t4[4], v4[4];
    orc_quat_mul_f64(w4, qd, t4);
    orc_quat_mul_f64(qc, t4, v4);
    for (int e = 0; e < n; ++e) v[c + e] = v4[1 + e];
  }
}

/* The IsoQuant front end of one vector ([IsoQuant §3.1]): rho = ||x|| (fp64
   sum of the exact squares in channel order, rounded to fp32), u = x / (rho +
   1e-8) in fp32, then the rotation of `rot` -- the 4-D sandwich w = qL (x)
   (u (x) qR) per block ([IsoQuant §2.2, §3.2]) or the 3-D sandwich of
   iso3_rotate_f32 ([IsoQuant §2.1]). */
static void iso_front(int rot, const uint16_t* xv, int D, const float* qL, const float* qR, float* w, float* rho_out) {
  double acc = 0.0;
  for (int j = 0; j < D; ++j) {
    float f = orc_half_to_float(xv[j]);
    acc += (double)f * (double)f;
  }
  float rho = (float)sqrt(acc);
  float den = rho + 1e-8f;
  float u[256];
  for (int j = 0; j < D; ++j) u[j] = orc_half_to_float(xv[j]) / den;
  if (rot == ORC_ROT_ISO3) {
    iso3_rotate_f32(u, qL, D, w);
  } else {
    for (int k = 0; k < D / 4; ++k) {
      float t4[4];
      orc_quat_mul_f32(u + 4 * k, qR + 4 * k, t4);
      orc_quat_mul_f32(qL + 4 * k, t4, w + 4 * k);
    }
  }
  *rho_out = rho;
}

int orc_encode(int B, int H, int T, int D, const int64_t* pos, int rot, int quant, int bits, int group,
               int group_heads, int rope, int n_sink, double base, const uint16_t* x, const int16_t* perm,
               const float* qL, const float* qR, const float* codebook, uint8_t* codes, uint16_t* sz,
               uint16_t* sink, float* norm, float* pre, const int32_t* sink_pos) {
  orc_shape s = {B, H, T, D, rot, quant, bits, group, group_heads, rope, n_sink, base, sink_pos};
  if (check_shape(&s)) return 1;
  size_t rb = rec_bytes(&s);
  int ng = D / (group > 0 ? group : D);
  float c[128], sn[128];
  float buf[2048], tmp[256];
  int hg = rot == ORC_ROT_FWHT_GROUP ? group_heads : 1;
  for (int b = 0; b < B; ++b)
    for (int h0 = 0; h0 < H; h0 += hg)
      for (int t = 0; t < T; ++t) {
        int64_t m = pos[t];
        if (rope) orc_rope_cs(m, D, base, rope, c, sn);
        const int ks = sink_slot(sink_pos, n_sink, b, m);
        for (int hl = 0; hl < hg; ++hl) {
          size_t v = ((size_t)(b * H + h0 + hl) * T + t);
          const uint16_t* xv = x + v * D;
          uint8_t* rec = codes + v * rb;
          if (ks >= 0) {
            memcpy(sink + ((size_t)(b * H + h0 + hl) * n_sink + ks) * D, xv, sizeof(uint16_t) * D);
            memset(rec, 0, rb);
            if (rot == ORC_ROT_ISO || rot == ORC_ROT_ISO3)
              norm[v] = 0.0f;
            else
              memset(sz + v * ng * 2, 0, sizeof(uint16_t) * ng * 2);
          }
        }
        if (ks >= 0) continue;

        if (rot == ORC_ROT_ISO || rot == ORC_ROT_ISO3) {
          /* [IsoQuant §3.1]: rho = ||x||, x_hat = x / (rho + eps); 4-D blocks
             w = qL (x) (v (x) qR) ([IsoQuant §2.2, §3.2]) or the 3-D sandwich
             on 3-channel blocks ([IsoQuant §2.1]); Lloyd-Max codes. */
          size_t v = ((size_t)(b * H + h0) * T + t);
          float rho, w[256];
          iso_front(rot, x + v * D, D, qL, qR, w, &rho);
          uint8_t cds[256];
          for (int j = 0; j < D; ++j) cds[j] = (uint8_t)codebook_code(w[j], codebook, bits);
          if (pre) memcpy(pre + v * D, w, sizeof(float) * D);
          orc_pack(cds, D, bits, codes + v * rb);
          norm[v] = rho;
          continue;
        }

        if (rot == ORC_ROT_FWHT_GROUP) {
          /* [RotateKV] pre-RoPE grouped-head rotation: the hg head vectors of
             the token are concatenated (index = local_head * D + j), channel-
             permuted per head, transformed by one FWHT of size hg*D, and only
             then rotated by RoPE, head slice by head slice. */
          int n = hg * D;
          for (int hl = 0; hl < hg; ++hl) {
            const uint16_t* xv = x + ((size_t)(b * H + h0 + hl) * T + t) * D;
            for (int j = 0; j < D; ++j) {
              int src = perm ? perm[(h0 + hl) * D + j] : j;
              buf[hl * D + j] = orc_half_to_float(xv[src]);
            }
          }
          orc_fwht_f32(buf, n);
          float r = orc_fwht_scale_f32(n);
          for (int e = 0; e < n; ++e) buf[e] = buf[e] * r;
          for (int hl = 0; hl < hg; ++hl) {
            float* ph = buf + hl * D;
            if (rope) {
              orc_rope_apply_f32_mode(tmp, ph, c, sn, D, rope);
              memcpy(ph, tmp, sizeof(float) * D);
            }
            size_t v = ((size_t)(b * H + h0 + hl) * T + t);
            if (pre) memcpy(pre + v * D, ph, sizeof(float) * D);
            quantize_head(&s, ph, codes + v * rb, sz + v * ng * 2);
          }
          continue;
        }

        /* head variant ([RotateKV] outlier-aware rotation): RoPE, channel
           permutation, FWHT over head_dim (or none), quantize. */
        {
          size_t v = ((size_t)(b * H + h0) * T + t);
          const uint16_t* xv = x + v * D;
          for (int j = 0; j < D; ++j) tmp[j] = orc_half_to_float(xv[j]);
          float y[256];
          if (rope)
            orc_rope_apply_f32_mode(y, tmp, c, sn, D, rope);
          else
            memcpy(y, tmp, sizeof(float) * D);
          for (int j = 0; j < D; ++j) buf[j] = y[perm ? perm[h0 * D + j] : j];
          if (rot == ORC_ROT_FWHT_HEAD) {
            orc_fwht_f32(buf, D);
            float r = orc_fwht_scale_f32(D);
            for (int j = 0; j < D; ++j) buf[j] = buf[j] * r;
          }
          if (pre) memcpy(pre + v * D, buf, sizeof(float) * D);
          quantize_head(&s, buf, codes + v * rb, sz + v * ng * 2);
        }
      }
  return 0;
}

/* ------------------------------------------------------------------------
 * Decode (fp64): dequantize, then invert each rotation in reverse order.
 *   min-max:  y = Z + c S          codebook: w = l_c
 *   head:     FWHT (an involution once normalised), inverse permutation,
 *             inverse RoPE
 *   group:    inverse RoPE per head, FWHT over the group, inverse permutation
 *   iso:      v = qL^-1 (x) w (x) qR^-1, x = v * rho   ([IsoQuant §3.1] step 3)
 * attn_space != 0 skips the inverse RoPE and returns the key in attention
 * space (used by the score).  Sink tokens come back verbatim.
 * ---------------------------------------------------------------------- */
static void dequant_head(const orc_shape* s, const uint8_t* rec, const uint16_t* szrow, double* y) {
  uint8_t cds[1024];
  orc_unpack(rec, s->D, s->bits, cds);
  for (int j = 0; j < s->D; ++j) {
    int g = j / s->group;
    double S = orc_half_to_float(szrow[2 * g]), Z = orc_half_to_float(szrow[2 * g + 1]);
    y[j] = Z + (double)cds[j] * S;
  }
}

static void quat_inv_f64(const float* q, double* o) {
  double n2 = (double)q[0] * q[0] + (double)q[1] * q[1] + (double)q[2] * q[2] + (double)q[3] * q[3];
  o[0] = q[0] / n2;
  o[1] = -q[1] / n2;
  o[2] = -q[2] / n2;
  o[3] = -q[3] / n2;
}

/* Inverse of iso_front in fp64 ([IsoQuant §3.1] step 3): the inverse
   rotation -- v = qL^-1 (x) (w (x) qR^-1) per 4-D block, or v = q* (x) (w (x)
   q) per 3-D block -- then the norm restored, out = v * rho. */
static void iso_back(int rot, const double* w, int D, const float* qL, const float* qR, float rho, double* out) {
  if (rot == ORC_ROT_ISO3) {
    double u[256];
    iso3_unrotate_f64(w, qL, D, u);
    for (int j = 0; j < D; ++j) out[j] = u[j] * (double)rho;
    return;
  }
  for (int k = 0; k < D / 4; ++k) {
    double li[4], ri[4], t4[4], v4[4];
    quat_inv_f64(qL + 4 * k, li);
    quat_inv_f64(qR + 4 * k, ri);
    orc_quat_mul_f64(w + 4 * k, ri, t4);
    orc_quat_mul_f64(li, t4, v4);
    for (int e = 0; e < 4; ++e) out[4 * k + e] = v4[e] * (double)rho;
  }
}

static int decode_impl(const orc_shape* s, const int64_t* pos, const uint8_t* codes, const uint16_t* sz,
                       const uint16_t* sink, const float* norm, const int16_t* perm, const float* qL,
                       const float* qR, const float* codebook, double* out, int attn_space) {
  if (check_shape(s)) return 1;
  int B = s->B, H = s->H, T = s->T, D = s->D;
  size_t rb = rec_bytes(s);
  int ng = D / (s->group > 0 ? s->group : D);
  int hg = s->rot == ORC_ROT_FWHT_GROUP ? s->group_heads : 1;
  double buf[2048], y[256];
  for (int b = 0; b < B; ++b)
    for (int h0 = 0; h0 < H; h0 += hg)
      for (int t = 0; t < T; ++t) {
        int64_t m = pos[t];
        const int ks = sink_slot(s->sink_pos, s->n_sink, b, m);
        if (ks >= 0) {
          for (int hl = 0; hl < hg; ++hl) {
            size_t v = ((size_t)(b * H + h0 + hl) * T + t);
            const uint16_t* sv = sink + ((size_t)(b * H + h0 + hl) * s->n_sink + ks) * D;
            for (int j = 0; j < D; ++j) y[j] = orc_half_to_float(sv[j]);
            if (attn_space && s->rope)
              orc_rope_apply_f64(out + v * D, y, m, D, s->base, s->rope, 0);
            else
              memcpy(out + v * D, y, sizeof(double) * D);
          }
          continue;
        }
        if (s->rot == ORC_ROT_ISO || s->rot == ORC_ROT_ISO3) {
          size_t v = ((size_t)(b * H + h0) * T + t);
          uint8_t cds[256];
          orc_unpack(codes + v * rb, D, s->bits, cds);
          double w[256];
          for (int j = 0; j < D; ++j) w[j] = codebook[cds[j]];
          iso_back(s->rot, w, D, qL, qR, norm[v], out + v * D);
          continue;
        }
        if (s->rot == ORC_ROT_FWHT_GROUP) {
          int n = hg * D;
          for (int hl = 0; hl < hg; ++hl) {
            size_t v = ((size_t)(b * H + h0 + hl) * T + t);
            dequant_head(s, codes + v * rb, sz + v * ng * 2, y);
            if (s->rope)
              orc_rope_apply_f64(buf + hl * D, y, m, D, s->base, s->rope, 1);
            else
              memcpy(buf + hl * D, y, sizeof(double) * D);
          }
          orc_fwht_f64(buf, n);
          double r = 1.0 / sqrt((double)n);
          for (int hl = 0; hl < hg; ++hl) {
            size_t v = ((size_t)(b * H + h0 + hl) * T + t);
            double x[256];
            for (int j = 0; j < D; ++j) {
              int dst = perm ? perm[(h0 + hl) * D + j] : j;
              x[dst] = buf[hl * D + j] * r;
            }
            if (attn_space && s->rope)
              orc_rope_apply_f64(out + v * D, x, m, D, s->base, s->rope, 0);
            else
              memcpy(out + v * D, x, sizeof(double) * D);
          }
          continue;
        }
        {
          size_t v = ((size_t)(b * H + h0) * T + t);
          dequant_head(s, codes + v * rb, sz + v * ng * 2, buf);
          if (s->rot == ORC_ROT_FWHT_HEAD) {
            orc_fwht_f64(buf, D);
            double r = 1.0 / sqrt((double)D);
            for (int j = 0; j < D; ++j) buf[j] *= r;
          }
          for (int j = 0; j < D; ++j) y[perm ? perm[h0 * D + j] : j] = buf[j];
          if (s->rope && !attn_space)
            orc_rope_apply_f64(out + v * D, y, m, D, s->base, s->rope, 1);
          else
            memcpy(out + v * D, y, sizeof(double) * D);
        }
      }
  return 0;
}

int orc_decode(int B, int H, int T, int D, const int64_t* pos, int rot, int quant, int bits, int group,
               int group_heads, int rope, int n_sink, double base, const uint8_t* codes, const uint16_t* sz,
               const uint16_t* sink, const float* norm, const int16_t* perm, const float* qL, const float* qR,
               const float* codebook, double* out, const int32_t* sink_pos) {
  orc_shape s = {B, H, T, D, rot, quant, bits, group, group_heads, rope, n_sink, base, sink_pos};
  return decode_impl(&s, pos, codes, sz, sink, norm, perm, qL, qR, codebook, out, 0);
}

/* ------------------------------------------------------------------------
 * Decode-step score ([EliteKV §2.2]: A_{m,n} = q_m^rot . k_n^rot / sqrt(d)).
 *   s[b][qh][i] = scale * sum_j q[b][qh][j] * khat[b][qh / (Hq/H)][n_i][j]
 * q is given in attention space (already rotated by RoPE at the query's
 * position). khat_n is the decoded key in attention space: the stored slot
 * n decoded without the inverse RoPE, or RoPE_n(sink_n) for n < n_sink.
 * Cache layouts are the encode layouts with T = t_cap; slot index = position.
 * tok[] lists the n_idx token positions to score (all of them, or a sample).
 * fp64 throughout.
 * ---------------------------------------------------------------------- */
int orc_score(int B, int H, int Hq, int D, int t_cap, int rot, int quant, int bits, int group, int group_heads,
              int rope, int n_sink, double base, const uint16_t* q, const uint8_t* codes, const uint16_t* sz,
              const uint16_t* sink, const float* norm, const int16_t* perm, const float* qL, const float* qR,
              const float* codebook, const int64_t* tok, int n_idx, double scale, double* out,
              const int32_t* sink_pos) {
  if (Hq % H) return 1;
  orc_shape s = {B, H, 1, D, rot, quant, bits, group, group_heads, rope, n_sink, base, NULL};
  if (check_shape(&s)) return 1;
  int hg = rot == ORC_ROT_FWHT_GROUP ? group_heads : 1;
  int ng = D / (group > 0 ? group : D);
  size_t rb = rec_bytes(&s);
  double* kh = (double*)malloc(sizeof(double) * (size_t)hg * D);
  for (int b = 0; b < B; ++b)
    for (int h0 = 0; h0 < H; h0 += hg)
      for (int i = 0; i < n_idx; ++i) {
        int64_t n = tok[i];
        /* decode the single slot n of heads h0..h0+hg-1 through a one-token
           view of the cache */
        orc_shape s1 = s;
        s1.B = 1;
        s1.H = hg;
        s1.T = 1;
        s1.sink_pos = sink_pos ? sink_pos + (size_t)b * n_sink : NULL;  /* the one-sequence view's list */
        uint8_t* c1 = (uint8_t*)malloc(rb * hg + 1);
        uint16_t* z1 = (uint16_t*)malloc(sizeof(uint16_t) * 2 * ng * hg + 2);
        uint16_t* k1 = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)hg * (n_sink > 0 ? n_sink : 1) * D));
        float nm[16];
        for (int hl = 0; hl < hg; ++hl) {
          size_t v = ((size_t)(b * H + h0 + hl) * t_cap + n);
          memcpy(c1 + hl * rb, codes + v * rb, rb);
          if (rot != ORC_ROT_ISO) memcpy(z1 + hl * 2 * ng, sz + v * 2 * ng, sizeof(uint16_t) * 2 * ng);
          if (rot == ORC_ROT_ISO) nm[hl] = norm[v];
          if (n_sink > 0)
            memcpy(k1 + (size_t)hl * n_sink * D, sink + (size_t)(b * H + h0 + hl) * n_sink * D,
                   sizeof(uint16_t) * n_sink * D);
        }
        const int16_t* p1 = perm ? perm + (size_t)h0 * D : NULL;
        decode_impl(&s1, &n, c1, z1, k1, nm, p1, qL, qR, codebook, kh, 1);
        for (int hl = 0; hl < hg; ++hl) {
          int h = h0 + hl;
          for (int r = 0; r < Hq / H; ++r) {
            int qh = h * (Hq / H) + r;
            const uint16_t* qv = q + ((size_t)b * Hq + qh) * D;
            double acc = 0.0;
            for (int j = 0; j < D; ++j) acc += (double)orc_half_to_float(qv[j]) * kh[hl * D + j];
            out[((size_t)b * Hq + qh) * n_idx + i] = scale * acc;
          }
        }
        free(c1);
        free(z1);
        free(k1);
      }
  free(kh);
  return 0;
}

/* ------------------------------------------------------------------------
 * Decode-step attention ("EliteKV - RoPE频率选择与低秩投影" §2.2: the score
 * of query m and key n is q_m^rot . k_n^rot / sqrt(d); §7.1: the softmax of
 * the scaled scores over the cached tokens weights the values). For query
 * head qh of batch b (KV head h = qh / (Hq/H)) over cache slots n < n_tok:
 *   s_n   = scale * q . khat_n          (as orc_score: attention-space keys)
 *   p_n   = exp(s_n - max s) / sum exp(s - max s)
 *   out   = sum_n p_n * vhat_n          (vhat_n: decoded V slot n; sinks verbatim)
 * K and V caches share the record shape (rot, bits, group, n_sink) and have
 * their own RoPE flag and permutation. sink_pos: NULL (the sinks are the
 * positions < n_sink) or the sink list [B][n_sink] of both caches, as
 * orc_score and orc_decode take it. fp64 throughout.
 * ---------------------------------------------------------------------- */
int orc_attend(int B, int H, int Hq, int D, int t_cap, int n_tok, int rot, int bits, int group, int n_sink,
               double base, const uint16_t* q, const uint8_t* kcodes, const uint16_t* ksz,
               const uint16_t* ksink, const int16_t* kperm, int krope, const uint8_t* vcodes,
               const uint16_t* vsz, const uint16_t* vsink, const int16_t* vperm, int vrope, double scale,
               double* out, const int32_t* sink_pos) {
  if (Hq % H || n_tok < 1 || n_tok > t_cap) return 1;
  if (rot != ORC_ROT_NONE && rot != ORC_ROT_FWHT_HEAD) return 1;
  int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)t_cap);
  for (int n = 0; n < t_cap; ++n) tok[n] = n;
  double* s = (double*)malloc(sizeof(double) * (size_t)B * Hq * n_tok);
  double* vh = (double*)malloc(sizeof(double) * (size_t)B * H * t_cap * D);
  int rc = orc_score(B, H, Hq, D, t_cap, rot, ORC_Q_MINMAX, bits, group, 1, krope, n_sink, base, q, kcodes, ksz,
                     ksink, NULL, kperm, NULL, NULL, NULL, tok, n_tok, scale, s, sink_pos);
  if (!rc)
    rc = orc_decode(B, H, t_cap, D, tok, rot, ORC_Q_MINMAX, bits, group, 1, vrope, n_sink, base, vcodes, vsz,
                    vsink, NULL, vperm, NULL, NULL, NULL, vh, sink_pos);
  if (!rc) {
    for (int b = 0; b < B; ++b)
      for (int qh = 0; qh < Hq; ++qh) {
        const double* sv = s + ((size_t)b * Hq + qh) * n_tok;
        double mx = sv[0];
        for (int n = 1; n < n_tok; ++n) mx = sv[n] > mx ? sv[n] : mx;
        double den = 0.0;
        for (int n = 0; n < n_tok; ++n) den += exp(sv[n] - mx);
        double* o = out + ((size_t)b * Hq + qh) * D;
        for (int j = 0; j < D; ++j) o[j] = 0.0;
        int h = qh / (Hq / H);
        for (int n = 0; n < n_tok; ++n) {
          double p = exp(sv[n] - mx) / den;
          const double* v = vh + (((size_t)b * H + h) * t_cap + n) * D;
          for (int j = 0; j < D; ++j) o[j] += p * v[j];
        }
      }
  }
  free(tok);
  free(s);
  free(vh);
  return rc;
}

/* ------------------------------------------------------------------------
 * Channel permutation by abs-max ([RotateKV] outlier-aware rotation:
 * channel reordering before the FWHT). For each head, a_j = max over
 * batches and non-sink tokens of |y_j|, y = the fp32 input to the
 * permutation (RoPE'd keys when rope != 0). perm lists channels in
 * descending a_j; equal a_j keep ascending channel order.
 * ---------------------------------------------------------------------- */
int orc_calibrate_perm(int B, int H, int T, int D, const int64_t* pos, int rope, int n_sink, double base,
                       const uint16_t* x, int16_t* perm, const int32_t* sink_pos) {
  float* a = (float*)calloc((size_t)H * D, sizeof(float));
  float c[128], sn[128], xf[256], y[256];
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int t = 0; t < T; ++t) {
        if (sink_slot(sink_pos, n_sink, b, pos[t]) >= 0) continue;
        const uint16_t* xv = x + ((size_t)(b * H + h) * T + t) * D;
        for (int j = 0; j < D; ++j) xf[j] = orc_half_to_float(xv[j]);
        if (rope) {
          orc_rope_cs(pos[t], D, base, rope, c, sn);
          orc_rope_apply_f32_mode(y, xf, c, sn, D, rope);
        } else {
          memcpy(y, xf, sizeof(float) * D);
        }
        for (int j = 0; j < D; ++j)
          if (fabsf(y[j]) > a[h * D + j]) a[h * D + j] = fabsf(y[j]);
      }
  for (int h = 0; h < H; ++h) {
    /* stable selection: rank_j = #{k : a_k > a_j or (a_k == a_j and k < j)} */
    for (int j = 0; j < D; ++j) {
      int rank = 0;
      for (int k = 0; k < D; ++k) {
        float ak = a[h * D + k], aj = a[h * D + j];
        if (ak > aj || (ak == aj && k < j)) ++rank;
      }
      perm[h * D + rank] = (int16_t)j;
    }
  }
  free(a);
  return 0;
}

/* ------------------------------------------------------------------------
 * Energy of each RoPE frequency pair ([EliteKV] §3.1 frequency energy
 * analysis): E_i = sum over the cached keys of |K_{2i}|^2 + |K_{2i+1}|^2,
 * here per head, summed over batches and tokens of the fp16 keys. A pair's
 * norm is what RoPE preserves, so the energy is taken on the keys as given.
 * Exact: an fp16 value is M 2^(e) with an 11-bit M, so its square is an
 * integer multiple of 2^-48 below 2^80; the sum is kept as an unsigned
 * 128-bit integer in units of 2^-48 (energy[2k] = low 64 bits, energy[2k+1]
 * = high 64 bits). rank lists the pairs by descending energy, equal
 * energies in ascending pair order.
 * ---------------------------------------------------------------------- */
static unsigned __int128 half_square_units(uint16_t h) {
  unsigned e = (h >> 10) & 31u, m = h & 1023u;
  if (e == 31) return 0; /* inf / nan: not a finite key, contributes nothing */
  uint64_t M = e ? (m | 1024u) : m;
  unsigned shift = e ? 2 * e - 2 : 0; /* v = M 2^(e-25) (normal) or M 2^-24 */
  return ((unsigned __int128)(M * M)) << shift;
}

int orc_pair_energy(int B, int H, int T, int D, const uint16_t* x, uint64_t* energy, int16_t* rank) {
  int P = D / 2;
  unsigned __int128* acc = (unsigned __int128*)calloc((size_t)H * P, sizeof(unsigned __int128));
  if (!acc) return 1;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int t = 0; t < T; ++t) {
        const uint16_t* xv = x + ((size_t)(b * H + h) * T + t) * D;
        for (int i = 0; i < P; ++i) acc[h * P + i] += half_square_units(xv[2 * i]) + half_square_units(xv[2 * i + 1]);
      }
  for (int h = 0; h < H; ++h)
    for (int i = 0; i < P; ++i) {
      unsigned __int128 v = acc[h * P + i];
      energy[2 * (h * P + i)] = (uint64_t)v;
      energy[2 * (h * P + i) + 1] = (uint64_t)(v >> 64);
      int r = 0;
      for (int k = 0; k < P; ++k) {
        unsigned __int128 w = acc[h * P + k];
        if (w > v || (w == v && k < i)) ++r;
      }
      rank[h * P + r] = (int16_t)i;
    }
  free(acc);
  return 0;
}

/* ------------------------------------------------------------------------
 * Sink detection by massive activations ([RotateKV] abstract (iii) and
 * 关键设计: attention sinks are identified from the activations, by their
 * massive magnitude, and protected). Per sequence b:
 *   a_t = max over heads h and channels j of |x[b][h][t][j]| (exact fp16),
 *   med = the lower median of a_0 .. a_{T-1} (rank floor((T-1)/2), ascending),
 *   sinks = the tokens with a_t > tau * med (exact: both sides in fp64),
 * at most max_sinks of them, the largest a_t first, equal a_t to the earlier
 * token; sink_pos[b] lists their positions pos[t] in ascending order, padded
 * with -1, and count[b] how many there are.
 * Pins: constructed sequences with known massive tokens, the median by
 * numpy, the cap, ties, the strict threshold.
 * ---------------------------------------------------------------------- */
static int cmp_f32(const void* pa, const void* pb) {
  float a = *(const float*)pa, b = *(const float*)pb;
  return a < b ? -1 : a > b ? 1 : 0;
}

int orc_detect_sinks(int B, int H, int T, int D, const int64_t* pos, const uint16_t* x, double tau, int max_sinks,
                     int32_t* sink_pos, int32_t* count) {
  if (T <= 0 || max_sinks < 1) return 1;
  float* a = (float*)malloc(sizeof(float) * (size_t)T);
  float* srt = (float*)malloc(sizeof(float) * (size_t)T);
  int* pick = (int*)malloc(sizeof(int) * (size_t)max_sinks);
  for (int b = 0; b < B; ++b) {
    for (int t = 0; t < T; ++t) {
      float m = 0.0f;
      for (int h = 0; h < H; ++h) {
        const uint16_t* xv = x + ((size_t)(b * H + h) * T + t) * D;
        for (int j = 0; j < D; ++j) {
          float v = fabsf(orc_half_to_float(xv[j]));
          if (v > m) m = v;
        }
      }
      a[t] = m;
    }
    memcpy(srt, a, sizeof(float) * (size_t)T);
    qsort(srt, (size_t)T, sizeof(float), cmp_f32);
    double thr = tau * (double)srt[(T - 1) / 2];
    int n = 0;
    for (int k = 0; k < max_sinks; ++k) {  /* the next largest a_t above the threshold */
      int best = -1;
      for (int t = 0; t < T; ++t) {
        if (!((double)a[t] > thr)) continue;
        int taken = 0;
        for (int i = 0; i < n; ++i) taken |= pick[i] == t;
        if (taken) continue;
        if (best < 0 || a[t] > a[best]) best = t;  /* equal a_t: the earlier t stays */
      }
      if (best < 0) break;
      pick[n++] = best;
    }
    for (int i = 1; i < n; ++i)  /* ascending positions */
      for (int j = i; j > 0 && pick[j] < pick[j - 1]; --j) {
        int tmp = pick[j];
        pick[j] = pick[j - 1];
        pick[j - 1] = tmp;
      }
    for (int k = 0; k < max_sinks; ++k) sink_pos[(size_t)b * max_sinks + k] = k < n ? (int32_t)pos[pick[k]] : -1;
    count[b] = n;
  }
  free(a);
  free(srt);
  free(pick);
  return 0;
}

/* ------------------------------------------------------------------------
 * Dynamic codebooks for IsoQuant ([IsoQuant §4.2] quantization error
 * control: per-channel value statistics gathered online, quantization
 * boundaries set by the KL divergence, codebooks of twice the size for
 * outlier channels). Readings:
 *  - the statistics are per head h and channel j of the rotated unit vectors
 *    w (the quantizer's input, iso_front), over the batches and the
 *    non-sink positions of the calibration tokens: m2[h][j] = sum w_j^2 / N
 *    in fp64, sequentially;
 *  - the candidate codebooks are the Lloyd-Max designs for N(0, sigma^2),
 *    i.e. the N(0,1) levels l_k scaled by sigma; the KL divergence from the
 *    channel's distribution to N(0, sigma^2) is
 *    const + log sigma + m2 / (2 sigma^2), smallest at sigma^2 = m2, so
 *    sigma[h][j] = (float)sqrt(m2) (fp32(1/sqrt(D)), the fixed codebook's
 *    scale, when N = 0);
 *  - outlier channels: sigma_j > 2 * the lower median of the head's sigmas
 *    (rank floor((D-1)/2)), at most D/8 of them, the largest first, equal
 *    sigmas to the lower channel; bit j of wide[h][j/32] marks them; they use
 *    the (bits+1)-bit levels (twice the codebook);
 *  - channel j's levels are L_k = fp32(sigma_j * l_k) and its boundaries the
 *    fp32 midpoints 0.5f * (L_k + L_{k+1}); code = number of boundaries
 *    strictly below w_j (ties to the lower code);
 *  - storage: the low `bits` bits of every code in the record (LSB-first, as
 *    the fixed codebook), and the top bit of each outlier channel's code in
 *    ext[slot] (uint16), in ascending channel order, LSB first.
 * Pins: sigma against a numerical KL minimisation (scipy) and numpy
 * moments of the encoder's w; the outlier rule by brute force; codes against
 * the nearest level by brute force; the fixed-codebook special case
 * (every sigma equal, no outlier) byte for byte.
 * ---------------------------------------------------------------------- */
static int dyn_is_wide(const uint32_t* wide, int h, int D, int j) {
  return (wide[(size_t)h * (D / 32) + j / 32] >> (j % 32)) & 1u;
}

static int dyn_code(float w, float sigma, const float* lv, int n) {
  int c = 0;
  for (int k = 0; k + 1 < n; ++k) {
    float a = sigma * lv[k], b = sigma * lv[k + 1];
    float beta = 0.5f * (a + b);
    if (w > beta) ++c;
  }
  return c;
}

int orc_dyn_calibrate(int B, int H, int T, int D, const int64_t* pos, int rot, int n_sink, const uint16_t* x,
                      const float* qL, const float* qR, const int32_t* sink_pos, double* m2, float* sigma,
                      uint32_t* wide) {
  if ((rot != ORC_ROT_ISO && rot != ORC_ROT_ISO3) || D < 32 || D > 256 || D % 32) return 1;
  for (int h = 0; h < H; ++h) {
    double* s = m2 + (size_t)h * D;
    for (int j = 0; j < D; ++j) s[j] = 0.0;
    long long n = 0;
    for (int b = 0; b < B; ++b)
      for (int t = 0; t < T; ++t) {
        if (sink_slot(sink_pos, n_sink, b, pos[t]) >= 0) continue;
        float w[256], rho;
        iso_front(rot, x + ((size_t)(b * H + h) * T + t) * D, D, qL, qR, w, &rho);
        for (int j = 0; j < D; ++j) s[j] += (double)w[j] * (double)w[j];
        ++n;
      }
    float* sg = sigma + (size_t)h * D;
    for (int j = 0; j < D; ++j) {
      if (n > 0) s[j] /= (double)n;
      sg[j] = n > 0 ? (float)sqrt(s[j]) : (float)(1.0 / sqrt((double)D));
    }
    /* lower median by counting ranks (ties to the lower channel) */
    float med = 0.0f;
    for (int j = 0; j < D; ++j) {
      int r = 0;
      for (int k = 0; k < D; ++k) r += sg[k] < sg[j] || (sg[k] == sg[j] && k < j);
      if (r == (D - 1) / 2) med = sg[j];
    }
    uint32_t* wd = wide + (size_t)h * (D / 32);
    for (int i = 0; i < D / 32; ++i) wd[i] = 0;
    for (int j = 0; j < D; ++j) {
      if (!(sg[j] > 2.0f * med)) continue;
      int above = 0; /* channels ahead of j in the outlier order */
      for (int k = 0; k < D; ++k) above += sg[k] > sg[j] || (sg[k] == sg[j] && k < j);
      if (above < D / 8) wd[j / 32] |= 1u << (j % 32);
    }
  }
  return 0;
}

int orc_dyn_encode(int B, int H, int T, int D, const int64_t* pos, int rot, int bits, int n_sink,
                   const uint16_t* x, const float* qL, const float* qR, const float* cb, const float* cbw,
                   const float* sigma, const uint32_t* wide, uint8_t* codes, uint16_t* ext, uint16_t* sink,
                   float* norm, float* pre, const int32_t* sink_pos) {
  if ((rot != ORC_ROT_ISO && rot != ORC_ROT_ISO3) || bits < 2 || bits > 4 || D < 32 || D > 256 || D % 32) return 1;
  size_t rb = (size_t)D * bits / 8;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int t = 0; t < T; ++t) {
        size_t v = (size_t)(b * H + h) * T + t;
        const int ks = sink_slot(sink_pos, n_sink, b, pos[t]);
        if (ks >= 0) {
          memcpy(sink + ((size_t)(b * H + h) * n_sink + ks) * D, x + v * D, sizeof(uint16_t) * D);
          memset(codes + v * rb, 0, rb);
          ext[v] = 0;
          norm[v] = 0.0f;
          continue;
        }
        float w[256], rho;
        iso_front(rot, x + v * D, D, qL, qR, w, &rho);
        uint8_t lo[256];
        uint16_t e = 0;
        int nw = 0;
        for (int j = 0; j < D; ++j) {
          const float sg = sigma[(size_t)h * D + j];
          if (dyn_is_wide(wide, h, D, j)) {
            int c = dyn_code(w[j], sg, cbw, 1 << (bits + 1));
            lo[j] = (uint8_t)(c & ((1 << bits) - 1));
            if (nw < 16) e |= (uint16_t)((c >> bits) << nw);
            ++nw;
          } else {
            lo[j] = (uint8_t)dyn_code(w[j], sg, cb, 1 << bits);
          }
        }
        orc_pack(lo, D, bits, codes + v * rb);
        ext[v] = e;
        norm[v] = rho;
        if (pre) memcpy(pre + v * D, w, sizeof(float) * D);
      }
  return 0;
}

int orc_dyn_decode(int B, int H, int T, int D, const int64_t* pos, int rot, int bits, int n_sink,
                   const uint8_t* codes, const uint16_t* ext, const uint16_t* sink, const float* norm,
                   const float* qL, const float* qR, const float* cb, const float* cbw, const float* sigma,
                   const uint32_t* wide, double* out, const int32_t* sink_pos) {
  if ((rot != ORC_ROT_ISO && rot != ORC_ROT_ISO3) || bits < 2 || bits > 4 || D < 32 || D > 256 || D % 32) return 1;
  size_t rb = (size_t)D * bits / 8;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int t = 0; t < T; ++t) {
        size_t v = (size_t)(b * H + h) * T + t;
        const int ks = sink_slot(sink_pos, n_sink, b, pos[t]);
        if (ks >= 0) {
          const uint16_t* sv = sink + ((size_t)(b * H + h) * n_sink + ks) * D;
          for (int j = 0; j < D; ++j) out[v * D + j] = orc_half_to_float(sv[j]);
          continue;
        }
        uint8_t lo[256];
        orc_unpack(codes + v * rb, D, bits, lo);
        double w[256];
        int nw = 0;
        for (int j = 0; j < D; ++j) {
          const float sg = sigma[(size_t)h * D + j];
          if (dyn_is_wide(wide, h, D, j)) {
            int c = lo[j] | (nw < 16 ? ((ext[v] >> nw) & 1) << bits : 0);
            w[j] = (double)(sg * cbw[c]);
            ++nw;
          } else {
            w[j] = (double)(sg * cb[lo[j]]);
          }
        }
        iso_back(rot, w, D, qL, qR, norm[v], out + v * D);
      }
  return 0;
}
