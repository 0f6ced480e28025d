// Head-variant encode / decode ("RotateKV: Accurate and Robust 2-Bit KV Cache
// Quantization for LLMs via Outlier-Aware Adaptive Rotations", abstract and
// 关键设计: channel reordering followed by the FWHT; 2-bit KV quantization;
// attention sinks):
//   RoPE (keys) -> channel permutation -> normalised FWHT over head_dim
//   -> per-group min-max quantization with fp16 (scale, zero) -> LSB-first packing.
// Decode is the inverse. The literal per-token score over the same cache
// (k_score_literal, at the end of this file) reuses the decode's unpacking
// and inverse transform.
//
// Two lanes of a warp share one token-head vector: lane 2i + s holds channels
// [sV, sV + V), V = D/2, loaded straight from global memory (256-bit loads).
// Warps work independently (no barriers): each takes 16 consecutive vectors.
// Without RoPE the order is (batch, head, token): 4 KB of contiguous rows of
// one head, which share that head's permutation. With RoPE it is (batch,
// token, head): the heads of a token share its cos/sin row in L1, which costs
// more than the permutation's bank conflicts. The FWHT strides 1 .. V/2 run in registers; the last stride V pairs
// the two lanes: each lane computes fma(own, +-1, partner), i.e. exactly
// a + b (lower lane) or a - b (upper lane), and so keeps final values of its
// own channels. Groups of G <= V channels are then whole inside one lane; a
// group of D channels takes one min/max exchange with the partner.
// The permutation gathers (decode: scatters) through a per-warp buffer of rows
// in shared memory; with one permutation per warp and rows 130 words apart,
// the 16 rows read at one channel fall on 16 distinct banks.
#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_qdigits.cuh"

namespace kvq {
namespace {

constexpr int kThreads = 128;  // 4 independent warps per CTA
constexpr int kVecW = 16;      // vectors per warp step

struct HeadArgs {
  int B, H, T, t0, t_cap, n_sink, rope, v8;
  uint32_t n_vec;        // B * H * T
  FastDiv div_t, div_h;  // tokens; heads
  float rscale;          // fp32(1/sqrt(D))
  const __half* x;       // encode input  [B][H][T][D]
  void* out;             // decode output [B][H][T][D], fp16 or fp32
  const int16_t* perm;
  const float* rope_cs;  // [rows][D/2][2]
  uint8_t* codes;
  __half2* sz;
  __half* sink;
};

// Rows of the per-warp permutation buffer: D floats plus two pad words (an
// odd number of 8-byte units, so row k starts 2k words into the banks);
// element e of a row is at row + 4e.
template <int D>
__host__ __device__ constexpr uint32_t row_pitch() {
  return D * 4 + 8;
}

// Store / load this lane's run of NBY packed bytes; ALN = the run's alignment.
template <int NBY, int ALN>
__device__ __forceinline__ void st_run(uint8_t* p, const uint32_t* w) {
  if constexpr (ALN >= 16) {
#pragma unroll
    for (int i = 0; i < NBY / 16; ++i)
      reinterpret_cast<uint4*>(p)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else if constexpr (ALN == 8) {
#pragma unroll
    for (int i = 0; i < NBY / 8; ++i) reinterpret_cast<uint2*>(p)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < NBY / 4; ++i) reinterpret_cast<uint32_t*>(p)[i] = w[i];
  }
}
template <int NBY, int ALN>
__device__ __forceinline__ void ld_run(const uint8_t* p, uint32_t* w) {
  if constexpr (ALN >= 16) {
#pragma unroll
    for (int i = 0; i < NBY / 16; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  } else if constexpr (ALN == 8) {
#pragma unroll
    for (int i = 0; i < NBY / 8; ++i) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p) + i);
      w[2 * i] = v.x;
      w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < NBY / 4; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(p) + i);
  }
}
__host__ __device__ constexpr int pow2_align(int n) { return (n & 15) == 0 ? 16 : (n & 7) == 0 ? 8 : 4; }

// (b * H + h, h, token) of vector v, ordered (batch, token, head) for RoPE
// without a permutation (the heads of a token share one (cos, sin) row in L1)
// and (batch, head, token) otherwise (a warp's 16 vectors share one
// permutation, so its gather is conflict-free; with RoPE their 16 rows are
// staged by stage_rope_rows).
__device__ __forceinline__ void vec_coords(const HeadArgs& a, uint32_t v, uint32_t& bh, int& h, int& tt) {
  if (a.rope && !a.perm) {
    const uint32_t bt = a.div_h.div(v);
    h = static_cast<int>(a.div_h.mod(v, bt));
    const uint32_t b = a.div_t.div(bt);
    tt = static_cast<int>(a.div_t.mod(bt, b));
    bh = b * static_cast<uint32_t>(a.H) + static_cast<uint32_t>(h);
  } else {
    bh = a.div_t.div(v);
    tt = static_cast<int>(a.div_t.mod(v, bh));
    h = static_cast<int>(a.div_h.mod(bh, a.div_h.div(bh)));
  }
}

// Staged (cos, sin) rows: 16-byte aligned rows of D floats.
template <int D>
__host__ __device__ constexpr uint32_t cs_pitch() {
  return D * 4 + 16;
}
// Per-warp shared memory: encode keeps the permutation rows and the staged
// (cos, sin) rows in one buffer (they are used one after the other); decode
// needs both at once (the rows are staged while the permutation is applied).
template <int D>
__host__ __device__ constexpr uint32_t warp_buf(bool enc) {
  return enc ? kVecW * cs_pitch<D>() : kVecW * (row_pitch<D>() + cs_pitch<D>());
}

// Start copying the (cos, sin) rows of the warp's 16 vectors into cs rows at
// csbuf (row k <- the position of slot k, taken from lane 2k): every lane
// copies one 16-byte chunk of every row, so each row is one coalesced
// transfer; cp.async keeps all 16 in flight without registers.
template <int D>
__device__ __forceinline__ void stage_rope_rows(const HeadArgs& a, uint32_t csbuf, int m, int lane) {
  constexpr int CH = D * 4 / 16;  // 16-byte chunks of a row: 32 (D = 128) or 16 (D = 64)
#pragma unroll
  for (int k = 0; k < kVecW; ++k) {
    const int mk = __shfl_sync(0xffffffffu, m, 2 * k);
    if (lane < CH)
      cp_async16(csbuf + k * cs_pitch<D>() + 16 * lane,
                 reinterpret_cast<const uint4*>(a.rope_cs + static_cast<size_t>(mk) * D) + lane, 16);
  }
  cp_async_commit();
}

// The staged rows have landed and every lane sees them.
__device__ __forceinline__ void staged_rows_ready() {
  cp_async_wait_all();
  __syncwarp();
}

template <int D, int BITS, int G, bool ROT>
__global__ void __launch_bounds__(kThreads, 4) k_encode_head(const HeadArgs a) {
  constexpr int V = D / 2;            // channels per lane
  constexpr int RB = D * BITS / 8;    // record bytes
  constexpr int NG = D / G;           // groups per record
  constexpr bool SHARED = G > V;      // one group spans both lanes
  constexpr int GS = SHARED ? V : G;  // channels of a group inside this lane
  constexpr int NGT = V / GS;         // groups inside this lane
  constexpr int NBY = V * BITS / 8;   // this lane's packed bytes
  constexpr int NW = NBY / 4;
  extern __shared__ uint8_t smem_raw[];  // permutation rows: 16 x D floats per warp
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s = lane & 1, slot = lane >> 1;
  const uint32_t wbuf = smem_u32(smem_raw) + warp * warp_buf<D>(true);
  const uint32_t row = wbuf + slot * row_pitch<D>();   // permutation staging
  const uint32_t csrow = wbuf + slot * cs_pitch<D>();  // staged (cos, sin) row, same buffer
  const float r = a.rscale;
  const bool v8 = a.v8 != 0;
  const bool staged = a.rope && a.perm;  // the warp's (cos, sin) rows in its buffer
  const uint32_t gw = blockIdx.x * (kThreads / 32) + warp, nw = gridDim.x * (kThreads / 32);

  for (uint32_t base = gw * kVecW; base < a.n_vec; base += nw * kVecW) {
    const uint32_t v = base + slot;
    const bool live = v < a.n_vec;
    uint32_t bh;
    int h, tt;
    vec_coords(a, live ? v : a.n_vec - 1, bh, h, tt);
    const int m = a.t0 + tt;
    const size_t vec = bh;
    const bool sink_tok = m < a.n_sink;
    if (staged) stage_rope_rows<D>(a, wbuf, m, lane);  // in flight while the row loads

    uint32_t raw[V / 2];
    ld_row<V / 2>(a.x + (vec * a.T + tt) * D + V * s, v8, raw);
    if (live && sink_tok) {  // attention sink: this lane's half row, verbatim
      uint4* dst = reinterpret_cast<uint4*>(a.sink + (vec * a.n_sink + m) * D + V * s);
#pragma unroll
      for (int c = 0; c < V / 8; ++c) dst[c] = make_uint4(raw[4 * c], raw[4 * c + 1], raw[4 * c + 2], raw[4 * c + 3]);
    }
    // P[2g + e] = (x[4g + e], x[4g + 2 + e]) over this lane's channels
    float2 P[V / 2];
#pragma unroll
    for (int g = 0; g < V / 4; ++g) {
      const float2 h01 = __half22float2(*reinterpret_cast<const __half2*>(&raw[2 * g]));
      const float2 h23 = __half22float2(*reinterpret_cast<const __half2*>(&raw[2 * g + 1]));
      P[2 * g] = f2(h01.x, h23.x);
      P[2 * g + 1] = f2(h01.y, h23.y);
    }
    if (staged) staged_rows_ready();
    if (a.rope == 1) {  // pairs (2i, 2i+1): y0 = fma(x0, c, -(x1*s)), y1 = fma(x0, s, x1*c)
      const uint4* rp = reinterpret_cast<const uint4*>(a.rope_cs + static_cast<size_t>(m) * D) + (V / 4) * s;
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {
        // (c, s) of pairs 2g and 2g+1 of this lane
        const uint4 cv = staged ? lds128(csrow + 16 * ((V / 4) * s + g)) : __ldg(rp + g);
        const float2 cc = f2(__uint_as_float(cv.x), __uint_as_float(cv.z));
        const float2 ss = f2(__uint_as_float(cv.y), __uint_as_float(cv.w));
        const float2 x0 = P[2 * g], x1 = P[2 * g + 1];
        P[2 * g] = fma2(x0, cc, mul2(x1, f2(-ss.x, -ss.y)));
        P[2 * g + 1] = fma2(x0, ss, mul2(x1, cc));
      }
    } else if (a.rope == 2) {  // half-split pairs (i, i + V): local channel j of both lanes, angle j
      const uint4* rp = reinterpret_cast<const uint4*>(a.rope_cs + static_cast<size_t>(m) * D);
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {
        // angles 4g .. 4g+1, 4g+2 .. 4g+3
        const uint4 c0 = staged ? lds128(csrow + 32 * g) : __ldg(rp + 2 * g);
        const uint4 c1 = staged ? lds128(csrow + 32 * g + 16) : __ldg(rp + 2 * g + 1);
        // P[2g] holds local channels 4g, 4g+2; P[2g+1] holds 4g+1, 4g+3
        P[2 * g] = rope_half_fwd2(P[2 * g], f2(__uint_as_float(c0.x), __uint_as_float(c1.x)),
                                  f2(__uint_as_float(c0.y), __uint_as_float(c1.y)), s != 0, 1);
        P[2 * g + 1] = rope_half_fwd2(P[2 * g + 1], f2(__uint_as_float(c0.z), __uint_as_float(c1.z)),
                                      f2(__uint_as_float(c0.w), __uint_as_float(c1.w)), s != 0, 1);
      }
    }
    if (a.perm) {  // p_j = y_perm[h][j]: stage the row, gather
      if (staged) __syncwarp();  // every lane has read its (cos, sin) row
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {
        sts64(row + 4 * (V * s + 4 * g), __float_as_uint(P[2 * g].x), __float_as_uint(P[2 * g + 1].x));
        sts64(row + 4 * (V * s + 4 * g + 2), __float_as_uint(P[2 * g].y), __float_as_uint(P[2 * g + 1].y));
      }
      __syncwarp();
      const int16_t* pr = a.perm + static_cast<size_t>(h) * D + V * s;
      float xv[V];
#pragma unroll
      for (int c = 0; c < V / 8; ++c) {
        const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
        const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
          xv[8 * c + i] = lds32f(row + 4 * ((pw[i >> 1] >> (16 * (i & 1))) & (D - 1)));
      }
      __syncwarp();  // the row buffer is free for the next step
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {
        P[2 * g] = f2(xv[4 * g], xv[4 * g + 2]);
        P[2 * g + 1] = f2(xv[4 * g + 1], xv[4 * g + 3]);
      }
    }
    if constexpr (ROT) {
      fwht_pairs<V>(P);
      // stride V across the lane pair: lower lane a + b, upper lane a - b
      const float sg = s ? -1.0f : 1.0f;
#pragma unroll
      for (int k = 0; k < V / 2; ++k) {
        const float2 o = P[k];
        const float2 p = f2(__shfl_xor_sync(0xffffffffu, o.x, 1), __shfl_xor_sync(0xffffffffu, o.y, 1));
        P[k] = fma2(o, f2(sg, sg), p);
      }
#pragma unroll
      for (int k = 0; k < V / 2; ++k) P[k] = mul2(P[k], f2(r, r));
    }

    // min-max per group, fp16 (scale, zero); a sink slot quantizes with Z = R = 0
    float Zg[NGT], Rg[NGT];
    __half2 szg[NGT];
#pragma unroll
    for (int gg = 0; gg < NGT; ++gg) {
      constexpr int QG = GS / 4;  // channel quads per group
      float lo = fminf(P[2 * QG * gg].x, P[2 * QG * gg].y), hi = fmaxf(P[2 * QG * gg].x, P[2 * QG * gg].y);
      lo = min3f(lo, P[2 * QG * gg + 1].x, P[2 * QG * gg + 1].y);
      hi = max3f(hi, P[2 * QG * gg + 1].x, P[2 * QG * gg + 1].y);
#pragma unroll
      for (int q = 1; q < QG; ++q) {
        const float2 e0 = P[2 * (QG * gg + q)], e1 = P[2 * (QG * gg + q) + 1];
        lo = min3f(lo, e0.x, e0.y);
        hi = max3f(hi, e0.x, e0.y);
        lo = min3f(lo, e1.x, e1.y);
        hi = max3f(hi, e1.x, e1.y);
      }
      if constexpr (SHARED) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, 1));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, 1));
      }
      const QParams p = minmax_params<BITS>(lo, hi);
      Zg[gg] = sink_tok ? 0.0f : p.Z;
      Rg[gg] = sink_tok ? 0.0f : p.R;
      szg[gg] = sink_tok ? __halves2half2(__ushort_as_half(0), __ushort_as_half(0)) : p.sz;
    }

    // quantize and pack this lane's V codes (LSB first)
    uint32_t w[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = 0u;
#pragma unroll
    for (int g = 0; g < V / 4; ++g) {
      const int gg = (4 * g) / GS;
      const float2 nZ = f2(-Zg[gg], -Zg[gg]), R2 = f2(Rg[gg], Rg[gg]), M2 = f2(kMagicRound, kMagicRound);
      const float2 ua = fma2(add2(P[2 * g], nZ), R2, M2);
      const float2 ub = fma2(add2(P[2 * g + 1], nZ), R2, M2);
      const uint32_t t4[4] = {__float_as_uint(ua.x), __float_as_uint(ub.x), __float_as_uint(ua.y),
                              __float_as_uint(ub.y)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int pos = (4 * g + e) * BITS;
        if constexpr (32 % BITS == 0) {
          w[pos >> 5] += t4[e] << (pos & 31);  // codes never straddle a word
        } else {
          const uint32_t c = t4[e] - kMagicBits;
          w[pos >> 5] |= c << (pos & 31);
          if ((pos & 31) + BITS > 32) w[(pos >> 5) + 1] |= c >> (32 - (pos & 31));
        }
      }
    }
    if constexpr (32 % BITS == 0) {
#pragma unroll
      for (int i = 0; i < NW; ++i) w[i] -= magic_offset<BITS, 32 / BITS>();
    }
    if (live) {
      const size_t slot_i = vec * a.t_cap + m;
      st_run<NBY, pow2_align(NBY)>(a.codes + slot_i * RB + NBY * s, w);
      if constexpr (SHARED) {
        if (s == 0) a.sz[slot_i] = szg[0];
      } else if constexpr (NGT == 1) {
        a.sz[slot_i * NG + s] = szg[0];
      } else {
        static_assert(NGT == 2, "at most two groups per lane");
        *reinterpret_cast<uint2*>(a.sz + slot_i * NG + 2 * s) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&szg[0]), *reinterpret_cast<const uint32_t*>(&szg[1]));
      }
    }
  }
}

// This lane's half record back to fp32: dequantize (S, Z per group, already
// multiplied by the normalisation when ROT) and undo the FWHT. Codes 0 and 2
// of a quad are masked in place at bit 0, codes 1 and 3 at bit BITS; read
// through the fp32 pattern 2^23 + v they give code * 2^p, and the power of two
// 2^p folds exactly into the scale. The transform is its own inverse: stride V
// across the lane pair, then strides 1 .. V/2 in registers. P ends in the
// register-pair layout of this lane's V channels of the permuted vector.
template <int D, int BITS, int G, bool ROT>
__device__ __forceinline__ void unpack_inverse(const uint32_t* w, const float* Sg, const float* Zg, int s,
                                               float2 (&P)[D / 4]) {
  constexpr int V = D / 2;
  constexpr int GS = G > V ? V : G;
  constexpr int NW = V * BITS / 32;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
#pragma unroll
  for (int g = 0; g < V / 4; ++g) {
    const int gg = (4 * g) / GS;
    const int pos = 4 * g * BITS;
    const uint32_t lo = w[pos >> 5] >> (pos & 31);
    const uint32_t w0 =
        (32 - (pos & 31) >= 4 * BITS || (pos >> 5) + 1 >= NW) ? lo : (lo | (w[(pos >> 5) + 1] << (32 - (pos & 31))));
    const uint32_t w1 = w0 >> (2 * BITS);
    const float2 c02 = f2(__uint_as_float(0x4B000000u | (w0 & MASK)), __uint_as_float(0x4B000000u | (w1 & MASK)));
    const float2 c13 = f2(__uint_as_float(0x4B000000u | (w0 & (MASK << BITS))),
                          __uint_as_float(0x4B000000u | (w1 & (MASK << BITS))));
    const float2 nM = f2(-8388608.0f, -8388608.0f), Z2 = f2(Zg[gg], Zg[gg]);
    const float S1 = Sg[gg] * (1.0f / (1 << BITS));
    P[2 * g] = fma2(add2(c02, nM), f2(Sg[gg], Sg[gg]), Z2);
    P[2 * g + 1] = fma2(add2(c13, nM), f2(S1, S1), Z2);
  }
  if constexpr (ROT) {
    const float sg = s ? -1.0f : 1.0f;
#pragma unroll
    for (int k = 0; k < V / 2; ++k) {
      const float2 o = P[k];
      const float2 p = f2(__shfl_xor_sync(0xffffffffu, o.x, 1), __shfl_xor_sync(0xffffffffu, o.y, 1));
      P[k] = fma2(o, f2(sg, sg), p);
    }
    fwht_pairs<V>(P);
  }
}

template <int D, int BITS, int G, bool ROT, bool F32>
__global__ void __launch_bounds__(kThreads, 3) k_decode_head(const HeadArgs a) {
  constexpr int V = D / 2;
  constexpr int RB = D * BITS / 8;
  constexpr int NG = D / G;
  constexpr bool SHARED = G > V;
  constexpr int GS = SHARED ? V : G;
  constexpr int NGT = V / GS;
  constexpr int NBY = V * BITS / 8;
  constexpr int NW = NBY / 4;
  constexpr int ES = F32 ? 4 : 2;
  extern __shared__ uint8_t smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s = lane & 1, slot = lane >> 1;
  const uint32_t wbuf = smem_u32(smem_raw) + warp * warp_buf<D>(false);
  const uint32_t row = wbuf + slot * row_pitch<D>();  // permutation staging
  const uint32_t csbuf = wbuf + kVecW * row_pitch<D>();
  const uint32_t csrow = csbuf + slot * cs_pitch<D>();  // staged (cos, sin) row
  const float r = a.rscale;
  const bool v8 = a.v8 != 0;
  const bool staged = a.rope && a.perm;  // the warp's (cos, sin) rows in its buffer
  const uint32_t gw = blockIdx.x * (kThreads / 32) + warp, nw = gridDim.x * (kThreads / 32);

  for (uint32_t base = gw * kVecW; base < a.n_vec; base += nw * kVecW) {
    const uint32_t v = base + slot;
    const bool live = v < a.n_vec;
    uint32_t bh;
    int h, tt;
    vec_coords(a, live ? v : a.n_vec - 1, bh, h, tt);
    const int m = a.t0 + tt;
    const size_t vec = bh;
    const size_t slot_i = vec * a.t_cap + m;
    const bool sink_tok = m < a.n_sink;
    if (staged) stage_rope_rows<D>(a, csbuf, m, lane);  // in flight while the codes are decoded

    uint32_t w[NW];
    ld_run<NBY, pow2_align(NBY)>(a.codes + slot_i * RB + NBY * s, w);
    float Sg[NGT], Zg[NGT];
#pragma unroll
    for (int gg = 0; gg < NGT; ++gg) {
      const float2 sz = __half22float2(a.sz[slot_i * NG + (SHARED ? 0 : NGT * s + gg)]);
      Sg[gg] = ROT ? __fmul_rn(sz.x, r) : sz.x;  // the normalisation folds into S and Z
      Zg[gg] = ROT ? __fmul_rn(sz.y, r) : sz.y;
    }
    float2 P[V / 2];
    unpack_inverse<D, BITS, G, ROT>(w, Sg, Zg, s, P);
    if (a.perm) {  // x[perm[h][j]] = p_j: scatter into the row, read this lane's half back
      const int16_t* pr = a.perm + static_cast<size_t>(h) * D + V * s;
#pragma unroll
      for (int c = 0; c < V / 8; ++c) {
        const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
        const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = 8 * c + i;  // local channel: P[2(j/4) + (j&1)], lane (j>>1)&1
          const float xv = ((j >> 1) & 1) ? P[2 * (j >> 2) + (j & 1)].y : P[2 * (j >> 2) + (j & 1)].x;
          sts32f(row + 4 * ((pw[i >> 1] >> (16 * (i & 1))) & (D - 1)), xv);
        }
      }
      __syncwarp();
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {
        const uint2 u = lds64(row + 4 * (V * s + 4 * g)), w2 = lds64(row + 4 * (V * s + 4 * g + 2));
        P[2 * g] = f2(__uint_as_float(u.x), __uint_as_float(w2.x));
        P[2 * g + 1] = f2(__uint_as_float(u.y), __uint_as_float(w2.y));
      }
      __syncwarp();  // the row buffer is free for the next step
    }
    if (staged) staged_rows_ready();
    if (a.rope == 1) {  // inverse pairs: x0 = y0 c + y1 s, x1 = y1 c - y0 s
      const uint4* rp = reinterpret_cast<const uint4*>(a.rope_cs + static_cast<size_t>(m) * D) + (V / 4) * s;
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {
        const uint4 cv = staged ? lds128(csrow + 16 * ((V / 4) * s + g)) : __ldg(rp + g);
        const float2 cc = f2(__uint_as_float(cv.x), __uint_as_float(cv.z));
        const float2 ss = f2(__uint_as_float(cv.y), __uint_as_float(cv.w));
        const float2 y0 = P[2 * g], y1 = P[2 * g + 1];
        P[2 * g] = fma2(y0, cc, mul2(y1, ss));
        P[2 * g + 1] = fma2(y1, cc, mul2(y0, f2(-ss.x, -ss.y)));
      }
    } else if (a.rope == 2) {  // half-split pairs across the lane pair
      const uint4* rp = reinterpret_cast<const uint4*>(a.rope_cs + static_cast<size_t>(m) * D);
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {
        const uint4 c0 = staged ? lds128(csrow + 32 * g) : __ldg(rp + 2 * g);
        const uint4 c1 = staged ? lds128(csrow + 32 * g + 16) : __ldg(rp + 2 * g + 1);
        P[2 * g] = rope_half_inv2(P[2 * g], f2(__uint_as_float(c0.x), __uint_as_float(c1.x)),
                                  f2(__uint_as_float(c0.y), __uint_as_float(c1.y)), s != 0, 1);
        P[2 * g + 1] = rope_half_inv2(P[2 * g + 1], f2(__uint_as_float(c0.z), __uint_as_float(c1.z)),
                                      f2(__uint_as_float(c0.w), __uint_as_float(c1.w)), s != 0, 1);
      }
    }
    if (staged) __syncwarp();  // every lane has read its (cos, sin) row: the buffer is free
    // output words of this lane's half row (a sink slot comes back verbatim)
    uint32_t ow[V * ES / 4];
    if (sink_tok) {
      uint32_t hv[V / 2];
      ld_row<V / 2>(a.sink + (vec * a.n_sink + m) * D + V * s, false, hv);
      if constexpr (F32) {
#pragma unroll
        for (int j = 0; j < V / 2; ++j) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hv[j]));
          ow[2 * j] = __float_as_uint(f.x);
          ow[2 * j + 1] = __float_as_uint(f.y);
        }
      } else {
#pragma unroll
        for (int j = 0; j < V / 2; ++j) ow[j] = hv[j];
      }
    } else if constexpr (F32) {
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {
        ow[4 * g] = __float_as_uint(P[2 * g].x);
        ow[4 * g + 1] = __float_as_uint(P[2 * g + 1].x);
        ow[4 * g + 2] = __float_as_uint(P[2 * g].y);
        ow[4 * g + 3] = __float_as_uint(P[2 * g + 1].y);
      }
    } else {
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {
        const __half2 h01 = __floats2half2_rn(P[2 * g].x, P[2 * g + 1].x);
        const __half2 h23 = __floats2half2_rn(P[2 * g].y, P[2 * g + 1].y);
        ow[2 * g] = *reinterpret_cast<const uint32_t*>(&h01);
        ow[2 * g + 1] = *reinterpret_cast<const uint32_t*>(&h23);
      }
    }
    if (live) st_row<V * ES / 4>(static_cast<uint8_t*>(a.out) + ((vec * a.T + tt) * D + V * s) * ES, v8, ow);
  }
}

// ---------------------------------------------------------------------------
// Literal decode-step score ("EliteKV - RoPE频率选择与低秩投影" §2.2 score over
// the head-variant cache): every key is decoded on the fly (unpack,
// dequantize, inverse FWHT per token) and dotted with the GQ query heads of
// its KV head. The permutation moves onto the query instead of the key
// (sum_i q_i khat_i = sum_j q_perm[j] p_j, the same products in another
// order); the transform is applied to every key. This is the reference form
// that the query-rotation kernels (which transform the query once) are
// measured against.
// A CTA owns a contiguous range of 16-token steps of one (batch, KV head)
// stream; its warps take every 8th step, two lanes per token as in the decode.
constexpr int kLitThreads = 256;
constexpr int kLitWarps = kLitThreads / 32;

struct LitArgs {
  int H, Hq, t_cap, n_tok, n_sink, rope;
  int splits, n_step;  // CTAs per stream; 16-token steps per stream
  float scale, rscale;
  const __half* q;  // [B][Hq][128]
  const int16_t* perm;
  const float* rope_cs;
  const uint8_t* codes;
  const __half2* sz;
  const __half* sink;
  float* scores;  // [B][Hq][n_tok]
};

// A query row in shared memory: lane half s (channels sV .. sV + V - 1) at
// s * (V + 4) floats, so the two halves read at once sit on distinct banks.
template <int D>
__host__ __device__ constexpr int lit_qpitch() {
  return 2 * (D / 2 + 4);
}

template <int BITS, int G, int GQ, bool ROT>
__global__ void __launch_bounds__(kLitThreads) k_score_literal(const LitArgs a) {
  constexpr int D = 128, V = D / 2;
  constexpr int RB = D * BITS / 8;
  constexpr int NG = D / G;
  constexpr bool SHARED = G > V;
  constexpr int GS = SHARED ? V : G;
  constexpr int NGT = V / GS;
  constexpr int NBY = V * BITS / 8;
  constexpr int NW = NBY / 4;
  constexpr int QP = lit_qpitch<D>();
  __shared__ __align__(16) float qraw[GQ][D];  // the queries as given (sink keys)
  __shared__ __align__(16) float qp[GQ][QP];   // q_perm[j] at the lane-half position of channel j
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = lane & 1, slot = lane >> 1;
  const int bh = static_cast<int>(blockIdx.x) / a.splits, part = static_cast<int>(blockIdx.x) % a.splits;
  const int b = bh / a.H, h = bh - b * a.H;
  for (int e = tid; e < GQ * D; e += kLitThreads) {
    const int r = e / D, j = e % D;
    const __half* qv = a.q + (static_cast<size_t>(b) * a.Hq + h * GQ + r) * D;
    const int pj = a.perm ? (__ldg(a.perm + static_cast<size_t>(h) * D + j) & (D - 1)) : j;
    qraw[r][j] = __half2float(qv[j]);
    qp[r][(j / V) * (V + 4) + (j % V)] = __half2float(qv[pj]);
  }
  __syncthreads();
  float* const out_h = a.scores + (static_cast<size_t>(b) * a.Hq + h * GQ) * a.n_tok;
  if (part == 0) {  // fp16 sinks: s = scale * q . RoPE_n(sink_n)
    for (int e = warp; e < min(a.n_sink, a.n_tok) * GQ; e += kLitWarps) {
      const int n = e / GQ, r = e % GQ;
      const float acc = sink_dot(qraw[r], a.sink + (static_cast<size_t>(bh) * a.n_sink + n) * D,
                                 a.rope ? a.rope_cs + static_cast<size_t>(n) * D : nullptr, lane, a.rope == 2);
      if (lane == 0) out_h[static_cast<size_t>(r) * a.n_tok + n] = acc * a.scale;
    }
  }
  const int st0 = static_cast<int>(static_cast<long long>(a.n_step) * part / a.splits);
  const int st1 = static_cast<int>(static_cast<long long>(a.n_step) * (part + 1) / a.splits);
  const size_t rec0 = static_cast<size_t>(bh) * a.t_cap;
  const uint32_t qbase = smem_u32(&qp[0][0]) + 4 * s * (V + 4);
  for (int stp = st0 + warp; stp < st1; stp += kLitWarps) {
    const int n = stp * kVecW + slot;
    const bool live = n < a.n_tok && n >= a.n_sink;
    const size_t slot_i = rec0 + (n < a.n_tok ? n : a.n_tok - 1);
    uint32_t w[NW];
    ld_run<NBY, pow2_align(NBY)>(a.codes + slot_i * RB + NBY * s, w);
    float Sg[NGT], Zg[NGT];
#pragma unroll
    for (int gg = 0; gg < NGT; ++gg) {
      const float2 sz = __half22float2(a.sz[slot_i * NG + (SHARED ? 0 : NGT * s + gg)]);
      Sg[gg] = ROT ? __fmul_rn(sz.x, a.rscale) : sz.x;
      Zg[gg] = ROT ? __fmul_rn(sz.y, a.rscale) : sz.y;
    }
    float2 P[V / 2];
    unpack_inverse<D, BITS, G, ROT>(w, Sg, Zg, s, P);
    float acc[GQ];
#pragma unroll
    for (int r = 0; r < GQ; ++r) {
      float2 a2 = f2(0.0f, 0.0f);
#pragma unroll
      for (int g = 0; g < V / 4; ++g) {  // channels 4g .. 4g + 3 of this lane's half
        const uint4 qv = lds128(qbase + 4 * (r * QP + 4 * g));
        a2 = fma2(P[2 * g], f2(__uint_as_float(qv.x), __uint_as_float(qv.z)), a2);
        a2 = fma2(P[2 * g + 1], f2(__uint_as_float(qv.y), __uint_as_float(qv.w)), a2);
      }
      acc[r] = a2.x + a2.y;
      acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 1);
    }
    if (live) {  // both lanes hold every sum: query head r is written by lane half r mod 2
#pragma unroll
      for (int r = 0; r < GQ; ++r)
        if ((GQ == 1 ? 0 : (r & 1)) == s) out_h[static_cast<size_t>(r) * a.n_tok + n] = acc[r] * a.scale;
    }
  }
}

template <int BITS, int G, int GQ, bool ROT>
kvq_status run_literal(const kvq_desc& d, const LitArgs& a0, const LaunchCtx& ctx, cudaStream_t st) {
  LitArgs a = a0;
  const void* fn = reinterpret_cast<const void*>(k_score_literal<BITS, G, GQ, ROT>);
  const int per_sm = occupancy_once(fn, kLitThreads, 0);
  const long long streams = static_cast<long long>(d.batch) * d.heads;
  a.n_step = (a.n_tok + kVecW - 1) / kVecW;
  // as many CTAs per stream as one wave holds, each with at least one step per warp
  long long splits = static_cast<long long>(ctx.num_sms) * per_sm / streams;
  const long long max_splits = (a.n_step + kLitWarps - 1) / kLitWarps;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  if (streams * splits >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
  a.splits = static_cast<int>(splits);
  k_score_literal<BITS, G, GQ, ROT><<<static_cast<unsigned>(streams * splits), kLitThreads, 0, st>>>(a);
  return launch_status();
}

template <int BITS, int G, bool ROT>
kvq_status literal_by_gq(const kvq_desc& d, const LitArgs& a, int gq, const LaunchCtx& ctx, cudaStream_t st) {
  switch (gq) {
    case 1: return run_literal<BITS, G, 1, ROT>(d, a, ctx, st);
    case 2: return run_literal<BITS, G, 2, ROT>(d, a, ctx, st);
    case 4: return run_literal<BITS, G, 4, ROT>(d, a, ctx, st);
    case 8: return run_literal<BITS, G, 8, ROT>(d, a, ctx, st);
    default: return KVQ_ERR_UNSUPPORTED;
  }
}

template <int D, int BITS, int G, bool ROT>
kvq_status run(bool enc, const HeadArgs& a, int out_fp32, const LaunchCtx& ctx, cudaStream_t st) {
  const size_t smem = a.perm ? static_cast<size_t>(kThreads / 32) * warp_buf<D>(enc) : 0;
  const void* fn = enc        ? reinterpret_cast<const void*>(k_encode_head<D, BITS, G, ROT>)
                   : out_fp32 ? reinterpret_cast<const void*>(k_decode_head<D, BITS, G, ROT, true>)
                              : reinterpret_cast<const void*>(k_decode_head<D, BITS, G, ROT, false>);
  if (smem && !set_smem_once(fn, smem)) return KVQ_ERR_CUDA;
  const int per_sm = occupancy_once(fn, kThreads, smem);
  const long long steps = (static_cast<long long>(a.n_vec) + kVecW * (kThreads / 32) - 1) / (kVecW * (kThreads / 32));
  const long long want = static_cast<long long>(ctx.num_sms) * per_sm;
  const unsigned grid = static_cast<unsigned>(steps < want ? steps : want);
  if (enc)
    k_encode_head<D, BITS, G, ROT><<<grid, kThreads, smem, st>>>(a);
  else if (out_fp32)
    k_decode_head<D, BITS, G, ROT, true><<<grid, kThreads, smem, st>>>(a);
  else
    k_decode_head<D, BITS, G, ROT, false><<<grid, kThreads, smem, st>>>(a);
  return launch_status();
}

kvq_status dispatch(bool enc, const kvq_desc& d, const HeadArgs& a, int out_fp32, const LaunchCtx& ctx,
                    cudaStream_t st) {
  const bool rot = d.rot == KVQ_ROT_FWHT_HEAD;
#define KVQ_CASE(D_, B_, G_)                                                  \
  if (d.head_dim == D_ && d.bits == B_ && d.group == G_)                     \
    return rot ? run<D_, B_, G_, true>(enc, a, out_fp32, ctx, st)            \
               : run<D_, B_, G_, false>(enc, a, out_fp32, ctx, st);
#define KVQ_BITS(D_, G_) KVQ_CASE(D_, 2, G_) KVQ_CASE(D_, 3, G_) KVQ_CASE(D_, 4, G_)
  KVQ_BITS(128, 128)
  KVQ_BITS(128, 64)
  KVQ_BITS(128, 32)
  KVQ_BITS(64, 64)
  KVQ_BITS(64, 32)
#undef KVQ_BITS
#undef KVQ_CASE
  return KVQ_ERR_UNSUPPORTED;
}

bool make_args(const kvq_desc& d, const kvq_tables& tb, const kvq_packed& p, HeadArgs& a) {
  const unsigned long long n = static_cast<unsigned long long>(d.batch) * d.heads * d.tokens;
  if (n >= (1ull << 31)) return false;  // vector indices are 31-bit
  a = HeadArgs{};
  a.B = d.batch;
  a.H = d.heads;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.t_cap = d.t_cap;
  a.n_sink = d.n_sink;
  a.rope = d.rope;
  a.n_vec = static_cast<uint32_t>(n);
  a.div_t = FastDiv(static_cast<uint32_t>(d.tokens));
  a.div_h = FastDiv(static_cast<uint32_t>(d.heads));
  a.rscale = static_cast<float>(1.0 / sqrt(static_cast<double>(d.head_dim)));
  a.perm = tb.perm;
  a.rope_cs = tb.rope_cs;
  a.codes = p.codes;
  a.sz = static_cast<__half2*>(p.scale_zero);
  a.sink = static_cast<__half*>(p.sink);
  return true;
}

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

}  // namespace

kvq_status launch_encode_head(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                              cudaStream_t st, const LaunchCtx& ctx) {
  HeadArgs a;
  if (!make_args(d, tb, out, a)) return KVQ_ERR_UNSUPPORTED;
  a.x = static_cast<const __half*>(x);
  a.v8 = aligned32(x);
  return dispatch(true, d, a, 0, ctx, st);
}

kvq_status launch_decode_head(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                              int out_fp32, cudaStream_t st, const LaunchCtx& ctx) {
  HeadArgs a;
  if (!make_args(d, tb, in, a)) return KVQ_ERR_UNSUPPORTED;
  a.out = x_out;
  a.v8 = aligned32(x_out);
  return dispatch(false, d, a, out_fp32, ctx, st);
}

kvq_status launch_score_literal(const kvq_desc& d, const void* q, int q_heads, const kvq_packed& cache,
                                const kvq_tables& tb, int n_tokens, float scale, float* scores, cudaStream_t st,
                                const LaunchCtx& ctx) {
  if (d.head_dim != 128 || d.quant != KVQ_Q_MINMAX) return KVQ_ERR_UNSUPPORTED;
  LitArgs a{};
  a.H = d.heads;
  a.Hq = q_heads;
  a.t_cap = d.t_cap;
  a.n_tok = n_tokens;
  a.n_sink = d.n_sink;
  a.rope = d.rope;
  a.scale = scale;
  a.rscale = static_cast<float>(1.0 / sqrt(128.0));
  a.q = static_cast<const __half*>(q);
  a.perm = tb.perm;
  a.rope_cs = tb.rope_cs;
  a.codes = cache.codes;
  a.sz = static_cast<const __half2*>(cache.scale_zero);
  a.sink = static_cast<const __half*>(cache.sink);
  a.scores = scores;
  const int gq = q_heads / d.heads;
  const bool rot = d.rot == KVQ_ROT_FWHT_HEAD;
#define KVQ_CASE(B_, G_)                                                                   \
  if (d.bits == B_ && d.group == G_)                                                     \
    return rot ? literal_by_gq<B_, G_, true>(d, a, gq, ctx, st) : literal_by_gq<B_, G_, false>(d, a, gq, ctx, st);
#define KVQ_BITS(G_) KVQ_CASE(2, G_) KVQ_CASE(3, G_) KVQ_CASE(4, G_)
  KVQ_BITS(128)
  KVQ_BITS(64)
  KVQ_BITS(32)
#undef KVQ_BITS
#undef KVQ_CASE
  return KVQ_ERR_UNSUPPORTED;
}

}  // namespace kvq
