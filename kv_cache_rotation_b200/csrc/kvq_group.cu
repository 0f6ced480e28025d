// Grouped-head encode / decode ("RotateKV: Accurate and Robust 2-Bit KV Cache
// Quantization for LLMs via Outlier-Aware Adaptive Rotations", abstract and
// 关键设计: pre-RoPE grouped-head rotation). The HG heads of one token are
// concatenated (index = local_head * 128 + channel), permuted per head,
// transformed by one normalised FWHT of size HG*128 in natural (Sylvester)
// stride order -- the 7 in-head strides first, then the log2(HG) cross-head
// strides -- and only then rotated by RoPE head slice by head slice; each
// head slice is quantized with per-group min-max and packed.
//
// Persistent CTAs of kThreads threads walk tiles of HG heads x NT tokens
// (HG * NT = kThreads / 2 head rows) of one batch. Every thread holds 64
// values:
//   phase 1: thread (half s, head, token) holds channels [64s, 64s + 64) of
//            one head row (loaded straight from global memory, the next
//            tile's row prefetched into registers) and runs the strides
//            1 .. 32;
//   exchange: the rows go through shared memory as fp32 in 16-byte chunks of
//            four channels (rows padded to 17 chunks: every access is a base
//            address plus a constant, and conflict-free);
//   phase 2: thread (token, k) holds, for every head of the group and both
//            halves, the 4Q channels [4kQ, 4kQ + 4Q) (Q = 8/HG), runs the
//            stride 64 and the cross-head strides, RoPE, the group min/max (a
//            transpose-reduce over the 2*HG lanes of the token; one lane per
//            group derives its fp16 scale/zero and publishes (Z, 1/S) in
//            shared memory), quantizes and packs.
// Decode streams the packed codes in by TMA and the scales by cp.async, runs
// the phases in reverse and stores its output rows straight to global memory.
// The kernels are bound by the fp32 pipe and shared-memory bandwidth, not by
// HBM: the exchange is the one transpose the stride order forces.
//
// Arithmetic is fp32 with the oracle's operation order, two lanes at a time
// (sm_100 packed fp32 add / mul / fma). The FWHT normalisation 1/sqrt(HG*128)
// is a power of two for HG = 2 and 8 and is then folded exactly into the RoPE
// cos/sin (keys) or into the quantizer's zero and reciprocal scale (values).
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int D = 128;
#ifndef KVQ_GROUP_CT
#define KVQ_GROUP_CT 64
#endif
constexpr int kThreads = KVQ_GROUP_CT;  // threads per CTA (64, 128 or 256)
constexpr int kRows = kThreads / 2;     // head rows per tile
constexpr int kPitch = 272;             // exchange row: 16 chunks of 16 bytes + one pad chunk
constexpr int kXch = kRows * kPitch;    // fp32 exchange of one 64-channel half
constexpr int kCodes = kRows * 64;      // packed codes of one tile (at most 64 bytes a row)
constexpr int kStage = 264;             // row pitch of the fp16 staging used by the permutation
constexpr int kHalf = kRows * 128;      // decode: one 64-channel half of the fp16 output tile (one TMA box)
constexpr int kXchS = kRows * 256;      // decode: XOR-swizzled fp32 exchange of one 64-channel half
static_assert(kRows >= 32 && kRows <= 128 && (kRows & (kRows - 1)) == 0, "unsupported CTA size");
#ifndef KVQ_GROUP_PRELOAD
#define KVQ_GROUP_PRELOAD 0
#endif
// 1: encode loads the next tile's rows into registers during phase 2 (more
// registers); 0: each tile's rows are loaded when the tile starts.
constexpr bool kPreload = KVQ_GROUP_PRELOAD != 0;

struct GroupArgs {
  int B, H, T, t0, t_cap, n_sink, rope, n_tblk, n_grp, n_tiles;
  int v8;                  // the fp16 / fp32 rows may be moved with 32-byte accesses
  FastDiv div_grp, div_b;  // head groups per batch; batches
  float rscale;            // fp32(1/sqrt(HG*128))
  const __half* x;         // encode input [B][H][T][128]
  void* out;               // decode output [B][H][T][128], fp16 or fp32
  const int16_t* perm;
  const float* rope_cs;    // [rows][128/2][2]
  uint8_t* codes;
  __half2* sz;
  __half* sink;
  uint32_t* err;
  uint64_t wait_ns;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

// Byte offset of 16-byte chunk g (0..15) inside a padded exchange row. Rows
// are kPitch = 17 chunks apart and chunks 8..15 skip one slot, so 8
// consecutive rows at one chunk, or one row at chunks 0..7, 8..15 or at every
// other chunk, fall on 8 distinct bank groups.
__host__ __device__ constexpr uint32_t xoff(int g) { return 16u * static_cast<uint32_t>(g + (g >> 3)); }

// Decode's exchange: byte offset of 16-byte chunk g (0..15) of row rho of an
// unpadded 256-byte-row buffer (it later holds the TMA output tile); r = head *
// NT + token. The chunk index is XOR-swizzled by a rotation of r's low 3 bits:
// 8 consecutive r at one chunk, or consecutive chunks of one or two tokens,
// fall on 8 distinct bank groups.
__device__ __forceinline__ uint32_t xaddr(uint32_t rho, uint32_t r, uint32_t g) {
  const uint32_t sig = ((r << 1) | ((r >> 2) & 1u)) & 7u;
  return rho * 256u + 16u * ((g & 8u) | ((g ^ (g >> 3) ^ sig) & 7u));
}

// Tiles are ordered (token block, batch, head group): the tiles that share a
// token block -- and so the same RoPE rows -- run at the same time.
__device__ __forceinline__ void tile_coords(const GroupArgs& a, int tile, int HG, int NT, int& b, int& h_base,
                                            int& t_base) {
  const uint32_t rest = a.div_grp.div(tile);
  const uint32_t grp = a.div_grp.mod(tile, rest);
  const uint32_t tb = a.div_b.div(rest);
  b = static_cast<int>(a.div_b.mod(rest, tb));
  t_base = static_cast<int>(tb) * NT;
  h_base = static_cast<int>(grp) * HG;
}

// fp16 words (h[2j], h[2j+1]) of 64 consecutive channels -> phase-1 pairs.
__device__ __forceinline__ void halves_to_pairs(const uint32_t (&w)[32], float2 (&P)[32]) {
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    const float2 h01 = __half22float2(*reinterpret_cast<const __half2*>(&w[2 * g]));
    const float2 h23 = __half22float2(*reinterpret_cast<const __half2*>(&w[2 * g + 1]));
    P[2 * g] = f2(h01.x, h23.x);
    P[2 * g + 1] = f2(h01.y, h23.y);
  }
}

// Min/max of NGP groups, each spread over the TPT lanes of one token (an
// aligned lane group). Halving exchanges (upper lanes keep the upper half of
// the groups) and, when TPT > NGP, a final butterfly: lane k ends with the
// totals of group k >> log2(TPT / NGP) in slot 0.
template <int NGP, int TPT>
__device__ __forceinline__ void group_reduce(float (&mn)[NGP], float (&mx)[NGP], int lane) {
#pragma unroll
  for (int i = 0; (TPT >> (i + 1)) >= 1; ++i) {
    const int o = TPT >> (i + 1);
    const int L = NGP >> i;  // groups held before this round
    if (L >= 2) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int j = 0; j < L / 2; ++j) {
        const float send_mn = upper ? mn[j] : mn[j + L / 2];
        const float send_mx = upper ? mx[j] : mx[j + L / 2];
        const float keep_mn = upper ? mn[j + L / 2] : mn[j];
        const float keep_mx = upper ? mx[j + L / 2] : mx[j];
        mn[j] = fminf(keep_mn, __shfl_xor_sync(0xffffffffu, send_mn, o));
        mx[j] = fmaxf(keep_mx, __shfl_xor_sync(0xffffffffu, send_mx, o));
      }
    } else {
      mn[0] = fminf(mn[0], __shfl_xor_sync(0xffffffffu, mn[0], o));
      mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], o));
    }
  }
}

// Store / load NBY bytes of packed codes (little-endian words w). The
// callers' offsets are multiples of the access width used.
template <int NBY>
__device__ __forceinline__ void st_code(uint8_t* p, const uint32_t* w) {
  if constexpr (NBY == 1) {
    *p = static_cast<uint8_t>(w[0]);
  } else if constexpr (NBY == 2) {
    *reinterpret_cast<uint16_t*>(p) = static_cast<uint16_t>(w[0]);
  } else if constexpr (NBY == 3) {
    p[0] = static_cast<uint8_t>(w[0]);
    p[1] = static_cast<uint8_t>(w[0] >> 8);
    p[2] = static_cast<uint8_t>(w[0] >> 16);
  } else if constexpr (NBY == 4) {
    *reinterpret_cast<uint32_t*>(p) = w[0];
  } else if constexpr (NBY == 6) {
    reinterpret_cast<uint16_t*>(p)[0] = static_cast<uint16_t>(w[0]);
    reinterpret_cast<uint16_t*>(p)[1] = static_cast<uint16_t>(w[0] >> 16);
    reinterpret_cast<uint16_t*>(p)[2] = static_cast<uint16_t>(w[1]);
  } else {
    static_assert(NBY == 8, "unsupported code run");
    *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
  }
}
template <int NBY>
__device__ __forceinline__ void ld_code(const uint8_t* p, uint32_t* w) {
  if constexpr (NBY == 1) {
    w[0] = *p;
  } else if constexpr (NBY == 2) {
    w[0] = *reinterpret_cast<const uint16_t*>(p);
  } else if constexpr (NBY == 3) {
    w[0] = static_cast<uint32_t>(p[0]) | (static_cast<uint32_t>(p[1]) << 8) | (static_cast<uint32_t>(p[2]) << 16);
  } else if constexpr (NBY == 4) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else if constexpr (NBY == 6) {
    const uint16_t* q = reinterpret_cast<const uint16_t*>(p);
    w[0] = static_cast<uint32_t>(q[0]) | (static_cast<uint32_t>(q[1]) << 16);
    w[1] = q[2];
  } else {
    static_assert(NBY == 8, "unsupported code run");
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x;
    w[1] = v.y;
  }
}

template <int HG, int BITS, int G>
__global__ void __launch_bounds__(kThreads, 512 / kThreads) k_encode_group(const GroupArgs a) {
  constexpr int NT = kRows / HG;     // tokens per tile
  constexpr int Q = 8 / HG;          // channel quads per phase-2 thread, head and half
  constexpr int TPT = 2 * HG;        // phase-2 threads per token
  constexpr int NG = D / G;          // min-max groups per head
  constexpr int NGP = HG * NG;       // groups per token
  constexpr int SH = TPT > NGP ? 1 : 0;
  constexpr int RB = D * BITS / 8;   // packed bytes per head row
  constexpr int NCB = 4 * Q * BITS;  // code bits per phase-2 thread, head and half
  constexpr int NWC = (NCB + 31) / 32;
  constexpr bool FOLD = (HG != 4);   // 1/sqrt(HG*128) is a power of two
  constexpr bool PRE_CS = (Q == 1);  // the thread's RoPE rows fit in registers early
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(16) float2 prm[NT * NGP];  // (Z, R) of every group of the tile
  const uint32_t x0_u = smem_u32(align1024(smem_raw));  // exchange, lower half
  const uint32_t x1_u = x0_u + kXch;                    // exchange, upper half
  const int tid = threadIdx.x, lane = tid & 31;
  const int s1 = tid / kRows, r1 = tid % kRows, h1 = r1 / NT, t1 = r1 % NT;  // phase-1 role
  const int t2 = tid / TPT, k2 = tid % TPT;                                    // phase-2 role
  const float r = a.rscale;
  const bool v8 = a.v8 != 0;

  // this thread's half row of a tile (zeros past the last token)
  uint32_t raw[32];
  auto load_raw = [&](int tile) {
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    const int tt = t_base + t1;
    if (tt < a.T) {
      ld_row<32>(a.x + ((static_cast<size_t>(b) * a.H + h_base + h1) * a.T + tt) * D + 64 * s1, v8, raw);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) raw[i] = 0u;
    }
  };
  if (kPreload && blockIdx.x < a.n_tiles) load_raw(blockIdx.x);

  for (int it = 0;; ++it) {
    const int tile = blockIdx.x + it * gridDim.x;
    if (tile >= a.n_tiles) break;
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    if (!kPreload) load_raw(tile);

    // RoPE rows of this thread's phase-2 channels (from L2)
    const uint4* rp =
        a.rope ? reinterpret_cast<const uint4*>(a.rope_cs + static_cast<size_t>(min(a.t0 + t_base + t2,
                                                                                    a.t0 + a.T - 1)) * D)
               : nullptr;
    uint4 cs_pre[2];
    if (PRE_CS && a.rope) {
      cs_pre[0] = __ldg(rp + k2);
      cs_pre[1] = __ldg(rp + 16 + k2);
    }

    // ---------------- phase 1: 64 channels of one head row, strides 1 .. 32
    float2 P[32];
    {
      const int tt = t_base + t1, m = a.t0 + tt;
      if (tt < a.T && m < a.n_sink) {
        uint4* dst = reinterpret_cast<uint4*>(
            a.sink + ((static_cast<size_t>(b) * a.H + h_base + h1) * a.n_sink + m) * D + 64 * s1);
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[c] = make_uint4(raw[4 * c], raw[4 * c + 1], raw[4 * c + 2], raw[4 * c + 3]);
      }
      if (a.perm) {  // the gather reads the whole row: stage the tile in shared memory
        __syncthreads();  // the previous tile's exchange reads are done
        const uint32_t row_u = x0_u + r1 * kStage;
#pragma unroll
        for (int i = 0; i < 16; ++i) sts64(row_u + 128 * s1 + 8 * i, raw[2 * i], raw[2 * i + 1]);
        __syncthreads();
        const int16_t* pr = a.perm + static_cast<size_t>(h_base + h1) * D + 64 * s1;
        float xv[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
          const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
            xv[8 * c + i] = __half2float(__ushort_as_half(lds16(row_u + 2 * e)));
          }
        }
#pragma unroll
        for (int g = 0; g < 16; ++g) {
          P[2 * g] = f2(xv[4 * g], xv[4 * g + 2]);
          P[2 * g + 1] = f2(xv[4 * g + 1], xv[4 * g + 3]);
        }
      } else {
        halves_to_pairs(raw, P);
      }
      fwht_pairs<64>(P);
    }
    __syncthreads();  // the previous tile's exchange reads (and the gathers) are done
    {
      const uint32_t rowp = (s1 == 0 ? x0_u : x1_u) + r1 * kPitch;
#pragma unroll
      for (int g = 0; g < 16; ++g)
        sts128(rowp + xoff(g), make_uint4(__float_as_uint(P[2 * g].x), __float_as_uint(P[2 * g].y),
                                          __float_as_uint(P[2 * g + 1].x), __float_as_uint(P[2 * g + 1].y)));
    }
    __syncthreads();
    // A[h][half][q][e] = (x[c + e], x[c + 2 + e]) of head h, c = 64 half + 4 (k2 Q + q)
    float2 A[HG][2][Q][2];
    {
      const uint32_t base = x0_u + t2 * kPitch + xoff(k2 * Q);
#pragma unroll
      for (int hs = 0; hs < 2; ++hs)
#pragma unroll
        for (int h = 0; h < HG; ++h)
#pragma unroll
          for (int q = 0; q < Q; ++q) {
            const uint4 u = lds128(base + hs * kXch + h * NT * kPitch + 16 * q);
            A[h][hs][q][0] = f2(__uint_as_float(u.x), __uint_as_float(u.y));
            A[h][hs][q][1] = f2(__uint_as_float(u.z), __uint_as_float(u.w));
          }
    }
    if (kPreload) {  // the next tile's rows arrive while this one finishes
      const int next = tile + gridDim.x;
      if (next < a.n_tiles) load_raw(next);
    }

    // ---------------- phase 2: stride 64, cross-head strides
#pragma unroll
    for (int h = 0; h < HG; ++h)
#pragma unroll
      for (int q = 0; q < Q; ++q)
#pragma unroll
        for (int e = 0; e < 2; ++e) bfly(A[h][0][q][e], A[h][1][q][e]);
#pragma unroll
    for (int sh = 1; sh < HG; sh <<= 1)
#pragma unroll
      for (int h = 0; h < HG; ++h)
        if ((h & sh) == 0)
#pragma unroll
          for (int hs = 0; hs < 2; ++hs)
#pragma unroll
            for (int q = 0; q < Q; ++q)
#pragma unroll
              for (int e = 0; e < 2; ++e) bfly(A[h][hs][q][e], A[h + sh][hs][q][e]);
    if (!FOLD) {
#pragma unroll
      for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int hs = 0; hs < 2; ++hs)
#pragma unroll
          for (int q = 0; q < Q; ++q)
#pragma unroll
            for (int e = 0; e < 2; ++e) A[h][hs][q][e] = mul2(A[h][hs][q][e], f2(r, r));
    }
    if (a.rope) {  // y0 = fma(x0, c, -(x1*s)), y1 = fma(x0, s, x1*c), two pairs at a time
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          // table chunk = (c_i, s_i, c_i+1, s_i+1) for channels c .. c+3; scaled by r when folding (exact)
          const uint4 cv = PRE_CS ? cs_pre[hs] : __ldg(rp + 16 * hs + k2 * Q + q);
          float2 cc = f2(__uint_as_float(cv.x), __uint_as_float(cv.z));
          float2 ss = f2(__uint_as_float(cv.y), __uint_as_float(cv.w));
          if (FOLD) {
            cc = mul2(cc, f2(r, r));
            ss = mul2(ss, f2(r, r));
          }
          const float2 nss = f2(-ss.x, -ss.y);
#pragma unroll
          for (int h = 0; h < HG; ++h) {
            const float2 x0 = A[h][hs][q][0], x1 = A[h][hs][q][1];
            A[h][hs][q][0] = fma2(x0, cc, mul2(x1, nss));
            A[h][hs][q][1] = fma2(x0, ss, mul2(x1, cc));
          }
        }
      }
    }
    // values are now p (keys, or every HG = 4 tensor) or p / r (values when folding)
    const bool unscaled = FOLD && !a.rope;
    float mn[NGP], mx[NGP];
#pragma unroll
    for (int h = 0; h < HG; ++h) {
#pragma unroll
      for (int grp = 0; grp < NG; ++grp) {
        float lo = 0.0f, hi = 0.0f;
        bool first = true;
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
          if (NG == 2 && hs != grp) continue;
#pragma unroll
          for (int q = 0; q < Q; ++q) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float2 v = A[h][hs][q][e];
              if (first) {
                lo = fminf(v.x, v.y);
                hi = fmaxf(v.x, v.y);
                first = false;
              } else {
                lo = min3f(lo, v.x, v.y);
                hi = max3f(hi, v.x, v.y);
              }
            }
          }
        }
        mn[h * NG + grp] = lo;
        mx[h * NG + grp] = hi;
      }
    }
    group_reduce<NGP, TPT>(mn, mx, lane);
    const int tt2 = t_base + t2, m2 = a.t0 + tt2;
    const bool store = tt2 < a.T;
    const bool sink_tok = m2 < a.n_sink;
    {
      const int gi = k2 >> SH;  // the group whose totals this lane holds
      float lo = mn[0], hi = mx[0];
      if (unscaled) {
        lo = __fmul_rn(lo, r);
        hi = __fmul_rn(hi, r);
      }
      const QParams p = minmax_params<BITS>(lo, hi);
      if ((k2 & ((1 << SH) - 1)) == 0) {
        // Z / r is exact (power of two). A sink slot quantizes with Z = R = 0:
        // every code of it comes out 0.
        prm[t2 * NGP + gi] = sink_tok ? f2(0.0f, 0.0f)
                                      : f2(unscaled ? __fdiv_rn(p.Z, r) : p.Z, unscaled ? __fmul_rn(p.R, r) : p.R);
        if (store) {
          const size_t slot = (static_cast<size_t>(b) * a.H + h_base + gi / NG) * a.t_cap + m2;
          a.sz[slot * NG + gi % NG] = sink_tok ? __halves2half2(__ushort_as_half(0), __ushort_as_half(0)) : p.sz;
        }
      }
    }
    __syncwarp();
    float4 zr4[NGP / 2];  // (Z, R) of groups 2j and 2j + 1
#pragma unroll
    for (int j = 0; j < NGP / 2; ++j) zr4[j] = *reinterpret_cast<const float4*>(&prm[t2 * NGP + 2 * j]);

    // ---------------- quantize and pack this thread's runs of 4Q channels
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      const size_t slot = (static_cast<size_t>(b) * a.H + h_base + h) * a.t_cap + m2;
      uint8_t* rec = a.codes + slot * RB;
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const int gi = h * NG + (NG == 2 ? hs : 0);
        const float Z = (gi & 1) ? zr4[gi >> 1].z : zr4[gi >> 1].x;
        const float R = (gi & 1) ? zr4[gi >> 1].w : zr4[gi >> 1].y;
        const float2 nZ = f2(-Z, -Z), R2 = f2(R, R), M2 = f2(kMagicRound, kMagicRound);
        // raw fp32 patterns kMagicBits + code of local channels 0 .. 4Q-1
        uint32_t t[4 * Q];
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          const float2 ua = fma2(add2(A[h][hs][q][0], nZ), R2, M2);
          const float2 ub = fma2(add2(A[h][hs][q][1], nZ), R2, M2);
          t[4 * q + 0] = __float_as_uint(ua.x);
          t[4 * q + 1] = __float_as_uint(ub.x);
          t[4 * q + 2] = __float_as_uint(ua.y);
          t[4 * q + 3] = __float_as_uint(ub.y);
        }
        uint32_t w[NWC];
        if constexpr (32 % BITS == 0) {
          constexpr int PER = 32 / BITS;  // codes per word
#pragma unroll
          for (int i = 0; i < NWC; ++i) {
            const int lo_c = i * PER;
            const int n_c = (4 * Q - lo_c) < PER ? (4 * Q - lo_c) : PER;
            uint32_t v = t[lo_c + n_c - 1];
#pragma unroll
            for (int j = n_c - 2; j >= 0; --j) v = (v << BITS) + t[lo_c + j];  // codes never straddle a word
            w[i] = v;
          }
          if constexpr (NCB > 22) {
#pragma unroll
            for (int i = 0; i < NWC; ++i)
              w[i] -= (NCB - 32 * i >= 32) ? magic_offset<BITS, PER>() : magic_offset<BITS, (NCB % 32) / BITS>();
          }
        } else {
#pragma unroll
          for (int i = 0; i < NWC; ++i) w[i] = 0u;
#pragma unroll
          for (int j = 0; j < 4 * Q; ++j) {
            const int pos = j * BITS;
            const uint32_t c = t[j] - kMagicBits;
            w[pos >> 5] |= c << (pos & 31);
            if ((pos & 31) + BITS > 32) w[(pos >> 5) + 1] |= c >> (32 - (pos & 31));
          }
        }
        if constexpr (NCB % 8 != 0) {
          // 12-bit runs (HG = 8, 3 bits): even lanes append their odd neighbour's run
          const uint32_t nb = __shfl_down_sync(0xffffffffu, w[0], 1);
          if (store && (k2 & 1) == 0) {
            const uint32_t v = w[0] | (nb << NCB);
            st_code<2 * NCB / 8>(rec + (64 * hs + 4 * k2 * Q) * BITS / 8, &v);
          }
        } else {
          if (store) st_code<NCB / 8>(rec + (64 * hs + 4 * k2 * Q) * BITS / 8, w);
        }
      }
    }
  }
}

template <int HG, int BITS, int G, bool F32>
__global__ void __launch_bounds__(kThreads, 512 / kThreads) k_decode_group(const __grid_constant__ CUtensorMap cmap,
                                                               const __grid_constant__ CUtensorMap omap,
                                                               const GroupArgs a) {
  constexpr int NT = kRows / HG;
  constexpr int Q = 8 / HG;
  constexpr int TPT = 2 * HG;
  constexpr int NG = D / G;
  constexpr int RB = D * BITS / 8;
  constexpr int NCB = 4 * Q * BITS;
  constexpr int NWC = (NCB + 31) / 32;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  constexpr bool PRE_CS = (Q == 1);
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[2];
  __shared__ __half2 szs[2][kRows * NG];  // scale/zero of the tile's rows, by cp.async
  uint8_t* sm = align1024(smem_raw);
  uint8_t* xr = sm + 2 * kCodes;  // exchange (two halves), then the output tile
  const uint32_t xr_u = smem_u32(xr);
  const int tid = threadIdx.x;
  const int s1 = tid / kRows, r1 = tid % kRows, h1 = r1 / NT, t1 = r1 % NT;
  const int t2 = tid / TPT, k2 = tid % TPT;
  const float r = a.rscale;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  auto issue = [&](int tile, int s) {
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    mbar_arrive_expect_tx(&full[s], kRows * RB);
    tma_load_3d(sm + s * kCodes, &cmap, 0, a.t0 + t_base, b * a.H + h_base, &full[s]);
  };
  // scale/zero of one tile's rows (zero-filled past the last token)
  auto fetch_sz = [&](int tile, int buf) {
    if (tid < kRows * NG) {
      int b, h_base, t_base;
      tile_coords(a, tile, HG, NT, b, h_base, t_base);
      const int rr = tid % kRows, grp = tid / kRows;
      const int h = rr / NT, t = rr % NT;
      const bool live = t_base + t < a.T;
      const size_t slot = (static_cast<size_t>(b) * a.H + h_base + h) * a.t_cap + a.t0 + t_base + t;
      cp_async4(smem_u32(&szs[buf][tid]), live ? static_cast<const void*>(a.sz + slot * NG + grp) : a.sz,
                live ? 4u : 0u);
    }
    cp_async_commit();
  };
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      const int tile = blockIdx.x + s * gridDim.x;
      if (tile < a.n_tiles) issue(tile, s);
    }
  }
  if (blockIdx.x < a.n_tiles) fetch_sz(blockIdx.x, 0);
  cp_async_wait_all();
  __syncthreads();
  bool ok = true;

  for (int it = 0;; ++it) {
    const int tile = blockIdx.x + it * gridDim.x;
    if (tile >= a.n_tiles) break;
    const int s = it & 1;
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    {
      const int next = tile + gridDim.x;
      if (next < a.n_tiles) fetch_sz(next, s ^ 1);
    }
    const uint4* rp =
        a.rope ? reinterpret_cast<const uint4*>(a.rope_cs + static_cast<size_t>(min(a.t0 + t_base + t2,
                                                                                    a.t0 + a.T - 1)) * D)
               : nullptr;
    uint4 cs_pre[2];
    if (PRE_CS && a.rope) {
      cs_pre[0] = __ldg(rp + k2);
      cs_pre[1] = __ldg(rp + 16 + k2);
    }
    ok = mbar_wait(&full[s], (it >> 1) & 1, a.wait_ns, a.err);

    // ---------------- phase 2 (reverse): dequantize (normalisation folded in), inverse RoPE, strides
    float2 A[HG][2][Q][2];
    const uint8_t* cst = sm + s * kCodes;
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      const uint8_t* rec = cst + (h * NT + t2) * RB;
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const float2 szf = __half22float2(szs[s][(NG == 2 ? hs : 0) * kRows + h * NT + t2]);
        const float S = __fmul_rn(szf.x, r), Z = __fmul_rn(szf.y, r);
        uint32_t w[NWC];
        if constexpr (NCB % 8 != 0) {  // 12-bit runs start half a byte in for odd k2
          const int bit = (64 * hs + 4 * k2 * Q) * BITS;
          const uint8_t* p = rec + (bit >> 3);
          w[0] = ((static_cast<uint32_t>(p[0]) | (static_cast<uint32_t>(p[1]) << 8)) >> (bit & 7)) & 0xfffu;
        } else {
          ld_code<NCB / 8>(rec + (64 * hs + 4 * k2 * Q) * BITS / 8, w);
        }
        // Codes 0 and 2 of a quad are masked in place at bit 0, codes 1 and 3
        // at bit BITS; read through the fp32 pattern 2^23 + v they give
        // code * 2^p, and the power of two 2^p is folded exactly into the scale.
        const float2 S0 = f2(S, S), S1 = f2(S * (1.0f / (1 << BITS)), S * (1.0f / (1 << BITS)));
        const float2 Z2 = f2(Z, Z), nM = f2(-8388608.0f, -8388608.0f);
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          const int pos = 4 * q * BITS;
          const uint32_t lo = w[pos >> 5] >> (pos & 31);
          const uint32_t w0 = (32 - (pos & 31) >= 4 * BITS || (pos >> 5) + 1 >= NWC)
                                  ? lo
                                  : (lo | (w[(pos >> 5) + 1] << (32 - (pos & 31))));
          const uint32_t w1 = w0 >> (2 * BITS);
          const float2 c02 =
              f2(__uint_as_float(0x4B000000u | (w0 & MASK)), __uint_as_float(0x4B000000u | (w1 & MASK)));
          const float2 c13 = f2(__uint_as_float(0x4B000000u | (w0 & (MASK << BITS))),
                                __uint_as_float(0x4B000000u | (w1 & (MASK << BITS))));
          A[h][hs][q][0] = fma2(add2(c02, nM), S0, Z2);
          A[h][hs][q][1] = fma2(add2(c13, nM), S1, Z2);
        }
      }
    }
    if (a.rope) {
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          const uint4 cv = PRE_CS ? cs_pre[hs] : __ldg(rp + 16 * hs + k2 * Q + q);
          const float2 cc = f2(__uint_as_float(cv.x), __uint_as_float(cv.z));
          const float2 ss = f2(__uint_as_float(cv.y), __uint_as_float(cv.w));
          const float2 nss = f2(-ss.x, -ss.y);
#pragma unroll
          for (int h = 0; h < HG; ++h) {  // x0 = y0 c + y1 s, x1 = y1 c - y0 s
            const float2 y0 = A[h][hs][q][0], y1 = A[h][hs][q][1];
            A[h][hs][q][0] = fma2(y0, cc, mul2(y1, ss));
            A[h][hs][q][1] = fma2(y1, cc, mul2(y0, nss));
          }
        }
      }
    }
#pragma unroll
    for (int sh = 1; sh < HG; sh <<= 1)
#pragma unroll
      for (int h = 0; h < HG; ++h)
        if ((h & sh) == 0)
#pragma unroll
          for (int hs = 0; hs < 2; ++hs)
#pragma unroll
            for (int q = 0; q < Q; ++q)
#pragma unroll
              for (int e = 0; e < 2; ++e) bfly(A[h][hs][q][e], A[h + sh][hs][q][e]);
#pragma unroll
    for (int h = 0; h < HG; ++h)
#pragma unroll
      for (int q = 0; q < Q; ++q)
#pragma unroll
        for (int e = 0; e < 2; ++e) bfly(A[h][0][q][e], A[h][1][q][e]);

    // The previous tile's output store has read the exchange region, and the
    // codes stage is consumed. A timed-out wait ends the CTA's work uniformly.
    if (tid == 0) bulk_wait_read<0>();
    if (!__syncthreads_and(ok)) {
      ok = false;
      break;
    }
    if (tid == 0 && tile + 2 * static_cast<int>(gridDim.x) < a.n_tiles) issue(tile + 2 * gridDim.x, s);

    // ---------------- exchange -> phase-1 registers
#pragma unroll
    for (int hs = 0; hs < 2; ++hs)
#pragma unroll
      for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int q = 0; q < Q; ++q)
          sts128(xr_u + hs * kXchS + xaddr(t2 * HG + h, h * NT + t2, k2 * Q + q),
                 make_uint4(__float_as_uint(A[h][hs][q][0].x), __float_as_uint(A[h][hs][q][0].y),
                            __float_as_uint(A[h][hs][q][1].x), __float_as_uint(A[h][hs][q][1].y)));
    __syncthreads();
    float2 P[32];
    {
      const uint32_t xb = xr_u + s1 * kXchS;
      const uint32_t rho = t1 * HG + h1;
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        const uint4 u = lds128(xb + xaddr(rho, r1, g));
        P[2 * g] = f2(__uint_as_float(u.x), __uint_as_float(u.y));
        P[2 * g + 1] = f2(__uint_as_float(u.z), __uint_as_float(u.w));
      }
    }
    __syncthreads();

    // ---------------- phase 1 (reverse): in-head strides, inverse permutation, output
    fwht_pairs<64>(P);
    const int tt = t_base + t1, m = a.t0 + tt;
    const bool sink_tok = tt < a.T && m < a.n_sink;
    const bool permute = a.perm != nullptr && !sink_tok;
    const int16_t* pr = a.perm ? a.perm + static_cast<size_t>(h_base + h1) * D + 64 * s1 : nullptr;
    float x[64];
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      x[4 * g] = P[2 * g].x;
      x[4 * g + 2] = P[2 * g].y;
      x[4 * g + 1] = P[2 * g + 1].x;
      x[4 * g + 3] = P[2 * g + 1].y;
    }
    if (sink_tok) {  // sink positions come back verbatim
      const uint4* src = reinterpret_cast<const uint4*>(
          a.sink + ((static_cast<size_t>(b) * a.H + h_base + h1) * a.n_sink + m) * D + 64 * s1);
#pragma unroll
      for (int c = 0; c < 8; ++c) h8_to_f32(__ldg(src + c), &x[8 * c]);
    }
    if constexpr (!F32) {
      if (permute) {  // x'[perm[j]] = x[j], written straight into the output row
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
          const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
            sts16(xr_u + (e >> 6) * kHalf + sw128(r1, (e & 63) >> 3) + (e & 7) * 2,
                  __half_as_ushort(__float2half_rn(x[8 * c + i])));
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) sts128(xr_u + s1 * kHalf + sw128(r1, c), f32_to_h8(&x[8 * c]));
      }
    } else {  // fp32: four 32-channel boxes of 16 KB
      if (permute) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
          const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
            sts32f(xr_u + (e >> 5) * kHalf + sw128(r1, (e & 31) >> 2) + (e & 3) * 4, x[8 * c + i]);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c)
          sts128(xr_u + (2 * s1 + (c >> 3)) * kHalf + sw128(r1, c & 7),
                 make_uint4(__float_as_uint(x[4 * c]), __float_as_uint(x[4 * c + 1]), __float_as_uint(x[4 * c + 2]),
                            __float_as_uint(x[4 * c + 3])));
      }
    }
    cp_async_wait_all();  // the next tile's scale/zero rows, published by the barrier below
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      if constexpr (!F32) {
        tma_store_3d(&omap, 0, t_base, b * a.H + h_base, xr);
        tma_store_3d(&omap, 64, t_base, b * a.H + h_base, xr + kHalf);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) tma_store_3d(&omap, 32 * j, t_base, b * a.H + h_base, xr + j * kHalf);
      }
      bulk_commit();
    }
  }
  if (tid == 0) {
    bulk_wait_read<0>();  // the last stores have read shared memory
    if (!ok)              // let copies in flight land (bounded) before the CTA exits
      for (int s = 0; s < 2; ++s)
        for (uint32_t p = 0; p < 2; ++p) mbar_wait(&full[s], p, a.wait_ns, a.err);
  }
  cp_async_wait_all();
}

template <int HG, int BITS, int G>
kvq_status run(bool enc, const GroupArgs& a, const CUtensorMap& cm, const CUtensorMap& om, int out_fp32,
               const LaunchCtx& ctx, cudaStream_t st) {
  const size_t smem =
      enc ? 1024 + 2 * static_cast<size_t>(kXch) : 1024 + 2 * static_cast<size_t>(kCodes) + 2 * kXchS;
  const void* fn = enc        ? reinterpret_cast<const void*>(k_encode_group<HG, BITS, G>)
                   : out_fp32 ? reinterpret_cast<const void*>(k_decode_group<HG, BITS, G, true>)
                              : reinterpret_cast<const void*>(k_decode_group<HG, BITS, G, false>);
  if (!set_smem_once(fn, smem)) return KVQ_ERR_CUDA;
  const int per_sm = occupancy_once(fn, kThreads, smem);
  const long long want = static_cast<long long>(ctx.num_sms) * per_sm;
  const unsigned grid = static_cast<unsigned>(a.n_tiles < want ? a.n_tiles : want);
  if (enc)
    k_encode_group<HG, BITS, G><<<grid, kThreads, smem, st>>>(a);
  else if (out_fp32)
    k_decode_group<HG, BITS, G, true><<<grid, kThreads, smem, st>>>(cm, om, a);
  else
    k_decode_group<HG, BITS, G, false><<<grid, kThreads, smem, st>>>(cm, om, a);
  return launch_status();
}

kvq_status dispatch(bool enc, const kvq_desc& d, const GroupArgs& a, const CUtensorMap& cm, const CUtensorMap& om,
                    int out_fp32, const LaunchCtx& ctx, cudaStream_t st) {
#define KVQ_CASE(HG_, B_, G_)                                    \
  if (d.group_heads == HG_ && d.bits == B_ && d.group == G_) \
    return run<HG_, B_, G_>(enc, a, cm, om, out_fp32, ctx, st);
#define KVQ_BITS(HG_, G_) KVQ_CASE(HG_, 2, G_) KVQ_CASE(HG_, 3, G_) KVQ_CASE(HG_, 4, G_)
  KVQ_BITS(8, 128)
  KVQ_BITS(8, 64)
  KVQ_BITS(4, 128)
  KVQ_BITS(4, 64)
  KVQ_BITS(2, 128)
  KVQ_BITS(2, 64)
#undef KVQ_BITS
#undef KVQ_CASE
  return KVQ_ERR_UNSUPPORTED;
}

GroupArgs make_args(const kvq_desc& d, const kvq_tables& tb, const kvq_packed& p, const LaunchCtx& ctx) {
  GroupArgs a{};
  a.B = d.batch;
  a.H = d.heads;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.t_cap = d.t_cap;
  a.n_sink = d.n_sink;
  a.rope = d.rope;
  const int NT = kRows / d.group_heads;
  a.n_tblk = (d.tokens + NT - 1) / NT;
  a.n_grp = d.heads / d.group_heads;
  a.n_tiles = d.batch * a.n_grp * a.n_tblk;
  a.div_grp = FastDiv(static_cast<uint32_t>(a.n_grp));
  a.div_b = FastDiv(static_cast<uint32_t>(d.batch));
  a.rscale = static_cast<float>(1.0 / sqrt(static_cast<double>(d.group_heads) * D));
  a.perm = tb.perm;
  a.rope_cs = tb.rope_cs;
  a.codes = p.codes;
  a.sz = static_cast<__half2*>(p.scale_zero);
  a.sink = static_cast<__half*>(p.sink);
  a.err = ctx.err;
  a.wait_ns = ctx.wait_ns;
  return a;
}

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

}  // namespace

kvq_status launch_encode_group(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                               cudaStream_t st, const LaunchCtx& ctx) {
  GroupArgs a = make_args(d, tb, out, ctx);
  a.x = static_cast<const __half*>(x);
  a.v8 = aligned32(x);
  CUtensorMap unused{};
  return dispatch(true, d, a, unused, unused, 0, ctx, st);
}

kvq_status launch_decode_group(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                               int out_fp32, cudaStream_t st, const LaunchCtx& ctx) {
  const GroupArgs a = make_args(d, tb, in, ctx);
  const int NT = kRows / d.group_heads;
  // packed codes: [B*H][t_cap][RB] bytes; one box = the tile's records
  CUtensorMap cm;
  const uint64_t rb = static_cast<uint64_t>(D) * d.bits / 8;
  const uint64_t cdims[3] = {rb, static_cast<uint64_t>(d.t_cap), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t cstrides[2] = {rb, static_cast<uint64_t>(d.t_cap) * rb};
  const uint32_t cbox[3] = {static_cast<uint32_t>(rb), static_cast<uint32_t>(NT),
                            static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&cm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, in.codes, cdims, cstrides, cbox, CU_TENSOR_MAP_SWIZZLE_NONE))
    return KVQ_ERR_CUDA;
  // output tile: boxes of 64 fp16 or 32 fp32 channels x NT tokens x HG heads
  CUtensorMap om;
  const uint64_t es = out_fp32 ? 4 : 2;
  const uint64_t dims[3] = {D, static_cast<uint64_t>(d.tokens), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t strides[2] = {D * es, static_cast<uint64_t>(d.tokens) * D * es};
  const uint32_t box[3] = {out_fp32 ? 32u : 64u, static_cast<uint32_t>(NT), static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&om, out_fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, x_out, dims,
                strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  return dispatch(false, d, a, cm, om, out_fp32, ctx, st);
}

}  // namespace kvq
