// Grouped-head encode / decode ("RotateKV: Accurate and Robust 2-Bit KV Cache
// Quantization for LLMs via Outlier-Aware Adaptive Rotations", abstract and
// 关键设计: pre-RoPE grouped-head rotation). The HG heads of one token are
// concatenated (index = local_head * 128 + channel), permuted per head,
// transformed by one normalised FWHT of size HG*128 in natural (Sylvester)
// stride order -- the 7 in-head strides first, then the log2(HG) cross-head
// strides -- and only then rotated by RoPE head slice by head slice; each
// head slice is quantized with per-group min-max and packed.
//
// Persistent CTAs of 128 threads walk tiles of HG heads x NT tokens
// (HG * NT = 128) of one batch. Each tile's fp16 rows and RoPE rows arrive
// by TMA into one of two shared-memory stages, so the next tile streams in
// while the current one is computed.
//   phase 1: thread (head, token) holds one 128-channel row in registers and
//            runs the 7 in-head FWHT strides;
//   exchange: the rows go through the stage's buffer in two halves of 64
//            channels (fp32, XOR-swizzled: conflict-free row writes and
//            column reads);
//   phase 2: thread (token, k) holds channels [k*C, (k+1)*C), C = 128/HG, of
//            all HG heads, runs the cross-head strides, RoPE, the group
//            min/max (a transpose-reduce across the lanes sharing a group,
//            so each lane derives one head's fp16 scale/zero), quantizes and
//            stores its slice of each head's packed record.
// Decode runs the phases in reverse, staging its output through the same
// buffers and writing it back by TMA.
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
constexpr int kStages = 2;
constexpr int kStageX = 32768;  // x tile, exchange half and output tile (fp16)

struct GroupArgs {
  int B, H, T, t0, t_cap, n_sink, rope, n_tblk, n_grp, n_tiles;
  FastDiv div_grp, div_b;  // head groups per batch; batches
  float rscale;  // fp32(1/sqrt(HG*128))
  const int16_t* perm;
  const float* rope_cs;  // [rows][128/2][2]
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

__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b as one packed fma: fma(b, -1, a) rounds a - b exactly once, like a subtraction.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// 16-byte chunk c (0..15) of the 64-channel exchange row (t, h) -> position.
__device__ __forceinline__ uint32_t xpos(int t, int c) {
  return (static_cast<uint32_t>(c & 1) << 3) | ((static_cast<uint32_t>(c >> 1) ^ static_cast<uint32_t>(t)) & 7u);
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

// Bytes of one stage: the x tile, which later carries the exchange halves
// and (decode) the output tile.
template <int HG>
__host__ __device__ constexpr int stage_bytes() {
  return kStageX;
}

// Sum over the codes of one packed word of (kMagicBits << bit position):
// the packer adds each code's raw fp32 pattern (kMagicBits + code) at its
// shift and subtracts this once per word.
template <int BITS>
__host__ __device__ constexpr uint32_t magic_word_offset() {
  uint32_t k = 0;
  for (int j = 0; j < 32 / BITS; ++j) k += kMagicBits << (BITS * j);
  return k;
}

template <int NB>
__device__ __forceinline__ void st_bytes(uint8_t* dst, const uint32_t* w) {
  if constexpr (NB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i)
      reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else if constexpr (NB % 8 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 8; ++i) reinterpret_cast<uint2*>(dst)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
  } else if constexpr (NB % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 4; ++i) reinterpret_cast<uint32_t*>(dst)[i] = w[i];
  } else {
#pragma unroll
    for (int i = 0; i < NB / 2; ++i)
      reinterpret_cast<uint16_t*>(dst)[i] = static_cast<uint16_t>(w[i >> 1] >> (16 * (i & 1)));
  }
}
template <int NB>
__device__ __forceinline__ void ld_bytes(const uint8_t* src, uint32_t* w) {
  if constexpr (NB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (NB % 8 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 8; ++i) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(src) + i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else if constexpr (NB % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 4; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(src) + i);
  } else {
#pragma unroll
    for (int i = 0; i < (NB + 3) / 4; ++i) w[i] = 0u;
#pragma unroll
    for (int i = 0; i < NB / 2; ++i)
      w[i >> 1] |= static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(src) + i)) << (16 * (i & 1));
  }
}

// Phase-1 register layout: P[2g + e] = (x[4g + e], x[4g + 2 + e]), g = 0..31.
// In-head FWHT strides 1, 2, 4, ..., 64 in ascending order.
__device__ __forceinline__ void fwht128_pairs(float2 (&P)[64]) {
#pragma unroll
  for (int g = 0; g < 32; ++g) {  // stride 1: x[4g] <-> x[4g+1], x[4g+2] <-> x[4g+3]
    const float2 a = P[2 * g], b = P[2 * g + 1];
    P[2 * g] = add2(a, b);
    P[2 * g + 1] = sub2(a, b);
  }
#pragma unroll
  for (int k = 0; k < 64; ++k) {  // stride 2: inside each pair
    const float a = P[k].x, b = P[k].y;
    P[k] = f2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
#pragma unroll
  for (int hs = 1; hs < 32; hs <<= 1) {  // strides 4 .. 64 = group strides 1 .. 16
#pragma unroll
    for (int g = 0; g < 32; ++g) {
      if ((g & hs) == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float2 a = P[2 * g + e], b = P[2 * (g + hs) + e];
          P[2 * g + e] = add2(a, b);
          P[2 * (g + hs) + e] = sub2(a, b);
        }
      }
    }
  }
}

// Transpose-reduce of per-head (min, max) across the TPG lanes that share a
// group: afterwards lane k (within its aligned TPG-lane group) holds the
// totals of heads [k*HG/TPG, (k+1)*HG/TPG).
template <int HG, int TPG>
__device__ __forceinline__ void transpose_reduce(float (&mn)[HG], float (&mx)[HG], int lane) {
  constexpr int L0 = HG;
#pragma unroll
  for (int o = TPG / 2, L = L0; o >= 1; o >>= 1, L >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < L / 2; ++i) {
      const float send_mn = upper ? mn[i] : mn[i + L / 2];
      const float send_mx = upper ? mx[i] : mx[i + L / 2];
      const float keep_mn = upper ? mn[i + L / 2] : mn[i];
      const float keep_mx = upper ? mx[i + L / 2] : mx[i];
      mn[i] = fminf(keep_mn, __shfl_xor_sync(0xffffffffu, send_mn, o));
      mx[i] = fmaxf(keep_mx, __shfl_xor_sync(0xffffffffu, send_mx, o));
    }
  }
}

template <int HG, int BITS, int G>
__global__ void __launch_bounds__(128) k_encode_group(const __grid_constant__ CUtensorMap xmap, const GroupArgs a) {
  constexpr int NT = 128 / HG;      // tokens per tile
  constexpr int C = D / HG;         // channels per phase-2 thread
  constexpr int NGL = C / 4;        // 4-channel groups per phase-2 thread
  constexpr int TPG = G / C;        // phase-2 lanes sharing one min-max group
  constexpr int HPL = HG / TPG;     // heads whose scale/zero one lane derives
  constexpr int NB = C * BITS / 8;  // packed bytes per phase-2 thread and head
  constexpr int RB = D * BITS / 8;
  constexpr int NG = D / G;
  constexpr int SB = stage_bytes<HG>();
  constexpr bool FOLD = (HG != 4);  // 1/sqrt(HG*128) is a power of two
  constexpr int L = (1 << BITS) - 1;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kStages];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x;
  const int hl = tid / NT, t = tid % NT;   // phase-1 role
  const int t2 = tid / HG, k = tid % HG;   // phase-2 role
  const int lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int tile, int s) {
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    uint8_t* st = sm + s * SB;
    mbar_arrive_expect_tx(&full[s], kStageX);
    tma_load_3d(st, &xmap, 0, t_base, b * a.H + h_base, &full[s]);
    tma_load_3d(st + 16384, &xmap, 64, t_base, b * a.H + h_base, &full[s]);
  };
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      const int tile = blockIdx.x + s * gridDim.x;
      if (tile < a.n_tiles) issue(tile, s);
    }
  }
  const float r = a.rscale;
  bool ok = true;

  for (int it = 0;; ++it) {
    const int tile = blockIdx.x + it * gridDim.x;
    if (tile >= a.n_tiles) break;
    const int s = it & 1;
    const uint32_t parity = (it >> 1) & 1;
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    uint8_t* st = sm + s * SB;
    const uint32_t st_u = smem_u32(st);
    ok = mbar_wait(&full[s], parity, a.wait_ns, a.err);  // on a timeout the tile is garbage; see below


    // ---------------- phase 1
    const int tt = t_base + t, m = a.t0 + tt;
    float2 P[64];
    {
      if (tt < a.T && m < a.n_sink) {
        uint4* dst = reinterpret_cast<uint4*>(a.sink + ((static_cast<size_t>(b) * a.H + h_base + hl) * a.n_sink + m) * D);
#pragma unroll
        for (int c = 0; c < 16; ++c) dst[c] = lds128(st_u + (c >> 3) * 16384 + sw128(tid, c & 7));
      }
      if (a.perm) {
        const int16_t* pr = a.perm + static_cast<size_t>(h_base + hl) * D;
        float xv[D];
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
          const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
            const uint32_t addr = st_u + (e >> 6) * 16384 + sw128(tid, (e & 63) >> 3) + (e & 7) * 2;
            xv[8 * c + i] = __half2float(__ushort_as_half(lds16(addr)));
          }
        }
#pragma unroll
        for (int g = 0; g < 32; ++g) {
          P[2 * g] = f2(xv[4 * g], xv[4 * g + 2]);
          P[2 * g + 1] = f2(xv[4 * g + 1], xv[4 * g + 3]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint4 raw = lds128(st_u + (c >> 3) * 16384 + sw128(tid, c & 7));
          const __half2* hp = reinterpret_cast<const __half2*>(&raw);
          const float2 h01 = __half22float2(hp[0]), h23 = __half22float2(hp[1]);
          const float2 h45 = __half22float2(hp[2]), h67 = __half22float2(hp[3]);
          P[4 * c + 0] = f2(h01.x, h23.x);
          P[4 * c + 1] = f2(h01.y, h23.y);
          P[4 * c + 2] = f2(h45.x, h67.x);
          P[4 * c + 3] = f2(h45.y, h67.y);
        }
      }
      fwht128_pairs(P);
    }
    // the x tile is consumed; its space carries the exchange. A timed-out wait
    // in any thread ends the CTA's work uniformly here.
    if (!__syncthreads_and(ok)) {
      ok = false;
      break;
    }

    // ---------------- exchange (two halves of 64 channels) -> phase-2 registers
    float2 A[HG][NGL], Bv[HG][NGL];  // A = (ch 4g, 4g+2), Bv = (ch 4g+1, 4g+3) of head h
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const uint32_t row1 = st_u + (t * HG + hl) * 256;
#pragma unroll
      for (int q = 0; q < 8; ++q) {  // 8-channel chunk q8 = 2q + h2 = groups 2*q8, 2*q8+1
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int g = 2 * (2 * q + h2) + e;
          sts128(row1 + xpos(t, 2 * q + e) * 16,
                 make_uint4(__float_as_uint(P[2 * g].x), __float_as_uint(P[2 * g].y), __float_as_uint(P[2 * g + 1].x),
                            __float_as_uint(P[2 * g + 1].y)));
        }
      }
      __syncthreads();
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const uint32_t row2 = st_u + (t2 * HG + h) * 256;
#pragma unroll
        for (int qq = 0; qq < C / 16; ++qq) {  // this thread's chunks of the half
          const int q8 = k * (C / 8) + 2 * qq + h2;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const uint4 u = lds128(row2 + xpos(t2, 2 * (q8 >> 1) + e) * 16);
            const int gl = 2 * (2 * qq + h2) + e;  // static: keeps A / Bv in registers
            A[h][gl] = f2(__uint_as_float(u.x), __uint_as_float(u.y));
            Bv[h][gl] = f2(__uint_as_float(u.z), __uint_as_float(u.w));
          }
        }
      }
      __syncthreads();
    }
    // the stage is free again: stream in the tile after next
    if (tid == 0 && tile + kStages * gridDim.x < a.n_tiles) issue(tile + kStages * gridDim.x, s);
    // RoPE (cos, sin) of this thread's phase-2 channels, straight from L2
    // (the tiles of one token block run together, so the rows stay hot)
    uint4 csr[NGL];
    if (a.rope) {
      const int mr = min(a.t0 + t_base + t2, a.t0 + a.T - 1);
      const uint4* rp = reinterpret_cast<const uint4*>(a.rope_cs + static_cast<size_t>(mr) * D) + k * NGL;
#pragma unroll
      for (int gl = 0; gl < NGL; ++gl) csr[gl] = __ldg(rp + gl);
    }

    // ---------------- phase 2
#pragma unroll
    for (int sh = 1; sh < HG; sh <<= 1) {  // cross-head strides
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        if ((h & sh) == 0) {
#pragma unroll
          for (int gl = 0; gl < NGL; ++gl) {
            const float2 pa = A[h][gl], qa = A[h + sh][gl];
            A[h][gl] = add2(pa, qa);
            A[h + sh][gl] = sub2(pa, qa);
            const float2 pb = Bv[h][gl], qb = Bv[h + sh][gl];
            Bv[h][gl] = add2(pb, qb);
            Bv[h + sh][gl] = sub2(pb, qb);
          }
        }
      }
    }
    if (!FOLD) {
#pragma unroll
      for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int gl = 0; gl < NGL; ++gl) {
          A[h][gl] = mul2(A[h][gl], f2(r, r));
          Bv[h][gl] = mul2(Bv[h][gl], f2(r, r));
        }
    }
    if (a.rope) {  // y0 = fma(x0, c, -(x1*s)), y1 = fma(x0, s, x1*c), two pairs at a time
#pragma unroll
      for (int gl = 0; gl < NGL; ++gl) {
        // table chunk g = (c_2g, s_2g, c_2g+1, s_2g+1); scaled by r when folding (exact)
        float2 cc = f2(__uint_as_float(csr[gl].x), __uint_as_float(csr[gl].z));
        float2 ss = f2(__uint_as_float(csr[gl].y), __uint_as_float(csr[gl].w));
        if (FOLD) {
          cc = mul2(cc, f2(r, r));
          ss = mul2(ss, f2(r, r));
        }
        const float2 nss = f2(-ss.x, -ss.y);
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const float2 x0 = A[h][gl], x1 = Bv[h][gl];
          const float2 t1n = mul2(x1, nss);
          const float2 t2c = mul2(x1, cc);
          A[h][gl] = fma2(x0, cc, t1n);
          Bv[h][gl] = fma2(x0, ss, t2c);
        }
      }
    }
    // values are now p (keys, or every HG = 4 tensor) or p / r (values when folding)
    const bool unscaled = FOLD && !a.rope;
    float mn[HG], mx[HG];
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      float lo = fminf(A[h][0].x, A[h][0].y), hi = fmaxf(A[h][0].x, A[h][0].y);
      lo = min3f(lo, Bv[h][0].x, Bv[h][0].y);
      hi = max3f(hi, Bv[h][0].x, Bv[h][0].y);
#pragma unroll
      for (int gl = 1; gl < NGL; ++gl) {
        lo = min3f(lo, A[h][gl].x, A[h][gl].y);
        hi = max3f(hi, A[h][gl].x, A[h][gl].y);
        lo = min3f(lo, Bv[h][gl].x, Bv[h][gl].y);
        hi = max3f(hi, Bv[h][gl].x, Bv[h][gl].y);
      }
      mn[h] = lo;
      mx[h] = hi;
    }
    transpose_reduce<HG, TPG>(mn, mx, lane);
    const int kg = lane & (TPG - 1);  // this lane's rank among the lanes of its group
    float Zq[HPL], Rq[HPL];
    __half2 szo[HPL];
#pragma unroll
    for (int i = 0; i < HPL; ++i) {
      float lo = mn[i], hi = mx[i];
      if (unscaled) {
        lo = __fmul_rn(lo, r);
        hi = __fmul_rn(hi, r);
      }
      const QParams p = minmax_params<BITS>(lo, hi);
      szo[i] = p.sz;
      Zq[i] = unscaled ? __fdiv_rn(p.Z, r) : p.Z;  // Z / r is exact (power of two)
      Rq[i] = unscaled ? __fmul_rn(p.R, r) : p.R;
    }
    const int tt2 = t_base + t2, m2 = a.t0 + tt2;
    const bool store = tt2 < a.T;
    const bool sink_tok = m2 < a.n_sink;
    const int lane0 = lane - kg;  // first lane of this thread's group
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      // (Z, R) of head h live in lane (lane0 + h / HPL), slot h % HPL
      const float Z = __shfl_sync(0xffffffffu, Zq[h % HPL], lane0 + h / HPL);
      const float R = __shfl_sync(0xffffffffu, Rq[h % HPL], lane0 + h / HPL);
      const float2 nZ = f2(-Z, -Z), R2 = f2(R, R), M2 = f2(kMagicRound, kMagicRound);
      constexpr int NWC = (C * BITS + 31) / 32;
      uint32_t w[NWC];
#pragma unroll
      for (int i = 0; i < NWC; ++i) w[i] = 0u;
#pragma unroll
      for (int gl = 0; gl < NGL; ++gl) {
        const float2 ua = fma2(add2(A[h][gl], nZ), R2, M2);
        const float2 ub = fma2(add2(Bv[h][gl], nZ), R2, M2);
        // raw fp32 patterns kMagicBits + code of local channels 4gl + 0, 1, 2, 3
        const uint32_t t4[4] = {__float_as_uint(ua.x), __float_as_uint(ub.x), __float_as_uint(ua.y),
                                __float_as_uint(ub.y)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int pos = (4 * gl + e) * BITS;
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
        for (int i = 0; i < NWC; ++i) w[i] -= magic_word_offset<BITS>();
      }
#pragma unroll
      for (int i = 0; i < NWC; ++i) w[i] = sink_tok ? 0u : w[i];
      if (store) {
        const size_t slot = (static_cast<size_t>(b) * a.H + h_base + h) * a.t_cap + m2;
        st_bytes<NB>(a.codes + slot * RB + k * NB, w);
      }
    }
    if (store) {
      const __half2 zero2 = __halves2half2(__ushort_as_half(0), __ushort_as_half(0));
#pragma unroll
      for (int i = 0; i < HPL; ++i) {
        const int h = kg * HPL + i;
        const size_t slot = (static_cast<size_t>(b) * a.H + h_base + h) * a.t_cap + m2;
        a.sz[slot * NG + (k * C) / G] = sink_tok ? zero2 : szo[i];
      }
    }
    (void)L;
  }
  if (!ok && tid == 0) {  // let copies in flight land (bounded) before the CTA exits
    for (int s = 0; s < kStages; ++s)
      for (uint32_t p = 0; p < 2; ++p) mbar_wait(&full[s], p, a.wait_ns, a.err);
  }
}

template <int HG, int BITS, int G>
__global__ void __launch_bounds__(128) k_decode_group(const __grid_constant__ CUtensorMap omap, const GroupArgs a,
                                                       int out_fp32) {
  constexpr int NT = 128 / HG;
  constexpr int C = D / HG;
  constexpr int NGL = C / 4;
  constexpr int NB = C * BITS / 8;
  constexpr int NW = (C * BITS + 31) / 32;
  constexpr int RB = D * BITS / 8;
  constexpr int NG = D / G;
  constexpr int SB = stage_bytes<HG>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x;
  const int hl = tid / NT, t = tid % NT;
  const int t2 = tid / HG, k = tid % HG;
  const float r = a.rscale;

  // this thread's packed codes, (S, Z) and RoPE (cos, sin) of one tile
  auto load_tile = [&](int tile, uint32_t (&cw)[HG][NW], __half2 (&szv)[HG], uint4 (&csr)[NGL]) {
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    const int tt2 = t_base + t2, m2 = a.t0 + tt2;
    const bool live = tt2 < a.T && m2 >= a.n_sink;
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      if (live) {
        const size_t slot = (static_cast<size_t>(b) * a.H + h_base + h) * a.t_cap + m2;
        ld_bytes<NB>(a.codes + slot * RB + k * NB, cw[h]);
        szv[h] = a.sz[slot * NG + (k * C) / G];
      } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) cw[h][i] = 0u;
        szv[h] = __halves2half2(__ushort_as_half(0), __ushort_as_half(0));
      }
    }
    if (a.rope) {
      const int mr = min(m2, a.t0 + a.T - 1);
      const uint4* rp = reinterpret_cast<const uint4*>(a.rope_cs + static_cast<size_t>(mr) * D) + k * NGL;
#pragma unroll
      for (int gl = 0; gl < NGL; ++gl) csr[gl] = __ldg(rp + gl);
    }
  };
  uint32_t cw[HG][NW];
  __half2 szv[HG];
  uint4 csr[NGL];
  if (blockIdx.x < a.n_tiles) load_tile(blockIdx.x, cw, szv, csr);

  for (int it = 0;; ++it) {
    const int tile = blockIdx.x + it * gridDim.x;
    if (tile >= a.n_tiles) break;
    const int s = it & 1;
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    uint8_t* st = sm + s * SB;
    const uint32_t st_u = smem_u32(st);

    // ---------------- phase 2 (reverse): dequantize (normalisation folded in), inverse RoPE, cross-head
    float2 A[HG][NGL], Bv[HG][NGL];
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      const float S = __fmul_rn(__low2float(szv[h]), r), Z = __fmul_rn(__high2float(szv[h]), r);
      const float2 S2 = f2(S, S), Z2 = f2(Z, Z);
#pragma unroll
      for (int gl = 0; gl < NGL; ++gl) {
        const float2 ca = f2(code_to_float(unpack_code<BITS, NW>(cw[h], 4 * gl + 0)),
                             code_to_float(unpack_code<BITS, NW>(cw[h], 4 * gl + 2)));
        const float2 cb = f2(code_to_float(unpack_code<BITS, NW>(cw[h], 4 * gl + 1)),
                             code_to_float(unpack_code<BITS, NW>(cw[h], 4 * gl + 3)));
        A[h][gl] = fma2(ca, S2, Z2);
        Bv[h][gl] = fma2(cb, S2, Z2);
      }
    }
    if (a.rope) {
#pragma unroll
      for (int gl = 0; gl < NGL; ++gl) {
        const float2 cc = f2(__uint_as_float(csr[gl].x), __uint_as_float(csr[gl].z));
        const float2 ss = f2(__uint_as_float(csr[gl].y), __uint_as_float(csr[gl].w));
        const float2 nss = f2(-ss.x, -ss.y);
#pragma unroll
        for (int h = 0; h < HG; ++h) {  // x0 = y0 c + y1 s, x1 = y1 c - y0 s
          const float2 y0 = A[h][gl], y1 = Bv[h][gl];
          A[h][gl] = fma2(y0, cc, mul2(y1, ss));
          Bv[h][gl] = fma2(y1, cc, mul2(y0, nss));
        }
      }
    }
#pragma unroll
    for (int sh = 1; sh < HG; sh <<= 1) {
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        if ((h & sh) == 0) {
#pragma unroll
          for (int gl = 0; gl < NGL; ++gl) {
            const float2 pa = A[h][gl], qa = A[h + sh][gl];
            A[h][gl] = add2(pa, qa);
            A[h + sh][gl] = sub2(pa, qa);
            const float2 pb = Bv[h][gl], qb = Bv[h + sh][gl];
            Bv[h][gl] = add2(pb, qb);
            Bv[h + sh][gl] = sub2(pb, qb);
          }
        }
      }
    }
    // the output store of two tiles ago must have read this stage
    if (tid == 0) bulk_wait_read<1>();
    __syncthreads();

    // ---------------- exchange (two halves) -> phase-1 registers
    float2 P[64];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const uint32_t row2 = st_u + (t2 * HG + h) * 256;
#pragma unroll
        for (int qq = 0; qq < C / 16; ++qq) {
          const int q8 = k * (C / 8) + 2 * qq + h2;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int gl = 2 * (2 * qq + h2) + e;  // static: keeps A / Bv in registers
            sts128(row2 + xpos(t2, 2 * (q8 >> 1) + e) * 16,
                   make_uint4(__float_as_uint(A[h][gl].x), __float_as_uint(A[h][gl].y),
                              __float_as_uint(Bv[h][gl].x), __float_as_uint(Bv[h][gl].y)));
          }
        }
      }
      __syncthreads();
      const uint32_t row1 = st_u + (t * HG + hl) * 256;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int g = 2 * (2 * q + h2) + e;
          const uint4 u = lds128(row1 + xpos(t, 2 * q + e) * 16);
          P[2 * g] = f2(__uint_as_float(u.x), __uint_as_float(u.y));
          P[2 * g + 1] = f2(__uint_as_float(u.z), __uint_as_float(u.w));
        }
      }
      __syncthreads();
    }

    // prefetch the next tile's codes, scales and RoPE rows while this one finishes
    const int next = tile + gridDim.x;
    if (next < a.n_tiles) load_tile(next, cw, szv, csr);

    // ---------------- phase 1 (reverse): in-head strides, inverse permutation, output
    fwht128_pairs(P);
    const int tt = t_base + t, m = a.t0 + tt;
    float x[D];
#pragma unroll
    for (int g = 0; g < 32; ++g) {
      x[4 * g] = P[2 * g].x;
      x[4 * g + 2] = P[2 * g].y;
      x[4 * g + 1] = P[2 * g + 1].x;
      x[4 * g + 3] = P[2 * g + 1].y;
    }
    const bool sink_tok = tt < a.T && m < a.n_sink;
    if (sink_tok) {
      const uint4* src = reinterpret_cast<const uint4*>(
          a.sink + ((static_cast<size_t>(b) * a.H + h_base + hl) * a.n_sink + m) * D);
#pragma unroll
      for (int c = 0; c < 16; ++c) h8_to_f32(__ldg(src + c), &x[8 * c]);
    }
    const bool permute = a.perm != nullptr && !sink_tok;
    const int16_t* pr = a.perm ? a.perm + static_cast<size_t>(h_base + hl) * D : nullptr;
    if (!out_fp32) {
      if (permute) {  // x'[perm[j]] = x[j], written straight into this thread's output row
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
          const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
            sts16(st_u + (e >> 6) * 16384 + sw128(tid, (e & 63) >> 3) + (e & 7) * 2,
                  __half_as_ushort(__float2half_rn(x[8 * c + i])));
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) sts128(st_u + (c >> 3) * 16384 + sw128(tid, c & 7), f32_to_h8(&x[8 * c]));
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        tma_store_3d(&omap, 0, t_base, b * a.H + h_base, st);
        tma_store_3d(&omap, 64, t_base, b * a.H + h_base, st + 16384);
        bulk_commit();
      }
    } else {
      // fp32 tile = 64 KB: two passes of 64 channels through the 32 KB stage
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1) {
          if (tid == 0) bulk_wait_read<0>();
          __syncthreads();
        }
        if (permute) {
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
            const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
              if ((e >> 6) == static_cast<uint32_t>(pass))
                sts32f(st_u + ((e & 63) >> 5) * 16384 + sw128(tid, (e & 31) >> 2) + (e & 3) * 4, x[8 * c + i]);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int cc = pass * 16 + c;
            sts128(st_u + (c >> 3) * 16384 + sw128(tid, c & 7),
                   make_uint4(__float_as_uint(x[4 * cc]), __float_as_uint(x[4 * cc + 1]),
                              __float_as_uint(x[4 * cc + 2]), __float_as_uint(x[4 * cc + 3])));
          }
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
          tma_store_3d(&omap, pass * 64, t_base, b * a.H + h_base, st);
          tma_store_3d(&omap, pass * 64 + 32, t_base, b * a.H + h_base, st + 16384);
          bulk_commit();
        }
      }
    }
  }
  if (tid == 0) bulk_wait_read<0>();  // the last stores have read shared memory
}

template <int HG, int BITS, int G>
kvq_status run(bool enc, const GroupArgs& a, const CUtensorMap& m0, int out_fp32,
               const LaunchCtx& ctx, cudaStream_t st) {
  const size_t smem = 1024 + static_cast<size_t>(kStages) * stage_bytes<HG>();
  const void* fn = enc ? reinterpret_cast<const void*>(k_encode_group<HG, BITS, G>)
                       : reinterpret_cast<const void*>(k_decode_group<HG, BITS, G>);
  if (!set_smem_once(reinterpret_cast<const void*>(fn), smem))
    return KVQ_ERR_CUDA;
  const int per_sm = occupancy_once(fn, 128, smem);
  const long long want = static_cast<long long>(ctx.num_sms) * per_sm;
  const unsigned grid = static_cast<unsigned>(a.n_tiles < want ? a.n_tiles : want);
  if (enc)
    k_encode_group<HG, BITS, G><<<grid, 128, smem, st>>>(m0, a);
  else
    k_decode_group<HG, BITS, G><<<grid, 128, smem, st>>>(m0, a, out_fp32);
  return launch_status();
}

kvq_status dispatch(bool enc, const kvq_desc& d, const GroupArgs& a, const CUtensorMap& m0, int out_fp32,
                    const LaunchCtx& ctx, cudaStream_t st) {
#define KVQ_CASE(HG_, B_, G_) \
  if (d.group_heads == HG_ && d.bits == B_ && d.group == G_) return run<HG_, B_, G_>(enc, a, m0, out_fp32, ctx, st);
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
  const int NT = 128 / d.group_heads;
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

}  // namespace

kvq_status launch_encode_group(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                               cudaStream_t st, const LaunchCtx& ctx) {
  const GroupArgs a = make_args(d, tb, out, ctx);
  const int NT = 128 / d.group_heads;
  CUtensorMap xm;
  const uint64_t dims[3] = {D, static_cast<uint64_t>(d.tokens), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t strides[2] = {D * 2, static_cast<uint64_t>(d.tokens) * D * 2};
  const uint32_t box[3] = {64, static_cast<uint32_t>(NT), static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&xm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  return dispatch(true, d, a, xm, 0, ctx, st);
}

kvq_status launch_decode_group(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                               int out_fp32, cudaStream_t st, const LaunchCtx& ctx) {
  const GroupArgs a = make_args(d, tb, in, ctx);
  const int NT = 128 / d.group_heads;
  CUtensorMap om;
  const uint64_t es = out_fp32 ? 4 : 2;
  const uint64_t dims[3] = {D, static_cast<uint64_t>(d.tokens), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t strides[2] = {D * es, static_cast<uint64_t>(d.tokens) * D * es};
  const uint32_t box[3] = {out_fp32 ? 32u : 64u, static_cast<uint32_t>(NT), static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&om, out_fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, x_out, dims,
                strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  return dispatch(false, d, a, om, out_fp32, ctx, st);
}

}  // namespace kvq
