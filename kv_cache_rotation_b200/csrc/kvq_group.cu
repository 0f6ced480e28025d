// Grouped-head encode / decode ("RotateKV: Accurate and Robust 2-Bit KV Cache
// Quantization for LLMs via Outlier-Aware Adaptive Rotations", abstract and
// 关键设计: pre-RoPE grouped-head rotation). The HG heads of one token are
// concatenated (index = local_head * 128 + channel), permuted per head,
// transformed by one normalised FWHT of size HG*128 in natural (Sylvester)
// stride order -- the 7 in-head strides first, then the log2(HG) cross-head
// strides -- and only then rotated by RoPE head slice by head slice; each
// head slice is quantized with per-group min-max and packed.
//
// Encode: warps work independently (no CTA barrier). A warp owns tiles of
// HG heads x 16/HG tokens of one batch (2048 values, 64 per lane) and keeps
// the next tile in flight while it computes: one lane issues one TMA copy of
// the tile's fp16 rows (a 4-D box: 64 channels x 2 halves x tokens x heads,
// 128-byte swizzle, zero-filled past the last token) into the warp's staging
// buffer, tracked by the warp's own mbarrier. Per tile:
//   phase 1: lane (head, token, half s) -- staged row (head * NT + token) * 2
//            + s, so 8 consecutive lanes read 8 distinct swizzle phases --
//            holds channels [64s, 64s + 64) of one head row; the strides 1
//            and 2 run in fp32 straight from the fp16 words (mixed-precision
//            add / sub), the strides 4 .. 32 packed;
//   exchange: the rows go through a per-warp shared buffer as fp32 in 16-byte
//            chunks of four channels (rows padded to 17 chunks: conflict-free);
//   phase 2: lane (token, k) holds, for every head of the group and both
//            halves, the 4Q channels [4kQ, 4kQ + 4Q) (Q = 8/HG), runs the
//            stride 64 and the cross-head strides, RoPE, the group min/max (a
//            transpose-reduce over the 2*HG lanes of the token; one lane per
//            group derives its fp16 scale/zero and publishes (-Z, 1/S) through
//            the warp's shared buffer), quantizes and packs.
// Decode runs the same tiles in reverse, warps again independent: one lane
// brings the tile's packed records in by TMA (the next tile's while this one
// computes), the lanes fetch its scale/zero words by cp.async; phase 2
// dequantizes (normalisation folded into S and Z), undoes RoPE and runs the
// cross-head strides and the stride 64; the exchange hands each phase-1 lane
// its 64 channels; phase 1 runs the strides 32 .. 1 and writes its row,
// fp16 or fp32, into a 128-byte-swizzled output box that overlays the
// exchange rows, and one lane stores the box by TMA.
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
// encode: independent warps, each with its own shared buffers
constexpr int kEncWarps = 4;
constexpr int kEncThreads = 32 * kEncWarps;
constexpr int kEncStage = 4096;                              // fp16 rows of one warp tile (TMA box)
constexpr int kEncXch = 32 * 272;                            // fp32 exchange, 17-chunk rows
constexpr int kEncPrm = 512;                                 // (-Z, -Z, 1/S, 1/S) of the tile's groups
constexpr int kEncWarpSmem = kEncStage + kEncXch + kEncPrm;  // 13312 bytes = 13 x 1024
static_assert(kEncWarpSmem % 1024 == 0, "each warp's staging box must stay 1024-byte aligned");
// decode: independent warps too; the output tile overlays the exchange rows
constexpr int kDecWarps = 4;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecXch = 9216;                                   // exchange rows, then the output box (<= 8 KB)
constexpr int kDecCodes = 1024;                                 // packed codes of one warp tile (TMA box)
constexpr int kDecSz = 256;                                     // scale/zero of the tile's groups (cp.async)
constexpr int kDecWarpSmem = 11264;                             // 11 x 1024
static_assert(kDecXch + kDecCodes + kDecSz <= kDecWarpSmem && kDecWarpSmem % 1024 == 0, "decode layout");

struct GroupArgs {
  int B, H, T, t0, t_cap, n_sink, rope, n_tblk, n_grp, n_tiles;
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
// are 17 chunks (272 bytes) apart and chunks 8..15 skip one slot, so 8
// consecutive rows at one chunk, or one row at chunks 0..7, 8..15 or at every
// other chunk, fall on 8 distinct bank groups.
__host__ __device__ constexpr uint32_t xoff(int g) { return 16u * static_cast<uint32_t>(g + (g >> 3)); }

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

// Table chunk (16 bytes: (c_i, s_i, c_i+1, s_i+1)) of a phase-2 lane's channel
// quad kk = k2 Q + q: interleaved pairs take the pairs of channels 4kk .. 4kk+3
// of half hs (chunk 16 hs + kk); half-split pairs (c, c + 64) take angles
// 4kk .. 4kk+3 (chunks 2kk and 2kk + 1, hs choosing which).
__device__ __forceinline__ int rope_chunk(bool half, int hs, int kk) { return half ? 2 * kk + hs : 16 * hs + kk; }

// Phase-1 values of 64 channels as 16 quads V[g] = (x[4g], x[4g+2], x[4g+1],
// x[4g+3]): each quad is one aligned register quad (the 16-byte exchange
// store) whose halves are the register pairs the packed butterflies use.
__device__ __forceinline__ float2 lo2(const float4& v) { return f2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4& v) { return f2(v.z, v.w); }
__device__ __forceinline__ void set_lo2(float4& v, float2 p) {
  v.x = p.x;
  v.y = p.y;
}
__device__ __forceinline__ void set_hi2(float4& v, float2 p) {
  v.z = p.x;
  v.w = p.y;
}

// Strides 4 .. 32 of the FWHT on the quads (strides 1 and 2 already applied).
__device__ __forceinline__ void fwht_quads_from4(float4 (&V)[16]) {
#pragma unroll
  for (int hs = 1; hs < 16; hs <<= 1) {
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      if ((g & hs) == 0) {
        float2 a0 = lo2(V[g]), b0 = lo2(V[g + hs]), a1 = hi2(V[g]), b1 = hi2(V[g + hs]);
        bfly(a0, b0);
        bfly(a1, b1);
        set_lo2(V[g], a0);
        set_lo2(V[g + hs], b0);
        set_hi2(V[g], a1);
        set_hi2(V[g + hs], b1);
      }
    }
  }
}

// Phase 1 from the staged fp16 words (w[q] = channels 2q, 2q + 1 of the half
// row): strides 1 and 2 in scalar fp32 (stride 1 by the mixed-precision
// butterfly), then strides 4 .. 32 packed.
__device__ __forceinline__ void phase1_from_halves(const uint32_t (&w)[32], float4 (&V)[16]) {
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    float y0, y1, y2, y3;
    bfly_h2(w[2 * g], y0, y1);      // (x0 + x1, x0 - x1)
    bfly_h2(w[2 * g + 1], y2, y3);  // (x2 + x3, x2 - x3)
    V[g] = make_float4(__fadd_rn(y0, y2), __fsub_rn(y0, y2), __fadd_rn(y1, y3), __fsub_rn(y1, y3));
  }
  fwht_quads_from4(V);
}

// The same from 64 fp32 channel values (the gathered, permuted row).
__device__ __forceinline__ void phase1_from_f32(const float (&x)[64], float4 (&V)[16]) {
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    const float y0 = __fadd_rn(x[4 * g], x[4 * g + 1]), y1 = __fsub_rn(x[4 * g], x[4 * g + 1]);
    const float y2 = __fadd_rn(x[4 * g + 2], x[4 * g + 3]), y3 = __fsub_rn(x[4 * g + 2], x[4 * g + 3]);
    V[g] = make_float4(__fadd_rn(y0, y2), __fsub_rn(y0, y2), __fadd_rn(y1, y3), __fsub_rn(y1, y3));
  }
  fwht_quads_from4(V);
}

template <int HG, int BITS, int G>
__global__ void __launch_bounds__(kEncThreads, 4)
    k_encode_group(const __grid_constant__ CUtensorMap xmap, const GroupArgs a) {
  constexpr int NT = 16 / HG;        // tokens per warp tile
  constexpr int Q = 8 / HG;          // channel quads per phase-2 lane, head and half
  constexpr int TPT = 2 * HG;        // lanes per token
  constexpr int NG = D / G;          // min-max groups per head
  constexpr int NGP = HG * NG;       // groups per token
  constexpr int SH = TPT > NGP ? 1 : 0;
  constexpr int RB = D * BITS / 8;   // packed bytes per head row
  constexpr int NCB = 4 * Q * BITS;  // code bits per phase-2 lane, head and half
  constexpr int NWC = (NCB + 31) / 32;
  constexpr bool FOLD = (HG != 4);   // 1/sqrt(HG*128) is a power of two
  constexpr bool PRE_CS = (Q <= 2);  // the lane's RoPE table chunks are loaded at the tile's start
  static_assert(NT * NGP * 16 <= kEncPrm, "parameter buffer too small");
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kEncWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* const wsm = align1024(smem_raw) + warp * kEncWarpSmem;
  uint8_t* const stg = wsm;                                              // staging (TMA box)
  uint8_t* const xch = wsm + kEncStage;                                  // exchange (fp32)
  float4* const prm = reinterpret_cast<float4*>(wsm + kEncStage + kEncXch);  // (-Z, -Z, R, R) per group
  uint64_t* const bar = &full[warp];
  const int s1 = lane & 1, t1 = (lane >> 1) % NT, h1 = lane / (2 * NT);  // phase-1 role
  const int t2 = lane / TPT, k2 = lane % TPT;                             // phase-2 role
  const float r = a.rscale;
  const int gw = blockIdx.x * kEncWarps + warp, n_gw = gridDim.x * kEncWarps;
  const size_t code_hstep = static_cast<size_t>(a.t_cap) * RB;  // bytes between heads' records
  const uint8_t* const row1 = stg + lane * 128;                    // this lane's staged half row
  const uint32_t sw1 = static_cast<uint32_t>(lane & 7) << 4;       // its swizzle phase
  uint8_t* const xrow1 = xch + lane * 272;                          // its exchange row
  const uint8_t* const xrd2 = xch + (t2 * 2) * 272 + xoff(k2 * Q);  // phase-2 reads: + (h NT 2 + hs) 272 + 16 q

  if (lane == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto issue = [&](int tile) {  // one lane: the tile's rows -> staging
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    mbar_arrive_expect_tx(bar, kEncStage);
    tma_load_4d(stg, &xmap, 0, 0, t_base, b * a.H + h_base, bar);
  };
  if (lane == 0 && gw < a.n_tiles) issue(gw);

  uint32_t parity = 0;
  for (int tile = gw; tile < a.n_tiles; tile += n_gw) {
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    const int tt2 = t_base + t2, m2 = a.t0 + tt2;
    // RoPE table row of this lane's phase-2 token: chunk (c_i, s_i, c_i+1, s_i+1) per channel quad
    const uint4* rp =
        a.rope ? reinterpret_cast<const uint4*>(a.rope_cs) + static_cast<size_t>(min(m2, a.t0 + a.T - 1)) * (D / 4)
               : nullptr;
    const bool half = a.rope == 2;  // half-split pairs (i, i + 64)
    uint4 cs_pre[2][Q];
    if (PRE_CS && a.rope) {
#pragma unroll
      for (int hs = 0; hs < 2; ++hs)
#pragma unroll
        for (int q = 0; q < Q; ++q) cs_pre[hs][q] = __ldg(rp + rope_chunk(half, hs, k2 * Q + q));
    }

    // the tile's rows are staged (bounded wait; a timeout ends the warp's work)
    const bool ok = mbar_wait(bar, parity, a.wait_ns, a.err);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) mbar_wait(bar, parity, a.wait_ns, a.err);  // let the copy in flight land
      break;
    }
    parity ^= 1u;
    const int tt1 = t_base + t1, m1 = a.t0 + tt1;
    const bool sink1 = tt1 < a.T && m1 < a.n_sink;

    // ---------------- phase 1: 64 channels of one head row, strides 1 .. 32
    float4 P[16];
    if (!a.perm) {
      uint32_t w[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 u = *reinterpret_cast<const uint4*>(row1 + ((static_cast<uint32_t>(j) << 4) ^ sw1));
        w[4 * j] = u.x;
        w[4 * j + 1] = u.y;
        w[4 * j + 2] = u.z;
        w[4 * j + 3] = u.w;
      }
      __syncwarp();  // every lane has read the staging buffer: refill it
      if (lane == 0 && tile + n_gw < a.n_tiles) {
        fence_async_smem();
        issue(tile + n_gw);
      }
      if (sink1) {
        uint4* dst = reinterpret_cast<uint4*>(
            a.sink + ((static_cast<size_t>(b) * a.H + h_base + h1) * a.n_sink + m1) * D + 64 * s1);
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      }
      phase1_from_halves(w, P);
    } else {
      // gather p_j = x[perm[h][64 s + j]] from the staged rows of (head, token)
      const int16_t* pr = a.perm + static_cast<size_t>(h_base + h1) * D + 64 * s1;
      float xv[64];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
        const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
          const uint32_t rr = static_cast<uint32_t>(lane & ~1) + (e >> 6);  // row of (head, token, half of e)
          const uint32_t off = rr * 128 + ((((e >> 3) & 7) ^ (rr & 7)) << 4) + (e & 7) * 2;
          xv[8 * c + i] = __half2float(*reinterpret_cast<const __half*>(stg + off));
        }
      }
      if (sink1) {
        uint4* dst = reinterpret_cast<uint4*>(
            a.sink + ((static_cast<size_t>(b) * a.H + h_base + h1) * a.n_sink + m1) * D + 64 * s1);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          dst[c] = *reinterpret_cast<const uint4*>(row1 + ((static_cast<uint32_t>(c) << 4) ^ sw1));
      }
      __syncwarp();  // every lane has read the staging buffer: refill it
      if (lane == 0 && tile + n_gw < a.n_tiles) {
        fence_async_smem();
        issue(tile + n_gw);
      }
      phase1_from_f32(xv, P);
    }

    // ---------------- exchange: row `lane`, 16 chunks (x[4g], x[4g+2], x[4g+1], x[4g+3])
#pragma unroll
    for (int g = 0; g < 16; ++g) *reinterpret_cast<float4*>(xrow1 + xoff(g)) = P[g];
    __syncwarp();
    // A[h][half][q][e] = (x[c + e], x[c + 2 + e]) of head h, c = 64 half + 4 (k2 Q + q)
    float2 A[HG][2][Q][2];
#pragma unroll
    for (int hs = 0; hs < 2; ++hs)
#pragma unroll
      for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          const float4 u = *reinterpret_cast<const float4*>(xrd2 + (h * NT * 2 + hs) * 272 + 16 * q);
          A[h][hs][q][0] = f2(u.x, u.y);
          A[h][hs][q][1] = f2(u.z, u.w);
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
    if (a.rope && !half) {  // pairs (2i, 2i+1): y0 = fma(x0, c, -(x1*s)), y1 = fma(x0, s, x1*c)
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          // table chunk = (c_i, s_i, c_i+1, s_i+1) for channels c .. c+3; scaled by r when folding (exact)
          const uint4 cv = PRE_CS ? cs_pre[hs][q] : __ldg(rp + rope_chunk(false, hs, k2 * Q + q));
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
    } else if (a.rope) {  // pairs (i, i+64): channel c of the lower half with c + 64, angle c
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        // chunks (c_i, s_i, c_i+1, s_i+1) of angles c .. c+1 and c+2 .. c+3
        const uint4 c0 = PRE_CS ? cs_pre[0][q] : __ldg(rp + rope_chunk(true, 0, k2 * Q + q));
        const uint4 c1 = PRE_CS ? cs_pre[1][q] : __ldg(rp + rope_chunk(true, 1, k2 * Q + q));
#pragma unroll
        for (int e = 0; e < 2; ++e) {  // A[.][.][q][e] holds channels c + e and c + 2 + e
          float2 cc = e ? f2(__uint_as_float(c0.z), __uint_as_float(c1.z)) : f2(__uint_as_float(c0.x), __uint_as_float(c1.x));
          float2 ss = e ? f2(__uint_as_float(c0.w), __uint_as_float(c1.w)) : f2(__uint_as_float(c0.y), __uint_as_float(c1.y));
          if (FOLD) {
            cc = mul2(cc, f2(r, r));
            ss = mul2(ss, f2(r, r));
          }
          const float2 nss = f2(-ss.x, -ss.y);
#pragma unroll
          for (int h = 0; h < HG; ++h) {
            const float2 x0 = A[h][0][q][e], x1 = A[h][1][q][e];
            A[h][0][q][e] = fma2(x0, cc, mul2(x1, nss));
            A[h][1][q][e] = fma2(x0, ss, mul2(x1, cc));
          }
        }
      }
    }
    // values are now p (keys, or every HG = 4 tensor) or p / r (values when folding)
    const bool unscaled = FOLD && !a.rope;
    // per-lane min/max of every group, the groups' chains interleaved (step outermost)
    float mn[NGP], mx[NGP];
    {
      constexpr int HSG = NG == 2 ? 1 : 2;  // halves per group
      constexpr int STEPS = HSG * Q * 2;    // value pairs per group in this lane
#pragma unroll
      for (int st = 0; st < STEPS; ++st) {
        const int e = st & 1, q = (st >> 1) % Q, hsl = st / (2 * Q);
#pragma unroll
        for (int h = 0; h < HG; ++h)
#pragma unroll
          for (int grp = 0; grp < NG; ++grp) {
            const float2 v = A[h][NG == 2 ? grp : hsl][q][e];
            const int gi = h * NG + grp;
            if (st == 0) {
              mn[gi] = fminf(v.x, v.y);
              mx[gi] = fmaxf(v.x, v.y);
            } else {
              mn[gi] = min3f(mn[gi], v.x, v.y);
              mx[gi] = max3f(mx[gi], v.x, v.y);
            }
          }
      }
    }
    group_reduce<NGP, TPT>(mn, mx, lane);
    const bool store = tt2 < a.T;
    const bool sink_tok = m2 < a.n_sink;
    const size_t slot0 = (static_cast<size_t>(b) * a.H + h_base) * a.t_cap + m2;  // head h_base's slot
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
        const float Zq = unscaled ? __fdiv_rn(p.Z, r) : p.Z, Rq = unscaled ? __fmul_rn(p.R, r) : p.R;
        prm[t2 * NGP + gi] = sink_tok ? make_float4(0.0f, 0.0f, 0.0f, 0.0f) : make_float4(-Zq, -Zq, Rq, Rq);
        if (store)
          a.sz[(slot0 + static_cast<size_t>(gi / NG) * a.t_cap) * NG + gi % NG] =
              sink_tok ? __halves2half2(__ushort_as_half(0), __ushort_as_half(0)) : p.sz;
      }
    }
    __syncwarp();

    // ---------------- quantize and pack this lane's runs of 4Q channels
    uint8_t* rec = a.codes + slot0 * RB + (4 * k2 * Q) * BITS / 8;
#pragma unroll
    for (int h = 0; h < HG; ++h) {
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const float4 zr = prm[t2 * NGP + h * NG + (NG == 2 ? hs : 0)];
        const float2 nZ = f2(zr.x, zr.y), R2 = f2(zr.z, zr.w), M2 = f2(kMagicRound, kMagicRound);
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
        uint32_t wc[NWC];
        if constexpr (32 % BITS == 0) {
          constexpr int PER = 32 / BITS;  // codes per word
#pragma unroll
          for (int i = 0; i < NWC; ++i) {
            const int lo_c = i * PER;
            const int n_c = (4 * Q - lo_c) < PER ? (4 * Q - lo_c) : PER;
            uint32_t v = t[lo_c + n_c - 1];
#pragma unroll
            for (int j = n_c - 2; j >= 0; --j) v = (v << BITS) + t[lo_c + j];  // codes never straddle a word
            wc[i] = v;
          }
          if constexpr (NCB > 22) {
#pragma unroll
            for (int i = 0; i < NWC; ++i)
              wc[i] -= (NCB - 32 * i >= 32) ? magic_offset<BITS, PER>() : magic_offset<BITS, (NCB % 32) / BITS>();
          }
        } else {
#pragma unroll
          for (int i = 0; i < NWC; ++i) wc[i] = 0u;
#pragma unroll
          for (int j = 0; j < 4 * Q; ++j) {
            const int pos = j * BITS;
            const uint32_t c = t[j] - kMagicBits;
            wc[pos >> 5] |= c << (pos & 31);
            if ((pos & 31) + BITS > 32) wc[(pos >> 5) + 1] |= c >> (32 - (pos & 31));
          }
        }
        if constexpr (NCB % 8 != 0) {
          // 12-bit runs (HG = 8, 3 bits): even lanes append their odd neighbour's run
          const uint32_t nb = __shfl_down_sync(0xffffffffu, wc[0], 1);
          if (store && (k2 & 1) == 0) {
            const uint32_t v = wc[0] | (nb << NCB);
            st_code<2 * NCB / 8>(rec + 64 * hs * BITS / 8, &v);
          }
        } else {
          if (store) st_code<NCB / 8>(rec + 64 * hs * BITS / 8, wc);
        }
      }
      rec += code_hstep;
    }
  }
}

// ---------------------------------------------------------------- decode building blocks
// (shared by the decode and the grouped-cache score)

// Phase 2 (reverse), dequantization: this lane's quads of every head of its
// token, A[h][half][q] = (y[c], y[c+2]), (y[c+1], y[c+3]), c = 64 half + 4 (k2 Q + q),
// with the normalisation r folded into S and Z. cst: staged records
// [head][token][RB]; szs: staged (S, Z) words [head][token][group].
template <int HG, int BITS, int G>
__device__ __forceinline__ void dec_dequant(const uint8_t* cst, const uint8_t* szs, int t2, int k2, float r,
                                            float2 (&A)[HG][2][8 / HG][2]) {
  constexpr int NT = 16 / HG, Q = 8 / HG, NG = D / G, RB = D * BITS / 8;
  constexpr int NCB = 4 * Q * BITS, NWC = (NCB + 31) / 32;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    const uint8_t* rec = cst + (h * NT + t2) * RB;
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      const __half2 szv = *reinterpret_cast<const __half2*>(szs + ((h * NT + t2) * NG + (NG == 2 ? hs : 0)) * 4);
      const float2 szf = __half22float2(szv);
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
}

// Phase 2 (reverse), rotations: inverse RoPE of the lane's token (keys), the
// cross-head strides and the stride 64. cs[half][q]: the table chunks
// (c_i, s_i, c_i+1, s_i+1) of the lane's channel quads.
// When PRE is false the chunks are read here from the table row rp instead.
template <int HG, bool PRE>
__device__ __forceinline__ void dec_phase2(float2 (&A)[HG][2][8 / HG][2], int rope, const uint4 (&cs)[2][8 / HG],
                                           const uint4* rp, int k2) {
  constexpr int Q = 8 / HG;
  if (rope == 2) {  // half-split pairs (c, c + 64), angle c: x0 = y0 c + y1 s, x1 = y1 c - y0 s
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const uint4 c0 = PRE ? cs[0][q] : __ldg(rp + rope_chunk(true, 0, k2 * Q + q));
      const uint4 c1 = PRE ? cs[1][q] : __ldg(rp + rope_chunk(true, 1, k2 * Q + q));
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float2 cc = e ? f2(__uint_as_float(c0.z), __uint_as_float(c1.z)) : f2(__uint_as_float(c0.x), __uint_as_float(c1.x));
        const float2 ss = e ? f2(__uint_as_float(c0.w), __uint_as_float(c1.w)) : f2(__uint_as_float(c0.y), __uint_as_float(c1.y));
        const float2 nss = f2(-ss.x, -ss.y);
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const float2 y0 = A[h][0][q][e], y1 = A[h][1][q][e];
          A[h][0][q][e] = fma2(y0, cc, mul2(y1, ss));
          A[h][1][q][e] = fma2(y1, cc, mul2(y0, nss));
        }
      }
    }
  } else if (rope) {
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        const uint4 cv = PRE ? cs[hs][q] : __ldg(rp + rope_chunk(false, hs, k2 * Q + q));
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
}

// The exchange (phase-2 quads -> phase-1 rows) and phase 1 (reverse): the
// strides 32 .. 1 of this lane's half row; x = its 64 channels in natural
// order. Ends with a __syncwarp (every exchange row has been read).
template <int HG>
__device__ __forceinline__ void dec_phase1(const float2 (&A)[HG][2][8 / HG][2], uint8_t* xch, int lane, int t2,
                                           int k2, float (&x)[64]) {
  constexpr int NT = 16 / HG, Q = 8 / HG;
  {
    uint8_t* const base = xch + (t2 * 2) * 272 + xoff(k2 * Q);
#pragma unroll
    for (int hs = 0; hs < 2; ++hs)
#pragma unroll
      for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int q = 0; q < Q; ++q)
          *reinterpret_cast<float4*>(base + (h * NT * 2 + hs) * 272 + 16 * q) =
              make_float4(A[h][hs][q][0].x, A[h][hs][q][0].y, A[h][hs][q][1].x, A[h][hs][q][1].y);
  }
  __syncwarp();
  float4 V[16];  // (x[4g], x[4g+2], x[4g+1], x[4g+3])
#pragma unroll
  for (int g = 0; g < 16; ++g) V[g] = *reinterpret_cast<const float4*>(xch + lane * 272 + xoff(g));
  __syncwarp();  // every exchange row has been read: the region may be reused
  fwht_quads_from4(V);
#pragma unroll
  for (int g = 0; g < 16; ++g) {  // stride 1 (packed), stride 2 (inside each pair)
    float2 p0 = lo2(V[g]), p1 = hi2(V[g]);
    bfly(p0, p1);
    V[g] = make_float4(__fadd_rn(p0.x, p0.y), __fsub_rn(p0.x, p0.y), __fadd_rn(p1.x, p1.y), __fsub_rn(p1.x, p1.y));
  }
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    x[4 * g] = V[g].x;
    x[4 * g + 2] = V[g].y;
    x[4 * g + 1] = V[g].z;
    x[4 * g + 3] = V[g].w;
  }
}

template <int HG, int BITS, int G, bool F32>
__global__ void __launch_bounds__(kDecThreads, 4)
    k_decode_group(const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap omap,
                   const GroupArgs a) {
  constexpr int NT = 16 / HG;        // tokens per warp tile
  constexpr int Q = 8 / HG;
  constexpr int TPT = 2 * HG;
  constexpr int NG = D / G;
  constexpr int NGP = HG * NG;
  constexpr int RB = D * BITS / 8;
  constexpr bool PRE_CS = (Q <= 2);
  static_assert(16 * RB <= kDecCodes && NT * NGP * 4 <= kDecSz, "decode buffers too small");
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kDecWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* const wsm = align1024(smem_raw) + warp * kDecWarpSmem;
  uint8_t* const xch = wsm;                        // exchange rows / output box
  uint8_t* const cst = wsm + kDecXch;              // packed records [head][token][RB]
  uint8_t* const szs = wsm + kDecXch + kDecCodes;  // (S, Z) words [head][token][group]
  uint64_t* const bar = &full[warp];
  const int s1 = lane & 1, t1 = (lane >> 1) % NT, h1 = lane / (2 * NT);  // phase-1 role (row `lane`)
  const int t2 = lane / TPT, k2 = lane % TPT;                             // phase-2 role
  const float r = a.rscale;
  const int gw = blockIdx.x * kDecWarps + warp, n_gw = gridDim.x * kDecWarps;

  if (lane == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto issue_codes = [&](int tile) {  // one lane
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    mbar_arrive_expect_tx(bar, 16 * RB);
    tma_load_3d(cst, &cmap, 0, a.t0 + t_base, b * a.H + h_base, bar);
  };
  auto fetch_sz = [&](int tile) {  // lanes < NT * NGP, one word each; zero past the last token
    if (lane < NT * NGP) {
      int b, h_base, t_base;
      tile_coords(a, tile, HG, NT, b, h_base, t_base);
      const int h = lane / (NT * NG), t = (lane / NG) % NT, g = lane % NG;
      const bool live = t_base + t < a.T;
      const size_t slot = (static_cast<size_t>(b) * a.H + h_base + h) * a.t_cap + a.t0 + t_base + t;
      cp_async4(smem_u32(szs + lane * 4), live ? static_cast<const void*>(a.sz + slot * NG + g) : a.sz,
                live ? 4u : 0u);
    }
    cp_async_commit();
  };
  if (gw < a.n_tiles) {
    if (lane == 0) issue_codes(gw);
    fetch_sz(gw);
  }

  uint32_t parity = 0;
  bool pending_store = false;
  for (int tile = gw; tile < a.n_tiles; tile += n_gw) {
    int b, h_base, t_base;
    tile_coords(a, tile, HG, NT, b, h_base, t_base);
    const int m2 = a.t0 + t_base + t2;
    const uint4* rp =
        a.rope ? reinterpret_cast<const uint4*>(a.rope_cs) + static_cast<size_t>(min(m2, a.t0 + a.T - 1)) * (D / 4)
               : nullptr;
    uint4 cs_pre[2][Q];
    if (PRE_CS && a.rope) {
#pragma unroll
      for (int hs = 0; hs < 2; ++hs)
#pragma unroll
        for (int q = 0; q < Q; ++q) cs_pre[hs][q] = __ldg(rp + rope_chunk(a.rope == 2, hs, k2 * Q + q));
    }
    const bool ok = mbar_wait(bar, parity, a.wait_ns, a.err);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) mbar_wait(bar, parity, a.wait_ns, a.err);  // let the copy in flight land
      break;
    }
    parity ^= 1u;
    cp_async_wait_all();
    __syncwarp();  // records and scale/zero words of the tile are staged

    // ---------------- phase 2 (reverse): dequantize (normalisation folded in), inverse RoPE, strides
    float2 A[HG][2][Q][2];
    dec_dequant<HG, BITS, G>(cst, szs, t2, k2, r, A);
    __syncwarp();  // every lane has read the staged records and words: fetch the next tile's
    if (tile + n_gw < a.n_tiles) {
      if (lane == 0) {
        fence_async_smem();
        issue_codes(tile + n_gw);
      }
      fetch_sz(tile + n_gw);
    }
    dec_phase2<HG, PRE_CS>(A, a.rope, cs_pre, rp, k2);

    // ---------------- exchange -> phase-1 rows (the previous output box must have been read)
    if (pending_store && lane == 0) bulk_wait_read<0>();
    __syncwarp();
    float x[64];  // natural channel order
    dec_phase1<HG>(A, xch, lane, t2, k2, x);

    // ---------------- phase 1 (reverse): sinks, inverse permutation, output box
    const int tt = t_base + t1, m = a.t0 + tt;
    const bool sink_tok = tt < a.T && m < a.n_sink;
    if (sink_tok) {  // sink positions come back verbatim
      const uint4* src = reinterpret_cast<const uint4*>(
          a.sink + ((static_cast<size_t>(b) * a.H + h_base + h1) * a.n_sink + m) * D + 64 * s1);
#pragma unroll
      for (int c = 0; c < 8; ++c) h8_to_f32(__ldg(src + c), &x[8 * c]);
    }
    const bool permute = a.perm != nullptr && !sink_tok;
    if constexpr (!F32) {  // box rows of 64 fp16 channels: row `lane`, chunk j at j ^ (lane & 7)
      if (!permute) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(xch + lane * 128 + ((c ^ (lane & 7)) << 4)) = f32_to_h8(&x[8 * c]);
      } else {  // x'[perm[j]] = x[j]: scatter into the row pair of (head, token)
        const int16_t* pr = a.perm + static_cast<size_t>(h_base + h1) * D + 64 * s1;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
          const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
            const uint32_t rr = static_cast<uint32_t>(lane & ~1) + (e >> 6);
            *reinterpret_cast<__half*>(xch + rr * 128 + ((((e >> 3) & 7) ^ (rr & 7)) << 4) + (e & 7) * 2) =
                __float2half_rn(x[8 * c + i]);
          }
        }
      }
    } else {  // box rows of 32 fp32 channels: rows 2 lane, 2 lane + 1
      if (!permute) {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t rr = 2 * lane + (c >> 3);
          *reinterpret_cast<float4*>(xch + rr * 128 + (((c & 7) ^ (rr & 7)) << 4)) =
              make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
        }
      } else {
        const int16_t* pr = a.perm + static_cast<size_t>(h_base + h1) * D + 64 * s1;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
          const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
            const uint32_t rr = 2 * (static_cast<uint32_t>(lane & ~1) + (e >> 6)) + ((e >> 5) & 1);
            *reinterpret_cast<float*>(xch + rr * 128 + ((((e >> 2) & 7) ^ (rr & 7)) << 4) + (e & 3) * 4) =
                x[8 * c + i];
          }
        }
      }
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_4d(&omap, 0, 0, t_base, b * a.H + h_base, xch);
      bulk_commit();
    }
    pending_store = true;
  }
  if (lane == 0) bulk_wait_all<0>();  // the output stores have completed
  cp_async_wait_all();
}

// ---------------------------------------------------------------- grouped-cache score
// Decode-step scores over a grouped-head cache ("RotateKV", pre-RoPE
// grouped-head rotation; "EliteKV - RoPE频率选择与低秩投影" §2.2 score): the key of
// head h at slot n in attention space is RoPE_n of its decode, and the decode
// mixes all heads of the group (inverse RoPE, the HG*128-point FWHT), so the
// query cannot be rotated once instead: every slot is decoded (the decode
// kernel's phases), turned by RoPE_n and dotted with the GQ query heads of
// its head. A CTA owns a contiguous token range of one (batch, head group);
// its queries sit in shared memory in fp32, rows padded so that the lanes of
// a quarter warp reading different (head, half) rows hit distinct banks.
struct ScoreGroupArgs {
  const __half* q;  // [B][Hq][128]
  float* scores;    // [B][Hq][n_tok]
  int Hq, n_tok, splits, n_tb;
  float scale;
};

template <int HG, int GQ>
__host__ __device__ constexpr int sg_qpitch() {  // bytes per (head, half) block of the queries in shared memory
  return GQ * 256 + 16;
}

template <int HG, int BITS, int G, int GQ>
__global__ void __launch_bounds__(kDecThreads)
    k_score_group(const __grid_constant__ CUtensorMap cmap, const GroupArgs a, const ScoreGroupArgs sa) {
  constexpr int NT = 16 / HG;
  constexpr int Q = 8 / HG;
  constexpr int TPT = 2 * HG;
  constexpr int NG = D / G;
  constexpr int NGP = HG * NG;
  constexpr int RB = D * BITS / 8;
  constexpr bool PRE_CS = (Q <= 2);
  constexpr int QP = sg_qpitch<HG, GQ>();
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kDecWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* const base = align1024(smem_raw);
  uint8_t* const wsm = base + warp * kDecWarpSmem;
  uint8_t* const xch = wsm;
  uint8_t* const cst = wsm + kDecXch;
  uint8_t* const szs = wsm + kDecXch + kDecCodes;
  uint8_t* const qs = base + kDecWarps * kDecWarpSmem;  // [HG][2][GQ][64] fp32, (head, half) rows QP apart
  uint64_t* const bar = &full[warp];
  const int s1 = lane & 1, t1 = (lane >> 1) % NT, h1 = lane / (2 * NT);
  const int t2 = lane / TPT, k2 = lane % TPT;
  const float r = a.rscale;
  const int sg = static_cast<int>(blockIdx.x) / sa.splits, part = static_cast<int>(blockIdx.x) % sa.splits;
  const int b = sg / a.n_grp, h_base = (sg % a.n_grp) * HG;
  const int tb0 = static_cast<int>(static_cast<long long>(sa.n_tb) * part / sa.splits);
  const int tb1 = static_cast<int>(static_cast<long long>(sa.n_tb) * (part + 1) / sa.splits);

  // the group's queries: q[b][(h_base + h) GQ + g][64 s + c] at qs + (h 2 + s) QP + g 256 + 4 c
  for (int e = threadIdx.x; e < HG * GQ * 32; e += blockDim.x) {
    const int hg = e / (GQ * 32), g = (e / 32) % GQ, c4 = e % 32;  // four channels c4*4 .. +3
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(
                                sa.q + (static_cast<size_t>(b) * sa.Hq + (h_base + hg) * GQ + g) * D) + c4);
    const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    const int s = c4 >> 4, c = (c4 & 15) * 4;
    *reinterpret_cast<float4*>(qs + (hg * 2 + s) * QP + g * 256 + c * 4) = make_float4(lo.x, lo.y, hi.x, hi.y);
  }
  if (lane == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto issue_codes = [&](int tb) {  // one lane
    mbar_arrive_expect_tx(bar, 16 * RB);
    tma_load_3d(cst, &cmap, 0, tb * NT, b * a.H + h_base, bar);
  };
  auto fetch_sz = [&](int tb) {
    if (lane < NT * NGP) {
      const int h = lane / (NT * NG), t = (lane / NG) % NT, g = lane % NG;
      const bool live = tb * NT + t < sa.n_tok;
      const size_t slot = (static_cast<size_t>(b) * a.H + h_base + h) * a.t_cap + tb * NT + t;
      cp_async4(smem_u32(szs + lane * 4), live ? static_cast<const void*>(a.sz + slot * NG + g) : a.sz,
                live ? 4u : 0u);
    }
    cp_async_commit();
  };
  const int tb_first = tb0 + warp;
  if (tb_first < tb1) {
    if (lane == 0) issue_codes(tb_first);
    fetch_sz(tb_first);
  }
  uint32_t parity = 0;
  for (int tb = tb_first; tb < tb1; tb += kDecWarps) {
    const int t_base = tb * NT;
    const int m2 = t_base + t2;
    const uint4* rp = reinterpret_cast<const uint4*>(a.rope_cs) + static_cast<size_t>(min(m2, sa.n_tok - 1)) * (D / 4);
    uint4 cs_pre[2][Q];
    if (PRE_CS) {
#pragma unroll
      for (int hs = 0; hs < 2; ++hs)
#pragma unroll
        for (int q = 0; q < Q; ++q) cs_pre[hs][q] = __ldg(rp + rope_chunk(a.rope == 2, hs, k2 * Q + q));
    }
    const bool ok = mbar_wait(bar, parity, a.wait_ns, a.err);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) mbar_wait(bar, parity, a.wait_ns, a.err);
      break;
    }
    parity ^= 1u;
    cp_async_wait_all();
    __syncwarp();
    float2 A[HG][2][Q][2];
    dec_dequant<HG, BITS, G>(cst, szs, t2, k2, r, A);
    __syncwarp();
    if (tb + kDecWarps < tb1) {
      if (lane == 0) {
        fence_async_smem();
        issue_codes(tb + kDecWarps);
      }
      fetch_sz(tb + kDecWarps);
    }
    dec_phase2<HG, PRE_CS>(A, a.rope, cs_pre, rp, k2);
    float x[64];  // the pre-RoPE key, channels [64 s1, 64 s1 + 64) of head h1 at slot n
    dec_phase1<HG>(A, xch, lane, t2, k2, x);
    const int n = t_base + t1;
    if (n < a.n_sink) {  // sinks: the stored fp16 key
      const uint4* src = reinterpret_cast<const uint4*>(
          a.sink + ((static_cast<size_t>(b) * a.H + h_base + h1) * a.n_sink + n) * D + 64 * s1);
#pragma unroll
      for (int c = 0; c < 8; ++c) h8_to_f32(__ldg(src + c), &x[8 * c]);
    }
    // RoPE_n of the key (fp32, the encoder's order)
    const float* row = a.rope_cs + static_cast<size_t>(min(n, sa.n_tok - 1)) * D;
    if (a.rope != 2) {  // pairs (2i, 2i + 1), i = 32 s1 + c / 2
      const float4* cs = reinterpret_cast<const float4*>(row) + 16 * s1;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 v = __ldg(cs + c);
        rope_fwd(x[4 * c], x[4 * c + 1], v.x, v.y);
        rope_fwd(x[4 * c + 2], x[4 * c + 3], v.z, v.w);
      }
    } else {  // pairs (c, c + 64) across the lane pair (lane ^ 1), angle c
      const float4* cs = reinterpret_cast<const float4*>(row);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float4 v = __ldg(cs + c);  // angles 2c, 2c + 1
        const float2 y = rope_half_fwd2(f2(x[2 * c], x[2 * c + 1]), f2(v.x, v.z), f2(v.y, v.w), s1 != 0, 1);
        x[2 * c] = y.x;
        x[2 * c + 1] = y.y;
      }
    }
    float dot[GQ];
#pragma unroll
    for (int g = 0; g < GQ; ++g) {
      const uint8_t* qrow = qs + (h1 * 2 + s1) * QP + g * 256;
      float acc = 0.0f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 qv = *reinterpret_cast<const float4*>(qrow + 16 * c);
        acc = __fmaf_rn(qv.x, x[4 * c], acc);
        acc = __fmaf_rn(qv.y, x[4 * c + 1], acc);
        acc = __fmaf_rn(qv.z, x[4 * c + 2], acc);
        acc = __fmaf_rn(qv.w, x[4 * c + 3], acc);
      }
      dot[g] = acc + __shfl_xor_sync(0xffffffffu, acc, 1);  // + the other half of the head
    }
    if (s1 == 0 && n < sa.n_tok) {
#pragma unroll
      for (int g = 0; g < GQ; ++g)
        sa.scores[(static_cast<size_t>(b) * sa.Hq + (h_base + h1) * GQ + g) * sa.n_tok + n] = dot[g] * sa.scale;
    }
  }
  cp_async_wait_all();
}

template <int HG, int BITS, int G, int GQ>
kvq_status run_score_group(const GroupArgs& a, const ScoreGroupArgs& sa0, const CUtensorMap& cm, const LaunchCtx& ctx,
                           cudaStream_t st) {
  ScoreGroupArgs sa = sa0;
  const void* fn = reinterpret_cast<const void*>(k_score_group<HG, BITS, G, GQ>);
  const size_t smem = 1024 + static_cast<size_t>(kDecWarps) * kDecWarpSmem + 2 * HG * sg_qpitch<HG, GQ>();
  if (!set_smem_once(fn, smem)) return KVQ_ERR_CUDA;
  const int per_sm = occupancy_once(fn, kDecThreads, smem);
  const long long streams = static_cast<long long>(a.B) * a.n_grp;
  sa.n_tb = (sa.n_tok + 16 / HG - 1) / (16 / HG);
  long long splits = static_cast<long long>(ctx.num_sms) * per_sm / streams;
  const long long max_splits = (sa.n_tb + kDecWarps - 1) / kDecWarps;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  if (streams * splits >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
  sa.splits = static_cast<int>(splits);
  k_score_group<HG, BITS, G, GQ><<<static_cast<unsigned>(streams * splits), kDecThreads, smem, st>>>(cm, a, sa);
  return launch_status();
}

template <int HG, int BITS, int G>
kvq_status run(bool enc, const GroupArgs& a, const CUtensorMap& cm, const CUtensorMap& om, int out_fp32,
               const LaunchCtx& ctx, cudaStream_t st) {
  if (enc) {
    const void* fn = reinterpret_cast<const void*>(k_encode_group<HG, BITS, G>);
    const size_t smem = 1024 + static_cast<size_t>(kEncWarps) * kEncWarpSmem;
    if (!set_smem_once(fn, smem)) return KVQ_ERR_CUDA;
    const int per_sm = occupancy_once(fn, kEncThreads, smem);
    const long long want = static_cast<long long>(ctx.num_sms) * per_sm;
    const long long ctas = (static_cast<long long>(a.n_tiles) + kEncWarps - 1) / kEncWarps;
    const unsigned grid = static_cast<unsigned>(ctas < want ? ctas : want);
    k_encode_group<HG, BITS, G><<<grid, kEncThreads, smem, st>>>(cm, a);
    return launch_status();
  }
  const size_t smem = 1024 + static_cast<size_t>(kDecWarps) * kDecWarpSmem;
  const void* fn = out_fp32 ? reinterpret_cast<const void*>(k_decode_group<HG, BITS, G, true>)
                            : reinterpret_cast<const void*>(k_decode_group<HG, BITS, G, false>);
  if (!set_smem_once(fn, smem)) return KVQ_ERR_CUDA;
  const int per_sm = occupancy_once(fn, kDecThreads, smem);
  const long long want = static_cast<long long>(ctx.num_sms) * per_sm;
  const long long ctas = (static_cast<long long>(a.n_tiles) + kDecWarps - 1) / kDecWarps;
  const unsigned grid = static_cast<unsigned>(ctas < want ? ctas : want);
  if (out_fp32)
    k_decode_group<HG, BITS, G, true><<<grid, kDecThreads, smem, st>>>(cm, om, a);
  else
    k_decode_group<HG, BITS, G, false><<<grid, kDecThreads, smem, st>>>(cm, om, a);
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

// NT tokens per tile (16 / HG: one warp tile of HG heads x NT tokens, 2048 values).
GroupArgs make_args(const kvq_desc& d, const kvq_tables& tb, const kvq_packed& p, const LaunchCtx& ctx, int NT) {
  GroupArgs a{};
  a.B = d.batch;
  a.H = d.heads;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.t_cap = d.t_cap;
  a.n_sink = d.n_sink;
  a.rope = d.rope;
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
  const int NT = 16 / d.group_heads;
  GroupArgs a = make_args(d, tb, out, ctx, NT);
  a.x = static_cast<const __half*>(x);
  // input as a 4-D tensor: 64 channels x 2 halves x T tokens x B*H heads; one box = one warp tile
  CUtensorMap xm;
  const uint64_t dims[4] = {64, 2, static_cast<uint64_t>(d.tokens), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t strides[3] = {128, 256, static_cast<uint64_t>(d.tokens) * 256};
  const uint32_t box[4] = {64, 2, static_cast<uint32_t>(NT), static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&xm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  return dispatch(true, d, a, xm, xm, 0, ctx, st);
}

kvq_status launch_decode_group(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                               int out_fp32, cudaStream_t st, const LaunchCtx& ctx) {
  const int NT = 16 / d.group_heads;
  const GroupArgs a = make_args(d, tb, in, ctx, NT);
  // packed codes: [B*H][t_cap][RB] bytes; one box = one warp tile's records
  CUtensorMap cm;
  const uint64_t rb = static_cast<uint64_t>(D) * d.bits / 8;
  const uint64_t cdims[3] = {rb, static_cast<uint64_t>(d.t_cap), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t cstrides[2] = {rb, static_cast<uint64_t>(d.t_cap) * rb};
  const uint32_t cbox[3] = {static_cast<uint32_t>(rb), static_cast<uint32_t>(NT),
                            static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&cm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, in.codes, cdims, cstrides, cbox, CU_TENSOR_MAP_SWIZZLE_NONE))
    return KVQ_ERR_CUDA;
  // output: rows of 128 bytes (64 fp16 or 32 fp32 channels) x row parts x tokens x heads,
  // one box = one warp tile, 128-byte swizzle
  CUtensorMap om;
  const uint64_t es = out_fp32 ? 4 : 2, inner = 128 / es, parts = D / inner;
  const uint64_t dims[4] = {inner, parts, static_cast<uint64_t>(d.tokens), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t strides[3] = {128, D * es, static_cast<uint64_t>(d.tokens) * D * es};
  const uint32_t box[4] = {static_cast<uint32_t>(inner), static_cast<uint32_t>(parts), static_cast<uint32_t>(NT),
                           static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&om, out_fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, x_out, dims,
                strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  return dispatch(false, d, a, cm, om, out_fp32, ctx, st);
}

kvq_status launch_score_group(const kvq_desc& d, const void* q, int q_heads, const kvq_packed& cache,
                              const kvq_tables& tb, int n_tokens, float scale, float* scores, cudaStream_t st,
                              const LaunchCtx& ctx) {
  const int NT = 16 / d.group_heads;
  kvq_desc dd = d;
  dd.tokens = n_tokens;
  dd.t0 = 0;
  const GroupArgs a = make_args(dd, tb, cache, ctx, NT);
  ScoreGroupArgs sa{};
  sa.q = static_cast<const __half*>(q);
  sa.scores = scores;
  sa.Hq = q_heads;
  sa.n_tok = n_tokens;
  sa.scale = scale;
  CUtensorMap cm;
  const uint64_t rb = static_cast<uint64_t>(D) * d.bits / 8;
  const uint64_t cdims[3] = {rb, static_cast<uint64_t>(d.t_cap), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t cstrides[2] = {rb, static_cast<uint64_t>(d.t_cap) * rb};
  const uint32_t cbox[3] = {static_cast<uint32_t>(rb), static_cast<uint32_t>(NT),
                            static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&cm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, cache.codes, cdims, cstrides, cbox, CU_TENSOR_MAP_SWIZZLE_NONE))
    return KVQ_ERR_CUDA;
  const int gq = q_heads / d.heads;
#define KVQ_SG(HG_, B_, G_, GQ_)                                                           \
  if (d.group_heads == HG_ && d.bits == B_ && d.group == G_ && gq == GQ_)                 \
    return run_score_group<HG_, B_, G_, GQ_>(a, sa, cm, ctx, st);
#define KVQ_SG_GQ(HG_, B_, G_) KVQ_SG(HG_, B_, G_, 1) KVQ_SG(HG_, B_, G_, 2) KVQ_SG(HG_, B_, G_, 4) KVQ_SG(HG_, B_, G_, 8)
  KVQ_SG_GQ(8, 2, 128)
  KVQ_SG_GQ(8, 4, 128)
  KVQ_SG_GQ(8, 2, 64)
  KVQ_SG_GQ(4, 2, 128)
  KVQ_SG_GQ(2, 2, 128)
#undef KVQ_SG_GQ
#undef KVQ_SG
  return KVQ_ERR_UNSUPPORTED;
}

}  // namespace kvq
