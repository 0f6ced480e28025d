// Decode-step score ("EliteKV - RoPE频率选择与低秩投影", §2.2:
// A_{m,n} = q_m^rot . k_n^rot / sqrt(d)) over the compressed cache.
//
// The keys were stored as y_n = H P RoPE_n(k_n) (normalised Sylvester H,
// permutation P) quantized per group to Z + c S. Since H and P are
// orthogonal, q . P^T H^T y = (H P q) . y, so the query is rotated once per
// (batch, query head) and every key needs only unpack + multiply-add:
//   s_n = scale * sum_g ( S_g * sum_{j in g} qt_j c_j + Z_g * sum_{j in g} qt_j ).
// Sink positions (n < n_sink) hold fp16 keys: s_n = scale * q . RoPE_n(sink_n).
//
// Grid: (token tiles of 256, KV head, batch); each CTA serves all GQ query
// heads that share its KV head (grouped-query attention), one token per
// thread, fp32 accumulation.
#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_qdigits.cuh"

namespace kvq {
namespace {

struct ScoreArgs {
  int B, H, Hq, t_cap, n_tok, n_sink, rope, rot;
  float scale, rscale;
  const __half* q;
  const int16_t* perm;
  const float* rope_cs;
  const uint8_t* codes;
  const __half2* sz;
  const __half* sink;
  float* scores;
};

constexpr int kThreads = 256;

template <int D, int BITS, int G, int GQ>
__global__ void __launch_bounds__(kThreads) k_score_simt(const ScoreArgs a) {
  constexpr int NG = D / G;
  constexpr int NW = D * BITS / 32;
  constexpr int RB = D * BITS / 8;
  __shared__ __align__(16) float qt[GQ][D];   // rotated queries H P q
  __shared__ __align__(16) float qr[GQ][D];   // raw queries (sink path)
  __shared__ float qsum[GQ][NG];
  const int tid = threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;

  if (tid < GQ) {
    const int qh = h * GQ + tid;
    const __half* qv = a.q + (static_cast<size_t>(b) * a.Hq + qh) * D;
    float v[D];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      float f[8];
      h8_to_f32(__ldg(reinterpret_cast<const uint4*>(qv) + c), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[8 * c + i] = f[i];
        qr[tid][8 * c + i] = f[i];
      }
    }
    if (a.perm) {
      const int16_t* pr = a.perm + static_cast<size_t>(h) * D;
#pragma unroll
      for (int j = 0; j < D; ++j) v[j] = __half2float(qv[__ldg(pr + j) & (D - 1)]);
    }
    if (a.rot == KVQ_ROT_FWHT_HEAD) {
      fwht_reg<D>(v);
#pragma unroll
      for (int j = 0; j < D; ++j) v[j] = __fmul_rn(v[j], a.rscale);
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float s = 0.0f;
#pragma unroll
      for (int j = 0; j < G; ++j) s = __fadd_rn(s, v[g * G + j]);
      qsum[tid][g] = s;
    }
#pragma unroll
    for (int j = 0; j < D; ++j) qt[tid][j] = v[j];
  }
  __syncthreads();

  const int n = blockIdx.x * kThreads + tid;
  if (n >= a.n_tok) return;
  float acc[GQ];
#pragma unroll
  for (int i = 0; i < GQ; ++i) acc[i] = 0.0f;
  const size_t vh = static_cast<size_t>(b) * a.H + h;

  if (n < a.n_sink) {
    const uint4* src = reinterpret_cast<const uint4*>(a.sink + (vh * a.n_sink + n) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      float k8[8];
      h8_to_f32(__ldg(src + c), k8);
      if (a.rope) {
        const float4* cs = reinterpret_cast<const float4*>(a.rope_cs + static_cast<size_t>(n) * D) + 2 * c;
        const float4 c0 = __ldg(cs), c1 = __ldg(cs + 1);
        rope_fwd(k8[0], k8[1], c0.x, c0.y);
        rope_fwd(k8[2], k8[3], c0.z, c0.w);
        rope_fwd(k8[4], k8[5], c1.x, c1.y);
        rope_fwd(k8[6], k8[7], c1.z, c1.w);
      }
#pragma unroll
      for (int i = 0; i < GQ; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i] = __fmaf_rn(qr[i][8 * c + e], k8[e], acc[i]);
    }
  } else {
    const size_t slot = vh * a.t_cap + n;
    uint32_t w[NW];
    const uint8_t* src = a.codes + slot * RB;
    if constexpr (RB % 16 == 0) {
#pragma unroll
      for (int i = 0; i < RB / 16; ++i) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(src) + i);
        w[4 * i] = u.x; w[4 * i + 1] = u.y; w[4 * i + 2] = u.z; w[4 * i + 3] = u.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < RB / 8; ++i) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(src) + i);
        w[2 * i] = u.x; w[2 * i + 1] = u.y;
      }
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const __half2 szv = a.sz[slot * NG + g];
      const float S = __low2float(szv), Z = __high2float(szv);
      float dg[GQ];
#pragma unroll
      for (int i = 0; i < GQ; ++i) dg[i] = 0.0f;
#pragma unroll
      for (int jj = 0; jj < G; ++jj) {
        const int j = g * G + jj;
        const float c = code_to_float(unpack_code<BITS, NW>(w, j));
#pragma unroll
        for (int i = 0; i < GQ; ++i) dg[i] = __fmaf_rn(c, qt[i][j], dg[i]);
      }
#pragma unroll
      for (int i = 0; i < GQ; ++i) acc[i] = __fmaf_rn(S, dg[i], __fmaf_rn(Z, qsum[i][g], acc[i]));
    }
  }
#pragma unroll
  for (int i = 0; i < GQ; ++i)
    a.scores[(static_cast<size_t>(b) * a.Hq + h * GQ + i) * a.n_tok + n] = __fmul_rn(acc[i], a.scale);
}

// ---------------------------------------------------------------------------
// Tensor-core score (head_dim 128, 2- or 4-bit codes).
//
// Per (batch, KV head) the rotated queries qt = H P q of the GQ query heads
// are quantized once to 16-bit integers Q = rint(qt / sq), sq = max|qt| / 32000,
// and split into two int8 digits Q = 256 hi + lo. A warp then scores 16
// tokens at a time with mma.sync m16n8k32 (u8 codes x s8 digits, exact int32
// accumulation): A = the codes expanded to one byte each by a shift and a
// mask per 4 codes, B = the digits, N = 2 columns (lo, hi) per query head.
//   s_n = scale * sum_g ( S_g * sq * (sum_j c_j lo_j + 256 sum_j c_j hi_j) + Z_g * sum_{j in g} qt_j ).
// The digit rounding moves each score by at most S * sq / 2 * sum_j c_j,
// i.e. below 2e-5 of the score's L1 magnitude. Codes stream through shared
// memory by bulk copy, two tiles of 128 tokens in flight; CTAs are
// persistent over a range of tiles of one (batch, KV head) so the query
// rotation is done once per CTA.
// Tiling: 2 m-tiles of 16 tokens per warp (256-token tiles), 4 tiles in
// flight per CTA, at most 4 CTAs per SM.
constexpr int kMmaThreads = 256;
constexpr int kMmaMT = 2;                  // 16-token m-tiles per warp per tile
constexpr int kMmaTile = 8 * 16 * kMmaMT;  // tokens per tile
constexpr int kMmaStages = 4;              // tiles in flight per CTA
constexpr int kMmaCtasPerSm = 4;

struct MmaArgs {
  ScoreArgs s;
  int chunks, tiles_per_chunk;
  FastDiv div_tpb, div_h;  // tiles per (batch, KV head); KV heads
  uint32_t* err;
  uint64_t wait_ns;
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int BITS, int G, int GQ>
__global__ void __launch_bounds__(kMmaThreads) k_score_mma(const MmaArgs ma) {
  constexpr int D = 128;
  constexpr int RB = D * BITS / 8;
  constexpr int NW = RB / 4;             // words per record
  constexpr int NTN = (2 * GQ + 7) / 8;  // n-tiles of 8 columns
  constexpr int NGK = D / G;             // quantization groups per record
  const ScoreArgs& a = ma.s;
  extern __shared__ __align__(128) uint8_t codes_dyn[];  // kMmaStages tiles of kMmaTile records
  __shared__ __align__(16) uint2 bfrag[NTN][4][4][8];
  __shared__ __align__(16) float qraw[GQ][D];
  __shared__ int8_t qd[GQ][2][D];
  __shared__ float qsum[GQ][NGK];
  __shared__ float sqh[GQ];
  __shared__ __align__(8) uint64_t full[kMmaStages];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  // this CTA's contiguous range of global tiles (batch-major, then KV head, then token tile)
  const int total = a.B * a.H * static_cast<int>(ma.div_tpb.d);
  const int gt0 = static_cast<int>(static_cast<long long>(total) * blockIdx.x / gridDim.x);
  const int gt1 = static_cast<int>(static_cast<long long>(total) * (blockIdx.x + 1) / gridDim.x);
  if (gt0 >= gt1) return;

  auto issue = [&](int gt, int st) {
    const int bh = static_cast<int>(ma.div_tpb.div(gt));
    const int n0 = static_cast<int>(ma.div_tpb.mod(gt, bh)) * kMmaTile;
    const uint32_t bytes = static_cast<uint32_t>(min(kMmaTile, a.n_tok - n0) * RB);
    mbar_arrive_expect_tx(&full[st], bytes);
    bulk_load(codes_dyn + st * (kMmaTile * RB), a.codes + (static_cast<size_t>(bh) * a.t_cap + n0) * RB, bytes,
              &full[st]);
  };
  if (tid == 0) {
    for (int i = 0; i < kMmaStages; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int i = 0; i < kMmaStages && gt0 + i < gt1; ++i) issue(gt0 + i, i);
  }

  // rotated, digit-split queries of one (batch, KV head); warp w < GQ handles query head w
  auto prologue = [&](int b, int h, bool with_sinks) {
    __syncthreads();  // previous (batch, head) fully consumed
    if (warp < GQ) {
      const int qh = h * GQ + warp;
      query_digits<G>(a.q + (static_cast<size_t>(b) * a.Hq + qh) * D,
                      a.perm ? a.perm + static_cast<size_t>(h) * D : nullptr, a.rot, a.rscale, lane, qraw[warp],
                      qd[warp][0], qd[warp][1], qsum[warp], &sqh[warp]);
    }
    __syncthreads();
    build_score_bfrag<BITS, GQ, NTN>(bfrag, qd, tid, kMmaThreads);  // column c = 2 * head + digit
    __syncthreads();
    // fp16 sinks of this (batch, head): s = scale * q . RoPE_n(sink_n); done by the
    // CTA that owns the (batch, head)'s first tile, one warp per (sink, query head)
    if (with_sinks) {
      const size_t vh = static_cast<size_t>(b) * a.H + h;
      for (int e = warp; e < min(a.n_sink, a.n_tok) * GQ; e += kMmaThreads / 32) {
        const int n = e / GQ, hh = e % GQ;
        const float acc = sink_dot(qraw[hh], a.sink + (vh * a.n_sink + n) * D,
                                   a.rope ? a.rope_cs + static_cast<size_t>(n) * D : nullptr, lane);
        if (lane == 0) a.scores[(static_cast<size_t>(b) * a.Hq + h * GQ + hh) * a.n_tok + n] = acc * a.scale;
      }
    }
  };
  // scale / zero of this thread's tokens of one tile (register prefetch)
  auto load_sz = [&](int gt, __half2 (&sza)[kMmaMT][NGK], __half2 (&szb)[kMmaMT][NGK]) {
    const int bh = static_cast<int>(ma.div_tpb.div(gt));
    const int n0 = static_cast<int>(ma.div_tpb.mod(gt, bh)) * kMmaTile;
#pragma unroll
    for (int mt = 0; mt < kMmaMT; ++mt) {
      const int na = n0 + warp * 16 * kMmaMT + mt * 16 + g, nb = na + 8;
#pragma unroll
      for (int q = 0; q < NGK; ++q) {
        sza[mt][q] = na < a.n_tok ? a.sz[(static_cast<size_t>(bh) * a.t_cap + na) * NGK + q] : __half2();
        szb[mt][q] = nb < a.n_tok ? a.sz[(static_cast<size_t>(bh) * a.t_cap + nb) * NGK + q] : __half2();
      }
    }
  };

  __half2 sza[kMmaMT][NGK], szb[kMmaMT][NGK];
  load_sz(gt0, sza, szb);
  int cur_bh = -1;
  bool ok = true;
  int gt_fail = gt1;  // first tile whose copy was not seen to land
  for (int gt = gt0; gt < gt1; ++gt) {
    const int it = gt - gt0;
    const int st = it % kMmaStages;
    const int bh = static_cast<int>(ma.div_tpb.div(gt));
    const int b = static_cast<int>(ma.div_h.div(bh)), h = bh - b * a.H;
    const int n0 = static_cast<int>(ma.div_tpb.mod(gt, bh)) * kMmaTile;
    if (bh != cur_bh) {
      prologue(b, h, n0 == 0);
      cur_bh = bh;
    }
    ok = mbar_wait(&full[st], (it / kMmaStages) & 1, ma.wait_ns, ma.err) && ok;
    const uint32_t base = smem_u32(codes_dyn + st * (kMmaTile * RB));
    int acc[kMmaMT][NGK][NTN][4];
#pragma unroll
    for (int mt = 0; mt < kMmaMT; ++mt) {
      const int ra = warp * 16 * kMmaMT + mt * 16 + g;  // tile rows ra and ra + 8
      uint32_t wa[NW], wb[NW];
#pragma unroll
      for (int i = 0; i < NW / 4; ++i) {
        const uint4 ua = lds128(base + ra * RB + 16 * i);
        const uint4 ub = lds128(base + (ra + 8) * RB + 16 * i);
        wa[4 * i] = ua.x; wa[4 * i + 1] = ua.y; wa[4 * i + 2] = ua.z; wa[4 * i + 3] = ua.w;
        wb[4 * i] = ub.x; wb[4 * i + 1] = ub.y; wb[4 * i + 2] = ub.z; wb[4 * i + 3] = ub.w;
      }
#pragma unroll
      for (int q = 0; q < NGK; ++q)
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[mt][q][nt][i] = 0;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t a0, a1, a2, a3;
        score_afrag<BITS, NW>(wa, wb, s, tig, a0, a1, a2, a3);
        constexpr int SPG = G / 32;  // k-steps per group
        const int q = s / SPG;
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt) mma_u8s8(acc[mt][q][nt], a0, a1, a2, a3, bfrag[nt][s][tig][g]);
      }
    }
    // every warp has read this stage: refill it with the tile kMmaStages ahead
    if (!__syncthreads_and(ok)) {
      gt_fail = gt;
      break;
    }
    if (tid == 0 && gt + kMmaStages < gt1) issue(gt + kMmaStages, st);
    __half2 pa[kMmaMT][NGK], pb[kMmaMT][NGK];
#pragma unroll
    for (int mt = 0; mt < kMmaMT; ++mt)
#pragma unroll
      for (int q = 0; q < NGK; ++q) {
        pa[mt][q] = sza[mt][q];
        pb[mt][q] = szb[mt][q];
      }
    if (gt + 1 < gt1) load_sz(gt + 1, sza, szb);  // next tile's scale / zero
    // epilogue: thread holds columns 2 tig (lo) and 2 tig + 1 (hi) = query head nt*4 + tig
#pragma unroll
    for (int mt = 0; mt < kMmaMT; ++mt) {
      const int na = n0 + warp * 16 * kMmaMT + mt * 16 + g, nb = na + 8;
#pragma unroll
      for (int nt = 0; nt < NTN; ++nt) {
        const int hh = nt * 4 + tig;
        if (hh >= GQ) continue;
        const float sq = sqh[hh];
        float sa = 0.0f, sb = 0.0f;
#pragma unroll
        for (int q = 0; q < NGK; ++q) {
          const float da = static_cast<float>(acc[mt][q][nt][0] + 256 * acc[mt][q][nt][1]);
          const float db = static_cast<float>(acc[mt][q][nt][2] + 256 * acc[mt][q][nt][3]);
          sa = __fmaf_rn(__low2float(pa[mt][q]) * sq, da, __fmaf_rn(__high2float(pa[mt][q]), qsum[hh][q], sa));
          sb = __fmaf_rn(__low2float(pb[mt][q]) * sq, db, __fmaf_rn(__high2float(pb[mt][q]), qsum[hh][q], sb));
        }
        float* out = a.scores + (static_cast<size_t>(b) * a.Hq + h * GQ + hh) * a.n_tok;
        if (na < a.n_tok && na >= a.n_sink) out[na] = sa * a.scale;
        if (nb < a.n_tok && nb >= a.n_sink) out[nb] = sb * a.scale;
      }
    }
  }
  // After a timed-out wait, let the copies still in flight land (bounded)
  // before the CTA exits: tiles gt_fail .. gt_fail + kMmaStages - 1 were
  // issued and not consumed; each is waited on once, at its stage and phase.
  if (gt_fail < gt1 && tid == 0) {
    for (int gt = gt_fail; gt < gt1 && gt < gt_fail + kMmaStages; ++gt) {
      const int it = gt - gt0;
      mbar_wait(&full[it % kMmaStages], (it / kMmaStages) & 1, ma.wait_ns, ma.err);
    }
  }
}

template <int BITS, int G, int GQ>
kvq_status run_mma(const ScoreArgs& a, const LaunchCtx& ctx, cudaStream_t st) {
  MmaArgs ma;
  ma.s = a;
  ma.err = ctx.err;
  ma.wait_ns = ctx.wait_ns;
  const size_t smem = static_cast<size_t>(kMmaStages) * kMmaTile * (128 * BITS / 8);
  if (!set_smem_once(reinterpret_cast<const void*>(k_score_mma<BITS, G, GQ>), smem)) return KVQ_ERR_CUDA;
  int per_sm = occupancy_once(reinterpret_cast<const void*>(k_score_mma<BITS, G, GQ>), kMmaThreads, smem);
  per_sm = per_sm > kMmaCtasPerSm ? kMmaCtasPerSm : per_sm;
  const int tpb = (a.n_tok + kMmaTile - 1) / kMmaTile;
  const long long total = static_cast<long long>(a.B) * a.H * tpb;
  if (total >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
  ma.div_tpb = FastDiv(static_cast<uint32_t>(tpb));
  ma.div_h = FastDiv(static_cast<uint32_t>(a.H));
  long long grid = static_cast<long long>(ctx.num_sms) * per_sm;
  if (grid > total) grid = total;
  ma.chunks = static_cast<int>(grid);
  ma.tiles_per_chunk = 0;
  k_score_mma<BITS, G, GQ><<<static_cast<unsigned>(grid), kMmaThreads, smem, st>>>(ma);
  return launch_status();
}

template <int BITS, int G>
kvq_status mma_by_gq(const ScoreArgs& a, int gq, const LaunchCtx& ctx, cudaStream_t st) {
  switch (gq) {
    case 1: return run_mma<BITS, G, 1>(a, ctx, st);
    case 2: return run_mma<BITS, G, 2>(a, ctx, st);
    case 4: return run_mma<BITS, G, 4>(a, ctx, st);
    case 8: return run_mma<BITS, G, 8>(a, ctx, st);
    default: return KVQ_ERR_UNSUPPORTED;
  }
}

template <int D, int BITS, int G, int GQ>
kvq_status run(const ScoreArgs& a, cudaStream_t st) {
  const dim3 grid((a.n_tok + kThreads - 1) / kThreads, a.H, a.B);
  k_score_simt<D, BITS, G, GQ><<<grid, kThreads, 0, st>>>(a);
  return launch_status();
}

template <int D, int BITS, int G>
kvq_status by_gq(const ScoreArgs& a, int gq, cudaStream_t st) {
  switch (gq) {
    case 1: return run<D, BITS, G, 1>(a, st);
    case 2: return run<D, BITS, G, 2>(a, st);
    case 4: return run<D, BITS, G, 4>(a, st);
    case 8: return run<D, BITS, G, 8>(a, st);
    default: return KVQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

kvq_status launch_score(const kvq_desc& d, const void* q, int q_heads, const kvq_packed& cache,
                        const kvq_tables& tb, int n_tokens, float scale, float* scores, cudaStream_t st,
                        const LaunchCtx& ctx) {
  ScoreArgs a{};
  a.B = d.batch;
  a.H = d.heads;
  a.Hq = q_heads;
  a.t_cap = d.t_cap;
  a.n_tok = n_tokens;
  a.n_sink = d.n_sink;
  a.rope = d.rope;
  a.rot = d.rot;
  a.scale = scale;
  a.rscale = static_cast<float>(1.0 / sqrt(static_cast<double>(d.head_dim)));
  a.q = static_cast<const __half*>(q);
  a.perm = tb.perm;
  a.rope_cs = tb.rope_cs;
  a.codes = cache.codes;
  a.sz = static_cast<const __half2*>(cache.scale_zero);
  a.sink = static_cast<const __half*>(cache.sink);
  a.scores = scores;
  const int gq = q_heads / d.heads;
  if (d.head_dim == 128 && (d.bits == 2 || d.bits == 4)) {
#define KVQ_MMA(B_, G_) \
  if (d.bits == B_ && d.group == G_) return mma_by_gq<B_, G_>(a, gq, ctx, st);
    KVQ_MMA(2, 128)
    KVQ_MMA(2, 64)
    KVQ_MMA(2, 32)
    KVQ_MMA(4, 128)
    KVQ_MMA(4, 64)
    KVQ_MMA(4, 32)
#undef KVQ_MMA
  }
#define KVQ_CASE(D_, B_, G_) \
  if (d.head_dim == D_ && d.bits == B_ && d.group == G_) return by_gq<D_, B_, G_>(a, gq, st);
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

}  // namespace kvq
