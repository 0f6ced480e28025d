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

  if (n < a.n_sink && a.rope == 2) {  // half-split pairs (c, c + D/2): chunks c and c + D/16 together
    const uint4* src = reinterpret_cast<const uint4*>(a.sink + (vh * a.n_sink + n) * D);
    const float4* cs = reinterpret_cast<const float4*>(a.rope_cs + static_cast<size_t>(n) * D);
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      float lo[8], hi[8];
      h8_to_f32(__ldg(src + c), lo);
      h8_to_f32(__ldg(src + c + D / 16), hi);
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // angles 8c + 2k, 8c + 2k + 1
        const float4 t = __ldg(cs + 4 * c + k);
        rope_fwd(lo[2 * k], hi[2 * k], t.x, t.y);
        rope_fwd(lo[2 * k + 1], hi[2 * k + 1], t.z, t.w);
      }
#pragma unroll
      for (int i = 0; i < GQ; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc[i] = __fmaf_rn(qr[i][8 * c + e], lo[e], acc[i]);
          acc[i] = __fmaf_rn(qr[i][D / 2 + 8 * c + e], hi[e], acc[i]);
        }
    }
  } else if (n < a.n_sink) {
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
// i.e. below 2e-5 of the score's L1 magnitude.
// A CTA owns a contiguous range of 64-token blocks of one (batch, KV head):
// it rotates and splits the queries once, then its 8 warps work independently
// (no CTA barrier in the loop), each streaming every 8th block through its
// own ring of kMmaStages stages: the records by one bulk copy (one mbarrier
// per stage), the scale/zero words by 4-byte cp.async spread over the lanes.
// A block is four m-tiles of 16 tokens.
constexpr int kMmaThreads = 256;
constexpr int kMmaWarps = kMmaThreads / 32;
constexpr int kMmaStages = 2;     // blocks in flight per warp (2 beat 3 and 4: less shared memory, 4 CTAs per SM)
constexpr int kMmaCtasPerSm = 4;
constexpr int kMmaBlk = 64;       // tokens per block

struct MmaArgs {
  ScoreArgs s;
  int splits;  // CTAs per (batch, KV head)
  int n_blk;   // 64-token blocks per (batch, KV head)
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

template <int BITS, int G>
__host__ __device__ constexpr int mma_stage_bytes() {
  return kMmaBlk * (128 * BITS / 8) + kMmaBlk * (128 / G) * 4;  // records + scale/zero words of a block
}

template <int BITS, int G, int GQ>
__global__ void __launch_bounds__(kMmaThreads) k_score_mma(const MmaArgs ma) {
  constexpr int D = 128;
  constexpr int RB = D * BITS / 8;
  constexpr int NW = RB / 4;             // words per record
  constexpr int NTN = (2 * GQ + 7) / 8;  // n-tiles of 8 columns
  constexpr int NGK = D / G;             // quantization groups per record
  constexpr int CB = kMmaBlk * RB;       // records of one block
  constexpr int NSZ = kMmaBlk * NGK;     // scale/zero words of one block
  constexpr int STB = mma_stage_bytes<BITS, G>();
  const ScoreArgs& a = ma.s;
  extern __shared__ __align__(128) uint8_t ring[];  // [warp][stage][STB]
  __shared__ __align__(16) uint2 bfrag[NTN][4][4][8];
  __shared__ __align__(16) float qraw[GQ][D];
  __shared__ int8_t qd[GQ][2][D];
  __shared__ float qsum[GQ][NGK];
  __shared__ float sqh[GQ];
  __shared__ __align__(8) uint64_t full[kMmaWarps][kMmaStages];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int bh = static_cast<int>(blockIdx.x) / ma.splits, part = static_cast<int>(blockIdx.x) % ma.splits;
  const int b = bh / a.H, h = bh - b * a.H;
  const int blk0 = static_cast<int>(static_cast<long long>(ma.n_blk) * part / ma.splits);
  const int blk1 = static_cast<int>(static_cast<long long>(ma.n_blk) * (part + 1) / ma.splits);
  const int n_my = blk1 - blk0 > warp ? (blk1 - blk0 - warp + kMmaWarps - 1) / kMmaWarps : 0;  // this warp's blocks
  uint8_t* const wring = ring + warp * (kMmaStages * STB);
  const size_t rec0 = static_cast<size_t>(bh) * a.t_cap;  // slot of token 0 of this stream

  // this warp's i-th block -> stage i % kMmaStages (records by bulk copy, words by cp.async)
  auto issue = [&](int i) {
    uint8_t* dst = wring + (i % kMmaStages) * STB;
    const int n0 = (blk0 + warp + i * kMmaWarps) * kMmaBlk;
    const int nv = i < n_my ? min(kMmaBlk, a.n_tok - n0) : 0;
    if (nv > 0 && lane == 0) {
      fence_async_smem();
      mbar_arrive_expect_tx(&full[warp][i % kMmaStages], static_cast<uint32_t>(nv * RB));
      bulk_load(dst, a.codes + (rec0 + n0) * RB, static_cast<uint32_t>(nv * RB), &full[warp][i % kMmaStages]);
    }
#pragma unroll
    for (int e = lane; e < NSZ; e += 32) {
      const bool live = e / NGK < nv;
      cp_async4(smem_u32(dst + CB + e * 4), live ? static_cast<const void*>(a.sz + (rec0 + n0) * NGK + e) : a.sz,
                live ? 4u : 0u);
    }
    cp_async_commit();
  };
  if (lane == 0) {
    for (int i = 0; i < kMmaStages; ++i) mbar_init(&full[warp][i], 1);
    fence_mbar_init();
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < kMmaStages; ++i) issue(i);

  // rotated, digit-split queries of this (batch, KV head); warp w < GQ handles query head w
  if (warp < GQ) {
    const int qh = h * GQ + warp;
    query_digits<G>(a.q + (static_cast<size_t>(b) * a.Hq + qh) * D, a.perm ? a.perm + static_cast<size_t>(h) * D : nullptr,
                    a.rot, a.rscale, lane, qraw[warp], qd[warp][0], qd[warp][1], qsum[warp], &sqh[warp]);
  }
  __syncthreads();
  build_score_bfrag<BITS, GQ, NTN>(bfrag, qd, tid, kMmaThreads);  // column c = 2 * head + digit
  __syncthreads();
  // fp16 sinks: s = scale * q . RoPE_n(sink_n), by the CTA that owns the stream's first block
  if (part == 0) {
    for (int e = warp; e < min(a.n_sink, a.n_tok) * GQ; e += kMmaWarps) {
      const int n = e / GQ, hh = e % GQ;
      const float acc = sink_dot(qraw[hh], a.sink + (static_cast<size_t>(bh) * a.n_sink + n) * D,
                                 a.rope ? a.rope_cs + static_cast<size_t>(n) * D : nullptr, lane, a.rope == 2);
      if (lane == 0) a.scores[(static_cast<size_t>(b) * a.Hq + h * GQ + hh) * a.n_tok + n] = acc * a.scale;
    }
  }
  uint2 bq[4][NTN];  // this lane's B fragments, kept in registers
#pragma unroll
  for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
    for (int s = 0; s < 4; ++s) bq[s][nt] = bfrag[nt][s][tig][g];
  float sqv[NTN], qsv[NTN][NGK];  // sq and the group sums of this lane's query head per n-tile
#pragma unroll
  for (int nt = 0; nt < NTN; ++nt) {
    const int hh = min(nt * 4 + tig, GQ - 1);
    sqv[nt] = sqh[hh];
#pragma unroll
    for (int q = 0; q < NGK; ++q) qsv[nt][q] = qsum[hh][q];
  }
  float* const out_h = a.scores + (static_cast<size_t>(b) * a.Hq + h * GQ) * a.n_tok;  // query head h*GQ

  int i_fail = -1;
  for (int i = 0; i < n_my; ++i) {
    const int st = i % kMmaStages;
    const bool ok = mbar_wait(&full[warp][st], (i / kMmaStages) & 1, ma.wait_ns, ma.err);
    if (!__all_sync(0xffffffffu, ok)) {
      i_fail = i;
      break;
    }
    cp_async_wait_group<kMmaStages - 1>();
    __syncwarp();  // the stage's records and words are visible to the whole warp
    const uint8_t* sb = wring + st * STB;
    const int n0 = (blk0 + warp + i * kMmaWarps) * kMmaBlk;
    const int nv = min(kMmaBlk, a.n_tok - n0);
#pragma unroll
    for (int mt = 0; mt < kMmaBlk / 16; ++mt) {
      if (mt * 16 >= nv) break;
      const int ra = mt * 16 + g;  // block rows ra and ra + 8
      uint32_t wa[NW], wb[NW];
#pragma unroll
      for (int k = 0; k < NW / 4; ++k) {
        const uint4 ua = *reinterpret_cast<const uint4*>(sb + ra * RB + 16 * k);
        const uint4 ub = *reinterpret_cast<const uint4*>(sb + (ra + 8) * RB + 16 * k);
        wa[4 * k] = ua.x; wa[4 * k + 1] = ua.y; wa[4 * k + 2] = ua.z; wa[4 * k + 3] = ua.w;
        wb[4 * k] = ub.x; wb[4 * k + 1] = ub.y; wb[4 * k + 2] = ub.z; wb[4 * k + 3] = ub.w;
      }
      float2 sza[NGK], szb[NGK];  // (S, Z) of rows ra and ra + 8
#pragma unroll
      for (int q = 0; q < NGK; ++q) {
        sza[q] = __half22float2(*reinterpret_cast<const __half2*>(sb + CB + (ra * NGK + q) * 4));
        szb[q] = __half22float2(*reinterpret_cast<const __half2*>(sb + CB + ((ra + 8) * NGK + q) * 4));
      }
      int acc[NGK][NTN][4];
#pragma unroll
      for (int q = 0; q < NGK; ++q)
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q][nt][e] = 0;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t a0, a1, a2, a3;
        score_afrag<BITS, NW>(wa, wb, s, tig, a0, a1, a2, a3);
        constexpr int SPG = G / 32;  // k-steps per group
        const int q = s / SPG;
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt) mma_u8s8(acc[q][nt], a0, a1, a2, a3, bq[s][nt]);
      }
      // epilogue: lane holds columns 2 tig (lo) and 2 tig + 1 (hi) = query head nt*4 + tig
      const int na = n0 + ra, nb = na + 8;
      const bool full_tile = n0 + mt * 16 >= a.n_sink && n0 + mt * 16 + 16 <= a.n_tok;
#pragma unroll
      for (int nt = 0; nt < NTN; ++nt) {
        const int hh = nt * 4 + tig;
        if (hh >= GQ) continue;
        float sa = 0.0f, sbv = 0.0f;
#pragma unroll
        for (int q = 0; q < NGK; ++q) {
          const float da = static_cast<float>(acc[q][nt][0] + 256 * acc[q][nt][1]);
          const float db = static_cast<float>(acc[q][nt][2] + 256 * acc[q][nt][3]);
          sa = __fmaf_rn(sza[q].x * sqv[nt], da, __fmaf_rn(sza[q].y, qsv[nt][q], sa));
          sbv = __fmaf_rn(szb[q].x * sqv[nt], db, __fmaf_rn(szb[q].y, qsv[nt][q], sbv));
        }
        float* out = out_h + static_cast<size_t>(hh) * a.n_tok;
        sa = sa * a.scale;
        sbv = sbv * a.scale;
        if (full_tile) {
          out[na] = sa;
          out[nb] = sbv;
        } else {
          if (na < a.n_tok && na >= a.n_sink) out[na] = sa;
          if (nb < a.n_tok && nb >= a.n_sink) out[nb] = sbv;
        }
      }
    }
    __syncwarp();  // every lane has read the stage: refill it with the block kMmaStages ahead
    issue(i + kMmaStages);
  }
  // After a timed-out wait, let this warp's copies still in flight land
  // (bounded) before the CTA exits: blocks i_fail .. i_fail + kMmaStages - 1
  // were issued and not consumed; each is waited on once, at its stage and phase.
  if (i_fail >= 0 && lane == 0) {
    for (int i = i_fail; i < n_my && i < i_fail + kMmaStages; ++i)
      mbar_wait(&full[warp][i % kMmaStages], (i / kMmaStages) & 1, ma.wait_ns, ma.err);
  }
  cp_async_wait_all();
}

template <int BITS, int G, int GQ>
kvq_status run_mma(const ScoreArgs& a, const LaunchCtx& ctx, cudaStream_t st) {
  MmaArgs ma;
  ma.s = a;
  ma.err = ctx.err;
  ma.wait_ns = ctx.wait_ns;
  const size_t smem = static_cast<size_t>(kMmaWarps) * kMmaStages * mma_stage_bytes<BITS, G>();
  const void* fn = reinterpret_cast<const void*>(k_score_mma<BITS, G, GQ>);
  if (!set_smem_once(fn, smem)) return KVQ_ERR_CUDA;
  int per_sm = occupancy_once(fn, kMmaThreads, smem);
  per_sm = per_sm > kMmaCtasPerSm ? kMmaCtasPerSm : per_sm;
  ma.n_blk = (a.n_tok + kMmaBlk - 1) / kMmaBlk;
  const long long streams = static_cast<long long>(a.B) * a.H;
  // as many CTAs per stream as one wave holds (rounded down: a partial second
  // wave would double the tail); each of a stream's CTAs takes at least one block per warp
  long long splits = static_cast<long long>(ctx.num_sms) * per_sm / streams;
  const long long max_splits = (ma.n_blk + kMmaWarps - 1) / kMmaWarps;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  if (streams * splits >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
  ma.splits = static_cast<int>(splits);
  k_score_mma<BITS, G, GQ><<<static_cast<unsigned>(streams * splits), kMmaThreads, smem, st>>>(ma);
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
