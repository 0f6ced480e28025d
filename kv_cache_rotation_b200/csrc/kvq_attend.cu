// Decode-step attention over the compressed cache ("EliteKV - RoPE频率选择与低秩投影"
// §2.2: the score of query m and cached key n is q_m^rot . k_n^rot / sqrt(d);
// §7.1: the softmax of the scaled scores over the cached tokens weights the
// values):
//   out[b][qh] = sum_n p_n vhat_n,   p = softmax_n(s_n),  s = the kvq_score scores.
// The value decode is linear in the dequantized codes y_n = S_g c_n + Z_g, so
//   sum_n p_n vhat_n = P^T H_norm (sum_n p_n y_n)  (+ the sink rows, verbatim):
// the inverse rotation runs once per output instead of once per token.
//
// Three launches on the caller's stream: the scores (kvq_score's kernel) into
// the workspace; k_attend_part, one CTA per (chunk of 512 tokens, batch, KV
// head), walks the chunk in sub-chunks of 128 with a running (online) softmax
// and writes the chunk's statistics (max m, sum l) and sum_n e^(s_n - m) y_n
// per query head of the group; k_attend_combine, one CTA
// per (batch, query head), merges the chunks (log-sum-exp), applies the
// inverse rotation and permutation and adds the sink rows.
#include <math.h>

#include <mutex>
#include <type_traits>

#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_qdigits.cuh"

namespace kvq {
namespace {

constexpr int D = 128;
constexpr int kCh = 128;       // tokens per sub-chunk (one per thread in the score pass)
constexpr int kSub = 4;        // sub-chunks per chunk: a chunk is 512 tokens (measured faster than 1024, equal to 256)
constexpr int kThreads = 128;  // part: one token each, then 32 channel quads x 4 token phases;
                               // combine: one thread per channel

struct AttnArgs {
  int B, H, Hq, GQ, t_cap, n_tok, n_chunks, n_sink, rot;
  const int32_t* list;  // sink positions [B][n_sink] (-1 unused), or nullptr: the positions < n_sink
  float rscale;  // fp32(1/sqrt(D))
  const float* scores;  // [B][Hq][n_tok]
  const uint8_t* vcodes;
  const __half2* vsz;
  const __half* vsink;
  const int16_t* vperm;
  float* part_acc;  // [B*Hq][n_chunks][D]
  float* part_ml;   // [B*Hq][n_chunks][2]
  float* out;       // [B][Hq][D]
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int BITS, int G, int GQ>
__global__ void __launch_bounds__(kThreads) k_attend_part(const AttnArgs a) {
  constexpr int NG = D / G;
  constexpr int RB = D * BITS / 8;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  __shared__ __align__(16) float wsm[kCh][NG][GQ];  // p_n * S_ng of the sub-chunk
  __shared__ __align__(16) uint32_t csm[2][kCh][RB / 4];  // value records: this sub-chunk's and the next one's
  __shared__ float red[4][GQ * (1 + NG)];
  __shared__ float mx_s[4][GQ];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  // accumulation role: thread (quad, phase) takes channels 4q..4q+3 of tokens n = phase mod 4
  const int q = tid >> 2, ph = tid & 3;
  const int g = (4 * q) / G;
  const int bit = 4 * q * BITS, wi = bit >> 5, sh = bit & 31;

  // running (online-softmax) state over the chunk's sub-chunks
  float m_run[GQ], l_run[GQ], z_run[GQ], acc[GQ][4];
#pragma unroll
  for (int r = 0; r < GQ; ++r) {
    m_run[r] = -INFINITY;
    l_run[r] = 0.0f;
    z_run[r] = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[r][e] = 0.0f;
  }

  // one sub-chunk ahead: its value records by cp.async into the other csm
  // buffer (zero past the last token), this thread's token's scores and
  // scale / zero words into registers
  float sv_n[GQ];
  float2 sz_n[NG];
  auto prefetch = [&](int sub) {
    const int n0 = (c * kSub + sub) * kCh;
    const int nn = min(kCh, a.n_tok - n0);
    const uint8_t* vsrc = a.vcodes + (static_cast<size_t>(bh) * a.t_cap + n0) * RB;
    const uint32_t dst = smem_u32(&csm[sub & 1][0][0]);
    for (int i = tid; i < kCh * RB / 16; i += kThreads) {
      const bool live = i / (RB / 16) < nn;
      cp_async16(dst + 16 * i, live ? vsrc + 16 * i : vsrc, live ? 16u : 0u);
    }
#pragma unroll
    for (int r = 0; r < GQ; ++r)
      sv_n[r] = tid < nn ? __ldg(a.scores + (static_cast<size_t>(b) * a.Hq + h * GQ + r) * a.n_tok + n0 + tid)
                         : -INFINITY;
#pragma unroll
    for (int gg = 0; gg < NG; ++gg)
      sz_n[gg] = tid < nn ? __half22float2(a.vsz[(static_cast<size_t>(bh) * a.t_cap + n0 + tid) * NG + gg])
                          : make_float2(0.0f, 0.0f);
  };
  if (c * kSub * kCh < a.n_tok) prefetch(0);
  cp_async_commit();

  for (int sub = 0; sub < kSub; ++sub) {
    const int n0 = (c * kSub + sub) * kCh;
    if (n0 >= a.n_tok) break;  // uniform over the CTA
    const int nn = min(kCh, a.n_tok - n0);
    float sv[GQ];
    float2 sz[NG];
#pragma unroll
    for (int r = 0; r < GQ; ++r) sv[r] = sv_n[r];
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) sz[gg] = sz_n[gg];
    __syncthreads();  // the previous sub-chunk's csm / wsm / red readers are done
    if (sub + 1 < kSub && n0 + kCh < a.n_tok) prefetch(sub + 1);
    cp_async_commit();  // one group per sub-chunk (empty at the end)
    const uint32_t(*cs)[RB / 4] = csm[sub & 1];

    // scores (thread = token), the sub-chunk max per query head
#pragma unroll
    for (int r = 0; r < GQ; ++r) {
      const float v = warp_max(sv[r]);
      if (lane == 0) mx_s[warp][r] = v;
    }
    __syncthreads();
    float m_new[GQ], f_old[GQ];
#pragma unroll
    for (int r = 0; r < GQ; ++r) {
      m_new[r] = fmaxf(m_run[r], fmaxf(fmaxf(mx_s[0][r], mx_s[1][r]), fmaxf(mx_s[2][r], mx_s[3][r])));
      f_old[r] = __expf(m_run[r] - m_new[r]);  // 0 on the first sub-chunk
    }
    // p_n = e^(s_n - m); w_n = p_n S_g; sub-chunk sums of p_n and p_n Z_g
    {
#pragma unroll
      for (int r = 0; r < GQ; ++r) {
        const float p = tid < nn ? __expf(sv[r] - m_new[r]) : 0.0f;
        const float l = warp_sum(p);
        if (lane == 0) red[warp][r] = l;
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) {
          wsm[tid][gg][r] = p * sz[gg].x;
          const float z = warp_sum(p * sz[gg].y);
          if (lane == 0) red[warp][GQ + r * NG + gg] = z;
        }
      }
    }
    cp_async_wait_group<1>();  // this sub-chunk's records (the next one's may still be in flight)
    __syncthreads();
#pragma unroll
    for (int r = 0; r < GQ; ++r) {
      const int zi = GQ + r * NG + g;
      l_run[r] = fmaf(l_run[r], f_old[r], red[0][r] + red[1][r] + red[2][r] + red[3][r]);
      z_run[r] = fmaf(z_run[r], f_old[r], red[0][zi] + red[1][zi] + red[2][zi] + red[3][zi]);
      m_run[r] = m_new[r];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][e] *= f_old[r];
    }
    // sum_n w_n c_n for this thread's channels and token phase
    for (int n = ph; n < nn; n += 4) {
      uint32_t v = cs[n][wi] >> sh;
      if constexpr ((4 * BITS) % 8 != 0 || 32 % (4 * BITS) != 0) {
        if (sh + 4 * BITS > 32) v |= cs[n][wi + 1] << (32 - sh);
      }
      float cf[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) cf[e] = __uint_as_float(0x4B000000u | ((v >> (BITS * e)) & MASK)) - 8388608.0f;
      float w[GQ];
#pragma unroll
      for (int r = 0; r < GQ; ++r) w[r] = wsm[n][g][r];
#pragma unroll
      for (int r = 0; r < GQ; ++r)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][e] = fmaf(w[r], cf[e], acc[r][e]);
    }
  }
  // the four token phases of a quad sit in adjacent lanes
#pragma unroll
  for (int r = 0; r < GQ; ++r)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[r][e] += __shfl_xor_sync(0xffffffffu, acc[r][e], 1);
      acc[r][e] += __shfl_xor_sync(0xffffffffu, acc[r][e], 2);
    }
  // add sum_n p_n Z_g; write the chunk's partials
  const size_t pc = static_cast<size_t>(a.n_chunks);
#pragma unroll
  for (int r = 0; r < GQ; ++r) {
    const size_t row = (static_cast<size_t>(b) * a.Hq + h * GQ + r) * pc + c;
    if (ph == 0)
      *reinterpret_cast<float4*>(a.part_acc + row * D + 4 * q) =
          make_float4(acc[r][0] + z_run[r], acc[r][1] + z_run[r], acc[r][2] + z_run[r], acc[r][3] + z_run[r]);
    if (tid == 0) {
      a.part_ml[row * 2] = m_run[r];
      a.part_ml[row * 2 + 1] = l_run[r];
    }
  }
}

__global__ void __launch_bounds__(kThreads) k_attend_combine(const AttnArgs a) {
  __shared__ float ys[2][D];
  __shared__ float nat[D];
  const int j = threadIdx.x;
  const int bq = blockIdx.x;  // b * Hq + qh
  const int b = bq / a.Hq, qh = bq % a.Hq, h = qh / a.GQ;
  const float* ml = a.part_ml + static_cast<size_t>(bq) * a.n_chunks * 2;
  const float* pa = a.part_acc + static_cast<size_t>(bq) * a.n_chunks * D;
  float M = -INFINITY;
  for (int c = 0; c < a.n_chunks; ++c) M = fmaxf(M, ml[2 * c]);
  float L = 0.0f, acc = 0.0f;
  for (int c = 0; c < a.n_chunks; ++c) {
    const float f = __expf(ml[2 * c] - M);
    L = fmaf(ml[2 * c + 1], f, L);
    acc = fmaf(pa[static_cast<size_t>(c) * D + j], f, acc);
  }
  const float invL = 1.0f / L;
  float y = acc * invL;  // sum_n p_n y_n, channel j of the rotated basis
  if (a.rot == KVQ_ROT_FWHT_HEAD) {  // x = H y / sqrt(D), Sylvester order, strides 1 .. 64
    int cur = 0;
    ys[0][j] = y;
    __syncthreads();
#pragma unroll
    for (int st = 1; st < D; st <<= 1) {
      const float u = ys[cur][j], w = ys[cur][j ^ st];
      ys[cur ^ 1][j] = (j & st) ? w - u : u + w;
      cur ^= 1;
      __syncthreads();
    }
    y = ys[cur][j] * a.rscale;
  }
  // inverse permutation: x[perm[j]] = y_j
  nat[a.vperm ? a.vperm[static_cast<size_t>(h) * D + j] & (D - 1) : j] = y;
  __syncthreads();
  float o = nat[j];
  // sink rows, verbatim values weighted by their softmax probability (their
  // scores are in the score array and their weights in L; their codes decode to 0)
  const int ns = a.list ? a.n_sink : min(a.n_sink, a.n_tok);
  const float* sv = a.scores + static_cast<size_t>(bq) * a.n_tok;
  for (int n = 0; n < ns; ++n) {
    const int m = a.list ? a.list[static_cast<size_t>(b) * a.n_sink + n] : n;
    if (m < 0 || m >= a.n_tok) continue;
    const float p = __expf(sv[m] - M) * invL;
    o = fmaf(p, __half2float(a.vsink[((static_cast<size_t>(b) * a.H + h) * a.n_sink + n) * D + j]), o);
  }
  a.out[static_cast<size_t>(bq) * D + j] = o;
}

template <int BITS, int G>
kvq_status run_part(const AttnArgs& a, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(a.n_chunks), static_cast<unsigned>(a.B * a.H));
  switch (a.GQ) {
    case 1: k_attend_part<BITS, G, 1><<<grid, kThreads, 0, st>>>(a); break;
    case 2: k_attend_part<BITS, G, 2><<<grid, kThreads, 0, st>>>(a); break;
    case 4: k_attend_part<BITS, G, 4><<<grid, kThreads, 0, st>>>(a); break;
    case 8: k_attend_part<BITS, G, 8><<<grid, kThreads, 0, st>>>(a); break;
    default: return KVQ_ERR_UNSUPPORTED;
  }
  return launch_status();
}

kvq_status dispatch_part(int bits, int group, const AttnArgs& a, cudaStream_t st) {
#define KVQ_CASE(B_, G_) \
  if (bits == B_ && group == G_) return run_part<B_, G_>(a, st);
  KVQ_CASE(2, 128) KVQ_CASE(2, 64) KVQ_CASE(2, 32)
  KVQ_CASE(3, 128) KVQ_CASE(3, 64) KVQ_CASE(3, 32)
  KVQ_CASE(4, 128) KVQ_CASE(4, 64) KVQ_CASE(4, 32)
#undef KVQ_CASE
  return KVQ_ERR_UNSUPPORTED;
}

size_t align256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// ---------------------------------------------------------------------------
// Fused path (head_dim 128, one quantization group per record, 2- or 4-bit
// codes): one pass over the K and V records of a chunk of tokens forms the
// scores, the running softmax statistics and sum_n p_n y_n, all products on
// the tensor cores; a small merge kernel then combines the chunks.
//
// Work split: CTA = (chunk of 16-token blocks, batch x KV head); its 8 warps
// take the chunk's blocks in turn and each streams its own blocks through a
// private ring of shared-memory stages filled by cp.async (no CTA barrier in
// the loop); the warps' running sums are merged once at the end.
//
// Scores: exactly the score kernel's arithmetic (u8 codes x s8 query digits,
// mma.sync m16n8k32, same fp32 epilogue), so they match kvq_score bit for bit.
//
// Values: out_rot = sum_n p_n (S_n c_n + Z_n) = sum_n w_n c_n + sum_n p_n Z_n
// with w_n = p_n S_n. sum_n w_n c_n runs on mma.sync m16n8k16 (fp16 in, fp32
// accumulate) with A = codes (channels x tokens) and B = weights (tokens x
// columns). Each weight is carried as two fp16 terms w = hi + lo (hi =
// fp16(w), lo = fp16(w - hi)), one column each, so the product keeps about 22
// bits of w; with N = 8 columns a group of four query heads fills one n-tile.
//
// Range: the running reference m tracks the largest key lambda_n = s_n log2(e)
// + log2(S_n) (S_n clamped to >= 2^-30), and p'_n = 2^(s_n log2(e) - m), so
// w'_n = p'_n S_n <= 2^8 (m is raised, and the sums rescaled, only when a key
// exceeds it by more than 2^8); p'_n and every sum stay in fp32 range. The
// partial of a chunk is (m, l = sum p'_n, sum_n p'_n y_n) in the log2 domain.
//
// A operand without a shift per m-tile: a lane's rows g and g + 8 of m-tile t
// are two channels whose codes sit at the same bit offset in the low and high
// 16-bit halves of one record word, and the two tokens of a register are
// paired by one byte permute per word pair. The code is masked in place:
// (y & (3 << 2t)) | 0x6400 is the fp16 1024 + c 4^t, minus 1024 exactly c 4^t
// (kept below 1024 by taking t >= 5 from y >> 10); 4^-t is applied once to the
// accumulators. (Leaving the masked field as an fp16 subnormal, c 4^t 2^-24,
// would save the subtraction, but its products with subnormal lo halves of
// small weights lost precision on the tensor cores.)
// Resident CTAs per SM the register budget of the fused kernel is sized for
// (GQ <= 4): 2 (<= 128 registers) measured faster than 3 (<= 80).
constexpr int kFMinBlocks = 2;
constexpr int kFWarps = 8;
constexpr int kFThreads = 32 * kFWarps;
constexpr int kFBlock = 16;           // tokens per warp step (one m16 tile of the score MMA)
constexpr int kFMaxChunks = 256;
constexpr int kFMaxSinks = 1024;      // merge keeps the sink scores in shared memory
constexpr float kFLazy = 8.0f;        // log2 headroom before the reference is raised
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kMinS = 9.3132257e-10f;  // 2^-30: floor of S in the reference key

template <int BITS>
struct FusedCfg {
  static constexpr int RB = 128 * BITS / 8;
  static constexpr int STAGES = BITS == 2 ? 6 : 4;                    // per warp
  static constexpr int STAGE = 2 * kFBlock * RB + 2 * kFBlock * 4;    // K codes, V codes, K sz, V sz
  static constexpr int SMEM = kFWarps * STAGES * STAGE;
};

struct FusedArgs {
  int B, H, Hq, t_cap, n_tok, n_sink, rot, blocks, blocks_per_chunk, n_chunks;
  const int32_t* list;  // listed sinks [B][n_list] (n_sink is then 0), or nullptr
  int n_list;           // <= 32: lane k holds entry k
  float scale, rscale;
  const __half* q;
  const int16_t* kperm;
  const uint8_t* kcodes;
  const uint32_t* ksz;  // (S, Z) fp16 pair per token
  const uint8_t* vcodes;
  const uint32_t* vsz;
  float* part_acc;  // [B*Hq][n_chunks][D]
  float* part_ml;   // [B*Hq][n_chunks][2]: (m, l), log2 domain
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// w as the fp16 pair (hi, lo) = (fp16(w), fp16(w - hi)): hi in the low half.
__device__ __forceinline__ uint32_t split_hi_lo(float w) {
  const __half hi = __float2half_rn(w);
  const __half lo = __float2half_rn(w - __half2float(hi));
  return static_cast<uint32_t>(__half_as_ushort(hi)) | (static_cast<uint32_t>(__half_as_ushort(lo)) << 16);
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ((y & msk) | 0x6400 per half) as fp16 pairs, minus 1024: the masked code values.
__device__ __forceinline__ uint32_t code_pair(uint32_t y, uint32_t msk) {
  const uint32_t x = (y & msk) | 0x64006400u;
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&x),
                            __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

__device__ __forceinline__ float2 h2f(uint32_t w) { return __half22float2(*reinterpret_cast<const __half2*>(&w)); }

// LIST: the sinks are a list (a.list), masked block by block; without it the
// kernel has no per-block list test at all.
template <int BITS, int GQ, bool LIST>
__global__ void __launch_bounds__(kFThreads, GQ <= 4 ? kFMinBlocks : 1) k_attend_fused(const FusedArgs a) {
  using C = FusedCfg<BITS>;
  constexpr int D = 128;
  constexpr int RB = C::RB;
  constexpr int NW = RB / 4;
  constexpr int NTN = (2 * GQ + 7) / 8;
  constexpr int S = C::STAGES;
  constexpr int CPL = kFBlock * RB / (32 * 16);  // 16-byte code copies per lane and tensor
  constexpr bool ALLQ = GQ % 4 == 0;             // every lane's query head exists
  extern __shared__ __align__(128) uint8_t fdyn[];  // per warp: S stages of {K codes, V codes, K sz, V sz}
  __shared__ __align__(16) uint2 bfrag[NTN][4][4][8];
  __shared__ __align__(16) float qraw[GQ][D];
  __shared__ int8_t qd[GQ][2][D];
  __shared__ float qsum[GQ][1];
  __shared__ float sqh[GQ];
  __shared__ float mw[kFWarps][GQ], lw[kFWarps][GQ], zw[kFWarps][GQ];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int c = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh - b * a.H;
  const int k_begin = c * a.blocks_per_chunk;
  const int nk = min(a.blocks_per_chunk, a.blocks - k_begin);
  const int my_n = nk > warp ? (nk - warp + kFWarps - 1) / kFWarps : 0;  // blocks k_begin + warp + 8 i
  const size_t rec0 = static_cast<size_t>(bh) * a.t_cap;
  const uint32_t wbase = smem_u32(fdyn) + warp * (S * C::STAGE);
  // listed sinks: lane k holds position k of this sequence's list (INT_MAX for none)
  int my_list = 0x7fffffff;
  if (LIST && lane < a.n_list) {
    const int m = __ldg(a.list + static_cast<size_t>(b) * a.n_list + lane);
    my_list = m >= 0 ? m : 0x7fffffff;
  }
  // The merge kernel may launch once every CTA of this grid has started (all are resident by then, so its
  // CTAs never hold slots this grid still needs); it runs its input-only prologue beside this grid and
  // waits for this grid's completion before reading any partial.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // block i of this warp into stage st: codes 16 bytes per lane, scale / zero 4 bytes (zero past n_tok)
  // per-lane sources of this warp's first block; consecutive blocks of a warp are kFWarps blocks apart
  constexpr size_t kStep = static_cast<size_t>(kFWarps) * kFBlock;  // records between a warp's blocks
  const int n_first = (k_begin + warp) * kFBlock;
  const size_t rec_first = rec0 + n_first;
  const uint8_t* kc_src = a.kcodes + rec_first * RB + 16 * lane;
  const uint8_t* vc_src = a.vcodes + rec_first * RB + 16 * lane;
  const uint32_t* sz_src = (lane < kFBlock ? a.ksz : a.vsz) + rec_first + (lane & (kFBlock - 1));
  const uint32_t sz_dst = 2 * kFBlock * RB + 4 * lane;
  auto issue = [&](int i, int st) {
    const int n0 = n_first + i * static_cast<int>(kStep);
    const size_t roff = static_cast<size_t>(i) * kStep;
    const uint32_t sb = wbase + st * C::STAGE;
    if (n0 + kFBlock <= a.n_tok) {  // the whole block exists (uniform over the warp)
#pragma unroll
      for (int r = 0; r < CPL; ++r) {
        cp_async16(sb + 512 * r + 16 * lane, kc_src + roff * RB + 512 * r, 16u);
        cp_async16(sb + kFBlock * RB + 512 * r + 16 * lane, vc_src + roff * RB + 512 * r, 16u);
      }
      cp_async4(sb + sz_dst, sz_src + roff, 4u);
    } else {  // last block: zero past n_tok, sources kept inside the cache
#pragma unroll
      for (int r = 0; r < CPL; ++r) {
        const int off = 16 * (lane + 32 * r);
        const bool live = n0 + off / RB < a.n_tok;
        const size_t src = (rec0 + n0) * RB + (live ? off : 0);
        cp_async16(sb + off, a.kcodes + src, live ? 16u : 0u);
        cp_async16(sb + kFBlock * RB + off, a.vcodes + src, live ? 16u : 0u);
      }
      const int tok = lane & (kFBlock - 1);
      const bool live = n0 + tok < a.n_tok;
      cp_async4(sb + sz_dst, (lane < kFBlock ? a.ksz : a.vsz) + rec0 + n0 + (live ? tok : 0), live ? 4u : 0u);
    }
  };
#pragma unroll
  for (int i = 0; i < S; ++i) {
    if (i < my_n) issue(i, i);
    cp_async_commit();
  }

  // the GQ query heads of this KV head, rotated and split into int8 digits
  if (warp < GQ)
    query_digits<128>(a.q + (static_cast<size_t>(b) * a.Hq + h * GQ + warp) * D,
                      a.kperm ? a.kperm + static_cast<size_t>(h) * D : nullptr, a.rot, a.rscale, lane, qraw[warp],
                      qd[warp][0], qd[warp][1], qsum[warp], &sqh[warp]);
  __syncthreads();
  build_score_bfrag<BITS, GQ, NTN>(bfrag, qd, tid, kFThreads);
  __syncthreads();
  uint2 bq[4][NTN];
  float sq[NTN], qs[NTN];
#pragma unroll
  for (int nt = 0; nt < NTN; ++nt) {
    const int qh = 4 * nt + tig;
#pragma unroll
    for (int s = 0; s < 4; ++s) bq[s][nt] = bfrag[nt][s][tig][g];
    sq[nt] = qh < GQ ? sqh[qh] : 0.0f;
    qs[nt] = qh < GQ ? qsum[qh][0] : 0.0f;
  }

  float acc[8][NTN][4];
  float m_run[NTN], l_run[NTN], z_run[NTN];
#pragma unroll
  for (int nt = 0; nt < NTN; ++nt) {
    m_run[nt] = -INFINITY;
    l_run[nt] = 0.0f;
    z_run[nt] = 0.0f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.0f;
  }
  // value B fragments come from the score lanes of rows 2 tig (+8) and 2 tig + 1 (+9)
  const int srcA = 8 * tig + (g >> 1), srcB = srcA + 4;
  const uint32_t sel = (g & 1) ? 0x7632u : 0x5410u;  // column g: digit hi (low halves) or lo

  // one 16-token block; INTERIOR: no sink and no position past n_tok in it;
  // lbits: the block's listed positions (bit t: position n0 + t)
  // shared-memory reads as plain loads, so the compiler may schedule them around the products
  auto ld4 = [](const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); };
  auto block = [&](auto interior, int n0, const uint8_t* kcb, uint32_t lbits) {
    constexpr bool INTERIOR = decltype(interior)::value;
    const uint8_t* vcb = kcb + kFBlock * RB;
    const uint8_t* kzb = vcb + kFBlock * RB;
    const uint8_t* vzb = kzb + 4 * kFBlock;
    // ---- scores of rows g and g + 8
    uint32_t wa[NW], wb[NW];
#pragma unroll
    for (int k = 0; k < NW / 4; ++k) {
      const uint4 ua = *reinterpret_cast<const uint4*>(kcb + g * RB + 16 * k);
      const uint4 ub = *reinterpret_cast<const uint4*>(kcb + (g + 8) * RB + 16 * k);
      wa[4 * k] = ua.x; wa[4 * k + 1] = ua.y; wa[4 * k + 2] = ua.z; wa[4 * k + 3] = ua.w;
      wb[4 * k] = ub.x; wb[4 * k + 1] = ub.y; wb[4 * k + 2] = ub.z; wb[4 * k + 3] = ub.w;
    }
    int sacc[NTN][4], sacc2[NTN][4];  // k-steps 0, 2 and 1, 3: two independent product chains
#pragma unroll
    for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = sacc2[nt][e] = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      uint32_t a0, a1, a2, a3;
      score_afrag<BITS, NW>(wa, wb, s, tig, a0, a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NTN; ++nt) mma_u8s8((s & 1) ? sacc2[nt] : sacc[nt], a0, a1, a2, a3, bq[s][nt]);
    }
#pragma unroll
    for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] += sacc2[nt][e];
    bool va = true, vb = true;
    if constexpr (!INTERIOR) {
      va = n0 + g >= a.n_sink && n0 + g < a.n_tok && !((lbits >> g) & 1u);
      vb = n0 + g + 8 >= a.n_sink && n0 + g + 8 < a.n_tok && !((lbits >> (g + 8)) & 1u);
    }
    const float2 kza = h2f(ld4(kzb + 4 * g)), kzb2 = h2f(ld4(kzb + 4 * (g + 8)));
    float2 vza = h2f(ld4(vzb + 4 * g)), vzb2 = h2f(ld4(vzb + 4 * (g + 8)));
    if constexpr (!INTERIOR) {
      if (!va) vza = make_float2(0.0f, 0.0f);
      if (!vb) vzb2 = make_float2(0.0f, 0.0f);
    }
    const float lga = lg2_approx(fmaxf(vza.x, kMinS)), lgb = lg2_approx(fmaxf(vzb2.x, kMinS));
    uint32_t hla[NTN], hlb[NTN];
#pragma unroll
    for (int nt = 0; nt < NTN; ++nt) {
      const bool qv = ALLQ || 4 * nt + tig < GQ;
      const float da = static_cast<float>(sacc[nt][0] + 256 * sacc[nt][1]);
      const float db = static_cast<float>(sacc[nt][2] + 256 * sacc[nt][3]);
      const float sa = __fmaf_rn(kza.x * sq[nt], da, __fmaf_rn(kza.y, qs[nt], 0.0f)) * a.scale;
      const float sb = __fmaf_rn(kzb2.x * sq[nt], db, __fmaf_rn(kzb2.y, qs[nt], 0.0f)) * a.scale;
      const bool oka = va && qv, okb = vb && qv;
      float blk = fmaxf(oka ? __fmaf_rn(sa, kLog2e, lga) : -INFINITY, okb ? __fmaf_rn(sb, kLog2e, lgb) : -INFINITY);
      blk = fmaxf(blk, __shfl_xor_sync(0xffffffffu, blk, 4));
      blk = fmaxf(blk, __shfl_xor_sync(0xffffffffu, blk, 8));
      blk = fmaxf(blk, __shfl_xor_sync(0xffffffffu, blk, 16));
      if (blk > m_run[nt] + kFLazy) {  // uniform over the lanes of this query head
        const float f = ex2_approx(m_run[nt] - blk);
        m_run[nt] = blk;
        l_run[nt] *= f;
        z_run[nt] *= f;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][nt][e] *= f;
      }
      const float pa = oka ? ex2_approx(__fmaf_rn(sa, kLog2e, -m_run[nt])) : 0.0f;
      const float pb = okb ? ex2_approx(__fmaf_rn(sb, kLog2e, -m_run[nt])) : 0.0f;
      l_run[nt] += pa + pb;
      z_run[nt] = __fmaf_rn(pa, vza.y, __fmaf_rn(pb, vzb2.y, z_run[nt]));
      hla[nt] = split_hi_lo(pa * vza.x);
      hlb[nt] = split_hi_lo(pb * vzb2.x);
    }
    // ---- value B fragments: tokens 2 tig, 2 tig + 1 (b0 b1) and + 8 (b2 b3), column g
    uint32_t bv0[NTN], bv1[NTN];
#pragma unroll
    for (int nt = 0; nt < NTN; ++nt) {
      const uint32_t x0 = __shfl_sync(0xffffffffu, hla[nt], srcA), x1 = __shfl_sync(0xffffffffu, hla[nt], srcB);
      const uint32_t x2 = __shfl_sync(0xffffffffu, hlb[nt], srcA), x3 = __shfl_sync(0xffffffffu, hlb[nt], srcB);
      bv0[nt] = __byte_perm(x0, x1, sel);
      bv1[nt] = __byte_perm(x2, x3, sel);
    }
    // ---- value A fragments and products
    const uint8_t* t0 = vcb + 2 * tig * RB;
    if constexpr (BITS == 2) {
      const uint32_t u0 = ld4(t0 + 4 * g), u1 = ld4(t0 + RB + 4 * g);
      const uint32_t u8 = ld4(t0 + 8 * RB + 4 * g), u9 = ld4(t0 + 9 * RB + 4 * g);
      uint32_t y[2][4];
      y[0][0] = __byte_perm(u0, u1, 0x5410);  // channel 16 g + t, tokens 2 tig, 2 tig + 1
      y[0][1] = __byte_perm(u0, u1, 0x7632);  // channel 16 g + 8 + t
      y[0][2] = __byte_perm(u8, u9, 0x5410);
      y[0][3] = __byte_perm(u8, u9, 0x7632);
#pragma unroll
      for (int r = 0; r < 4; ++r) y[1][r] = y[0][r] >> 10;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int hs = mt < 5 ? 0 : 1;
        const uint32_t msk = 0x00030003u << (2 * (mt < 5 ? mt : mt - 5));
        const uint32_t a0 = code_pair(y[hs][0], msk), a1 = code_pair(y[hs][1], msk);
        const uint32_t a2 = code_pair(y[hs][2], msk), a3 = code_pair(y[hs][3], msk);
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt) mma_f16(acc[mt][nt], a0, a1, a2, a3, bv0[nt], bv1[nt]);
      }
    } else {
      uint32_t y[2][2][4];  // [word g / g + 8][shift 0 / 8][register]
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int o = 4 * (g + 8 * w);
        const uint32_t u0 = ld4(t0 + o), u1 = ld4(t0 + RB + o);
        const uint32_t u8 = ld4(t0 + 8 * RB + o), u9 = ld4(t0 + 9 * RB + o);
        y[w][0][0] = __byte_perm(u0, u1, 0x5410);
        y[w][0][1] = __byte_perm(u0, u1, 0x7632);
        y[w][0][2] = __byte_perm(u8, u9, 0x5410);
        y[w][0][3] = __byte_perm(u8, u9, 0x7632);
#pragma unroll
        for (int r = 0; r < 4; ++r) y[w][1][r] = y[w][0][r] >> 8;
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int w = mt >> 2, p = mt & 3, hs = p >> 1;
        const uint32_t msk = 0x000F000Fu << (4 * (p & 1));
        const uint32_t a0 = code_pair(y[w][hs][0], msk), a1 = code_pair(y[w][hs][1], msk);
        const uint32_t a2 = code_pair(y[w][hs][2], msk), a3 = code_pair(y[w][hs][3], msk);
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt) mma_f16(acc[mt][nt], a0, a1, a2, a3, bv0[nt], bv1[nt]);
      }
    }
  };

  int st = 0;
  for (int i = 0; i < my_n; ++i) {
    cp_async_wait_group<S - 1>();  // this lane's copies of block i
    __syncwarp();                  // ... and every other lane's
    const int n0 = n_first + i * static_cast<int>(kStep);
    const uint8_t* kcb = fdyn + (warp * S + st) * C::STAGE;
    uint32_t lbits = 0;
    if constexpr (LIST) {
      const bool in = my_list >= n0 && my_list < n0 + kFBlock;
      lbits = __reduce_or_sync(0xffffffffu, in ? 1u << (my_list - n0) : 0u);
    }
    if (lbits == 0 && n0 >= a.n_sink && n0 + kFBlock <= a.n_tok) block(std::true_type{}, n0, kcb, 0u);
    else block(std::false_type{}, n0, kcb, lbits);
    __syncwarp();  // every lane has read the stage
    if (i + S < my_n) issue(i + S, st);
    cp_async_commit();
    st = st + 1 == S ? 0 : st + 1;
  }
  cp_async_wait_all();
#pragma unroll
  for (int nt = 0; nt < NTN; ++nt) {
#pragma unroll
    for (int o = 4; o <= 16; o <<= 1) {
      l_run[nt] += __shfl_xor_sync(0xffffffffu, l_run[nt], o);
      z_run[nt] += __shfl_xor_sync(0xffffffffu, z_run[nt], o);
    }
  }
  __syncthreads();  // every warp is done with its stages: the stage memory now holds the per-warp sums
  float* accw = reinterpret_cast<float*>(fdyn);  // [kFWarps][GQ][D]
#pragma unroll
  for (int nt = 0; nt < NTN; ++nt) {
    const int qh = 4 * nt + tig;
    if (qh >= GQ) continue;
    float* dst = accw + (warp * GQ + qh) * D;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      int cha, chb;
      float sc;
      if constexpr (BITS == 2) {
        cha = 16 * g + mt;
        chb = cha + 8;
        sc = 1.0f / static_cast<float>(1 << (2 * (mt < 5 ? mt : mt - 5)));
      } else {
        const int j = g + 8 * (mt >> 2), p = mt & 3;
        cha = 8 * j + p;
        chb = cha + 4;
        sc = (p & 1) ? 0.0625f : 1.0f;
      }
      dst[cha] = (acc[mt][nt][0] + acc[mt][nt][1]) * sc;
      dst[chb] = (acc[mt][nt][2] + acc[mt][nt][3]) * sc;
    }
    if (g == 0) {
      mw[warp][qh] = m_run[nt];
      lw[warp][qh] = l_run[nt];
      zw[warp][qh] = z_run[nt];
    }
  }
  __syncthreads();
  if (tid < GQ) {  // per query head: the chunk's reference, each warp's factor, l and the Z term
    const int qh = tid;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) M = fmaxf(M, mw[w][qh]);
    float L = 0.0f, Z = 0.0f;
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) {
      const float f = mw[w][qh] == -INFINITY ? 0.0f : ex2_approx(mw[w][qh] - M);
      mw[w][qh] = f;
      L = __fmaf_rn(f, lw[w][qh], L);
      Z = __fmaf_rn(f, zw[w][qh], Z);
    }
    zw[0][qh] = Z;
    const size_t row = (static_cast<size_t>(b) * a.Hq + h * GQ + qh) * a.n_chunks + c;
    *reinterpret_cast<float2*>(a.part_ml + 2 * row) = make_float2(M, L);
  }
  __syncthreads();
  for (int e = tid; e < GQ * D; e += kFThreads) {
    const int qh = e / D, j = e - qh * D;
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) s = __fmaf_rn(mw[w][qh], accw[(w * GQ + qh) * D + j], s);
    const size_t row = (static_cast<size_t>(b) * a.Hq + h * GQ + qh) * a.n_chunks + c;
    a.part_acc[row * D + j] = s + zw[0][qh];
  }
}

struct MergeArgs {
  int B, H, Hq, GQ, n_tok, n_sink, n_chunks, rot, krope;
  const int32_t* list;  // sink positions [B][n_sink] (-1 unused), or nullptr: the positions < n_sink
  float scale, rscale;
  const __half* q;
  const __half* ksink;
  const float* rope_cs;
  const __half* vsink;
  const int16_t* vperm;
  const float* part_acc;
  const float* part_ml;
  float* out;
};

// One CTA per (batch, query head): sink scores (fp16 keys, exactly as the
// score kernel forms them), the log-sum-exp merge of the chunks and sinks, the
// inverse rotation and permutation, and the sink values. Launched as a
// programmatic dependent of the fused kernel: everything up to the grid
// dependency wait reads only the caller's inputs.
__global__ void __launch_bounds__(kThreads) k_attend_merge(const MergeArgs a) {
  __shared__ __align__(16) float qraw[D];
  __shared__ float ts[kFMaxSinks];
  __shared__ float2 mls[kFMaxChunks];
  __shared__ float ys[2][D];
  __shared__ float nat[D];
  __shared__ float red[4];
  const int j = threadIdx.x, lane = j & 31, warp = j >> 5;
  const int bq = blockIdx.x;
  const int b = bq / a.Hq, qh = bq % a.Hq, h = qh / a.GQ;
  // sink n sits at position n, or at list entry n (skipped when -1 or past n_tok: score -inf)
  const int ns = a.list ? a.n_sink : min(a.n_sink, a.n_tok);
  const int32_t* lst = a.list ? a.list + static_cast<size_t>(b) * a.n_sink : nullptr;
  auto sink_at = [&](int n) { return lst ? lst[n] : n; };
  const size_t vh = static_cast<size_t>(b) * a.H + h;
  const int pj = a.vperm ? a.vperm[static_cast<size_t>(h) * D + j] & (D - 1) : j;
  qraw[j] = __half2float(a.q[static_cast<size_t>(bq) * D + j]);
  __syncthreads();
  float mloc = -INFINITY;
  for (int n = warp; n < ns; n += kThreads / 32) {
    const int m = sink_at(n);
    if (m < 0 || m >= a.n_tok) {
      if (lane == 0) ts[n] = -INFINITY;
      continue;
    }
    const float s = sink_dot(qraw, a.ksink + (vh * a.n_sink + n) * D,
                             a.krope ? a.rope_cs + static_cast<size_t>(m) * D : nullptr, lane, a.krope == 2) *
                    a.scale;
    if (lane == 0) ts[n] = s;
    mloc = fmaxf(mloc, s * kLog2e);
  }
  constexpr int kPre = 4;  // sink values held in registers from before the wait
  float sv[kPre];
#pragma unroll
  for (int n = 0; n < kPre; ++n) {
    const int m = n < ns ? sink_at(n) : -1;
    sv[n] = m >= 0 && m < a.n_tok ? __half2float(a.vsink[(vh * a.n_sink + n) * D + j]) : 0.0f;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the fused kernel's partials are complete
  const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + static_cast<size_t>(bq) * a.n_chunks;
  const float* pa = a.part_acc + static_cast<size_t>(bq) * a.n_chunks * D;
  for (int c = j; c < a.n_chunks; c += kThreads) {
    const float2 v = ml[c];
    mls[c] = v;
    mloc = fmaxf(mloc, v.x);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if (lane == 0) red[warp] = mloc;
  __syncthreads();
  const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  float L = 0.0f, acc = 0.0f;
  for (int c0 = 0; c0 < a.n_chunks; c0 += 16) {  // sixteen loads in flight, then their weights
    float v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = c0 + u < a.n_chunks ? pa[static_cast<size_t>(c0 + u) * D + j] : 0.0f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      if (c0 + u >= a.n_chunks) break;
      const float2 m = mls[c0 + u];
      const float f = m.x == -INFINITY ? 0.0f : ex2_approx(m.x - M);
      L = __fmaf_rn(m.y, f, L);
      acc = __fmaf_rn(v[u], f, acc);
    }
  }
  for (int n = 0; n < ns; ++n)
    if (ts[n] > -INFINITY) L += ex2_approx(__fmaf_rn(ts[n], kLog2e, -M));
  const float invL = 1.0f / L;
  float y = acc * invL;  // sum_n p_n y_n, channel j of the rotated basis
  if (a.rot == KVQ_ROT_FWHT_HEAD) {  // x = H y / sqrt(D), Sylvester order, strides 1 .. 64
    int cur = 0;
    ys[0][j] = y;
    __syncthreads();
#pragma unroll
    for (int st = 1; st < D; st <<= 1) {
      const float u = ys[cur][j], w = ys[cur][j ^ st];
      ys[cur ^ 1][j] = (j & st) ? w - u : u + w;
      cur ^= 1;
      __syncthreads();
    }
    y = ys[cur][j] * a.rscale;
  }
  nat[pj] = y;  // x[perm[j]] = y_j
  __syncthreads();
  float o = nat[j];
#pragma unroll
  for (int n = 0; n < kPre; ++n)
    if (n < ns && ts[n] > -INFINITY) o = __fmaf_rn(ex2_approx(__fmaf_rn(ts[n], kLog2e, -M)) * invL, sv[n], o);
  for (int n = kPre; n < ns; ++n) {
    if (!(ts[n] > -INFINITY)) continue;
    const float p = ex2_approx(__fmaf_rn(ts[n], kLog2e, -M)) * invL;
    o = __fmaf_rn(p, __half2float(a.vsink[(vh * a.n_sink + n) * D + j]), o);
  }
  a.out[static_cast<size_t>(bq) * D + j] = o;
}

template <int BITS, int GQ, bool LIST>
kvq_status run_fused(FusedArgs& fa, const LaunchCtx& ctx, cudaStream_t st) {
  constexpr size_t smem = FusedCfg<BITS>::SMEM;
  const void* fn = reinterpret_cast<const void*>(k_attend_fused<BITS, GQ, LIST>);
  if (!set_smem_once(fn, smem)) return KVQ_ERR_CUDA;
  const int per_sm = occupancy_once(fn, kFThreads, smem);
  const int bh = fa.B * fa.H;
  int want = ctx.num_sms * per_sm / bh;  // chunks per (batch, KV head) for about one wave
  want = want < 1 ? 1 : (want > kFMaxChunks ? kFMaxChunks : want);
  fa.blocks_per_chunk = (fa.blocks + want - 1) / want;
  fa.n_chunks = (fa.blocks + fa.blocks_per_chunk - 1) / fa.blocks_per_chunk;
  k_attend_fused<BITS, GQ, LIST><<<dim3(static_cast<unsigned>(fa.n_chunks), static_cast<unsigned>(bh)), kFThreads,
                             smem, st>>>(fa);
  return launch_status();
}

template <int BITS>
kvq_status fused_by_gq(FusedArgs& fa, int gq, const LaunchCtx& ctx, cudaStream_t st) {
  switch (gq) {
    case 1: return fa.list ? run_fused<BITS, 1, true>(fa, ctx, st) : run_fused<BITS, 1, false>(fa, ctx, st);
    case 2: return fa.list ? run_fused<BITS, 2, true>(fa, ctx, st) : run_fused<BITS, 2, false>(fa, ctx, st);
    case 4: return fa.list ? run_fused<BITS, 4, true>(fa, ctx, st) : run_fused<BITS, 4, false>(fa, ctx, st);
    case 8: return fa.list ? run_fused<BITS, 8, true>(fa, ctx, st) : run_fused<BITS, 8, false>(fa, ctx, st);
    default: return KVQ_ERR_UNSUPPORTED;
  }
}

// The merge as a programmatic dependent launch of the fused kernel.
kvq_status launch_merge(const MergeArgs& ma, unsigned grid, cudaStream_t st) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_attend_merge, ma) != cudaSuccess) return KVQ_ERR_CUDA;
  return launch_status();
}

// Listed sinks take the fused path up to 32 entries (one per lane of a warp).
constexpr int kFMaxListed = 32;
bool fused_path(int bits, int group, int n_sink, bool listed) {
  return (bits == 2 || bits == 4) && group == 128 && n_sink <= (listed ? kFMaxListed : kFMaxSinks);
}

int fused_tiles(int n_tokens) { return (n_tokens + kFBlock - 1) / kFBlock; }

// Fixed scratch of kvq_attend_noalloc: a file-scope device array, reserved when
// the module is loaded, so that entry point never allocates. 40 MiB holds the
// workspace of either form: chunk partials (at most 256 chunks per query head
// in the fused form: 4 sequences x 32 query heads x 32769 tokens take 17 MB),
// or scores plus partials (about 5 bytes per query head and cached token,
// 21 MB for the same shape). Nothing in it has to start at zero: every byte a
// call reads was written earlier in that call.
constexpr size_t kAttendScratchBytes = size_t{40} << 20;
__device__ __align__(256) uint8_t g_attend_scratch[kAttendScratchBytes];

}  // namespace

size_t attend_scratch_bytes() { return kAttendScratchBytes; }

// Device address of the fixed scratch on the current device, looked up once
// per device (with that device current) and cached; nullptr on a CUDA error.
void* attend_scratch() {
  constexpr int kDevices = 64;
  static std::mutex mu;
  static void* ptr[kDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attend_scratch) != cudaSuccess) return nullptr;
    ptr[dev] = p;
  }
  return ptr[dev];
}

size_t attend_workspace_bytes(const kvq_desc& dk, int q_heads, int n_tokens) {
  // enough for the prefix and the list form of these sinks (they take different paths above 32 sinks)
  const size_t bq = static_cast<size_t>(dk.batch) * q_heads;
  size_t fused = 0, other = 0;
  if (fused_path(dk.bits, dk.group, dk.n_sink, false)) {  // chunk partials only; chunks <= min(tiles, kFMaxChunks)
    const int tiles = fused_tiles(n_tokens);
    const size_t n_chunks = static_cast<size_t>(tiles < kFMaxChunks ? tiles : kFMaxChunks);
    fused = align256(bq * n_chunks * D * 4) + align256(bq * n_chunks * 2 * 4);
  }
  if (!fused_path(dk.bits, dk.group, dk.n_sink, true)) {
    const size_t n_chunks = (static_cast<size_t>(n_tokens) + kCh * kSub - 1) / (kCh * kSub);
    other = align256(bq * n_tokens * 4) + align256(bq * n_chunks * D * 4) + align256(bq * n_chunks * 2 * 4);
  }
  return fused > other ? fused : other;
}

kvq_status launch_attend(const kvq_desc& dk, const kvq_desc& dv, const void* q, int q_heads,
                         const kvq_packed& kc, const kvq_tables& tk, const kvq_packed& vc, const kvq_tables& tv,
                         int n_tokens, float scale, float* out, void* ws, cudaStream_t st, const LaunchCtx& ctx) {
  const size_t bq = static_cast<size_t>(dk.batch) * q_heads;
  const int32_t* list = dk.n_sink > 0 ? tk.sink_pos : nullptr;  // listed sinks (both caches' list)
  if (fused_path(dk.bits, dk.group, dk.n_sink, list != nullptr)) {
    const int tiles = fused_tiles(n_tokens);
    const int max_chunks = tiles < kFMaxChunks ? tiles : kFMaxChunks;
    FusedArgs fa{};
    fa.B = dk.batch;
    fa.H = dk.heads;
    fa.Hq = q_heads;
    fa.t_cap = dk.t_cap;
    fa.n_tok = n_tokens;
    fa.n_sink = list ? 0 : dk.n_sink;
    fa.list = list;
    fa.n_list = list ? dk.n_sink : 0;
    fa.rot = dk.rot;
    fa.blocks = tiles;
    fa.scale = scale;
    fa.rscale = static_cast<float>(1.0 / sqrt(static_cast<double>(D)));
    fa.q = static_cast<const __half*>(q);
    fa.kperm = tk.perm;
    fa.kcodes = kc.codes;
    fa.ksz = static_cast<const uint32_t*>(kc.scale_zero);
    fa.vcodes = vc.codes;
    fa.vsz = static_cast<const uint32_t*>(vc.scale_zero);
    uint8_t* w = static_cast<uint8_t*>(ws);
    fa.part_acc = reinterpret_cast<float*>(w);
    fa.part_ml = reinterpret_cast<float*>(w + align256(bq * max_chunks * D * 4));
    const int gq = q_heads / dk.heads;
    kvq_status s = dk.bits == 2 ? fused_by_gq<2>(fa, gq, ctx, st) : fused_by_gq<4>(fa, gq, ctx, st);
    if (s != KVQ_OK) return s;
    MergeArgs ma{};
    ma.B = dk.batch;
    ma.H = dk.heads;
    ma.Hq = q_heads;
    ma.GQ = gq;
    ma.n_tok = n_tokens;
    ma.n_sink = dk.n_sink;
    ma.list = list;
    ma.n_chunks = fa.n_chunks;
    ma.rot = dv.rot;
    ma.krope = dk.rope;
    ma.scale = scale;
    ma.rscale = fa.rscale;
    ma.q = fa.q;
    ma.ksink = static_cast<const __half*>(kc.sink);
    ma.rope_cs = tk.rope_cs;
    ma.vsink = static_cast<const __half*>(vc.sink);
    ma.vperm = tv.perm;
    ma.part_acc = fa.part_acc;
    ma.part_ml = fa.part_ml;
    ma.out = out;
    return launch_merge(ma, static_cast<unsigned>(bq), st);
  }
  AttnArgs a{};
  a.B = dk.batch;
  a.H = dk.heads;
  a.Hq = q_heads;
  a.GQ = q_heads / dk.heads;
  a.t_cap = dk.t_cap;
  a.n_tok = n_tokens;
  a.n_chunks = (n_tokens + kCh * kSub - 1) / (kCh * kSub);
  a.n_sink = dv.n_sink;
  a.list = list;
  a.rot = dv.rot;
  a.rscale = static_cast<float>(1.0 / sqrt(static_cast<double>(D)));
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* scores = reinterpret_cast<float*>(w);
  w += align256(bq * n_tokens * 4);
  a.part_acc = reinterpret_cast<float*>(w);
  w += align256(bq * a.n_chunks * D * 4);
  a.part_ml = reinterpret_cast<float*>(w);
  a.scores = scores;
  a.vcodes = vc.codes;
  a.vsz = static_cast<const __half2*>(vc.scale_zero);
  a.vsink = static_cast<const __half*>(vc.sink);
  a.vperm = tv.perm;
  a.out = out;
  // scores of every slot from its codes; with a list, the listed slots' exact scores
  // over them (their codes are zero, so their values enter only through the combine)
  kvq_desc dm = dk;
  if (list) dm.n_sink = 0;
  kvq_status s = launch_score(dm, q, q_heads, kc, tk, n_tokens, scale, scores, st, ctx);
  if (s != KVQ_OK) return s;
  if (list && (s = launch_sink_fix_score(dk, q, q_heads, kc, tk, n_tokens, scale, scores, st)) != KVQ_OK) return s;
  if ((s = dispatch_part(dv.bits, dv.group, a, st)) != KVQ_OK) return s;
  k_attend_combine<<<static_cast<unsigned>(bq), kThreads, 0, st>>>(a);
  return launch_status();
}

}  // namespace kvq
