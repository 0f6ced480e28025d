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
// the workspace; k_attend_part, one CTA per (chunk of 1024 tokens, batch, KV
// head), walks the chunk in sub-chunks of 128 with a running (online) softmax
// and writes the chunk's statistics (max m, sum l) and sum_n e^(s_n - m) y_n
// per query head of the group; k_attend_combine, one CTA
// per (batch, query head), merges the chunks (log-sum-exp), applies the
// inverse rotation and permutation and adds the sink rows.
#include <math.h>

#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int D = 128;
constexpr int kCh = 128;       // tokens per sub-chunk (one per thread in the score pass)
constexpr int kSub = 8;        // sub-chunks per chunk: a chunk is 1024 tokens
constexpr int kThreads = 128;  // part: one token each, then 32 channel quads x 4 token phases;
                               // combine: one thread per channel

struct AttnArgs {
  int B, H, Hq, GQ, t_cap, n_tok, n_chunks, n_sink, rot;
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
  __shared__ __align__(16) uint32_t csm[kCh][RB / 4];
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

  for (int sub = 0; sub < kSub; ++sub) {
    const int n0 = (c * kSub + sub) * kCh;
    if (n0 >= a.n_tok) break;  // uniform over the CTA
    const int nn = min(kCh, a.n_tok - n0);
    __syncthreads();  // the previous sub-chunk's csm / wsm / red readers are done

    // packed value records (zero past the last token)
    const uint4* vsrc = reinterpret_cast<const uint4*>(a.vcodes + (static_cast<size_t>(bh) * a.t_cap + n0) * RB);
    for (int i = tid; i < kCh * RB / 16; i += kThreads) {
      const int n = i / (RB / 16);
      reinterpret_cast<uint4*>(&csm[0][0])[i] = n < nn ? __ldg(vsrc + i) : make_uint4(0, 0, 0, 0);
    }
    // scores (thread = token), the sub-chunk max per query head
    float sv[GQ];
#pragma unroll
    for (int r = 0; r < GQ; ++r) {
      const float* sp = a.scores + (static_cast<size_t>(b) * a.Hq + h * GQ + r) * a.n_tok + n0;
      sv[r] = tid < nn ? __ldg(sp + tid) : -INFINITY;
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
      float2 sz[NG];
#pragma unroll
      for (int gg = 0; gg < NG; ++gg)
        sz[gg] = tid < nn ? __half22float2(a.vsz[(static_cast<size_t>(bh) * a.t_cap + n0 + tid) * NG + gg])
                          : make_float2(0.0f, 0.0f);
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
      uint32_t v = csm[n][wi] >> sh;
      if constexpr ((4 * BITS) % 8 != 0 || 32 % (4 * BITS) != 0) {
        if (sh + 4 * BITS > 32) v |= csm[n][wi + 1] << (32 - sh);
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
  // sink rows, verbatim values weighted by their softmax probability
  const int ns = min(a.n_sink, a.n_tok);
  const float* sv = a.scores + static_cast<size_t>(bq) * a.n_tok;
  for (int n = 0; n < ns; ++n) {
    const float p = __expf(sv[n] - M) * invL;
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

// Fixed scratch of kvq_attend_noalloc: a file-scope device array, reserved when
// the module is loaded, so that entry point never allocates. 40 MiB holds the
// scores and chunk partials of about 9 M (query head x cached token) pairs
// (4 bytes of score + 0.5 byte of chunk partials each), e.g. 4 sequences x 32
// query heads x 32769 tokens (19 MB). Nothing in it has
// to start at zero: every byte a call reads was written earlier in that call.
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

size_t attend_workspace_bytes(int B, int q_heads, int n_tokens) {
  const size_t bq = static_cast<size_t>(B) * q_heads;
  const size_t n_chunks = (static_cast<size_t>(n_tokens) + kCh * kSub - 1) / (kCh * kSub);
  return align256(bq * n_tokens * 4) + align256(bq * n_chunks * D * 4) + align256(bq * n_chunks * 2 * 4);
}

kvq_status launch_attend(const kvq_desc& dk, const kvq_desc& dv, const void* q, int q_heads,
                         const kvq_packed& kc, const kvq_tables& tk, const kvq_packed& vc, const kvq_tables& tv,
                         int n_tokens, float scale, float* out, void* ws, cudaStream_t st, const LaunchCtx& ctx) {
  const size_t bq = static_cast<size_t>(dk.batch) * q_heads;
  AttnArgs a{};
  a.B = dk.batch;
  a.H = dk.heads;
  a.Hq = q_heads;
  a.GQ = q_heads / dk.heads;
  a.t_cap = dk.t_cap;
  a.n_tok = n_tokens;
  a.n_chunks = (n_tokens + kCh * kSub - 1) / (kCh * kSub);
  a.n_sink = dv.n_sink;
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
  kvq_status s = launch_score(dk, q, q_heads, kc, tk, n_tokens, scale, scores, st, ctx);
  if (s != KVQ_OK) return s;
  if ((s = dispatch_part(dv.bits, dv.group, a, st)) != KVQ_OK) return s;
  k_attend_combine<<<static_cast<unsigned>(bq), kThreads, 0, st>>>(a);
  return launch_status();
}

}  // namespace kvq
