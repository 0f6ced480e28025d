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
__global__ void __launch_bounds__(kThreads) k_score(const ScoreArgs a) {
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

template <int D, int BITS, int G, int GQ>
kvq_status run(const ScoreArgs& a, cudaStream_t st) {
  const dim3 grid((a.n_tok + kThreads - 1) / kThreads, a.H, a.B);
  k_score<D, BITS, G, GQ><<<grid, kThreads, 0, st>>>(a);
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
                        const LaunchCtx&) {
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
