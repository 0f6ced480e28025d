// Attention sinks: detection by massive activations, and the list form of
// the sink set.
//
// "RotateKV: Accurate and Robust 2-Bit KV Cache Quantization for LLMs via
// Outlier-Aware Adaptive Rotations", abstract (iii) and 关键设计: the tokens
// that draw attention sinks carry massive activations; they are found from the
// activations and kept at high precision. Detection, per sequence b:
//   a_t  = max over heads and channels of |x[b][h][t][j]| (exact in fp16),
//   med  = the lower median of a_0 .. a_{T-1},
//   sink = a_t > tau * med (compared in fp64), at most max_sinks of them, the
//          largest first, equal a_t to the earlier token; listed ascending.
//
// Two kernels: k_token_absmax streams x once (HBM-bound) and leaves one
// 16-bit key per token, the fp16 magnitude bits, which order like the values;
// k_sink_select takes one CTA per sequence, finds the median and the cut-off
// key by a two-level radix select (256 + 128 bins in shared memory) and
// writes the list with an ordered block compaction.
//
// The list form of the cache (kvq_tables.sink_pos) reuses the prefix-free
// kernels unchanged: encode, decode and score run on every slot, then the
// k_sink_fix_* kernels overwrite what a listed sink changes (its fp16 row and
// zeroed record on encode, its verbatim row on decode, its exact score). The
// result equals the per-token definition because quantization is per token
// (per token and head group for FWHT_GROUP, whose heads share the decision).
#include <cuda_fp16.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kAbsThreads = 256;
constexpr int kSelThreads = 1024;

__device__ __forceinline__ uint32_t mag_max8(uint4 r) {
  const uint32_t m = __vmaxu2(__vmaxu2(r.x & 0x7fff7fffu, r.y & 0x7fff7fffu),
                              __vmaxu2(r.z & 0x7fff7fffu, r.w & 0x7fff7fffu));
  return max(m & 0xffffu, m >> 16);
}

// key[b][t] = max over heads and channels of the fp16 magnitude bits of
// x[b][h][t][:]. A tile is TPB tokens of one sequence; a token row is D/8
// lanes of 16 bytes; each thread walks the heads with four rows in flight.
// Persistent CTAs (one wave) stride over the B * ceil(T / TPB) tiles.
template <int D>
__global__ void __launch_bounds__(kAbsThreads) k_token_absmax(const uint4* __restrict__ x, uint16_t* key, int H,
                                                              int T, int tiles_per_seq, int n_tiles) {
  constexpr int LPT = D / 8;
  constexpr int TPB = kAbsThreads / LPT;
  const int c = threadIdx.x % LPT;
  const size_t hs = static_cast<size_t>(T) * LPT;  // uint4 per head slice
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int b = tile / tiles_per_seq;
    const int t = (tile - b * tiles_per_seq) * TPB + static_cast<int>(threadIdx.x) / LPT;
    uint32_t m = 0;
    if (t < T) {
      const uint4* p = x + (static_cast<size_t>(b) * H * T + t) * LPT + c;
      int h = 0;
      for (; h + 4 <= H; h += 4) {
        uint4 r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) r[u] = __ldcs(p + (h + u) * hs);
#pragma unroll
        for (int u = 0; u < 4; ++u) m = max(m, mag_max8(r[u]));
      }
      for (; h < H; ++h) m = max(m, mag_max8(__ldcs(p + h * hs)));
    }
#pragma unroll
    for (int o = LPT / 2; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (c == 0 && t < T) key[static_cast<size_t>(b) * T + t] = static_cast<uint16_t>(m);
  }
}

__device__ __forceinline__ double key_value(uint32_t k) {
  return static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(k))));
}

// Exclusive prefix of v over the CTA in thread order (kSelThreads threads),
// and the CTA total. `wsum` holds kSelThreads / 32 words.
__device__ __forceinline__ uint32_t cta_exclusive(uint32_t v, uint32_t* wsum, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  uint32_t off = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) {
    const uint32_t s = wsum[w];
    off += w < warp ? s : 0u;
    tot += s;
  }
  __syncthreads();
  total = tot;
  return off + inc - v;
}

// Warp 0 finds the bin of ascending rank r in hist[0 .. NB) (NB / 32 bins per
// lane) and writes (bin, count of keys in the bins below it) to out.
template <int NB>
__device__ __forceinline__ void warp_find_rank(const uint32_t* hist, uint32_t r, uint32_t* out) {
  constexpr int PER = NB / 32;
  const int lane = threadIdx.x & 31;
  uint32_t loc[PER], sum = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    loc[j] = hist[lane * PER + j];
    sum += loc[j];
  }
  uint32_t inc = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  uint32_t run = inc - sum;
  if (r >= run && r < inc) {
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      if (r < run + loc[j]) {
        out[0] = static_cast<uint32_t>(lane * PER + j);
        out[1] = run;
        break;
      }
      run += loc[j];
    }
  }
}

// The key of ascending rank r (0-based) among key[0 .. T): a two-level radix
// select, 256 bins on bits 14..7 of the 15-bit key, then 128 bins on bits 6..0
// of the keys in the chosen bin.
__device__ uint32_t radix_select(const uint16_t* key, int T, uint32_t r, uint32_t* h1, uint32_t* h2,
                                 uint32_t* sh) {
  const int tid = threadIdx.x;
  for (int i = tid; i < 256; i += kSelThreads) h1[i] = 0;
  for (int i = tid; i < 128; i += kSelThreads) h2[i] = 0;
  __syncthreads();
  for (int t = tid; t < T; t += kSelThreads) atomicAdd(&h1[(key[t] & 0x7fffu) >> 7], 1u);
  __syncthreads();
  if (tid < 32) warp_find_rank<256>(h1, r, sh);
  __syncthreads();
  const uint32_t hi = sh[0], below = sh[1];
  for (int t = tid; t < T; t += kSelThreads) {
    const uint32_t k = key[t] & 0x7fffu;
    if ((k >> 7) == hi) atomicAdd(&h2[k & 127u], 1u);
  }
  __syncthreads();
  if (tid < 32) warp_find_rank<128>(h2, r - below, sh);
  __syncthreads();
  const uint32_t k = (hi << 7) | sh[0];
  __syncthreads();  // sh is free again
  return k;
}

struct SelArgs {
  int T, t0, max_sinks;
  double tau;
  const uint16_t* key;
  int32_t* sink_pos;
  int32_t* count;
};

// One CTA per sequence. Thread i owns the contiguous token segment
// [i * S, (i + 1) * S), S = ceil(T / kSelThreads), so the ordered compaction
// needs one CTA scan for the ranks among equal keys and one for the output
// slots.
__global__ void __launch_bounds__(kSelThreads) k_sink_select(const SelArgs a, int staged) {
  __shared__ uint32_t h1[256], h2[128], wsum[kSelThreads / 32], sh[2], cnt;
  extern __shared__ uint16_t skey[];  // the sequence's keys when they fit (staged != 0)
  const int b = blockIdx.x, tid = threadIdx.x;
  const uint16_t* gkey = a.key + static_cast<size_t>(b) * a.T;
  const uint16_t* key = gkey;
  if (staged) {  // every later pass reads shared memory instead of L2
    constexpr int U = 8;
    for (int t0 = 0; t0 < a.T; t0 += U * kSelThreads) {
      uint16_t v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + u * kSelThreads + tid;
        v[u] = t < a.T ? gkey[t] : 0;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + u * kSelThreads + tid;
        if (t < a.T) skey[t] = v[u];
      }
    }
    __syncthreads();
    key = skey;
  }
  const uint32_t T = static_cast<uint32_t>(a.T), M = static_cast<uint32_t>(a.max_sinks);
  const double thr = a.tau * key_value(radix_select(key, a.T, (T - 1) / 2, h1, h2, sh));

  const int S = (a.T + kSelThreads - 1) / kSelThreads;
  const int s0 = min(tid * S, a.T), s1 = min(s0 + S, a.T);
  // C = tokens above the threshold
  if (tid == 0) cnt = 0;
  __syncthreads();
  uint32_t c = 0;
  for (int t = s0; t < s1; ++t) c += key_value(key[t] & 0x7fffu) > thr;
  if (c) atomicAdd(&cnt, c);
  __syncthreads();
  const uint32_t C = cnt;
  __syncthreads();
  // More candidates than room: keep those above the M-th largest key kc and
  // the earliest `need` tokens equal to it.
  const bool capped = C > M;
  uint32_t kc = 0, need = 0;
  if (capped) {
    kc = radix_select(key, a.T, T - M, h1, h2, sh);
    if (tid == 0) cnt = 0;
    __syncthreads();
    uint32_t g = 0;
    for (int t = s0; t < s1; ++t) g += (key[t] & 0x7fffu) > kc;
    if (g) atomicAdd(&cnt, g);
    __syncthreads();
    need = M - cnt;
  }
  auto selected = [&](uint32_t k, uint32_t eq_rank, bool& eq) {
    eq = capped && k == kc;
    if (!capped) return key_value(k) > thr;
    return k > kc || (eq && eq_rank < need);
  };
  uint32_t n_eq = 0;
  if (capped)
    for (int t = s0; t < s1; ++t) n_eq += (key[t] & 0x7fffu) == kc;
  uint32_t tot;
  const uint32_t eq0 = cta_exclusive(n_eq, wsum, tot);
  uint32_t n_sel = 0;
  {
    uint32_t er = eq0;
    for (int t = s0; t < s1; ++t) {
      bool eq;
      n_sel += selected(key[t] & 0x7fffu, er, eq);
      er += eq;
    }
  }
  uint32_t n;
  uint32_t idx = cta_exclusive(n_sel, wsum, n);
  int32_t* out = a.sink_pos + static_cast<size_t>(b) * M;
  {
    uint32_t er = eq0;
    for (int t = s0; t < s1 && n_sel; ++t) {
      bool eq;
      if (selected(key[t] & 0x7fffu, er, eq)) {
        if (idx < M) out[idx] = a.t0 + t;
        ++idx;
        --n_sel;
      }
      er += eq;
    }
  }
  if (n > M) n = M;
  for (uint32_t i = n + tid; i < M; i += kSelThreads) out[i] = -1;
  if (tid == 0 && a.count) a.count[b] = static_cast<int32_t>(n);
}

// ------------------------------------------------------------ list form fixes
struct FixArgs {
  int B, H, Hq, D, T, t0, t_cap, n_sink, rec_bytes, sz_words, n_tok, rope, out_fp32;
  float scale;
  const int32_t* list;  // [B][n_sink]
  const __half* x;      // encode input / score queries
  const float* rope_cs;
  uint8_t* codes;
  uint32_t* sz;  // scale/zero words of a record
  float* norm;
  uint16_t* ext;  // dynamic codebooks: the outlier channels' top bits
  __half* sink;
  void* out;      // decode output
  float* scores;  // [B][Hq][n_tok]
};

// Encode: the listed positions of this call keep their fp16 rows in the sink
// buffer (slot = index in the list) and a zero record.
__global__ void k_sink_fix_encode(const FixArgs a) {
  const int lane = threadIdx.x & 31;
  const int e = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // (b, k, h)
  if (e >= a.B * a.n_sink * a.H) return;
  const int h = e % a.H, bk = e / a.H, b = bk / a.n_sink, k = bk % a.n_sink;
  const int m = a.list[bk];
  if (m < a.t0 || m >= a.t0 + a.T) return;
  const size_t vh = static_cast<size_t>(b) * a.H + h;
  const uint4* src = reinterpret_cast<const uint4*>(a.x + (vh * a.T + (m - a.t0)) * a.D);
  uint4* dst = reinterpret_cast<uint4*>(a.sink + (vh * a.n_sink + k) * a.D);
  for (int i = lane; i < a.D / 8; i += 32) dst[i] = src[i];
  const size_t slot = vh * a.t_cap + m;
  for (int i = lane; i < a.rec_bytes; i += 32) a.codes[slot * a.rec_bytes + i] = 0;
  if (a.sz)
    for (int i = lane; i < a.sz_words; i += 32) a.sz[slot * a.sz_words + i] = 0u;
  if (a.norm && lane == 0) a.norm[slot] = 0.0f;
  if (a.ext && lane == 0) a.ext[slot] = 0;
}

// Decode: the listed positions of this call decode to their fp16 rows.
__global__ void k_sink_fix_decode(const FixArgs a) {
  const int lane = threadIdx.x & 31;
  const int e = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (e >= a.B * a.n_sink * a.H) return;
  const int h = e % a.H, bk = e / a.H, b = bk / a.n_sink, k = bk % a.n_sink;
  const int m = a.list[bk];
  if (m < a.t0 || m >= a.t0 + a.T) return;
  const size_t vh = static_cast<size_t>(b) * a.H + h;
  const __half* src = a.sink + (vh * a.n_sink + k) * a.D;
  const size_t row = (vh * a.T + (m - a.t0)) * a.D;
  if (a.out_fp32) {
    float* o = static_cast<float*>(a.out) + row;
    for (int i = lane; i < a.D; i += 32) o[i] = __half2float(src[i]);
  } else {
    __half* o = static_cast<__half*>(a.out) + row;
    for (int i = lane; i < a.D; i += 32) o[i] = src[i];
  }
}

// Score: scale * q . RoPE_m(sink row) for each listed m < n_tok, one warp per
// (b, k, query head); pair i is (2i, 2i+1) for rope 1, (i, i + D/2) for rope 2.
__global__ void k_sink_fix_score(const FixArgs a) {
  const int lane = threadIdx.x & 31;
  const int e = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (e >= a.B * a.n_sink * a.Hq) return;
  const int qh = e % a.Hq, bk = e / a.Hq, b = bk / a.n_sink, k = bk % a.n_sink;
  const int m = a.list[bk];
  if (m < 0 || m >= a.n_tok) return;
  const int h = qh / (a.Hq / a.H);
  const __half* kr = a.sink + ((static_cast<size_t>(b) * a.H + h) * a.n_sink + k) * a.D;
  const __half* qv = a.x + (static_cast<size_t>(b) * a.Hq + qh) * a.D;
  float acc = 0.0f;
  for (int i = lane; i < a.D / 2; i += 32) {
    const int c0 = a.rope == 2 ? i : 2 * i, c1 = a.rope == 2 ? i + a.D / 2 : 2 * i + 1;
    float k0 = __half2float(kr[c0]), k1 = __half2float(kr[c1]);
    if (a.rope) {
      const float2 cs = reinterpret_cast<const float2*>(a.rope_cs + static_cast<size_t>(m) * a.D)[i];
      const float r0 = __fsub_rn(__fmul_rn(k0, cs.x), __fmul_rn(k1, cs.y));
      const float r1 = __fadd_rn(__fmul_rn(k0, cs.y), __fmul_rn(k1, cs.x));
      k0 = r0;
      k1 = r1;
    }
    acc = __fmaf_rn(__half2float(qv[c0]), k0, acc);
    acc = __fmaf_rn(__half2float(qv[c1]), k1, acc);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) a.scores[(static_cast<size_t>(b) * a.Hq + qh) * a.n_tok + m] = a.scale * acc;
}

FixArgs fix_args(const kvq_desc& d, const kvq_tables& tb, const kvq_packed& p) {
  FixArgs a{};
  a.B = d.batch;
  a.H = d.heads;
  a.D = d.head_dim;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.t_cap = d.t_cap;
  a.n_sink = d.n_sink;
  a.rec_bytes = d.head_dim * d.bits / 8;
  a.rope = d.rope;
  a.list = tb.sink_pos;
  a.rope_cs = tb.rope_cs;
  a.codes = p.codes;
  if (d.quant == KVQ_Q_MINMAX) {
    a.sz = static_cast<uint32_t*>(p.scale_zero);
    a.sz_words = d.head_dim / d.group;  // one (scale, zero) half pair per group
  }
  if (d.rot == KVQ_ROT_ISO_SO4 || d.rot == KVQ_ROT_ISO_SO3) a.norm = p.norm;
  if (d.quant == KVQ_Q_CODEBOOK_DYN) a.ext = p.ext;
  a.sink = static_cast<__half*>(p.sink);
  return a;
}

int warps_grid(int64_t warps) { return static_cast<int>((warps * 32 + 255) / 256); }

}  // namespace

size_t detect_sinks_workspace_bytes(const kvq_desc& d) {
  return (static_cast<size_t>(d.batch) * d.tokens * 2 + 15) & ~size_t(15);
}

kvq_status launch_detect_sinks(const kvq_desc& d, const void* x, double tau, int max_sinks, int32_t* sink_pos,
                               int32_t* count, void* ws, cudaStream_t st, int num_sms) {
  uint16_t* key = static_cast<uint16_t*>(ws);
  const int D = d.head_dim;
  const int tpb = kAbsThreads / (D / 8);
  const long long tiles_per_seq = (d.tokens + tpb - 1) / tpb;
  const long long n_tiles = tiles_per_seq * d.batch;
  if (n_tiles >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
  const auto fn = D == 128 ? k_token_absmax<128> : k_token_absmax<64>;
  const int per_sm = occupancy_once(reinterpret_cast<const void*>(fn), kAbsThreads, 0);
  const long long wave = static_cast<long long>(num_sms) * per_sm;
  const unsigned grid = static_cast<unsigned>(n_tiles < wave ? n_tiles : wave);
  fn<<<grid, kAbsThreads, 0, st>>>(static_cast<const uint4*>(x), key, d.heads, d.tokens,
                                   static_cast<int>(tiles_per_seq), static_cast<int>(n_tiles));
  if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
  SelArgs a{d.tokens, d.t0, max_sinks, tau, key, sink_pos, count};
  // stage a sequence's keys in shared memory when they fit in 96 KB
  const size_t kbytes = static_cast<size_t>(d.tokens) * sizeof(uint16_t);
  const int staged = kbytes <= 96 * 1024 ? 1 : 0;
  const size_t smem = staged ? kbytes : 0;
  if (smem && !set_smem_once(reinterpret_cast<const void*>(k_sink_select), smem)) return KVQ_ERR_CUDA;
  k_sink_select<<<d.batch, kSelThreads, smem, st>>>(a, staged);
  return launch_status();
}

kvq_status launch_sink_fix_encode(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                                  cudaStream_t st) {
  FixArgs a = fix_args(d, tb, out);
  a.x = static_cast<const __half*>(x);
  k_sink_fix_encode<<<warps_grid(int64_t(d.batch) * d.n_sink * d.heads), 256, 0, st>>>(a);
  return launch_status();
}

kvq_status launch_sink_fix_decode(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                                  int out_fp32, cudaStream_t st) {
  FixArgs a = fix_args(d, tb, in);
  a.out = x_out;
  a.out_fp32 = out_fp32;
  k_sink_fix_decode<<<warps_grid(int64_t(d.batch) * d.n_sink * d.heads), 256, 0, st>>>(a);
  return launch_status();
}

kvq_status launch_sink_fix_score(const kvq_desc& d, const void* q, int q_heads, const kvq_packed& cache,
                                 const kvq_tables& tb, int n_tokens, float scale, float* scores, cudaStream_t st) {
  FixArgs a = fix_args(d, tb, cache);
  a.x = static_cast<const __half*>(q);
  a.Hq = q_heads;
  a.n_tok = n_tokens;
  a.scale = scale;
  a.scores = scores;
  k_sink_fix_score<<<warps_grid(int64_t(d.batch) * d.n_sink * q_heads), 256, 0, st>>>(a);
  return launch_status();
}

}  // namespace kvq
