// Channel permutation by abs-max ("RotateKV: Accurate and Robust 2-Bit KV Cache
// Quantization for LLMs via Outlier-Aware Adaptive Rotations": outlier-aware
// rotation, channel reordering before the FWHT). For each head h,
//   a_j = max over the batches and the non-sink positions of |y_j|,
// y = the fp32 input of the permutation step: RoPE_m(x) for keys of the
// head-dim variants (the permutation follows RoPE there), x itself otherwise
// (values, and the grouped variant, whose permutation acts on the raw input).
// perm[h] lists the channels by descending a_j; equal a_j keep ascending
// channel order.
//
// A memset and two launches. k_absmax: CTA = (chunk of token rows, head);
// each thread owns 8 channels of a row (16-byte loads, four rows in flight),
// applies RoPE in registers with the encoder's fp32 order, and keeps a running
// |y| maximum; the CTA's maxima go to the zeroed [H][D] workspace by atomicMax
// on the fp32 bit patterns (for non-negative floats the unsigned order is the
// numeric order, and a maximum does not depend on the order of the updates).
// k_perm_rank: one CTA per head ranks the channels,
// rank_j = #{k : a_k > a_j or (a_k = a_j and k < j)}, perm[rank_j] = j.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxChunks = 64;
constexpr int kMinRows = 256;  // token rows per chunk, at least

struct CalArgs {
  int H, T, t0, n_sink, rope, rows, rows_per_chunk;
  const int32_t* sink_pos;  // [B][n_sink] listed sink positions, or nullptr: positions < n_sink
  FastDiv div_t;
  const __half* x;
  const float* rope_cs;
  uint32_t* amax;  // [H][D]: fp32 bit patterns of the running maxima (zeroed before k_absmax)
  int16_t* perm;
};

__device__ __forceinline__ bool is_sink(const CalArgs& a, int b, int pos) {
  if (!a.sink_pos) return pos < a.n_sink;
  bool hit = false;
  for (int k = 0; k < a.n_sink; ++k) hit |= __ldg(a.sink_pos + static_cast<size_t>(b) * a.n_sink + k) == pos;
  return hit;
}

// ROPE: 0 none, 1 interleaved pairs, 2 half-split pairs (the only mode whose
// threads exchange channels, so the only one that needs a uniform trip count).
template <int D, int ROPE>
__global__ void __launch_bounds__(kThreads) k_absmax(const CalArgs a) {
  constexpr int TPR = D / 8;           // threads per row
  constexpr int RPI = kThreads / TPR;  // rows in flight per CTA iteration
  __shared__ float red[RPI][D];
  const int tid = threadIdx.x, cg = tid % TPR, rl = tid / TPR;
  const int h = blockIdx.y;
  const int r0 = blockIdx.x * a.rows_per_chunk;
  const int r1 = min(r0 + a.rows_per_chunk, a.rows);
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0.0f;
  constexpr int U = 4;  // rows per thread in flight
  // with half-split pairs the trip count is the same for every thread (rows
  // past r1 are not live), so the pairs may exchange channels between threads
  const int rstart = ROPE == 2 ? r0 : r0 + rl;
  for (int rs = rstart; rs < r1; rs += U * RPI) {  // row r = (batch b, token t)
    const int r = ROPE == 2 ? rs + rl : rs;
    uint4 raw[U];
    float4 c0[U], c1[U];
    int posu[U];
    bool live[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int rr = r + u * RPI;
      const int b = static_cast<int>(a.div_t.div(static_cast<uint32_t>(min(rr, r1 - 1))));
      const int t = min(rr, r1 - 1) - b * a.T;
      const int pos = a.t0 + t;
      posu[u] = pos;
      live[u] = rr < r1 && !is_sink(a, b, pos);
      raw[u] = live[u] ? __ldg(reinterpret_cast<const uint4*>(
                             a.x + ((static_cast<size_t>(b) * a.H + h) * a.T + t) * D) + cg)
                       : make_uint4(0, 0, 0, 0);
      if (ROPE == 1 && live[u]) {  // pairs 4 cg .. 4 cg + 3 of position pos
        const float4* cs = reinterpret_cast<const float4*>(a.rope_cs + static_cast<size_t>(pos) * D) + 2 * cg;
        c0[u] = __ldg(cs);
        c1[u] = __ldg(cs + 1);
      } else {
        c0[u] = c1[u] = make_float4(1.0f, 0.0f, 1.0f, 0.0f);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float v[8];
      h8_to_f32(raw[u], v);
      if constexpr (ROPE == 1) {
        rope_fwd(v[0], v[1], c0[u].x, c0[u].y);
        rope_fwd(v[2], v[3], c0[u].z, c0[u].w);
        rope_fwd(v[4], v[5], c1[u].x, c1[u].y);
        rope_fwd(v[6], v[7], c1[u].z, c1[u].w);
      } else if constexpr (ROPE == 2) {
        // half-split pairs (c, c + D/2): this thread's channel 8 (cg mod TPR/2) + i pairs with the same
        // channel of thread cg ^ TPR/2 (the other half of the row), angle 8 (cg mod TPR/2) + i
        const float4* cs = reinterpret_cast<const float4*>(a.rope_cs + static_cast<size_t>(posu[u]) * D) +
                           4 * (cg & (TPR / 2 - 1));
        const bool upper = (cg & (TPR / 2)) != 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // channels 2k, 2k + 1 of the eight: angles +2k, +2k + 1
          const float4 c = live[u] ? __ldg(cs + k) : make_float4(1.0f, 0.0f, 1.0f, 0.0f);
          const float2 y = rope_half_fwd2(f2(v[2 * k], v[2 * k + 1]), f2(c.x, c.z), f2(c.y, c.w), upper, TPR / 2);
          v[2 * k] = y.x;
          v[2 * k + 1] = y.y;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(v[i]));  // rows not live hold zeros
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[rl][8 * cg + i] = m[i];
  __syncthreads();
  if (tid < D) {
    float mx = 0.0f;
#pragma unroll 8
    for (int k = 0; k < RPI; ++k) mx = fmaxf(mx, red[k][tid]);
    atomicMax(a.amax + static_cast<size_t>(h) * D + tid, __float_as_uint(mx));
  }
}

template <int D>
__global__ void __launch_bounds__(D) k_perm_rank(const CalArgs a) {
  __shared__ float s_a[D];
  const int j = threadIdx.x, h = blockIdx.x;
  const float aj = __uint_as_float(a.amax[static_cast<size_t>(h) * D + j]);
  s_a[j] = aj;
  __syncthreads();
  int rank = 0;
#pragma unroll 8
  for (int k = 0; k < D; ++k) {
    const float ak = s_a[k];
    rank += (ak > aj || (ak == aj && k < j)) ? 1 : 0;
  }
  a.perm[static_cast<size_t>(h) * D + rank] = static_cast<int16_t>(j);
}

// Row chunks per head: at least kMinRows rows each, at most kMaxChunks, and
// no more than one wave of CTAs over all heads (a second, partial wave would
// leave most SMs idle for its whole length).
int chunks_for(int64_t rows, int heads, int wave) {
  int64_t c = (rows + kMinRows - 1) / kMinRows;
  if (c > kMaxChunks) c = kMaxChunks;
  const int64_t fit = wave / heads;
  if (fit >= 1 && c > fit) c = fit;
  return static_cast<int>(c < 1 ? 1 : c);
}

template <int D>
const void* absmax_fn(int rope) {
  return rope == 1 ? reinterpret_cast<const void*>(k_absmax<D, 1>)
                   : rope == 2 ? reinterpret_cast<const void*>(k_absmax<D, 2>)
                               : reinterpret_cast<const void*>(k_absmax<D, 0>);
}

template <int D>
kvq_status run(CalArgs& a, int chunks, cudaStream_t st) {
  if (cudaMemsetAsync(a.amax, 0, static_cast<size_t>(a.H) * D * sizeof(uint32_t), st) != cudaSuccess)
    return KVQ_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>(chunks), static_cast<unsigned>(a.H));
  if (a.rope == 1)
    k_absmax<D, 1><<<grid, kThreads, 0, st>>>(a);
  else if (a.rope == 2)
    k_absmax<D, 2><<<grid, kThreads, 0, st>>>(a);
  else
    k_absmax<D, 0><<<grid, kThreads, 0, st>>>(a);
  kvq_status s = launch_status();
  if (s != KVQ_OK) return s;
  k_perm_rank<D><<<static_cast<unsigned>(a.H), D, 0, st>>>(a);
  return launch_status();
}

}  // namespace

bool calibrate_rope(const kvq_desc& d) {
  return d.rope != 0 && (d.rot == KVQ_ROT_NONE || d.rot == KVQ_ROT_FWHT_HEAD);
}

size_t calibrate_workspace_bytes(const kvq_desc& d) { return static_cast<size_t>(d.heads) * d.head_dim * 4; }

kvq_status launch_calibrate(const kvq_desc& d, const void* x, const kvq_tables& tb, int16_t* perm, void* ws,
                            cudaStream_t st, int num_sms) {
  const int64_t rows = static_cast<int64_t>(d.batch) * d.tokens;
  if (rows >= (int64_t(1) << 31)) return KVQ_ERR_UNSUPPORTED;
  CalArgs a{};
  a.H = d.heads;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.n_sink = d.n_sink;
  a.sink_pos = tb.sink_pos;
  a.rope = calibrate_rope(d) ? d.rope : 0;  // 1 interleaved pairs, 2 half-split pairs
  a.rows = static_cast<int>(rows);
  const int rope = calibrate_rope(d) ? d.rope : 0;
  const void* fn = d.head_dim == 128 ? absmax_fn<128>(rope) : absmax_fn<64>(rope);
  const int chunks = chunks_for(rows, d.heads, num_sms * occupancy_once(fn, kThreads, 0));
  a.rows_per_chunk = static_cast<int>((rows + chunks - 1) / chunks);
  a.div_t = FastDiv(static_cast<uint32_t>(d.tokens > 0 ? d.tokens : 1));
  a.x = static_cast<const __half*>(x);
  a.rope_cs = tb.rope_cs;
  a.amax = static_cast<uint32_t*>(ws);
  a.perm = perm;
  return d.head_dim == 128 ? run<128>(a, chunks, st) : run<64>(a, chunks, st);
}

}  // namespace kvq
