// Energy of each RoPE frequency pair ("EliteKV - RoPE频率选择与低秩投影" §3.1,
// frequency energy analysis): per head,
//   E_i = sum over batches and cached tokens of |K_{2i}|^2 + |K_{2i+1}|^2,
// on the fp16 keys as given (RoPE rotates each pair without changing its
// norm), and the pairs ranked by descending E_i (equal energies in ascending
// pair order) — the ordering from which the elite frequencies are taken.
//
// Exact integer arithmetic: an fp16 value is M 2^(e - 25) (M = 1024 + the
// 10-bit fraction, biased exponent e >= 1) or M 2^-24 (subnormal), so its
// square is M^2 2^s units of 2^-48 with s = 2e - 2 (or 0), below 2^80. Each
// square is one 32x32 -> 64-bit product M^2 2^(s mod 32) (< 2^53) added to one
// of two 64-bit windows (weights 1 and 2^32), which are folded into the
// unsigned 128-bit sums (two words with carries) every 64 row steps, long
// before a window could overflow. The result does not depend on the order of
// the additions, and the ranking is decided on exact values.
//
// A memset and two launches: k_pair_energy, CTA = (chunk of token rows,
// head), each thread owns 4 pairs of a row with four rows' 16-byte loads in
// flight, then adds its CTA's sums into the zeroed output with 64-bit atomics
// (low word, then high word plus the low word's carry);
// k_pair_rank, one CTA per head, ranks the pairs.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxChunks = 64;
constexpr int kMinRows = 256;

struct EnergyArgs {
  int H, T, rows, rows_per_chunk;
  FastDiv div_t;
  const __half* x;
  unsigned long long* energy;  // [H][D/2][2]: low, high 64 bits, units of 2^-48
  int16_t* rank;               // [H][D/2]
};

// (a0, a1) += square of the fp16 value h: a0 in units of 2^-48, a1 in units of 2^-16 (inf / nan add nothing).
__device__ __forceinline__ void add_square(uint64_t& a0, uint64_t& a1, uint32_t h) {
  const uint32_t e = (h >> 10) & 31u, f = h & 1023u;
  const uint32_t M = e == 31u ? 0u : (e ? (f | 1024u) : f);
  const uint32_t s = e ? 2u * e - 2u : 0u;  // 0 .. 58
  const uint64_t t = static_cast<uint64_t>(M * M) * static_cast<uint64_t>(1u << (s & 31u));  // < 2^53
  const uint64_t m = s >= 32u ? ~0ull : 0ull;
  a1 += t & m;
  a0 += t & ~m;
}

__device__ __forceinline__ void add128(uint64_t& lo, uint64_t& hi, uint64_t blo, uint64_t bhi) {
  lo += blo;
  hi += bhi + (lo < blo ? 1u : 0u);
}

template <int D>
__global__ void __launch_bounds__(kThreads) k_pair_energy(const EnergyArgs a) {
  constexpr int P = D / 2;
  constexpr int TPR = D / 8;           // threads per row: 8 channels = 4 pairs each
  constexpr int RPI = kThreads / TPR;  // rows per CTA iteration
  constexpr int U = 4;                 // rows per thread in flight
  __shared__ uint64_t red[RPI][P][2];
  const int tid = threadIdx.x, cg = tid % TPR, rl = tid / TPR;
  const int h = blockIdx.y;
  const int r0 = blockIdx.x * a.rows_per_chunk;
  const int r1 = min(r0 + a.rows_per_chunk, a.rows);
  uint64_t lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};  // 128-bit sums per pair
  uint64_t a0[4] = {0, 0, 0, 0}, a1[4] = {0, 0, 0, 0};  // windows of weight 1 and 2^32
  int n_it = 0;
  for (int r = r0 + rl; r < r1; r += U * RPI) {  // row r = (batch b, token t)
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int rr = r + u * RPI;
      const int b = static_cast<int>(a.div_t.div(static_cast<uint32_t>(rr)));
      const int t = rr - b * a.T;
      raw[u] = rr < r1 ? __ldg(reinterpret_cast<const uint4*>(
                             a.x + ((static_cast<size_t>(b) * a.H + h) * a.T + t) * D) + cg)
                       : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};  // word k = pair 4 cg + k
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        add_square(a0[k], a1[k], w[k] & 0xFFFFu);
        add_square(a0[k], a1[k], w[k] >> 16);
      }
    }
    if (++n_it == 64) {  // fold before a window could overflow (64 x 8 terms < 2^53 each)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        add128(lo[k], hi[k], a0[k], 0);
        add128(lo[k], hi[k], a1[k] << 32, a1[k] >> 32);
        a0[k] = a1[k] = 0;
      }
      n_it = 0;
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    add128(lo[k], hi[k], a0[k], 0);
    add128(lo[k], hi[k], a1[k] << 32, a1[k] >> 32);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    red[rl][4 * cg + k][0] = lo[k];
    red[rl][4 * cg + k][1] = hi[k];
  }
  __syncthreads();
  if (tid < P) {
    uint64_t slo = 0, shi = 0;
    for (int k = 0; k < RPI; ++k) add128(slo, shi, red[k][tid][0], red[k][tid][1]);
    unsigned long long* dst = a.energy + (static_cast<size_t>(h) * P + tid) * 2;
    const unsigned long long old = atomicAdd(dst, static_cast<unsigned long long>(slo));
    const uint64_t carry = old + slo < slo ? 1u : 0u;
    atomicAdd(dst + 1, static_cast<unsigned long long>(shi + carry));
  }
}

template <int D>
__global__ void __launch_bounds__(D / 2) k_pair_rank(const EnergyArgs a) {
  constexpr int P = D / 2;
  __shared__ uint64_t elo[P], ehi[P];
  const int i = threadIdx.x, h = blockIdx.x;
  const unsigned long long* e = a.energy + (static_cast<size_t>(h) * P + i) * 2;
  const uint64_t li = e[0], hi = e[1];
  elo[i] = li;
  ehi[i] = hi;
  __syncthreads();
  int r = 0;
#pragma unroll 8
  for (int k = 0; k < P; ++k) {
    const uint64_t hk = ehi[k], lk = elo[k];
    const bool above = hk > hi || (hk == hi && (lk > li || (lk == li && k < i)));
    r += above ? 1 : 0;
  }
  a.rank[static_cast<size_t>(h) * P + r] = static_cast<int16_t>(i);
}

int chunks_for(int64_t rows) {
  int64_t c = (rows + kMinRows - 1) / kMinRows;
  if (c < 1) c = 1;
  return static_cast<int>(c < kMaxChunks ? c : kMaxChunks);
}

template <int D>
kvq_status run(EnergyArgs& a, int chunks, cudaStream_t st) {
  if (cudaMemsetAsync(a.energy, 0, static_cast<size_t>(a.H) * D * sizeof(uint64_t), st) != cudaSuccess)
    return KVQ_ERR_CUDA;
  if (a.rows > 0) {
    k_pair_energy<D><<<dim3(static_cast<unsigned>(chunks), static_cast<unsigned>(a.H)), kThreads, 0, st>>>(a);
    const kvq_status s = launch_status();
    if (s != KVQ_OK) return s;
  }
  k_pair_rank<D><<<static_cast<unsigned>(a.H), D / 2, 0, st>>>(a);
  return launch_status();
}

}  // namespace

kvq_status launch_pair_energy(const kvq_desc& d, const void* x, uint64_t* energy, int16_t* rank, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(d.batch) * d.tokens;
  if (rows >= (int64_t(1) << 31)) return KVQ_ERR_UNSUPPORTED;
  EnergyArgs a{};
  a.H = d.heads;
  a.T = d.tokens;
  a.rows = static_cast<int>(rows);
  const int chunks = chunks_for(rows);
  a.rows_per_chunk = static_cast<int>((rows + chunks - 1) / chunks);
  a.div_t = FastDiv(static_cast<uint32_t>(d.tokens > 0 ? d.tokens : 1));
  a.x = static_cast<const __half*>(x);
  a.energy = reinterpret_cast<unsigned long long*>(energy);
  a.rank = rank;
  return d.head_dim == 128 ? run<128>(a, chunks, st) : run<64>(a, chunks, st);
}

}  // namespace kvq
