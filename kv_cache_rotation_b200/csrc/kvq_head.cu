// Head-variant encode / decode: one thread per token-head vector, the whole
// vector in registers.
//
// Encode ("RotateKV: Accurate and Robust 2-Bit KV Cache Quantization for LLMs
// via Outlier-Aware Adaptive Rotations", abstract and 关键设计: channel
// reordering followed by the FWHT; 2-bit KV quantization; attention sinks):
//   RoPE (keys) -> channel permutation -> normalised FWHT over head_dim
//   -> per-group min-max quantization with fp16 (scale, zero) -> LSB-first packing.
// Decode is the exact inverse.
//
// A CTA owns a tile of HT heads x NT tokens of one batch (HT * NT = 128).
// The fp16 rows arrive in shared memory by one 3-D TMA copy per 64-channel
// half (128-byte swizzle, so the per-thread row reads are bank-conflict
// free); the RoPE cos/sin rows of the tile's NT positions arrive by 2-D TMA
// copies and are shared by the HT heads.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

struct HeadArgs {
  int B, H, T, t0, t_cap, n_sink, rope, HT, NT, n_tblk, n_hblk;
  float rscale;  // fp32(1/sqrt(D))
  const int16_t* perm;
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

template <int BYTES>
__device__ __forceinline__ void store_words(uint8_t* dst, const uint32_t* w) {
  if constexpr (BYTES % 16 == 0) {
#pragma unroll
    for (int i = 0; i < BYTES / 16; ++i)
      reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < BYTES / 8; ++i) reinterpret_cast<uint2*>(dst)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
  }
}
template <int BYTES>
__device__ __forceinline__ void load_words(const uint8_t* src, uint32_t* w) {
  if constexpr (BYTES % 16 == 0) {
#pragma unroll
    for (int i = 0; i < BYTES / 16; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < BYTES / 8; ++i) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(src) + i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  }
}
template <int NG>
__device__ __forceinline__ void store_sz(__half2* dst, const __half2* v) {
  if constexpr (NG == 1) {
    *dst = v[0];
  } else if constexpr (NG == 2) {
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&v[0]);
    u.y = *reinterpret_cast<const uint32_t*>(&v[1]);
    *reinterpret_cast<uint2*>(dst) = u;
  } else {
#pragma unroll
    for (int i = 0; i < NG; i += 4) {
      uint4 u;
      u.x = *reinterpret_cast<const uint32_t*>(&v[i]);
      u.y = *reinterpret_cast<const uint32_t*>(&v[i + 1]);
      u.z = *reinterpret_cast<const uint32_t*>(&v[i + 2]);
      u.w = *reinterpret_cast<const uint32_t*>(&v[i + 3]);
      *reinterpret_cast<uint4*>(dst + i) = u;
    }
  }
}

// Permutation through a thread-private shared-memory row of D floats
// (16-byte chunks XOR-swizzled by the thread index).
template <int D>
__device__ __forceinline__ uint32_t perm_addr(uint32_t row, int e, int tid) {
  return row + ((((e >> 2) ^ (tid & 7)) << 4) | ((e & 3) << 2));
}
// gather: v[j] <- v[perm[j]]
template <int D>
__device__ __forceinline__ void perm_gather(float (&v)[D], const int16_t* perm_row, uint32_t row, int tid) {
#pragma unroll
  for (int c = 0; c < D / 4; ++c)
    sts128(row + ((c ^ (tid & 7)) << 4), make_uint4(__float_as_uint(v[4 * c]), __float_as_uint(v[4 * c + 1]),
                                                    __float_as_uint(v[4 * c + 2]), __float_as_uint(v[4 * c + 3])));
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 pk = __ldg(reinterpret_cast<const uint4*>(perm_row) + c);
    const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = static_cast<int>((pw[i >> 1] >> (16 * (i & 1))) & (D - 1));
      v[8 * c + i] = lds32f(perm_addr<D>(row, e, tid));
    }
  }
}
// scatter: v'[perm[j]] <- v[j]
template <int D>
__device__ __forceinline__ void perm_scatter(float (&v)[D], const int16_t* perm_row, uint32_t row, int tid) {
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 pk = __ldg(reinterpret_cast<const uint4*>(perm_row) + c);
    const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = static_cast<int>((pw[i >> 1] >> (16 * (i & 1))) & (D - 1));
      sts32f(perm_addr<D>(row, e, tid), v[8 * c + i]);
    }
  }
#pragma unroll
  for (int c = 0; c < D / 4; ++c) {
    const uint4 u = lds128(row + ((c ^ (tid & 7)) << 4));
    v[4 * c] = __uint_as_float(u.x);
    v[4 * c + 1] = __uint_as_float(u.y);
    v[4 * c + 2] = __uint_as_float(u.z);
    v[4 * c + 3] = __uint_as_float(u.w);
  }
}

// Tile index -> (b, head base, token base).
__device__ __forceinline__ void tile_coords(const HeadArgs& a, int& b, int& h_base, int& t_base) {
  int blk = blockIdx.x;
  const int tb = blk % a.n_tblk;
  blk /= a.n_tblk;
  const int hb = blk % a.n_hblk;
  b = blk / a.n_hblk;
  h_base = hb * a.HT;
  t_base = tb * a.NT;
}

template <int D, int BITS, int G, bool ROT>
__global__ void __launch_bounds__(128) k_encode_head(const __grid_constant__ CUtensorMap xmap,
                                                      const __grid_constant__ CUtensorMap rmap, const HeadArgs a) {
  constexpr int RB = D * BITS / 8;  // record bytes
  constexpr int NG = D / G;
  constexpr int NW = D * BITS / 32;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar;
  uint8_t* xs = align1024(smem_raw);   // D/64 swizzled halves of 128 rows x 128 B
  uint8_t* rs = xs + D * 256;          // D/32 quarters of NT rows x 128 B
  uint8_t* ps = rs + a.NT * D * 4;     // permutation rows (128 x D floats)
  const int tid = threadIdx.x;
  int b, h_base, t_base;
  tile_coords(a, b, h_base, t_base);

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    const uint32_t bytes = D * 256 + (a.rope ? a.NT * D * 4 : 0);
    mbar_arrive_expect_tx(&bar, bytes);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) tma_load_3d(xs + hh * 16384, &xmap, hh * 64, t_base, b * a.H + h_base, &bar);
    if (a.rope)
      for (int q = 0; q < D / 32; ++q) tma_load_2d(rs + q * a.NT * 128, &rmap, q * 32, a.t0 + t_base, &bar);
  }
  if (!mbar_wait(&bar, 0, a.wait_ns, a.err)) {
    if (tid == 0) mbar_wait(&bar, 0, a.wait_ns, a.err);  // let an in-flight copy land before exiting
    return;
  }

  const int hl = tid / a.NT, t = tid % a.NT;
  const int h = h_base + hl, tt = t_base + t;
  if (h >= a.H || tt >= a.T) return;
  const int m = a.t0 + tt;
  const size_t v = static_cast<size_t>(b) * a.H + h;
  const size_t slot = v * a.t_cap + m;
  const uint32_t xs_u = smem_u32(xs);

  if (m < a.n_sink) {  // attention sink: verbatim fp16, zero codes / scale / zero
    uint4* dst = reinterpret_cast<uint4*>(a.sink + (v * a.n_sink + m) * D);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh)
#pragma unroll
      for (int c = 0; c < 8; ++c) dst[hh * 8 + c] = lds128(xs_u + hh * 16384 + sw128(tid, c));
    uint32_t z[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) z[i] = 0u;
    store_words<RB>(a.codes + slot * RB, z);
    __half2 zs[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) zs[g] = __half2(__ushort_as_half(0), __ushort_as_half(0));
    store_sz<NG>(a.sz + slot * NG, zs);
    return;
  }

  float x[D];
#pragma unroll
  for (int hh = 0; hh < D / 64; ++hh)
#pragma unroll
    for (int c = 0; c < 8; ++c) h8_to_f32(lds128(xs_u + hh * 16384 + sw128(tid, c)), &x[hh * 64 + c * 8]);

  if (a.rope) {
    const uint32_t rs_u = smem_u32(rs);
#pragma unroll
    for (int k = 0; k < D / 4; ++k) {  // chunk k = pairs 2k, 2k+1 = channels 4k..4k+3
      const uint4 cs = lds128(rs_u + (k >> 3) * a.NT * 128 + sw128(t, k & 7));
      rope_fwd(x[4 * k], x[4 * k + 1], __uint_as_float(cs.x), __uint_as_float(cs.y));
      rope_fwd(x[4 * k + 2], x[4 * k + 3], __uint_as_float(cs.z), __uint_as_float(cs.w));
    }
  }
  if (a.perm) perm_gather<D>(x, a.perm + static_cast<size_t>(h) * D, smem_u32(ps) + tid * D * 4, tid);
  if constexpr (ROT) {
    fwht_reg<D>(x);
#pragma unroll
    for (int j = 0; j < D; ++j) x[j] = __fmul_rn(x[j], a.rscale);
  }

  uint32_t w[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = 0u;
  __half2 szv[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    float mn, mx;
    minmax_range<D>(x, g * G, G, mn, mx);
    const QParams p = minmax_params<BITS>(mn, mx);
    szv[g] = p.sz;
#pragma unroll
    for (int jj = 0; jj < G; ++jj) {
      const int j = g * G + jj;
      const uint32_t c = quant_code(x[j], p.Z, p.R);
      const int pos = j * BITS;
      w[pos >> 5] |= c << (pos & 31);
      if ((pos & 31) + BITS > 32) w[(pos >> 5) + 1] |= c >> (32 - (pos & 31));
    }
  }
  store_words<RB>(a.codes + slot * RB, w);
  store_sz<NG>(a.sz + slot * NG, szv);
}

template <int D, int BITS, int G, bool ROT>
__global__ void __launch_bounds__(128) k_decode_head(const __grid_constant__ CUtensorMap omap,
                                                      const __grid_constant__ CUtensorMap rmap, const HeadArgs a,
                                                      int out_fp32) {
  constexpr int RB = D * BITS / 8;
  constexpr int NG = D / G;
  constexpr int NW = D * BITS / 32;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar;
  uint8_t* os = align1024(smem_raw);                   // output tile: fp16 D*256 B or fp32 D*512 B
  uint8_t* rs = os + D * 512;                          // rope rows
  uint8_t* ps = rs + a.NT * D * 4;                     // permutation rows
  const int tid = threadIdx.x;
  int b, h_base, t_base;
  tile_coords(a, b, h_base, t_base);

  if (a.rope) {
    if (tid == 0) {
      mbar_init(&bar, 1);
      fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
      mbar_arrive_expect_tx(&bar, a.NT * D * 4);
      for (int q = 0; q < D / 32; ++q) tma_load_2d(rs + q * a.NT * 128, &rmap, q * 32, a.t0 + t_base, &bar);
    }
  }

  const int hl = tid / a.NT, t = tid % a.NT;
  const int h = h_base + hl, tt = t_base + t;
  const bool active = (h < a.H) && (tt < a.T);
  const int m = a.t0 + tt;
  const size_t v = static_cast<size_t>(b) * a.H + h;
  const size_t slot = v * a.t_cap + m;
  float x[D];

  if (active && m < a.n_sink) {
    const uint4* src = reinterpret_cast<const uint4*>(a.sink + (v * a.n_sink + m) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) h8_to_f32(__ldg(src + c), &x[8 * c]);
  } else if (active) {
    uint32_t w[NW];
    load_words<RB>(a.codes + slot * RB, w);
    __half2 szv[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) szv[g] = a.sz[slot * NG + g];
#pragma unroll
    for (int j = 0; j < D; ++j) {
      const float S = __low2float(szv[j / G]), Z = __high2float(szv[j / G]);
      x[j] = __fmaf_rn(code_to_float(unpack_code<BITS, NW>(w, j)), S, Z);
    }
    if constexpr (ROT) {
      fwht_reg<D>(x);
#pragma unroll
      for (int j = 0; j < D; ++j) x[j] = __fmul_rn(x[j], a.rscale);
    }
    if (a.perm) perm_scatter<D>(x, a.perm + static_cast<size_t>(h) * D, smem_u32(ps) + tid * D * 4, tid);
  }
  // Every thread waits for the RoPE rows (so no copy is in flight when the
  // CTA exits); on a timeout the kernel still reaches its barrier and exits.
  const bool rope_ok = a.rope ? mbar_wait(&bar, 0, a.wait_ns, a.err) : true;
  if (active && m >= a.n_sink && a.rope && rope_ok) {
    {
      const uint32_t rs_u = smem_u32(rs);
#pragma unroll
      for (int k = 0; k < D / 4; ++k) {
        const uint4 cs = lds128(rs_u + (k >> 3) * a.NT * 128 + sw128(t, k & 7));
        rope_inv(x[4 * k], x[4 * k + 1], __uint_as_float(cs.x), __uint_as_float(cs.y));
        rope_inv(x[4 * k + 2], x[4 * k + 3], __uint_as_float(cs.z), __uint_as_float(cs.w));
      }
    }
  }

  const uint32_t os_u = smem_u32(os);
  if (active) {
    if (out_fp32) {
#pragma unroll
      for (int c = 0; c < D / 4; ++c)
        sts128(os_u + (c >> 3) * 16384 + sw128(tid, c & 7),
               make_uint4(__float_as_uint(x[4 * c]), __float_as_uint(x[4 * c + 1]), __float_as_uint(x[4 * c + 2]),
                          __float_as_uint(x[4 * c + 3])));
    } else {
#pragma unroll
      for (int c = 0; c < D / 8; ++c) sts128(os_u + (c >> 3) * 16384 + sw128(tid, c & 7), f32_to_h8(&x[8 * c]));
    }
  }
  fence_async_smem();
  __syncthreads();
  if (tid == 0 && a.rope && !rope_ok) mbar_wait(&bar, 0, a.wait_ns, a.err);
  if (tid == 0) {
    const int nbox = out_fp32 ? D / 32 : D / 64;
    const int step = out_fp32 ? 32 : 64;
    for (int i = 0; i < nbox; ++i) tma_store_3d(&omap, i * step, t_base, b * a.H + h_base, os + i * 16384);
    bulk_commit();
    bulk_wait_read0();
  }
}

template <int D, int BITS, int G, bool ROT>
kvq_status run_encode(const HeadArgs& a, const CUtensorMap& xm, const CUtensorMap& rm, size_t smem,
                      cudaStream_t st) {
  auto k = k_encode_head<D, BITS, G, ROT>;
  if (!set_smem_once(reinterpret_cast<const void*>(k), smem))
    return KVQ_ERR_CUDA;
  const size_t grid = static_cast<size_t>(a.B) * a.n_hblk * a.n_tblk;
  k<<<static_cast<unsigned>(grid), 128, smem, st>>>(xm, rm, a);
  return launch_status();
}
template <int D, int BITS, int G, bool ROT>
kvq_status run_decode(const HeadArgs& a, const CUtensorMap& om, const CUtensorMap& rm, size_t smem, int out_fp32,
                      cudaStream_t st) {
  auto k = k_decode_head<D, BITS, G, ROT>;
  if (!set_smem_once(reinterpret_cast<const void*>(k), smem))
    return KVQ_ERR_CUDA;
  const size_t grid = static_cast<size_t>(a.B) * a.n_hblk * a.n_tblk;
  k<<<static_cast<unsigned>(grid), 128, smem, st>>>(om, rm, a, out_fp32);
  return launch_status();
}

// Dispatch over (D, BITS, G, ROT).
template <bool ENC>
kvq_status dispatch(const kvq_desc& d, const HeadArgs& a, const CUtensorMap& m0, const CUtensorMap& rm, size_t smem,
                    int out_fp32, cudaStream_t st) {
  const bool rot = d.rot == KVQ_ROT_FWHT_HEAD;
#define KVQ_CASE(D_, B_, G_)                                                                     \
  if (d.head_dim == D_ && d.bits == B_ && d.group == G_) {                                      \
    if constexpr (ENC) {                                                                        \
      return rot ? run_encode<D_, B_, G_, true>(a, m0, rm, smem, st)                            \
                 : run_encode<D_, B_, G_, false>(a, m0, rm, smem, st);                          \
    } else {                                                                                    \
      return rot ? run_decode<D_, B_, G_, true>(a, m0, rm, smem, out_fp32, st)                  \
                 : run_decode<D_, B_, G_, false>(a, m0, rm, smem, out_fp32, st);                \
    }                                                                                           \
  }
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

HeadArgs make_args(const kvq_desc& d, const kvq_tables& tb, const kvq_packed& p, const LaunchCtx& ctx) {
  HeadArgs a{};
  a.B = d.batch;
  a.H = d.heads;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.t_cap = d.t_cap;
  a.n_sink = d.n_sink;
  a.rope = d.rope;
  a.HT = heads_per_tile(d.heads);
  a.NT = 128 / a.HT;
  a.n_tblk = (d.tokens + a.NT - 1) / a.NT;
  a.n_hblk = d.heads / a.HT;
  a.rscale = static_cast<float>(1.0 / sqrt(static_cast<double>(d.head_dim)));
  a.perm = tb.perm;
  a.codes = p.codes;
  a.sz = static_cast<__half2*>(p.scale_zero);
  a.sink = static_cast<__half*>(p.sink);
  a.err = ctx.err;
  a.wait_ns = ctx.wait_ns;
  return a;
}

bool rope_map(CUtensorMap* m, const kvq_desc& d, const kvq_tables& tb, int NT) {
  if (!d.rope) {
    *m = CUtensorMap{};
    return true;
  }
  const uint64_t dims[2] = {static_cast<uint64_t>(d.head_dim), static_cast<uint64_t>(tb.rope_rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(d.head_dim) * 4};
  const uint32_t box[2] = {32, static_cast<uint32_t>(NT)};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, tb.rope_cs, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

kvq_status launch_encode_head(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                              cudaStream_t st, const LaunchCtx& ctx) {
  const HeadArgs a = make_args(d, tb, out, ctx);
  CUtensorMap xm, rm;
  const uint64_t dims[3] = {static_cast<uint64_t>(d.head_dim), static_cast<uint64_t>(d.tokens),
                            static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t strides[2] = {static_cast<uint64_t>(d.head_dim) * 2,
                               static_cast<uint64_t>(d.tokens) * d.head_dim * 2};
  const uint32_t box[3] = {64, static_cast<uint32_t>(a.NT), static_cast<uint32_t>(a.HT)};
  if (!make_map(&xm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  if (!rope_map(&rm, d, tb, a.NT)) return KVQ_ERR_CUDA;
  const size_t smem = 1024 + static_cast<size_t>(d.head_dim) * 256 + static_cast<size_t>(a.NT) * d.head_dim * 4 +
                      (tb.perm ? static_cast<size_t>(128) * d.head_dim * 4 : 0);
  return dispatch<true>(d, a, xm, rm, smem, 0, st);
}

kvq_status launch_decode_head(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                              int out_fp32, cudaStream_t st, const LaunchCtx& ctx) {
  HeadArgs a = make_args(d, tb, in, ctx);
  CUtensorMap om, rm;
  const uint64_t es = out_fp32 ? 4 : 2;
  const uint64_t dims[3] = {static_cast<uint64_t>(d.head_dim), static_cast<uint64_t>(d.tokens),
                            static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t strides[2] = {static_cast<uint64_t>(d.head_dim) * es,
                               static_cast<uint64_t>(d.tokens) * d.head_dim * es};
  const uint32_t box[3] = {out_fp32 ? 32u : 64u, static_cast<uint32_t>(a.NT), static_cast<uint32_t>(a.HT)};
  if (!make_map(&om, out_fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, x_out, dims,
                strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  if (!rope_map(&rm, d, tb, a.NT)) return KVQ_ERR_CUDA;
  const size_t smem = 1024 + static_cast<size_t>(d.head_dim) * 512 + static_cast<size_t>(a.NT) * d.head_dim * 4 +
                      (tb.perm ? static_cast<size_t>(128) * d.head_dim * 4 : 0);
  return dispatch<false>(d, a, om, rm, smem, out_fp32, st);
}

}  // namespace kvq
