// Grouped-head encode / decode ("RotateKV: Accurate and Robust 2-Bit KV Cache
// Quantization for LLMs via Outlier-Aware Adaptive Rotations", abstract and
// 关键设计: pre-RoPE grouped-head rotation). The HG heads of one token are
// concatenated (index = local_head * 128 + channel), permuted per head,
// transformed by one normalised FWHT of size HG*128 in natural (Sylvester)
// stride order -- the 7 in-head strides first, then the log2(HG) cross-head
// strides -- and only then rotated by RoPE head slice by head slice; each
// head slice is quantized with per-group min-max and packed.
//
// A CTA owns HG heads x NT tokens (HG * NT = 128 threads) of one batch.
//   phase 1: thread (head, token) holds one 128-channel row in registers and
//            runs the 7 in-head FWHT strides;
//   exchange: rows go through shared memory (fp32, XOR-swizzled so both the
//            row writes and the column reads are bank-conflict free);
//   phase 2: thread (token, k) holds channels [k*C, (k+1)*C), C = 128/HG, of
//            all HG heads, runs the cross-head strides, RoPE, the min-max
//            reductions (warp shuffles over the threads sharing a group),
//            quantizes and stores its slice of each head's packed record.
// Decode runs the same two phases in reverse order.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int D = 128;

struct GroupArgs {
  int B, H, T, t0, t_cap, n_sink, rope, NT, n_tblk, n_grp;
  float rscale;  // fp32(1/sqrt(HG*128))
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

// 16-byte chunk c (0..31) of exchange row (t, h) -> chunk position in the row.
__device__ __forceinline__ uint32_t xpos(int t, int c) {
  return (static_cast<uint32_t>(c & 3) << 3) | ((static_cast<uint32_t>(c >> 2) ^ static_cast<uint32_t>(t)) & 7u);
}

// Store / load NB bytes (NB*8 <= 128 bits) at an NB-aligned address.
template <int NB>
__device__ __forceinline__ void st_bytes(uint8_t* dst, const uint32_t* w) {
  if constexpr (NB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i)
      reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else if constexpr (NB % 8 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 8; ++i) reinterpret_cast<uint2*>(dst)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
  } else if constexpr (NB % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 4; ++i) reinterpret_cast<uint32_t*>(dst)[i] = w[i];
  } else {
#pragma unroll
    for (int i = 0; i < NB / 2; ++i)
      reinterpret_cast<uint16_t*>(dst)[i] = static_cast<uint16_t>(w[i >> 1] >> (16 * (i & 1)));
  }
}
template <int NB>
__device__ __forceinline__ void ld_bytes(const uint8_t* src, uint32_t* w) {
  if constexpr (NB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (NB % 8 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 8; ++i) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(src) + i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else if constexpr (NB % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 4; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(src) + i);
  } else {
#pragma unroll
    for (int i = 0; i < (NB + 3) / 4; ++i) w[i] = 0u;
#pragma unroll
    for (int i = 0; i < NB / 2; ++i)
      w[i >> 1] |= static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(src) + i)) << (16 * (i & 1));
  }
}

__device__ __forceinline__ void tile_coords(const GroupArgs& a, int& b, int& g, int& t_base) {
  int blk = blockIdx.x;
  const int tb = blk % a.n_tblk;
  blk /= a.n_tblk;
  g = blk % a.n_grp;
  b = blk / a.n_grp;
  t_base = tb * a.NT;
}

template <int HG, int BITS, int G>
__global__ void __launch_bounds__(128) k_encode_group(const __grid_constant__ CUtensorMap xmap,
                                                       const __grid_constant__ CUtensorMap rmap, const GroupArgs a) {
  constexpr int NT = 128 / HG;    // tokens per tile
  constexpr int C = D / HG;       // channels per phase-2 thread
  constexpr int TPG = G / C;      // phase-2 threads sharing one min-max group
  constexpr int NB = C * BITS / 8;  // packed bytes per phase-2 thread and head
  constexpr int RB = D * BITS / 8;
  constexpr int NG = D / G;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar;
  uint8_t* xs = align1024(smem_raw);  // x tile (32 KB), then the exchange rows (64 KB) over it
  uint8_t* rs = xs + 65536;           // RoPE rows: 4 quarters x NT x 128 B
  const int tid = threadIdx.x;
  int b, grp, t_base;
  tile_coords(a, b, grp, t_base);
  const int h_base = grp * HG;

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar, 32768 + (a.rope ? NT * D * 4 : 0));
    tma_load_3d(xs, &xmap, 0, t_base, b * a.H + h_base, &bar);
    tma_load_3d(xs + 16384, &xmap, 64, t_base, b * a.H + h_base, &bar);
    if (a.rope)
      for (int q = 0; q < 4; ++q) tma_load_2d(rs + q * NT * 128, &rmap, q * 32, a.t0 + t_base, &bar);
  }
  const bool ok = mbar_wait(&bar, 0, a.wait_ns, a.err);

  // ---------------- phase 1: thread (hl, t) owns one head row
  const int hl = tid / NT, t = tid % NT;
  const int tt = t_base + t, m = a.t0 + tt;
  const size_t v1 = static_cast<size_t>(b) * a.H + h_base + hl;
  const uint32_t xs_u = smem_u32(xs);
  float x[D];
  if (ok) {
    if (tt < a.T && m < a.n_sink) {
      uint4* dst = reinterpret_cast<uint4*>(a.sink + (v1 * a.n_sink + m) * D);
#pragma unroll
      for (int c = 0; c < 16; ++c) dst[c] = lds128(xs_u + (c >> 3) * 16384 + sw128(tid, c & 7));
    }
    if (a.perm) {
      const int16_t* pr = a.perm + static_cast<size_t>(h_base + hl) * D;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
        const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t e = (pw[i >> 1] >> (16 * (i & 1))) & (D - 1);
          const uint32_t addr = xs_u + (e >> 6) * 16384 + sw128(tid, (e & 63) >> 3) + (e & 7) * 2;
          x[8 * c + i] = __half2float(__ushort_as_half(lds16(addr)));
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) h8_to_f32(lds128(xs_u + (c >> 3) * 16384 + sw128(tid, c & 7)), &x[8 * c]);
    }
    fwht_reg<D>(x);
  }
  __syncthreads();  // every x row is in registers: the exchange may overwrite the tile
  {
    const uint32_t row = xs_u + (t * HG + hl) * 512;
#pragma unroll
    for (int c = 0; c < 32; ++c)
      sts128(row + xpos(t, c) * 16, make_uint4(__float_as_uint(x[4 * c]), __float_as_uint(x[4 * c + 1]),
                                               __float_as_uint(x[4 * c + 2]), __float_as_uint(x[4 * c + 3])));
  }
  __syncthreads();

  // ---------------- phase 2: thread (t2, k) owns channels [k*C, (k+1)*C) of every head
  const int t2 = tid / HG, k = tid % HG;
  const int tt2 = t_base + t2, m2 = a.t0 + tt2;
  float vv[HG][C];
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    const uint32_t row = xs_u + (t2 * HG + h) * 512;
#pragma unroll
    for (int i = 0; i < C / 4; ++i) {
      const uint4 u = lds128(row + xpos(t2, k * (C / 4) + i) * 16);
      vv[h][4 * i] = __uint_as_float(u.x);
      vv[h][4 * i + 1] = __uint_as_float(u.y);
      vv[h][4 * i + 2] = __uint_as_float(u.z);
      vv[h][4 * i + 3] = __uint_as_float(u.w);
    }
  }
  // cross-head strides of the FWHT, then the normalisation
#pragma unroll
  for (int s = 1; s < HG; s <<= 1) {
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      if ((h & s) == 0) {
#pragma unroll
        for (int j = 0; j < C; ++j) {
          const float p = vv[h][j], q = vv[h + s][j];
          vv[h][j] = __fadd_rn(p, q);
          vv[h + s][j] = __fsub_rn(p, q);
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < HG; ++h)
#pragma unroll
    for (int j = 0; j < C; ++j) vv[h][j] = __fmul_rn(vv[h][j], a.rscale);
  if (a.rope && ok) {
    const uint32_t rs_u = smem_u32(rs);
#pragma unroll
    for (int i = 0; i < C / 4; ++i) {
      const int cc = k * (C / 4) + i;  // table chunk = pairs 2cc, 2cc+1 = channels 4cc..4cc+3
      const uint4 cs = lds128(rs_u + (cc >> 3) * NT * 128 + sw128(t2, cc & 7));
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        rope_fwd(vv[h][4 * i], vv[h][4 * i + 1], __uint_as_float(cs.x), __uint_as_float(cs.y));
        rope_fwd(vv[h][4 * i + 2], vv[h][4 * i + 3], __uint_as_float(cs.z), __uint_as_float(cs.w));
      }
    }
  }
  const bool store = ok && tt2 < a.T;
  const bool sink_tok = m2 < a.n_sink;
  const int g = (k * C) / G;
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    float mn, mx;
    minmax_range<C>(vv[h], 0, C, mn, mx);
#pragma unroll
    for (int off = 1; off < TPG; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    const QParams p = minmax_params<BITS>(mn, mx);
    uint32_t w[(C * BITS + 31) / 32];
#pragma unroll
    for (int i = 0; i < (C * BITS + 31) / 32; ++i) w[i] = 0u;
#pragma unroll
    for (int j = 0; j < C; ++j) {
      const uint32_t c = sink_tok ? 0u : quant_code(vv[h][j], p.Z, p.R);
      const int pos = j * BITS;
      w[pos >> 5] |= c << (pos & 31);
      if ((pos & 31) + BITS > 32) w[(pos >> 5) + 1] |= c >> (32 - (pos & 31));
    }
    if (store) {
      const size_t slot = (static_cast<size_t>(b) * a.H + h_base + h) * a.t_cap + m2;
      st_bytes<NB>(a.codes + slot * RB + k * NB, w);
      if ((k * C) % G == 0) {
        const __half2 zero2 = __halves2half2(__ushort_as_half(0), __ushort_as_half(0));
        a.sz[slot * NG + g] = sink_tok ? zero2 : p.sz;
      }
    }
  }
  if (!ok && tid == 0) mbar_wait(&bar, 0, a.wait_ns, a.err);  // let an in-flight copy land before exiting
}

template <int HG, int BITS, int G>
__global__ void __launch_bounds__(128) k_decode_group(const __grid_constant__ CUtensorMap omap,
                                                       const __grid_constant__ CUtensorMap rmap, const GroupArgs a,
                                                       int out_fp32) {
  constexpr int NT = 128 / HG;
  constexpr int C = D / HG;
  constexpr int NB = C * BITS / 8;
  constexpr int RB = D * BITS / 8;
  constexpr int NG = D / G;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar;
  uint8_t* xs = align1024(smem_raw);  // exchange rows (64 KB), then the output tile over them
  uint8_t* rs = xs + 65536;
  const int tid = threadIdx.x;
  int b, grp, t_base;
  tile_coords(a, b, grp, t_base);
  const int h_base = grp * HG;
  const uint32_t xs_u = smem_u32(xs);

  bool ok = true;
  if (a.rope) {
    if (tid == 0) {
      mbar_init(&bar, 1);
      fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
      mbar_arrive_expect_tx(&bar, NT * D * 4);
      for (int q = 0; q < 4; ++q) tma_load_2d(rs + q * NT * 128, &rmap, q * 32, a.t0 + t_base, &bar);
    }
  }

  // ---------------- phase 2 (reverse): dequantize, inverse RoPE, cross-head strides
  const int t2 = tid / HG, k = tid % HG;
  const int tt2 = t_base + t2, m2 = a.t0 + tt2;
  const bool live2 = tt2 < a.T && m2 >= a.n_sink;
  float vv[HG][C];
  const int g = (k * C) / G;
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    if (live2) {
      const size_t slot = (static_cast<size_t>(b) * a.H + h_base + h) * a.t_cap + m2;
      uint32_t w[(C * BITS + 31) / 32];
      ld_bytes<NB>(a.codes + slot * RB + k * NB, w);
      const __half2 sz = a.sz[slot * NG + g];
      const float S = __low2float(sz), Z = __high2float(sz);
#pragma unroll
      for (int j = 0; j < C; ++j) vv[h][j] = __fmaf_rn(code_to_float(unpack_code<BITS>(w, j)), S, Z);
    } else {
#pragma unroll
      for (int j = 0; j < C; ++j) vv[h][j] = 0.0f;
    }
  }
  if (a.rope) {
    ok = mbar_wait(&bar, 0, a.wait_ns, a.err);
    if (ok) {
      const uint32_t rs_u = smem_u32(rs);
#pragma unroll
      for (int i = 0; i < C / 4; ++i) {
        const int cc = k * (C / 4) + i;
        const uint4 cs = lds128(rs_u + (cc >> 3) * NT * 128 + sw128(t2, cc & 7));
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          rope_inv(vv[h][4 * i], vv[h][4 * i + 1], __uint_as_float(cs.x), __uint_as_float(cs.y));
          rope_inv(vv[h][4 * i + 2], vv[h][4 * i + 3], __uint_as_float(cs.z), __uint_as_float(cs.w));
        }
      }
    }
  }
#pragma unroll
  for (int s = 1; s < HG; s <<= 1) {
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      if ((h & s) == 0) {
#pragma unroll
        for (int j = 0; j < C; ++j) {
          const float p = vv[h][j], q = vv[h + s][j];
          vv[h][j] = __fadd_rn(p, q);
          vv[h + s][j] = __fsub_rn(p, q);
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    const uint32_t row = xs_u + (t2 * HG + h) * 512;
#pragma unroll
    for (int i = 0; i < C / 4; ++i)
      sts128(row + xpos(t2, k * (C / 4) + i) * 16,
             make_uint4(__float_as_uint(vv[h][4 * i]), __float_as_uint(vv[h][4 * i + 1]),
                        __float_as_uint(vv[h][4 * i + 2]), __float_as_uint(vv[h][4 * i + 3])));
  }
  __syncthreads();

  // ---------------- phase 1 (reverse): in-head strides, normalisation, inverse permutation
  const int hl = tid / NT, t = tid % NT;
  const int tt = t_base + t, m = a.t0 + tt;
  const size_t v1 = static_cast<size_t>(b) * a.H + h_base + hl;
  float x[D];
  const uint32_t row = xs_u + (t * HG + hl) * 512;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const uint4 u = lds128(row + xpos(t, c) * 16);
    x[4 * c] = __uint_as_float(u.x);
    x[4 * c + 1] = __uint_as_float(u.y);
    x[4 * c + 2] = __uint_as_float(u.z);
    x[4 * c + 3] = __uint_as_float(u.w);
  }
  fwht_reg<D>(x);
#pragma unroll
  for (int j = 0; j < D; ++j) x[j] = __fmul_rn(x[j], a.rscale);
  if (a.perm) {  // x'[perm[j]] = x[j], through this thread's own exchange row
    const int16_t* pr = a.perm + static_cast<size_t>(h_base + hl) * D;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 pk = __ldg(reinterpret_cast<const uint4*>(pr) + c);
      const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = static_cast<int>((pw[i >> 1] >> (16 * (i & 1))) & (D - 1));
        sts32f(row + xpos(t, e >> 2) * 16 + (e & 3) * 4, x[8 * c + i]);
      }
    }
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const uint4 u = lds128(row + xpos(t, c) * 16);
      x[4 * c] = __uint_as_float(u.x);
      x[4 * c + 1] = __uint_as_float(u.y);
      x[4 * c + 2] = __uint_as_float(u.z);
      x[4 * c + 3] = __uint_as_float(u.w);
    }
  }
  if (tt < a.T && m < a.n_sink) {
    const uint4* src = reinterpret_cast<const uint4*>(a.sink + (v1 * a.n_sink + m) * D);
#pragma unroll
    for (int c = 0; c < 16; ++c) h8_to_f32(__ldg(src + c), &x[8 * c]);
  }
  __syncthreads();  // all exchange reads done: the output tile reuses the space
  if (out_fp32) {
#pragma unroll
    for (int c = 0; c < 32; ++c)
      sts128(xs_u + (c >> 3) * 16384 + sw128(tid, c & 7),
             make_uint4(__float_as_uint(x[4 * c]), __float_as_uint(x[4 * c + 1]), __float_as_uint(x[4 * c + 2]),
                        __float_as_uint(x[4 * c + 3])));
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c) sts128(xs_u + (c >> 3) * 16384 + sw128(tid, c & 7), f32_to_h8(&x[8 * c]));
  }
  fence_async_smem();
  __syncthreads();
  if (tid == 0) {
    if (a.rope && !ok) mbar_wait(&bar, 0, a.wait_ns, a.err);
    const int nbox = out_fp32 ? 4 : 2;
    const int step = out_fp32 ? 32 : 64;
    for (int i = 0; i < nbox; ++i) tma_store_3d(&omap, i * step, t_base, b * a.H + h_base, xs + i * 16384);
    bulk_commit();
    bulk_wait_read0();
  }
}

template <int HG, int BITS, int G>
kvq_status run(bool enc, const GroupArgs& a, const CUtensorMap& m0, const CUtensorMap& rm, size_t smem, int out_fp32,
               cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(static_cast<size_t>(a.B) * a.n_grp * a.n_tblk);
  if (enc) {
    auto k = k_encode_group<HG, BITS, G>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
      return KVQ_ERR_CUDA;
    k<<<grid, 128, smem, st>>>(m0, rm, a);
  } else {
    auto k = k_decode_group<HG, BITS, G>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
      return KVQ_ERR_CUDA;
    k<<<grid, 128, smem, st>>>(m0, rm, a, out_fp32);
  }
  return launch_status();
}

kvq_status dispatch(bool enc, const kvq_desc& d, const GroupArgs& a, const CUtensorMap& m0, const CUtensorMap& rm,
                    size_t smem, int out_fp32, cudaStream_t st) {
#define KVQ_CASE(HG_, B_, G_) \
  if (d.group_heads == HG_ && d.bits == B_ && d.group == G_) return run<HG_, B_, G_>(enc, a, m0, rm, smem, out_fp32, st);
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

GroupArgs make_args(const kvq_desc& d, const kvq_tables& tb, const kvq_packed& p, const LaunchCtx& ctx) {
  GroupArgs a{};
  a.B = d.batch;
  a.H = d.heads;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.t_cap = d.t_cap;
  a.n_sink = d.n_sink;
  a.rope = d.rope;
  a.NT = 128 / d.group_heads;
  a.n_tblk = (d.tokens + a.NT - 1) / a.NT;
  a.n_grp = d.heads / d.group_heads;
  a.rscale = static_cast<float>(1.0 / sqrt(static_cast<double>(d.group_heads) * D));
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
  const uint64_t dims[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(tb.rope_rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(D) * 4};
  const uint32_t box[2] = {32, static_cast<uint32_t>(NT)};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, tb.rope_cs, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t smem_bytes(int NT) { return 1024 + 65536 + static_cast<size_t>(NT) * D * 4; }

}  // namespace

kvq_status launch_encode_group(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                               cudaStream_t st, const LaunchCtx& ctx) {
  const GroupArgs a = make_args(d, tb, out, ctx);
  CUtensorMap xm, rm;
  const uint64_t dims[3] = {D, static_cast<uint64_t>(d.tokens), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t strides[2] = {D * 2, static_cast<uint64_t>(d.tokens) * D * 2};
  const uint32_t box[3] = {64, static_cast<uint32_t>(a.NT), static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&xm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  if (!rope_map(&rm, d, tb, a.NT)) return KVQ_ERR_CUDA;
  return dispatch(true, d, a, xm, rm, smem_bytes(a.NT), 0, st);
}

kvq_status launch_decode_group(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                               int out_fp32, cudaStream_t st, const LaunchCtx& ctx) {
  const GroupArgs a = make_args(d, tb, in, ctx);
  CUtensorMap om, rm;
  const uint64_t es = out_fp32 ? 4 : 2;
  const uint64_t dims[3] = {D, static_cast<uint64_t>(d.tokens), static_cast<uint64_t>(d.batch) * d.heads};
  const uint64_t strides[2] = {D * es, static_cast<uint64_t>(d.tokens) * D * es};
  const uint32_t box[3] = {out_fp32 ? 32u : 64u, static_cast<uint32_t>(a.NT), static_cast<uint32_t>(d.group_heads)};
  if (!make_map(&om, out_fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, x_out, dims,
                strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  if (!rope_map(&rm, d, tb, a.NT)) return KVQ_ERR_CUDA;
  return dispatch(false, d, a, om, rm, smem_bytes(a.NT), out_fp32, st);
}

}  // namespace kvq
