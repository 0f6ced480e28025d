// IsoQuant encode / decode ("KV缓存压缩技术：IsoQuant在大语言模型中的应用",
// §2.2 SO(4) isoclinic decomposition, §3.1 pipeline, §3.2 IsoQuant-Full):
//   rho = ||x||, u = x / (rho + 1e-8), per 4-D block v: w = qL (x) v (x) qR,
//   scalar Lloyd-Max codes against a fixed codebook, LSB-first packing, and
//   rho stored as fp32. Decode applies the inverse rotation and restores rho.
// The 3-D variant (§2.1: T(v) = q v q* on pure quaternions; §1: 3-channel
// blocks leave 42 blocks and a 2-D tail at d = 128) rotates blocks of three
// channels, turns a 2-channel tail in its own plane with the same sandwich
// and keeps a 1-channel tail.
//
// One thread per vector. The quaternion sandwich of block k is applied as
// its matrix, built once per CTA in shared memory: M_k = L(qL_k) R(qR_k)
// (left / right multiplication matrices of the Hamilton product), 16
// multiply-adds per 4-D block instead of two quaternion products, or the 3x3
// vector part of L(q_k) R(q_k*) for the 3-D sandwich. The matrices are
// orthogonal, so the inverse is the transpose. The division by rho + eps is a
// multiplication by its reciprocal. Both reorder fp32 rounding relative to
// the literal sandwich, so a code can differ by one level where w sits
// within a few ulps of a decision boundary.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

struct IsoArgs {
  long long rows;  // B*H*T vectors in this call
  int T, t0, t_cap, n_sink;
  const float* qL;
  const float* qR;
  const float* codebook;
  uint8_t* codes;
  float* norm;
  __half* sink;
  uint32_t* err;
  uint64_t wait_ns;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

// M_k = L(qL) R(qR), row-major 4x4, for k = tid < D/4.
__device__ __forceinline__ void build_m(const float* qL, const float* qR, float* M, int nblk) {
  for (int k = threadIdx.x; k < nblk; k += blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(qL)[k];
    const float4 b = reinterpret_cast<const float4*>(qR)[k];
    const float L[4][4] = {{a.x, -a.y, -a.z, -a.w}, {a.y, a.x, -a.w, a.z}, {a.z, a.w, a.x, -a.y},
                           {a.w, -a.z, a.y, a.x}};
    const float R[4][4] = {{b.x, -b.y, -b.z, -b.w}, {b.y, b.x, b.w, -b.z}, {b.z, -b.w, b.x, b.y},
                           {b.w, b.z, -b.y, b.x}};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float s = __fmul_rn(L[i][0], R[0][j]);
#pragma unroll
        for (int t = 1; t < 4; ++t) s = __fmaf_rn(L[i][t], R[t][j], s);
        M[k * 16 + i * 4 + j] = s;
      }
  }
}

// The 3-D sandwich's matrix of entry k (k < nblk = ceil(D/3)): rows / columns
// i, j channels (i, j, k parts) of L(q) R(q*), row-major 3x3.
__device__ __forceinline__ void build_m3(const float* q, float* M, int nblk) {
  for (int k = threadIdx.x; k < nblk; k += blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(q)[k];
    const float4 b = make_float4(a.x, -a.y, -a.z, -a.w);  // q*
    const float L[4][4] = {{a.x, -a.y, -a.z, -a.w}, {a.y, a.x, -a.w, a.z}, {a.z, a.w, a.x, -a.y},
                           {a.w, -a.z, a.y, a.x}};
    const float R[4][4] = {{b.x, -b.y, -b.z, -b.w}, {b.y, b.x, b.w, -b.z}, {b.z, -b.w, b.x, b.y},
                           {b.w, b.z, -b.y, b.x}};
#pragma unroll
    for (int i = 1; i < 4; ++i)
#pragma unroll
      for (int j = 1; j < 4; ++j) {
        float s = __fmul_rn(L[i][0], R[0][j]);
#pragma unroll
        for (int t = 1; t < 4; ++t) s = __fmaf_rn(L[i][t], R[t][j], s);
        M[k * 9 + (i - 1) * 3 + (j - 1)] = s;
      }
  }
}

// code = number of midpoints strictly below w (binary search)
template <int NL>
__device__ __forceinline__ uint32_t cb_code(float w, const float* beta) {
  uint32_t c = 0;
#pragma unroll
  for (int s = NL / 2; s >= 1; s >>= 1)
    if (w > beta[c + s - 1]) c += s;
  return c;
}

template <int BITS, int NW>
__device__ __forceinline__ void put_code(uint32_t (&w)[NW], int j, uint32_t c) {
  const int pos = j * BITS;
  w[pos >> 5] |= c << (pos & 31);
  if ((pos & 31) + BITS > 32) w[(pos >> 5) + 1] |= c >> (32 - (pos & 31));
}

template <int D, int BITS, bool SO3>
__global__ void __launch_bounds__(128) k_encode_iso(const __grid_constant__ CUtensorMap xmap, const IsoArgs a) {
  constexpr int NB = D / 4;
  constexpr int NB3 = D / 3, TAIL = D % 3;  // 3-D sandwich blocks, tail channels
  constexpr int NL = 1 << BITS;
  constexpr int NW = D * BITS / 32;
  constexpr int RB = D * BITS / 8;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ __align__(16) float Ms[NB * 16];  // holds the 3x3 matrices too (9 * ceil(D/3) < 4 D)
  __shared__ float beta[NL];
  uint8_t* xs = align1024(smem_raw);
  const int tid = threadIdx.x;
  const long long r0 = static_cast<long long>(blockIdx.x) * 128;

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar, D * 256);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) tma_load_2d(xs + hh * 16384, &xmap, hh * 64, static_cast<int>(r0), &bar);
  }
  if constexpr (SO3)
    build_m3(a.qL, Ms, NB3 + (TAIL ? 1 : 0));
  else
    build_m(a.qL, a.qR, Ms, NB);
  if (tid < NL - 1) beta[tid] = __fmul_rn(0.5f, __fadd_rn(a.codebook[tid], a.codebook[tid + 1]));
  __syncthreads();
  if (!mbar_wait(&bar, 0, a.wait_ns, a.err)) {
    if (tid == 0) mbar_wait(&bar, 0, a.wait_ns, a.err);
    return;
  }
  const long long vid = r0 + tid;
  if (vid >= a.rows) return;
  const long long bh = vid / a.T;
  const int tt = static_cast<int>(vid - bh * a.T);
  const int m = a.t0 + tt;
  const size_t slot = static_cast<size_t>(bh) * a.t_cap + m;
  const uint32_t xs_u = smem_u32(xs);
  if (m < a.n_sink) {
    uint4* dst = reinterpret_cast<uint4*>(a.sink + (static_cast<size_t>(bh) * a.n_sink + m) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) dst[c] = lds128(xs_u + (c >> 3) * 16384 + sw128(tid, c & 7));
#pragma unroll
    for (int i = 0; i < RB / 8; ++i) reinterpret_cast<uint2*>(a.codes + slot * RB)[i] = make_uint2(0, 0);
    a.norm[slot] = 0.0f;
    return;
  }
  float x[D];
#pragma unroll
  for (int c = 0; c < D / 8; ++c) h8_to_f32(lds128(xs_u + (c >> 3) * 16384 + sw128(tid, c & 7)), &x[8 * c]);
  // rho from the fp64 sum of squares in channel order (each square is exact in fp64)
  double acc = 0.0;
#pragma unroll
  for (int j = 0; j < D; ++j) acc = __fma_rn(static_cast<double>(x[j]), static_cast<double>(x[j]), acc);
  const float rho = __double2float_rn(__dsqrt_rn(acc));
  const float inv = __frcp_rn(__fadd_rn(rho, 1e-8f));
  uint32_t w[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = 0u;
  if constexpr (!SO3) {
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      float u[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) u[e] = __fmul_rn(x[4 * k + e], inv);
      const float4* Mk = reinterpret_cast<const float4*>(Ms + k * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 row = Mk[i];
        float wi = __fmul_rn(row.x, u[0]);
        wi = __fmaf_rn(row.y, u[1], wi);
        wi = __fmaf_rn(row.z, u[2], wi);
        wi = __fmaf_rn(row.w, u[3], wi);
        put_code<BITS, NW>(w, 4 * k + i, cb_code<NL>(wi, beta));
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < NB3; ++k) {
      float u[3];
#pragma unroll
      for (int e = 0; e < 3; ++e) u[e] = __fmul_rn(x[3 * k + e], inv);
      const float* Mk = Ms + k * 9;
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        float wi = __fmul_rn(Mk[3 * i], u[0]);
        wi = __fmaf_rn(Mk[3 * i + 1], u[1], wi);
        wi = __fmaf_rn(Mk[3 * i + 2], u[2], wi);
        put_code<BITS, NW>(w, 3 * k + i, cb_code<NL>(wi, beta));
      }
    }
    if constexpr (TAIL == 2) {  // the tail in its own plane: the matrix's upper-left 2x2 block
      const float u0 = __fmul_rn(x[D - 2], inv), u1 = __fmul_rn(x[D - 1], inv);
      const float* Mk = Ms + NB3 * 9;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float wi = __fmaf_rn(Mk[3 * i + 1], u1, __fmul_rn(Mk[3 * i], u0));
        put_code<BITS, NW>(w, D - 2 + i, cb_code<NL>(wi, beta));
      }
    } else if constexpr (TAIL == 1) {  // a single channel is kept
      put_code<BITS, NW>(w, D - 1, cb_code<NL>(__fmul_rn(x[D - 1], inv), beta));
    }
  }
  uint8_t* dst = a.codes + slot * RB;
  if constexpr (RB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < RB / 16; ++i)
      reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < RB / 8; ++i) reinterpret_cast<uint2*>(dst)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
  }
  a.norm[slot] = rho;
}

template <int D, int BITS, bool SO3>
__global__ void __launch_bounds__(128) k_decode_iso(const __grid_constant__ CUtensorMap omap, const IsoArgs a,
                                                     int out_fp32) {
  constexpr int NB = D / 4;
  constexpr int NB3 = D / 3, TAIL = D % 3;
  constexpr int NL = 1 << BITS;
  constexpr int NW = D * BITS / 32;
  constexpr int RB = D * BITS / 8;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(16) float Ms[NB * 16];
  __shared__ float lv[NL];
  uint8_t* os = align1024(smem_raw);
  const int tid = threadIdx.x;
  const long long r0 = static_cast<long long>(blockIdx.x) * 128;
  if constexpr (SO3)
    build_m3(a.qL, Ms, NB3 + (TAIL ? 1 : 0));
  else
    build_m(a.qL, a.qR, Ms, NB);
  if (tid < NL) lv[tid] = a.codebook[tid];
  __syncthreads();
  const long long vid = r0 + tid;
  float x[D];
  if (vid < a.rows) {
    const long long bh = vid / a.T;
    const int tt = static_cast<int>(vid - bh * a.T);
    const int m = a.t0 + tt;
    const size_t slot = static_cast<size_t>(bh) * a.t_cap + m;
    if (m < a.n_sink) {
      const uint4* src = reinterpret_cast<const uint4*>(a.sink + (static_cast<size_t>(bh) * a.n_sink + m) * D);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) h8_to_f32(__ldg(src + c), &x[8 * c]);
    } else {
      uint32_t w[NW];
      const uint8_t* srcb = a.codes + slot * RB;
      if constexpr (RB % 16 == 0) {
#pragma unroll
        for (int i = 0; i < RB / 16; ++i) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(srcb) + i);
          w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < RB / 8; ++i) {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(srcb) + i);
          w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
      }
      const float rho = a.norm[slot];
      if constexpr (!SO3) {
#pragma unroll
        for (int k = 0; k < NB; ++k) {
          float wh[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) wh[e] = lv[unpack_code<BITS, NW>(w, 4 * k + e)];
          const float* Mk = Ms + k * 16;
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // v = M^T w
            float vi = __fmul_rn(Mk[i], wh[0]);
            vi = __fmaf_rn(Mk[4 + i], wh[1], vi);
            vi = __fmaf_rn(Mk[8 + i], wh[2], vi);
            vi = __fmaf_rn(Mk[12 + i], wh[3], vi);
            x[4 * k + i] = __fmul_rn(vi, rho);
          }
        }
      } else {
#pragma unroll
        for (int k = 0; k < NB3; ++k) {
          float wh[3];
#pragma unroll
          for (int e = 0; e < 3; ++e) wh[e] = lv[unpack_code<BITS, NW>(w, 3 * k + e)];
          const float* Mk = Ms + k * 9;
#pragma unroll
          for (int i = 0; i < 3; ++i) {  // v = M^T w
            float vi = __fmul_rn(Mk[i], wh[0]);
            vi = __fmaf_rn(Mk[3 + i], wh[1], vi);
            vi = __fmaf_rn(Mk[6 + i], wh[2], vi);
            x[3 * k + i] = __fmul_rn(vi, rho);
          }
        }
        if constexpr (TAIL == 2) {
          const float w0 = lv[unpack_code<BITS, NW>(w, D - 2)], w1 = lv[unpack_code<BITS, NW>(w, D - 1)];
          const float* Mk = Ms + NB3 * 9;
#pragma unroll
          for (int i = 0; i < 2; ++i)
            x[D - 2 + i] = __fmul_rn(__fmaf_rn(Mk[3 + i], w1, __fmul_rn(Mk[i], w0)), rho);
        } else if constexpr (TAIL == 1) {
          x[D - 1] = __fmul_rn(lv[unpack_code<BITS, NW>(w, D - 1)], rho);
        }
      }
    }
    const uint32_t os_u = smem_u32(os);
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
  if (tid == 0) {
    const int nbox = out_fp32 ? D / 32 : D / 64;
    const int step = out_fp32 ? 32 : 64;
    for (int i = 0; i < nbox; ++i) tma_store_2d(&omap, i * step, static_cast<int>(r0), os + i * 16384);
    bulk_commit();
    bulk_wait_read0();
  }
}

IsoArgs make_args(const kvq_desc& d, const kvq_tables& tb, const kvq_packed& p, const LaunchCtx& ctx) {
  IsoArgs a{};
  a.rows = static_cast<long long>(d.batch) * d.heads * d.tokens;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.t_cap = d.t_cap;
  a.n_sink = d.n_sink;
  a.qL = tb.qL;
  a.qR = tb.qR;
  a.codebook = tb.codebook;
  a.codes = p.codes;
  a.norm = p.norm;
  a.sink = static_cast<__half*>(p.sink);
  a.err = ctx.err;
  a.wait_ns = ctx.wait_ns;
  return a;
}

template <int D, int BITS, bool SO3>
kvq_status run(bool enc, const IsoArgs& a, const CUtensorMap& m0, int out_fp32, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((a.rows + 127) / 128);
  if (enc) {
    const size_t smem = 1024 + D * 256;
    auto k = k_encode_iso<D, BITS, SO3>;
    if (!set_smem_once(reinterpret_cast<const void*>(k), smem))
      return KVQ_ERR_CUDA;
    k<<<grid, 128, smem, st>>>(m0, a);
  } else {
    const size_t smem = 1024 + D * 512;
    auto k = k_decode_iso<D, BITS, SO3>;
    if (!set_smem_once(reinterpret_cast<const void*>(k), smem))
      return KVQ_ERR_CUDA;
    k<<<grid, 128, smem, st>>>(m0, a, out_fp32);
  }
  return launch_status();
}

kvq_status dispatch(bool enc, const kvq_desc& d, const IsoArgs& a, const CUtensorMap& m0, int out_fp32,
                    cudaStream_t st) {
#define KVQ_CASE(D_, B_)                                                                  \
  if (d.head_dim == D_ && d.bits == B_)                                                   \
    return d.rot == KVQ_ROT_ISO_SO3 ? run<D_, B_, true>(enc, a, m0, out_fp32, st)         \
                                    : run<D_, B_, false>(enc, a, m0, out_fp32, st);
  KVQ_CASE(128, 2)
  KVQ_CASE(128, 3)
  KVQ_CASE(128, 4)
  KVQ_CASE(64, 2)
  KVQ_CASE(64, 3)
  KVQ_CASE(64, 4)
#undef KVQ_CASE
  return KVQ_ERR_UNSUPPORTED;
}

}  // namespace

kvq_status launch_encode_iso(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                             cudaStream_t st, const LaunchCtx& ctx) {
  const IsoArgs a = make_args(d, tb, out, ctx);
  if (a.rows > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  CUtensorMap xm;
  const uint64_t dims[2] = {static_cast<uint64_t>(d.head_dim), static_cast<uint64_t>(a.rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(d.head_dim) * 2};
  const uint32_t box[2] = {64, 128};
  if (!make_map(&xm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  return dispatch(true, d, a, xm, 0, st);
}

kvq_status launch_decode_iso(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                             int out_fp32, cudaStream_t st, const LaunchCtx& ctx) {
  const IsoArgs a = make_args(d, tb, in, ctx);
  if (a.rows > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  CUtensorMap om;
  const uint64_t es = out_fp32 ? 4 : 2;
  const uint64_t dims[2] = {static_cast<uint64_t>(d.head_dim), static_cast<uint64_t>(a.rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(d.head_dim) * es};
  const uint32_t box[2] = {out_fp32 ? 32u : 64u, 128};
  if (!make_map(&om, out_fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x_out, dims,
                strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return KVQ_ERR_CUDA;
  return dispatch(false, d, a, om, out_fp32, st);
}

}  // namespace kvq
