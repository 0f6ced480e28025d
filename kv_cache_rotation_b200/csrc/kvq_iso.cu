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
//
// Dynamic codebooks (§4.2: per-channel statistics, boundaries set by the KL
// divergence, twice the codebook for outlier channels): channel j of head h
// quantizes against the levels fp32(sigma[h][j] * l_k) of the N(0,1)
// Lloyd-Max design l (2^bits levels, or 2^(bits+1) for the channels marked in
// ch_wide), with fp32 midpoints as boundaries; the top bit of each outlier
// channel's code goes to a per-slot 16-bit word. sigma is the square root of
// the channel's mean square over the calibration tokens, the minimiser of the
// KL divergence from the channel's values to N(0, sigma^2): k_dyn_stats sums
// the squares of the rotated values per (sequence, head, 1024-token chunk) in
// a fixed order, k_dyn_finish adds the chunks in order and marks the outlier
// channels (sigma > 2 x the lower median, at most D/8).
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

struct IsoArgs {
  long long rows;  // B*H*T vectors in this call
  int H, T, t0, t_cap, n_sink;
  const float* qL;
  const float* qR;
  const float* codebook;  // fixed: the levels; dynamic: the 2^bits N(0,1) levels
  const float* cb_wide;   // dynamic: the 2^(bits+1) N(0,1) levels
  const float* ch_scale;  // dynamic: [H][D]
  const uint32_t* ch_wide;  // dynamic: [H][D/32]
  uint8_t* codes;
  float* norm;
  uint16_t* ext;  // dynamic: [B][H][t_cap]
  __half* sink;
  uint32_t* err;
  uint64_t wait_ns;
};

constexpr int kStatChunk = 1024;  // tokens per k_dyn_stats CTA

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

// The same search over boundaries held in registers (NL <= 8): each step's
// boundary is chosen by selects on the bits found so far, so there is no
// data-dependent shared-memory load.
template <int NL>
__device__ __forceinline__ uint32_t cb_code_reg(float w, const float (&b)[NL > 1 ? NL - 1 : 1]) {
  static_assert(NL == 4 || NL == 8, "2- or 3-bit codes");
  if constexpr (NL == 4) {
    const bool hi = w > b[1];
    const bool lo = w > (hi ? b[2] : b[0]);
    return (hi ? 2u : 0u) + (lo ? 1u : 0u);
  } else {
    const bool b2 = w > b[3];
    const bool b1 = w > (b2 ? b[5] : b[1]);
    const float t = b2 ? (b1 ? b[6] : b[4]) : (b1 ? b[2] : b[0]);
    const bool b0 = w > t;
    return (b2 ? 4u : 0u) + (b1 ? 2u : 0u) + (b0 ? 1u : 0u);
  }
}

// Dynamic codebook: code of w against the levels fp32(s * lv[k]) with fp32
// midpoints as boundaries (ties to the lower code).
template <int NL>
__device__ __forceinline__ uint32_t dyn_code(float w, float s, const float* lv) {
  uint32_t c = 0;
#pragma unroll
  for (int st = NL / 2; st >= 1; st >>= 1) {
    const float a = __fmul_rn(s, lv[c + st - 1]), b = __fmul_rn(s, lv[c + st]);
    if (w > __fmul_rn(0.5f, __fadd_rn(a, b))) c += st;
  }
  return c;
}

// The rotated unit vector: w = M_k (x * inv) per block (4-D, or 3-D with its
// tail), handed to emit(j, w_j) in ascending channel order.
template <int D, bool SO3, class Emit>
__device__ __forceinline__ void iso_rotate(const float (&x)[D], float inv, const float* Ms, Emit&& emit) {
  constexpr int NB = D / 4;
  constexpr int NB3 = D / 3, TAIL = D % 3;
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
        emit(4 * k + i, wi);
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
        emit(3 * k + i, wi);
      }
    }
    if constexpr (TAIL == 2) {  // the tail in its own plane: the matrix's upper-left 2x2 block
      const float u0 = __fmul_rn(x[D - 2], inv), u1 = __fmul_rn(x[D - 1], inv);
      const float* Mk = Ms + NB3 * 9;
#pragma unroll
      for (int i = 0; i < 2; ++i) emit(D - 2 + i, __fmaf_rn(Mk[3 * i + 1], u1, __fmul_rn(Mk[3 * i], u0)));
    } else if constexpr (TAIL == 1) {  // a single channel is kept
      emit(D - 1, __fmul_rn(x[D - 1], inv));
    }
  }
}

// iso_rotate on a row read chunk by chunk (ld(c, v) fills v[0..7] with the
// channels 8c .. 8c+7): the same operations in the same order, with only the
// channels of the current blocks live in registers. 4-D blocks take one chunk
// per two blocks; 3-D blocks take three chunks per eight blocks, then the
// remaining channels (two or five blocks and the tail).
template <int D, bool SO3, class Ld, class Emit>
__device__ __forceinline__ void iso_rotate_chunks(Ld&& ld, float inv, const float* Ms, Emit&& emit) {
  if constexpr (!SO3) {
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      float v[8];
      ld(c, v);
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        const int k = 2 * c + kb;
        float u[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) u[e] = __fmul_rn(v[4 * kb + e], inv);
        const float4* Mk = reinterpret_cast<const float4*>(Ms + k * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 row = Mk[i];
          float wi = __fmul_rn(row.x, u[0]);
          wi = __fmaf_rn(row.y, u[1], wi);
          wi = __fmaf_rn(row.z, u[2], wi);
          wi = __fmaf_rn(row.w, u[3], wi);
          emit(4 * k + i, wi);
        }
      }
    }
  } else {
    constexpr int NG = D / 24;           // groups of 24 channels = 8 blocks
    constexpr int R0 = 24 * NG, RN = D - R0, RB = RN / 3, TAIL = D % 3;
    auto block3 = [&](int k, const float* v3) {  // channels 3k .. 3k+2 from v3[0..2]
      float u[3];
#pragma unroll
      for (int e = 0; e < 3; ++e) u[e] = __fmul_rn(v3[e], inv);
      const float* Mk = Ms + k * 9;
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        float wi = __fmul_rn(Mk[3 * i], u[0]);
        wi = __fmaf_rn(Mk[3 * i + 1], u[1], wi);
        wi = __fmaf_rn(Mk[3 * i + 2], u[2], wi);
        emit(3 * k + i, wi);
      }
    };
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float v[24];
      ld(3 * g, v);
      ld(3 * g + 1, v + 8);
      ld(3 * g + 2, v + 16);
#pragma unroll
      for (int kb = 0; kb < 8; ++kb) block3(8 * g + kb, v + 3 * kb);
    }
    float v[RN];
#pragma unroll
    for (int c = 0; c < RN / 8; ++c) ld(R0 / 8 + c, v + 8 * c);
#pragma unroll
    for (int kb = 0; kb < RB; ++kb) block3(8 * NG + kb, v + 3 * kb);
    if constexpr (TAIL == 2) {  // the tail in its own plane: the matrix's upper-left 2x2 block
      const float u0 = __fmul_rn(v[RN - 2], inv), u1 = __fmul_rn(v[RN - 1], inv);
      const float* Mk = Ms + (D / 3) * 9;
#pragma unroll
      for (int i = 0; i < 2; ++i) emit(D - 2 + i, __fmaf_rn(Mk[3 * i + 1], u1, __fmul_rn(Mk[3 * i], u0)));
    } else if constexpr (TAIL == 1) {  // a single channel is kept
      emit(D - 1, __fmul_rn(v[RN - 1], inv));
    }
  }
}

// iso_norm on a row read chunk by chunk (the same sum in the same order).
template <int D, class Ld>
__device__ __forceinline__ float iso_norm_chunks(Ld&& ld, float& inv) {
  double acc = 0.0;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    float v[8];
    ld(c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc = __fma_rn(static_cast<double>(v[i]), static_cast<double>(v[i]), acc);
  }
  const float rho = __double2float_rn(__dsqrt_rn(acc));
  inv = __frcp_rn(__fadd_rn(rho, 1e-8f));
  return rho;
}

// rho = ||x|| from the fp64 sum of squares in channel order (each square is
// exact in fp64), and the reciprocal of rho + 1e-8.
template <int D>
__device__ __forceinline__ float iso_norm(const float (&x)[D], float& inv) {
  double acc = 0.0;
#pragma unroll
  for (int j = 0; j < D; ++j) acc = __fma_rn(static_cast<double>(x[j]), static_cast<double>(x[j]), acc);
  const float rho = __double2float_rn(__dsqrt_rn(acc));
  inv = __frcp_rn(__fadd_rn(rho, 1e-8f));
  return rho;
}

// Dynamic codebooks: the head shared by all of this CTA's vectors (rows r0 ..
// r0 + 127, ordered (batch, head, token)), or -1 when they span two heads.
__device__ __forceinline__ int cta_head(const IsoArgs& a, long long r0) {
  const long long last = min(r0 + 127, a.rows - 1);
  const long long bh0 = r0 / a.T, bh1 = last / a.T;
  return (a.H == 1 || bh0 == bh1) ? static_cast<int>(bh0 % a.H) : -1;
}

// Per-channel tables of head h in shared memory, row pitch 2 NL floats:
// encode (LEVELS = false) the boundaries fp32(0.5 (L_k + L_k+1)), decode
// (LEVELS = true) the levels L_k = fp32(sigma_j l_k) -- the same fp32 values
// dyn_code and the decode's level() form one by one.
template <int D, int NL, bool LEVELS>
__device__ __forceinline__ void dyn_tables(const IsoArgs& a, int h, const float* lv, const float* lvw, float* tab) {
  const float* sc = a.ch_scale + static_cast<size_t>(h) * D;
  const uint32_t* wd = a.ch_wide + static_cast<size_t>(h) * (D / 32);
  for (int e = threadIdx.x; e < D * 2 * NL; e += blockDim.x) {
    const int j = e / (2 * NL), k = e % (2 * NL);
    const bool wide = (__ldg(wd + (j >> 5)) >> (j & 31)) & 1u;
    const int n = wide ? 2 * NL : NL;
    const float* l = wide ? lvw : lv;
    const float sj = __ldg(sc + j);
    float v = 0.0f;
    if (LEVELS) {
      if (k < n) v = __fmul_rn(sj, l[k]);
    } else if (k + 1 < n) {
      v = __fmul_rn(0.5f, __fadd_rn(__fmul_rn(sj, l[k]), __fmul_rn(sj, l[k + 1])));
    }
    tab[e] = v;
  }
}

template <bool SO3>
__device__ __forceinline__ void build_mats(const IsoArgs& a, float* Ms, int D) {
  if constexpr (SO3)
    build_m3(a.qL, Ms, D / 3 + (D % 3 ? 1 : 0));
  else
    build_m(a.qL, a.qR, Ms, D / 4);
}

template <int BITS, int NW>
__device__ __forceinline__ void put_code(uint32_t (&w)[NW], int j, uint32_t c) {
  const int pos = j * BITS;
  w[pos >> 5] |= c << (pos & 31);
  if ((pos & 31) + BITS > 32) w[(pos >> 5) + 1] |= c >> (32 - (pos & 31));
}

// DYN: 0 fixed codebook; 1 dynamic, channel levels formed per element; 2
// dynamic, the channel boundaries / levels of the CTA's one head in shared
// memory (the host picks 2 when no CTA spans two heads: H = 1 or T % 128 = 0).
template <int D, int BITS, bool SO3, int DYN>
__global__ void __launch_bounds__(128) k_encode_iso(const __grid_constant__ CUtensorMap xmap, const IsoArgs a) {
  constexpr int NB = D / 4;
  constexpr int NL = 1 << BITS;
  constexpr int NW = D * BITS / 32;
  constexpr int RB = D * BITS / 8;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ __align__(16) float Ms[NB * 16];  // holds the 3x3 matrices too (9 * ceil(D/3) < 4 D)
  __shared__ float beta[NL];    // fixed: the midpoints; dynamic: the N(0,1) levels
  __shared__ float lvw[2 * NL];  // dynamic: the wide N(0,1) levels
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
  build_mats<SO3>(a, Ms, D);
  float* tab = reinterpret_cast<float*>(xs + D * 256);  // DYN == 2: the channel boundaries
  if constexpr (DYN != 0) {
    if (tid < NL) beta[tid] = a.codebook[tid];
    if (tid < 2 * NL) lvw[tid] = a.cb_wide[tid];
    if constexpr (DYN == 2) {
      __syncthreads();
      dyn_tables<D, NL, false>(a, cta_head(a, r0), beta, lvw, tab);
    }
  } else {
    if (tid < NL - 1) beta[tid] = __fmul_rn(0.5f, __fadd_rn(a.codebook[tid], a.codebook[tid + 1]));
  }
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
    if constexpr (DYN != 0) a.ext[slot] = 0;
    return;
  }
  // the staged row is read from shared memory twice (norm, then rotation), so
  // only a few channels are live in registers at a time
  auto ld = [&](int c, float* v) { h8_to_f32(lds128(xs_u + (c >> 3) * 16384 + sw128(tid, c & 7)), v); };
  float inv;
  const float rho = iso_norm_chunks<D>(ld, inv);
  // keep the second pass's shared-memory loads after the norm (they would
  // otherwise be hoisted and hold the whole row in registers again)
  asm volatile("" : "+f"(inv));
  uint32_t w[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = 0u;
  if constexpr (DYN == 0) {
    if constexpr (NL <= 8) {  // the boundaries in registers
      float br[NL - 1];
#pragma unroll
      for (int k = 0; k < NL - 1; ++k) br[k] = beta[k];
      iso_rotate_chunks<D, SO3>(ld, inv, Ms,
                                [&](int j, float wj) { put_code<BITS, NW>(w, j, cb_code_reg<NL>(wj, br)); });
    } else {
      iso_rotate_chunks<D, SO3>(ld, inv, Ms, [&](int j, float wj) { put_code<BITS, NW>(w, j, cb_code<NL>(wj, beta)); });
    }
  } else {
    const int h = static_cast<int>(bh % a.H);
    const float* sc = a.ch_scale + static_cast<size_t>(h) * D;
    uint32_t wd[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) wd[i] = __ldg(a.ch_wide + static_cast<size_t>(h) * (D / 32) + i);
    uint32_t ext = 0;
    int nw = 0;
    iso_rotate_chunks<D, SO3>(ld, inv, Ms, [&](int j, float wj) {
      uint32_t c;
      const bool wide = (wd[j >> 5] >> (j & 31)) & 1u;
      if constexpr (DYN == 2) {  // the channel's boundaries from shared memory
        // one code path for both codebook sizes: the wide channels take the first
        // step of the 2 NL search (boundary NL - 1), then both run the NL steps
        const float* row = tab + j * 2 * NL;
        c = (wide && wj > row[NL - 1]) ? static_cast<uint32_t>(NL) : 0u;
#pragma unroll
        for (int st = NL / 2; st >= 1; st >>= 1)
          if (wj > row[c + st - 1]) c += st;
      } else {
        const float sj = __ldg(sc + j);
        c = wide ? dyn_code<2 * NL>(wj, sj, lvw) : dyn_code<NL>(wj, sj, beta);
      }
      if (wide) {
        if (nw < 16) ext |= (c >> BITS) << nw;
        ++nw;
        c &= NL - 1;
      }
      put_code<BITS, NW>(w, j, c);
    });
    a.ext[slot] = static_cast<uint16_t>(ext);
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

template <int D, int BITS, bool SO3, int DYN>
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
  __shared__ float lvw[2 * NL];  // dynamic: the wide N(0,1) levels
  uint8_t* os = align1024(smem_raw);
  const int tid = threadIdx.x;
  const long long r0 = static_cast<long long>(blockIdx.x) * 128;
  build_mats<SO3>(a, Ms, D);
  if (tid < NL) lv[tid] = a.codebook[tid];
  // DYN == 2: the channel levels, after the output tile (fp32: D * 512 bytes, fp16: D * 256)
  float* tab = reinterpret_cast<float*>(os + D * (out_fp32 ? 512 : 256));
  if constexpr (DYN != 0) {
    if (tid < 2 * NL) lvw[tid] = a.cb_wide[tid];
    if constexpr (DYN == 2) {
      __syncthreads();
      dyn_tables<D, NL, true>(a, cta_head(a, r0), lv, lvw, tab);
    }
  }
  __syncthreads();
  const long long vid = r0 + tid;
  if (vid < a.rows) {
    const long long bh = vid / a.T;
    const int tt = static_cast<int>(vid - bh * a.T);
    const int m = a.t0 + tt;
    const size_t slot = static_cast<size_t>(bh) * a.t_cap + m;
    const uint32_t os_u = smem_u32(os);
    // chunk c = channels 8c .. 8c+7 of this thread's output row, into the tile
    auto st = [&](int c, const float* v) {
      if (out_fp32) {
        sts128(os_u + ((2 * c) >> 3) * 16384 + sw128(tid, (2 * c) & 7),
               make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3])));
        sts128(os_u + ((2 * c + 1) >> 3) * 16384 + sw128(tid, (2 * c + 1) & 7),
               make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]), __float_as_uint(v[7])));
      } else {
        sts128(os_u + (c >> 3) * 16384 + sw128(tid, c & 7), f32_to_h8(v));
      }
    };
    if (m < a.n_sink) {
      const uint4* src = reinterpret_cast<const uint4*>(a.sink + (static_cast<size_t>(bh) * a.n_sink + m) * D);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        float v[8];
        h8_to_f32(__ldg(src + c), v);
        st(c, v);
      }
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
      // level of channel j (called in ascending channel order)
      const float* sc = nullptr;
      uint32_t wd[D / 32], ext = 0;
      int nw = 0;
      if constexpr (DYN != 0) {
        const int h = static_cast<int>(bh % a.H);
        sc = a.ch_scale + static_cast<size_t>(h) * D;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) wd[i] = __ldg(a.ch_wide + static_cast<size_t>(h) * (D / 32) + i);
        ext = a.ext[slot];
      }
      auto level = [&](int j) -> float {
        uint32_t c = unpack_code<BITS, NW>(w, j);
        if constexpr (DYN == 0) {
          return lv[c];
        } else {
          const bool wide = (wd[j >> 5] >> (j & 31)) & 1u;
          if (wide) {
            if (nw < 16) c |= ((ext >> nw) & 1u) << BITS;
            ++nw;
          }
          if constexpr (DYN == 2) return tab[j * 2 * NL + c];
          const float sj = __ldg(sc + j);
          return __fmul_rn(sj, wide ? lvw[c] : lv[c]);
        }
      };
      if constexpr (!SO3) {
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {  // blocks 2c, 2c+1
          float x8[8];
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
            const int k = 2 * c + kb;
            float wh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) wh[e] = level(4 * k + e);
            const float* Mk = Ms + k * 16;
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // v = M^T w
              float vi = __fmul_rn(Mk[i], wh[0]);
              vi = __fmaf_rn(Mk[4 + i], wh[1], vi);
              vi = __fmaf_rn(Mk[8 + i], wh[2], vi);
              vi = __fmaf_rn(Mk[12 + i], wh[3], vi);
              x8[4 * kb + i] = __fmul_rn(vi, rho);
            }
          }
          st(c, x8);
        }
      } else {
        constexpr int NG = D / 24;  // groups of 24 channels = 8 blocks
        constexpr int R0 = 24 * NG, RN = D - R0, RB3 = RN / 3;
        auto block3 = [&](int k, float* x3) {  // channels 3k .. 3k+2 into x3[0..2]
          float wh[3];
#pragma unroll
          for (int e = 0; e < 3; ++e) wh[e] = level(3 * k + e);
          const float* Mk = Ms + k * 9;
#pragma unroll
          for (int i = 0; i < 3; ++i) {  // v = M^T w
            float vi = __fmul_rn(Mk[i], wh[0]);
            vi = __fmaf_rn(Mk[3 + i], wh[1], vi);
            vi = __fmaf_rn(Mk[6 + i], wh[2], vi);
            x3[i] = __fmul_rn(vi, rho);
          }
        };
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          float x24[24];
#pragma unroll
          for (int kb = 0; kb < 8; ++kb) block3(8 * g + kb, x24 + 3 * kb);
          st(3 * g, x24);
          st(3 * g + 1, x24 + 8);
          st(3 * g + 2, x24 + 16);
        }
        float xr[RN];
#pragma unroll
        for (int kb = 0; kb < RB3; ++kb) block3(8 * NG + kb, xr + 3 * kb);
        if constexpr (TAIL == 2) {
          const float w0 = level(D - 2);
          const float w1 = level(D - 1);
          const float* Mk = Ms + NB3 * 9;
#pragma unroll
          for (int i = 0; i < 2; ++i) xr[RN - 2 + i] = __fmul_rn(__fmaf_rn(Mk[3 + i], w1, __fmul_rn(Mk[i], w0)), rho);
        } else if constexpr (TAIL == 1) {
          xr[RN - 1] = __fmul_rn(level(D - 1), rho);
        }
#pragma unroll
        for (int c = 0; c < RN / 8; ++c) st(R0 / 8 + c, xr + 8 * c);
      }
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

// ------------------------------------------------------- dynamic statistics
struct DynStatArgs {
  int H, T, t0, n_sink, nchunk;
  const __half* x;
  const int32_t* sink_pos;  // [B][n_sink] or nullptr (positions < n_sink)
  const float* qL;
  const float* qR;
  double* part;  // [B*H][nchunk][D] sums of squares
  int* cnt;      // [B*H][nchunk] vectors counted
};

// Sum over the CTA's tokens of w_j^2 (fp64, token order) for every channel:
// the rotated rows go through shared memory (pitch D + 1 words, so the row
// writes and the column reads are both conflict-free); thread j adds column j.
template <int D, bool SO3>
__global__ void __launch_bounds__(128) k_dyn_stats(const DynStatArgs a) {
  extern __shared__ float wsm[];  // [128][D + 1]
  __shared__ __align__(16) float Ms[D * 4];
  const int tid = threadIdx.x;
  const int bh = blockIdx.y, b = bh / a.H;
  IsoArgs ia{};
  ia.qL = a.qL;
  ia.qR = a.qR;
  build_mats<SO3>(ia, Ms, D);
  __syncthreads();
  const int tbeg = blockIdx.x * kStatChunk;
  const int tend = min(tbeg + kStatChunk, a.T);
  double acc = 0.0;
  int cnt = 0;
  for (int tc = tbeg; tc < tend; tc += 128) {  // the same trip count for every thread
    const int t = tc + tid;
    bool live = t < tend;
    if (live) {
      const int pos = a.t0 + t;
      if (!a.sink_pos) {
        live = pos >= a.n_sink;
      } else {
        for (int k = 0; k < a.n_sink; ++k) live &= __ldg(a.sink_pos + static_cast<size_t>(b) * a.n_sink + k) != pos;
      }
    }
    float* row = wsm + tid * (D + 1);
    if (live) {
      float x[D];
      const uint4* src = reinterpret_cast<const uint4*>(a.x + (static_cast<size_t>(bh) * a.T + t) * D);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) h8_to_f32(__ldg(src + c), &x[8 * c]);
      float inv;
      (void)iso_norm<D>(x, inv);
      iso_rotate<D, SO3>(x, inv, Ms, [&](int j, float wj) { row[j] = wj; });
    } else {
#pragma unroll 8
      for (int j = 0; j < D; ++j) row[j] = 0.0f;
    }
    cnt += __syncthreads_count(live);
    if (tid < D)
      for (int r = 0; r < 128; ++r) {
        const double v = static_cast<double>(wsm[r * (D + 1) + tid]);
        acc = __fma_rn(v, v, acc);
      }
    __syncthreads();
  }
  const size_t pr = static_cast<size_t>(bh) * a.nchunk + blockIdx.x;
  if (tid < D) a.part[pr * D + tid] = acc;
  if (tid == 0) a.cnt[pr] = cnt;
}

// One CTA of D threads per head: the chunk sums in order, sigma, the lower
// median of the head's sigmas, and the outlier mask (sigma > 2 x median, the
// D/8 largest at most, equal sigmas to the lower channel).
template <int D>
__global__ void __launch_bounds__(D) k_dyn_finish(int B, int H, int nchunk, const double* part, const int* cnt,
                                                  float* ch_scale, uint32_t* ch_wide) {
  __shared__ float sg[D];
  __shared__ float med;
  const int h = blockIdx.x, j = threadIdx.x;
  double s = 0.0;
  long long n = 0;
  for (int b = 0; b < B; ++b)
    for (int c = 0; c < nchunk; ++c) {
      const size_t r = (static_cast<size_t>(b) * H + h) * nchunk + c;
      s = __dadd_rn(s, part[r * D + j]);
      n += cnt[r];
    }
  const float sigma = n > 0 ? __double2float_rn(__dsqrt_rn(__ddiv_rn(s, static_cast<double>(n))))
                            : __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(static_cast<double>(D))));
  sg[j] = sigma;
  __syncthreads();
  int below = 0, above = 0;
  for (int k = 0; k < D; ++k) {
    const float v = sg[k];
    below += v < sigma || (v == sigma && k < j);
    above += v > sigma || (v == sigma && k < j);
  }
  if (below == (D - 1) / 2) med = sigma;
  __syncthreads();
  const bool wide = sigma > __fmul_rn(2.0f, med) && above < D / 8;
  const uint32_t word = __ballot_sync(0xffffffffu, wide);
  ch_scale[static_cast<size_t>(h) * D + j] = sigma;
  if ((j & 31) == 0) ch_wide[static_cast<size_t>(h) * (D / 32) + (j >> 5)] = word;
}

IsoArgs make_args(const kvq_desc& d, const kvq_tables& tb, const kvq_packed& p, const LaunchCtx& ctx) {
  IsoArgs a{};
  a.rows = static_cast<long long>(d.batch) * d.heads * d.tokens;
  a.H = d.heads;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.t_cap = d.t_cap;
  a.n_sink = d.n_sink;
  a.qL = tb.qL;
  a.qR = tb.qR;
  a.codebook = tb.codebook;
  a.cb_wide = tb.codebook_wide;
  a.ch_scale = tb.ch_scale;
  a.ch_wide = tb.ch_wide;
  a.codes = p.codes;
  a.norm = p.norm;
  a.ext = p.ext;
  a.sink = static_cast<__half*>(p.sink);
  a.err = ctx.err;
  a.wait_ns = ctx.wait_ns;
  return a;
}

template <int D, int BITS, bool SO3, int DYN>
kvq_status run(bool enc, const IsoArgs& a, const CUtensorMap& m0, int out_fp32, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((a.rows + 127) / 128);
  // dynamic codebooks: the channel table after the staging tile, D rows of
  // 2 NL = 2^(BITS+1) floats (dyn_tables writes entries 0 .. D * 2 NL - 1;
  // lookups read row j at most entry 2 NL - 1); the 1024 bytes cover align1024
  constexpr size_t kTab = DYN == 2 ? static_cast<size_t>(D) * (2 << BITS) * sizeof(float) : 0;
  if (enc) {
    const size_t smem = 1024 + D * 256 + kTab;
    auto k = k_encode_iso<D, BITS, SO3, DYN>;
    if (!set_smem_once(reinterpret_cast<const void*>(k), smem))
      return KVQ_ERR_CUDA;
    k<<<grid, 128, smem, st>>>(m0, a);
  } else {
    const size_t smem = 1024 + D * (out_fp32 ? 512 : 256) + kTab;
    auto k = k_decode_iso<D, BITS, SO3, DYN>;
    if (!set_smem_once(reinterpret_cast<const void*>(k), smem))
      return KVQ_ERR_CUDA;
    k<<<grid, 128, smem, st>>>(m0, a, out_fp32);
  }
  return launch_status();
}

kvq_status dispatch(bool enc, const kvq_desc& d, const IsoArgs& a, const CUtensorMap& m0, int out_fp32,
                    cudaStream_t st) {
  // dynamic codebooks: the shared-memory tables when no 128-vector CTA spans two heads
  const bool one_head = d.heads == 1 || d.tokens % 128 == 0;
#define KVQ_RUN(D_, B_, DYN_)                                                                         \
  return d.rot == KVQ_ROT_ISO_SO3 ? run<D_, B_, true, DYN_>(enc, a, m0, out_fp32, st)                 \
                                  : run<D_, B_, false, DYN_>(enc, a, m0, out_fp32, st);
#define KVQ_CASE(D_, B_)                                                                              \
  if (d.head_dim == D_ && d.bits == B_) {                                                             \
    if (d.quant != KVQ_Q_CODEBOOK_DYN) { KVQ_RUN(D_, B_, 0) }                                         \
    if (one_head) { KVQ_RUN(D_, B_, 2) }                                                              \
    KVQ_RUN(D_, B_, 1)                                                                                \
  }
  KVQ_CASE(128, 2)
  KVQ_CASE(128, 3)
  KVQ_CASE(128, 4)
  KVQ_CASE(64, 2)
  KVQ_CASE(64, 3)
  KVQ_CASE(64, 4)
#undef KVQ_CASE
#undef KVQ_RUN
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

size_t dyn_stats_chunks(const kvq_desc& d) {
  return d.tokens > 0 ? (static_cast<size_t>(d.tokens) + kStatChunk - 1) / kStatChunk : 1;
}

size_t calibrate_codebook_workspace_bytes(const kvq_desc& d) {
  const size_t rows = static_cast<size_t>(d.batch) * d.heads * dyn_stats_chunks(d);
  return rows * d.head_dim * 8 + ((rows * 4 + 255) & ~size_t(255));
}

kvq_status launch_calibrate_codebook(const kvq_desc& d, const void* x, const kvq_tables& tb, float* ch_scale,
                                     uint32_t* ch_wide, void* ws, cudaStream_t st) {
  const size_t nchunk = dyn_stats_chunks(d);
  const size_t rows = static_cast<size_t>(d.batch) * d.heads * nchunk;
  if (static_cast<size_t>(d.batch) * d.heads > 65535 || nchunk > 0x7fffffff) return KVQ_ERR_UNSUPPORTED;
  DynStatArgs a{};
  a.H = d.heads;
  a.T = d.tokens;
  a.t0 = d.t0;
  a.n_sink = d.n_sink;
  a.nchunk = static_cast<int>(nchunk);
  a.x = static_cast<const __half*>(x);
  a.sink_pos = tb.sink_pos;
  a.qL = tb.qL;
  a.qR = tb.qR;
  a.part = static_cast<double*>(ws);
  a.cnt = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + rows * d.head_dim * 8);
  const dim3 grid(static_cast<unsigned>(nchunk), static_cast<unsigned>(d.batch * d.heads));
  const bool so3 = d.rot == KVQ_ROT_ISO_SO3;
  auto go = [&](auto kstats, auto kfin, int D) -> kvq_status {
    const size_t smem = static_cast<size_t>(128) * (D + 1) * 4;
    if (!set_smem_once(reinterpret_cast<const void*>(kstats), smem)) return KVQ_ERR_CUDA;
    kstats<<<grid, 128, smem, st>>>(a);
    if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
    kfin<<<d.heads, D, 0, st>>>(d.batch, d.heads, a.nchunk, a.part, a.cnt, ch_scale, ch_wide);
    return launch_status();
  };
  if (d.head_dim == 128)
    return so3 ? go(k_dyn_stats<128, true>, k_dyn_finish<128>, 128) : go(k_dyn_stats<128, false>, k_dyn_finish<128>, 128);
  return so3 ? go(k_dyn_stats<64, true>, k_dyn_finish<64>, 64) : go(k_dyn_stats<64, false>, k_dyn_finish<64>, 64);
}

}  // namespace kvq
