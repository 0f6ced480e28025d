// Device-side building blocks shared by the libkvq kernels (sm_100a):
// mbarrier + TMA (cp.async.bulk.tensor) staging with bounded waits, the
// in-register FWHT, RoPE, the min-max quantizer and bit packing.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace kvq {

// Error word bits, read and cleared by kvq_check. Kernels receive the
// address of the per-device error word as an argument.
constexpr uint32_t kErrTimeout = 1u;

constexpr float kMagicRound = 12582912.0f;  // 1.5 * 2^23: fp32 ulp = 1 on [2^23, 2^24)
constexpr uint32_t kMagicBits = 0x4B400000u;

// Division of n < 2^31 by a fixed divisor 1 <= d < 2^31 as a multiply and a
// shift: with s = ceil(log2 d) and M = ceil(2^(31+s) / d) < 2^32,
// floor(n / d) = (n * M) >> (31 + s) exactly (the rounding error of M stays
// below 1/d for n < 2^31). Precomputed on the host, two instructions on the GPU.
struct FastDiv {
  uint32_t d, m, s;
  __host__ __device__ FastDiv() : d(1), m(0x80000000u), s(0) {}
  __host__ explicit FastDiv(uint32_t div) : d(div) {
    s = 0;
    while ((1ull << s) < div) ++s;
    m = static_cast<uint32_t>(((1ull << (31 + s)) + div - 1) / div);
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    return static_cast<uint32_t>((static_cast<uint64_t>(n) * m) >> (31 + s));
  }
  __device__ __forceinline__ uint32_t mod(uint32_t n, uint32_t q) const { return n - q * d; }
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait on an mbarrier phase: gives up after limit_ns of wall time
// (and in any case after 2^30 polls), sets the error word, returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns, uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0 && global_ns() - t0 > limit_ns) break;
  }
  atomicOr(err, kErrTimeout);
  return false;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}
// Pull a tensor tile into L2 ahead of its TMA load (no shared memory, no barrier).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, int x, int y, int z, int w, const void* src) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until at most N committed bulk-store groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N committed bulk-store groups are still incomplete
// (their global writes done, not only their shared-memory reads).
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Make generic-proxy smem writes visible to the TMA (async proxy).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 4-byte asynchronous global -> shared copy; n = 0 reads nothing and
// writes zeros. Completion: cp_async_wait_all in the issuing thread, then a
// barrier before other threads read the data.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t n) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
// 16-byte async copy through L2 only; n < 16 fills the rest with zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t n) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- smem access
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ float lds32f(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts32f(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Byte offset of 16-byte chunk c of row r in a TMA tile written with
// CU_TENSOR_MAP_SWIZZLE_128B (128-byte rows, tile base 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t c) { return r * 128u + ((c ^ (r & 7u)) << 4); }

// ---------------------------------------------------------------- fp16
__device__ __forceinline__ void h8_to_f32(uint4 raw, float* f) {
  const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __half22float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ uint4 f32_to_h8(const float* f) {
  uint4 raw;
  __half2* h = reinterpret_cast<__half2*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  return raw;
}

// ---------------------------------------------------------------- FWHT
// Unnormalised Sylvester FWHT on a register array, strides 1, 2, ..., N/2
// in ascending order; each pair (i, i+h), (i & h) == 0 becomes (a+b, a-b).
template <int N>
__device__ __forceinline__ void fwht_reg(float (&v)[N]) {
#pragma unroll
  for (int h = 1; h < N; h <<= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
    }
  }
}

// ---------------------------------------------------------------- packed fp32 (sm_100 FADD2 / FFMA2 / FMUL2)
// Same IEEE rounding per lane as the scalar operations.
__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b as one packed fma: fma(b, -1, a) rounds a - b exactly once, like a subtraction.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ void bfly(float2& a, float2& b) {
  const float2 p = a, q = b;
  a = add2(p, q);
  b = sub2(p, q);
}

// Stride-1 butterfly of the two fp16 channels held in one word w = (x0 | x1 << 16):
// s = x0 + x1 and d = x0 - x1, each rounded once to fp32. The sm_100 mixed-
// precision add / sub take x0 as fp16 (its conversion is exact), so only x1 is
// converted: the same fp32 results as converting both and adding, in one
// conversion fewer.
__device__ __forceinline__ void bfly_h2(uint32_t w, float& s, float& d) {
  asm("{\n\t.reg .b16 lo, hi;\n\t.reg .f32 f1;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "cvt.f32.f16 f1, hi;\n\t"
      "add.rn.f32.f16 %0, lo, f1;\n\t"
      "sub.rn.f32.f16 %1, lo, f1;\n\t}"
      : "=f"(s), "=f"(d)
      : "r"(w));
}

// Register-pair layout of V consecutive channels: P[2g + e] = (x[4g + e],
// x[4g + 2 + e]), g < V/4. Unnormalised Sylvester FWHT strides 1, 2, 4, ...,
// V/2 in ascending order; stride 2 falls inside a pair (scalar ops), every
// other stride is one packed add and one packed subtract per two pairs.
template <int V>
__device__ __forceinline__ void fwht_pairs(float2 (&P)[V / 2]) {
#pragma unroll
  for (int g = 0; g < V / 4; ++g) bfly(P[2 * g], P[2 * g + 1]);  // stride 1
#pragma unroll
  for (int k = 0; k < V / 2; ++k) {  // stride 2
    const float a = P[k].x, b = P[k].y;
    P[k] = f2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
#pragma unroll
  for (int hs = 1; hs < V / 4; hs <<= 1) {  // strides 4 .. V/2
#pragma unroll
    for (int g = 0; g < V / 4; ++g) {
      if ((g & hs) == 0) {
        bfly(P[2 * g], P[2 * (g + hs)]);
        bfly(P[2 * g + 1], P[2 * (g + hs) + 1]);
      }
    }
  }
}

// N words (N a multiple of 8) of global memory <-> registers: 256-bit accesses
// when the address is 32-byte aligned, 128-bit ones otherwise. Loads use the
// read-only path and do not allocate in L1.
template <int N>
__device__ __forceinline__ void ld_row(const void* p, bool v8, uint32_t* w) {
  if (v8) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i)
      asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=r"(w[8 * i]), "=r"(w[8 * i + 1]), "=r"(w[8 * i + 2]), "=r"(w[8 * i + 3]),
                     "=r"(w[8 * i + 4]), "=r"(w[8 * i + 5]), "=r"(w[8 * i + 6]), "=r"(w[8 * i + 7])
                   : "l"(static_cast<const uint8_t*>(p) + 32 * i));
  } else {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const uint4 v = __ldg(static_cast<const uint4*>(p) + i);
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  }
}
template <int N>
__device__ __forceinline__ void st_row(void* p, bool v8, const uint32_t* w) {
  if (v8) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i)
      asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(static_cast<uint8_t*>(p) + 32 * i),
                   "r"(w[8 * i]), "r"(w[8 * i + 1]), "r"(w[8 * i + 2]), "r"(w[8 * i + 3]), "r"(w[8 * i + 4]),
                   "r"(w[8 * i + 5]), "r"(w[8 * i + 6]), "r"(w[8 * i + 7])
                   : "memory");
  } else {
#pragma unroll
    for (int i = 0; i < N / 4; ++i)
      static_cast<uint4*>(p)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  }
}

// Sum of kMagicBits << (BITS * j) over the N codes of one packed word: a packer
// that adds each code's raw fp32 pattern (kMagicBits + code) at its shift
// subtracts this once per word. The constant only touches bits 22 and up, so
// runs of at most 22 bits need no correction.
template <int BITS, int N>
__host__ __device__ constexpr uint32_t magic_offset() {
  uint32_t k = 0;
  for (int j = 0; j < N; ++j) k += kMagicBits << (BITS * j);
  return k;
}

// ---------------------------------------------------------------- RoPE
// Forward rotation of one pair with fp32 (c, s):
//   y0 = fma(x0, c, -(x1*s)),  y1 = fma(x0, s, x1*c)
__device__ __forceinline__ void rope_fwd(float& x0, float& x1, float c, float s) {
  const float t1 = __fmul_rn(x1, s);
  const float t2 = __fmul_rn(x1, c);
  const float y0 = __fmaf_rn(x0, c, -t1);
  const float y1 = __fmaf_rn(x0, s, t2);
  x0 = y0;
  x1 = y1;
}
// Half-split RoPE pairs (i, i + D/2) held by two lanes (partner = lane ^ pm):
// this lane holds two channels of the lower half (upper == false) or of the
// upper half, and (cc, ss) are the cosines and sines of their pairs' angles.
// Forward, the encoder's fp32 order: lower y0 = fma(x0, c, -(x1*s)), upper
// y1 = fma(x0, s, x1*c), x0 / x1 the lower / upper channel of the pair.
__device__ __forceinline__ float2 rope_half_fwd2(float2 own, float2 cc, float2 ss, bool upper, int pm) {
  const float2 oth = f2(__shfl_xor_sync(0xffffffffu, own.x, pm), __shfl_xor_sync(0xffffffffu, own.y, pm));
  return upper ? fma2(oth, ss, mul2(own, cc)) : fma2(own, cc, mul2(oth, f2(-ss.x, -ss.y)));
}
// Inverse: lower x0 = y0 c + y1 s, upper x1 = y1 c - y0 s.
__device__ __forceinline__ float2 rope_half_inv2(float2 own, float2 cc, float2 ss, bool upper, int pm) {
  const float2 oth = f2(__shfl_xor_sync(0xffffffffu, own.x, pm), __shfl_xor_sync(0xffffffffu, own.y, pm));
  return upper ? fma2(own, cc, mul2(oth, f2(-ss.x, -ss.y))) : fma2(own, cc, mul2(oth, ss));
}

// ---------------------------------------------------------------- min/max
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Scale / zero of one min-max group from its (canonicalised) min and max:
// Z = largest half <= mn, S = smallest half >= fp32((mx - Z)/L), R = 1/S.
struct QParams {
  float Z, R;
  __half2 sz;  // (S, Z)
};
template <int BITS>
__device__ __forceinline__ QParams minmax_params(float mn, float mx) {
  mn = __fadd_rn(mn, 0.0f);
  mx = __fadd_rn(mx, 0.0f);
  const __half zh = __float2half_rd(mn);
  const float Z = __half2float(zh);
  const float w = __fsub_rn(mx, Z);
  const float q = __fdiv_rn(w, static_cast<float>((1 << BITS) - 1));
  const __half sh = __float2half_ru(q);
  const float S = __half2float(sh);
  QParams p;
  p.Z = Z;
  p.R = S > 0.0f ? __frcp_rn(S) : 0.0f;
  p.sz = __halves2half2(sh, zh);
  return p;
}

// ---------------------------------------------------------------- packing
// Code j of a packed word array.
template <int BITS, int NW>
__device__ __forceinline__ uint32_t unpack_code(const uint32_t (&w)[NW], int j) {
  const int p = j * BITS;
  uint32_t c = w[p >> 5] >> (p & 31);
  if ((p & 31) + BITS > 32) c |= w[(p >> 5) + 1] << (32 - (p & 31));
  return c & ((1u << BITS) - 1u);
}
// Exact small integer -> float without the conversion pipe.
__device__ __forceinline__ float code_to_float(uint32_t c) {
  return __fsub_rn(__uint_as_float(0x4B000000u | c), 8388608.0f);
}

}  // namespace kvq
