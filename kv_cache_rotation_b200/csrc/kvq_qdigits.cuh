// Rotated, digit-split queries for the tensor-core scores (head_dim 128).
//
// "EliteKV - RoPE频率选择与低秩投影" §2.2: the score of query m and cached key
// n is q_m . k_n (times the softmax scale). The keys are stored as
// y_n = H P RoPE_n(k_n) quantized per group to Z + c S; H (normalised
// Sylvester) and P (channel permutation) are orthogonal, so
// q . P^T H^T y = (H P q) . y and each query is rotated once, qt = H P q.
// qt is quantized to 16-bit integers Q = rint(qt / sq), sq = max|qt| / 32000,
// and split into two int8 digits Q = 256 hi + lo, so that an exact
// u8 x s8 -> s32 tensor-core product forms sum_j c_j Q_j per group.
//
// Shared by the score kernel and the fused attention kernel: both compute a
// key's score with the same integer products and the same fp32 epilogue, so
// their scores agree bit for bit.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

// Channel that K index (k-step s, lane quad position tig, byte l, upper half u)
// of the m16n8k32 A fragment carries when the codes are expanded one byte per
// code by `(w >> BITS * tig) & mask`; the B fragment uses the same map.
template <int BITS>
__device__ __forceinline__ int kchan(int s, int tig, int l, int u) {
  if constexpr (BITS == 2) return 32 * s + 16 * u + 4 * l + tig;
  else return 32 * s + 16 * u + 8 * (tig >> 1) + 2 * l + (tig & 1);
}

// One warp, one query head: qraw = q (fp32), qd = the two int8 digits of
// rint(H P q / sq), qsum[g] = sum over group g of H P q, *sqh = sq.
// qv: the query head's 128 fp16 values (16-byte aligned); perm_h: this KV
// head's permutation row or nullptr; lane holds channels 4 lane .. 4 lane + 3.
template <int G>
__device__ __forceinline__ void query_digits(const __half* qv, const int16_t* perm_h, int rot, float rscale,
                                             int lane, float* qraw, int8_t* qd_lo, int8_t* qd_hi, float* qsum,
                                             float* sqh) {
  constexpr int D = 128;
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qv) + lane);  // channels 4 lane .. 4 lane + 3
  const float2 r01 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
  const float2 r23 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
  float v[4] = {r01.x, r01.y, r23.x, r23.y};
  *reinterpret_cast<float4*>(qraw + 4 * lane) = make_float4(v[0], v[1], v[2], v[3]);
  if (perm_h) {
    const uint2 pk = __ldg(reinterpret_cast<const uint2*>(perm_h) + lane);
    const uint32_t pw[2] = {pk.x, pk.y};
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __half2float(qv[(pw[i >> 1] >> (16 * (i & 1))) & (D - 1)]);
  }
  if (rot == KVQ_ROT_FWHT_HEAD) {
    const float t0 = v[0] + v[1], t1 = v[0] - v[1], t2 = v[2] + v[3], t3 = v[2] - v[3];
    v[0] = t0 + t2; v[2] = t0 - t2; v[1] = t1 + t3; v[3] = t1 - t3;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float p = __shfl_xor_sync(0xffffffffu, v[i], m);
        v[i] = (lane & m) ? (p - v[i]) : (v[i] + p);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] *= rscale;
  }
  float mx = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
  const float sq = mx > 0.0f ? mx / 32000.0f : 1.0f;
  const float rsq = 1.0f / sq;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int Q = __float2int_rn(v[i] * rsq);
    const int lo = ((Q + 128) & 255) - 128;
    qd_lo[4 * lane + i] = static_cast<int8_t>(lo);
    qd_hi[4 * lane + i] = static_cast<int8_t>((Q - lo) >> 8);
  }
  float ps = (v[0] + v[1]) + (v[2] + v[3]);
#pragma unroll
  for (int m = 1; m < G / 4; m <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, m);
  if ((lane & (G / 4 - 1)) == 0) qsum[lane / (G / 4)] = ps;
  if (lane == 0) *sqh = sq;
}

// B fragments of the m16n8k32 score MMA: column c = 2 * query head + digit
// (0 = lo, 1 = hi) of n-tile c / 8; entry [nt][s][tig][n] is the (b0, b1)
// register pair of lane 4 n + tig for k-step s.
template <int BITS, int GQ, int NTN>
__device__ __forceinline__ void build_score_bfrag(uint2 (&bfrag)[NTN][4][4][8], const int8_t (&qd)[GQ][2][128],
                                                  int tid, int nthreads) {
  for (int e = tid; e < NTN * 128; e += nthreads) {
    const int nt = e >> 7, s = (e >> 5) & 3, tg = (e >> 3) & 3, n = e & 7;
    const int c = nt * 8 + n, hh = c >> 1, dg = c & 1;
    uint32_t b0 = 0, b1 = 0;
    if (hh < GQ) {
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        b0 |= static_cast<uint32_t>(static_cast<uint8_t>(qd[hh][dg][kchan<BITS>(s, tg, l, 0)])) << (8 * l);
        b1 |= static_cast<uint32_t>(static_cast<uint8_t>(qd[hh][dg][kchan<BITS>(s, tg, l, 1)])) << (8 * l);
      }
    }
    bfrag[nt][s][tg][n] = make_uint2(b0, b1);
  }
}

// A fragment of k-step s of the m16n8k32 score MMA for this lane's two token
// rows (words wa of row g, wb of row g + 8): every code expanded to one byte.
template <int BITS, int NW>
__device__ __forceinline__ void score_afrag(const uint32_t (&wa)[NW], const uint32_t (&wb)[NW], int s, int tig,
                                            uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) {
  if constexpr (BITS == 2) {
    constexpr uint32_t MASK = 0x03030303u;
    a0 = (wa[2 * s] >> (2 * tig)) & MASK;
    a1 = (wb[2 * s] >> (2 * tig)) & MASK;
    a2 = (wa[2 * s + 1] >> (2 * tig)) & MASK;
    a3 = (wb[2 * s + 1] >> (2 * tig)) & MASK;
  } else {
    constexpr uint32_t MASK = 0x0F0F0F0Fu;
    const bool odd = (tig & 2) != 0;  // word 4s + (tig >> 1), selected without dynamic indexing
    const int sh = 4 * (tig & 1);
    a0 = ((odd ? wa[4 * s + 1] : wa[4 * s]) >> sh) & MASK;
    a1 = ((odd ? wb[4 * s + 1] : wb[4 * s]) >> sh) & MASK;
    a2 = ((odd ? wa[4 * s + 3] : wa[4 * s + 2]) >> sh) & MASK;
    a3 = ((odd ? wb[4 * s + 3] : wb[4 * s + 2]) >> sh) & MASK;
  }
}

// q . RoPE_n(sink_n) for an fp16 sink key by one warp (fp32; every lane gets
// the sum): lane takes channels 4 lane .. 4 lane + 3, the lane sums are added
// by an xor butterfly. rope_row: the position's (cos, sin) pairs, or nullptr;
// half: the half-split pairs (c, c + 64) (lane ^ 16 holds the partner
// channels) instead of the interleaved (2i, 2i + 1).
__device__ __forceinline__ float sink_dot(const float* qraw, const __half* sink_row, const float* rope_row,
                                          int lane, bool half = false) {
  const uint2 kr = __ldg(reinterpret_cast<const uint2*>(sink_row) + lane);
  const float2 k01 = __half22float2(*reinterpret_cast<const __half2*>(&kr.x));
  const float2 k23 = __half22float2(*reinterpret_cast<const __half2*>(&kr.y));
  float k4[4] = {k01.x, k01.y, k23.x, k23.y};
  if (rope_row && !half) {  // pairs 2 lane and 2 lane + 1 of the sink's position
    const float4 cs = __ldg(reinterpret_cast<const float4*>(rope_row) + lane);
    rope_fwd(k4[0], k4[1], cs.x, cs.y);
    rope_fwd(k4[2], k4[3], cs.z, cs.w);
  } else if (rope_row) {  // angles 4 (lane mod 16) .. + 3
    const float4 c0 = __ldg(reinterpret_cast<const float4*>(rope_row) + 2 * (lane & 15));
    const float4 c1 = __ldg(reinterpret_cast<const float4*>(rope_row) + 2 * (lane & 15) + 1);
    const float2 y01 = rope_half_fwd2(f2(k4[0], k4[1]), f2(c0.x, c0.z), f2(c0.y, c0.w), lane >= 16, 16);
    const float2 y23 = rope_half_fwd2(f2(k4[2], k4[3]), f2(c1.x, c1.z), f2(c1.y, c1.w), lane >= 16, 16);
    k4[0] = y01.x;
    k4[1] = y01.y;
    k4[2] = y23.x;
    k4[3] = y23.y;
  }
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) acc = __fmaf_rn(qraw[4 * lane + i], k4[i], acc);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  return acc;
}

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint2 b) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
}

}  // namespace kvq
