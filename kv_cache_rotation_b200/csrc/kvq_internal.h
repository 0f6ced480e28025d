// Host-side internals shared by the libkvq translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

// Per-call launch context prepared by the C-ABI layer.
struct LaunchCtx {
  uint32_t* err;     // device address of this device's error word
  uint64_t wait_ns;  // bound on every in-kernel wait
  int num_sms;
};

// Tensor-map construction (driver entry point resolved through the runtime).
bool make_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes /* rank-1 entries */, const uint32_t* box, CUtensorMapSwizzle swz);

// Heads per tile for the head-variant kernels: the largest power of two
// <= 8 that divides H (so a tile never spans two batches).
inline int heads_per_tile(int H) {
  int ht = 8;
  while (ht > 1 && H % ht) ht >>= 1;
  return ht;
}

kvq_status launch_encode_head(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                              cudaStream_t st, const LaunchCtx& ctx);
kvq_status launch_decode_head(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                              int out_fp32, cudaStream_t st, const LaunchCtx& ctx);
kvq_status launch_encode_group(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                               cudaStream_t st, const LaunchCtx& ctx);
kvq_status launch_decode_group(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                               int out_fp32, cudaStream_t st, const LaunchCtx& ctx);
kvq_status launch_encode_iso(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                             cudaStream_t st, const LaunchCtx& ctx);
kvq_status launch_decode_iso(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                             int out_fp32, cudaStream_t st, const LaunchCtx& ctx);
kvq_status launch_score(const kvq_desc& d, const void* q, int q_heads, const kvq_packed& cache,
                        const kvq_tables& tb, int n_tokens, float scale, float* scores, cudaStream_t st,
                        const LaunchCtx& ctx);
kvq_status launch_score_literal(const kvq_desc& d, const void* q, int q_heads, const kvq_packed& cache,
                                const kvq_tables& tb, int n_tokens, float scale, float* scores, cudaStream_t st,
                                const LaunchCtx& ctx);
kvq_status launch_score_group(const kvq_desc& d, const void* q, int q_heads, const kvq_packed& cache,
                              const kvq_tables& tb, int n_tokens, float scale, float* scores, cudaStream_t st,
                              const LaunchCtx& ctx);
kvq_status launch_debug_wait(uint64_t limit_ns, cudaStream_t st, const LaunchCtx& ctx);
size_t attend_workspace_bytes(const kvq_desc& dk, int q_heads, int n_tokens);
size_t attend_scratch_bytes();
kvq_status launch_pair_energy(const kvq_desc& d, const void* x, uint64_t* energy, int16_t* rank, cudaStream_t st);
bool calibrate_rope(const kvq_desc& d);
size_t calibrate_workspace_bytes(const kvq_desc& d);
kvq_status launch_calibrate(const kvq_desc& d, const void* x, const kvq_tables& tb, int16_t* perm, void* ws,
                            cudaStream_t st, int num_sms);
void* attend_scratch();
size_t calibrate_codebook_workspace_bytes(const kvq_desc& d);
kvq_status launch_calibrate_codebook(const kvq_desc& d, const void* x, const kvq_tables& tb, float* ch_scale,
                                     uint32_t* ch_wide, void* ws, cudaStream_t st);
size_t detect_sinks_workspace_bytes(const kvq_desc& d);
kvq_status launch_detect_sinks(const kvq_desc& d, const void* x, double tau, int max_sinks, int32_t* sink_pos,
                               int32_t* count, void* ws, cudaStream_t st, int num_sms);
// The list form of the sink set (kvq_tables.sink_pos): run after the kernels of
// encode / decode / score were launched with n_sink = 0.
kvq_status launch_sink_fix_encode(const kvq_desc& d, const void* x, const kvq_tables& tb, const kvq_packed& out,
                                  cudaStream_t st);
kvq_status launch_sink_fix_decode(const kvq_desc& d, const kvq_packed& in, const kvq_tables& tb, void* x_out,
                                  int out_fp32, cudaStream_t st);
kvq_status launch_sink_fix_score(const kvq_desc& d, const void* q, int q_heads, const kvq_packed& cache,
                                 const kvq_tables& tb, int n_tokens, float scale, float* scores, cudaStream_t st);
kvq_status launch_attend(const kvq_desc& dk, const kvq_desc& dv, const void* q, int q_heads,
                         const kvq_packed& kc, const kvq_tables& tk, const kvq_packed& vc, const kvq_tables& tv,
                         int n_tokens, float scale, float* out, void* ws, cudaStream_t st, const LaunchCtx& ctx);

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) only when a kernel needs
// more dynamic shared memory on this device than it was last granted (the
// attribute persists per device). A small per-thread cache of (kernel,
// device, bytes) keeps the host cost of repeated launches low.
inline bool set_smem_once(const void* fn, size_t bytes) {
  struct Entry {
    const void* fn;
    int dev;
    size_t bytes;
  };
  static thread_local Entry cache[32];
  static thread_local int n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  for (int i = 0; i < n; ++i)
    if (cache[i].fn == fn && cache[i].dev == dev && bytes <= cache[i].bytes) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
      cudaSuccess)
    return false;
  for (int i = 0; i < n; ++i)
    if (cache[i].fn == fn && cache[i].dev == dev) {
      cache[i].bytes = bytes;
      return true;
    }
  cache[n < 32 ? n++ : 31] = Entry{fn, dev, bytes};
  return true;
}

// Resident CTAs per SM of a kernel (cached per kernel, device and smem size).
inline int occupancy_once(const void* fn, int threads, size_t smem) {
  struct Entry {
    const void* fn;
    int dev, threads;
    size_t smem;
    int per_sm;
  };
  static thread_local Entry cache[32];
  static thread_local int n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  for (int i = 0; i < n; ++i)
    if (cache[i].fn == fn && cache[i].dev == dev && cache[i].threads == threads && cache[i].smem == smem)
      return cache[i].per_sm;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  cache[n < 32 ? n++ : 31] = Entry{fn, dev, threads, smem, per_sm};
  return per_sm;
}

// Finish a launch: map a launch error to a status.
inline kvq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
