// C-ABI layer of libkvq: argument validation, per-device error word,
// tensor-map construction, dispatch to the kernels, and the host helpers
// (RoPE table, Lloyd-Max codebook).
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

__device__ uint32_t g_error_word;

namespace {

constexpr int kMaxDevices = 64;
uint32_t* g_err_addr[kMaxDevices];
int g_num_sms[kMaxDevices];
std::mutex g_mu;

// Bound on every in-kernel wait (TMA copies normally land in microseconds).
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

kvq_status get_ctx(LaunchCtx* ctx) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return KVQ_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return KVQ_ERR_CUDA;
    g_err_addr[dev] = static_cast<uint32_t*>(p);
    g_num_sms[dev] = sms;
    // Resolve kvq_attend_noalloc's fixed scratch now, on the first call of any
    // entry point on this device: under lazy module loading this is when the
    // array is reserved, so a later kvq_attend_noalloc call finds it ready and
    // reserves nothing. A failure here is reported by kvq_attend_noalloc alone
    // (it returns KVQ_ERR_CUDA); every other entry point keeps working.
    (void)attend_scratch();
  }
  ctx->err = g_err_addr[dev];
  ctx->num_sms = g_num_sms[dev];
  ctx->wait_ns = kWaitNs;
  return KVQ_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Shape / parameter validation common to every entry point.
kvq_status check_desc(const kvq_desc* d) {
  if (!d) return KVQ_ERR_INVALID;
  if (d->batch <= 0 || d->heads <= 0 || d->tokens < 0 || d->t0 < 0 || d->t_cap <= 0 || d->n_sink < 0)
    return KVQ_ERR_INVALID;
  if (static_cast<int64_t>(d->t0) + d->tokens > d->t_cap) return KVQ_ERR_INVALID;
  if (d->rope < 0 || d->rope > 2) return KVQ_ERR_INVALID;
  if (d->bits < 2 || d->bits > 4) return KVQ_ERR_UNSUPPORTED;
  if (d->head_dim != 64 && d->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->batch) * d->heads * d->t_cap * d->head_dim > (int64_t(1) << 40))
    return KVQ_ERR_UNSUPPORTED;
  switch (d->rot) {
    case KVQ_ROT_NONE:
    case KVQ_ROT_FWHT_HEAD:
      if (d->quant != KVQ_Q_MINMAX) return KVQ_ERR_UNSUPPORTED;
      if (d->group != 32 && d->group != 64 && d->group != 128) return KVQ_ERR_UNSUPPORTED;
      if (d->head_dim % d->group) return KVQ_ERR_INVALID;
      break;
    case KVQ_ROT_FWHT_GROUP:
      if (d->quant != KVQ_Q_MINMAX) return KVQ_ERR_UNSUPPORTED;
      if (d->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
      if (d->group_heads != 2 && d->group_heads != 4 && d->group_heads != 8) return KVQ_ERR_UNSUPPORTED;
      if (d->heads % d->group_heads) return KVQ_ERR_INVALID;
      if (d->group != 64 && d->group != 128) return KVQ_ERR_UNSUPPORTED;
      if (d->group < 128 / d->group_heads) return KVQ_ERR_UNSUPPORTED;
      break;
    case KVQ_ROT_ISO_SO4:
    case KVQ_ROT_ISO_SO3:
      if (d->quant != KVQ_Q_CODEBOOK && d->quant != KVQ_Q_CODEBOOK_DYN) return KVQ_ERR_UNSUPPORTED;
      if (d->rope) return KVQ_ERR_UNSUPPORTED;
      break;
    default:
      return KVQ_ERR_INVALID;
  }
  if (d->quant != KVQ_Q_MINMAX && d->quant != KVQ_Q_CODEBOOK && d->quant != KVQ_Q_CODEBOOK_DYN)
    return KVQ_ERR_INVALID;
  return KVQ_OK;
}

kvq_status check_tables(const kvq_desc* d, const kvq_tables* tb, int64_t rope_rows_needed) {
  if (!tb) return KVQ_ERR_INVALID;
  if (d->rope) {
    if (!tb->rope_cs) return KVQ_ERR_INVALID;
    if (!aligned(tb->rope_cs, 16)) return KVQ_ERR_ALIGN;
    if (tb->rope_rows < rope_rows_needed || tb->rope_rows <= 0) return KVQ_ERR_INVALID;
  }
  if (tb->perm && !aligned(tb->perm, 16)) return KVQ_ERR_ALIGN;
  if (tb->sink_pos && !aligned(tb->sink_pos, 4)) return KVQ_ERR_ALIGN;
  if (d->rot == KVQ_ROT_ISO_SO4) {
    if (!tb->qL || !tb->qR || !tb->codebook) return KVQ_ERR_INVALID;
    if (!aligned(tb->qL, 16) || !aligned(tb->qR, 16) || !aligned(tb->codebook, 4)) return KVQ_ERR_ALIGN;
  }
  if (d->rot == KVQ_ROT_ISO_SO3) {
    if (!tb->qL || !tb->codebook) return KVQ_ERR_INVALID;
    if (!aligned(tb->qL, 16) || !aligned(tb->codebook, 4)) return KVQ_ERR_ALIGN;
  }
  if (d->quant == KVQ_Q_CODEBOOK_DYN) {
    if (!tb->codebook_wide || !tb->ch_scale || !tb->ch_wide) return KVQ_ERR_INVALID;
    if (!aligned(tb->codebook_wide, 4) || !aligned(tb->ch_scale, 16) || !aligned(tb->ch_wide, 4))
      return KVQ_ERR_ALIGN;
  }
  return KVQ_OK;
}

kvq_status check_packed(const kvq_desc* d, const kvq_packed* p) {
  if (!p || !p->codes) return KVQ_ERR_INVALID;
  if (!aligned(p->codes, 16)) return KVQ_ERR_ALIGN;
  if (d->quant == KVQ_Q_MINMAX) {
    if (!p->scale_zero) return KVQ_ERR_INVALID;
    if (!aligned(p->scale_zero, 16)) return KVQ_ERR_ALIGN;
  }
  if (d->rot == KVQ_ROT_ISO_SO4 || d->rot == KVQ_ROT_ISO_SO3) {
    if (!p->norm) return KVQ_ERR_INVALID;
    if (!aligned(p->norm, 4)) return KVQ_ERR_ALIGN;
  }
  if (d->quant == KVQ_Q_CODEBOOK_DYN) {
    if (!p->ext) return KVQ_ERR_INVALID;
    if (!aligned(p->ext, 2)) return KVQ_ERR_ALIGN;
  }
  if (d->n_sink > 0) {
    if (!p->sink) return KVQ_ERR_INVALID;
    if (!aligned(p->sink, 16)) return KVQ_ERR_ALIGN;
  }
  return KVQ_OK;
}

// Lloyd-Max levels of N(0,1): boundaries are midpoints of neighbouring
// levels; each level moves to the mean of its cell,
// (phi(a) - phi(b)) / (Phi(b) - Phi(a)), until it stops moving.
double phi_pdf(double x) { return isinf(x) ? 0.0 : 0.3989422804014327 * exp(-0.5 * x * x); }
double cell_mass(double a, double b) {
  const double r2 = 0.7071067811865476;
  if (a >= 0) return 0.5 * (erfc(a * r2) - erfc(b * r2));
  if (b <= 0) return 0.5 * (erfc(-b * r2) - erfc(-a * r2));
  return 1.0 - 0.5 * erfc(-a * r2) - 0.5 * erfc(b * r2);
}

}  // namespace

bool make_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bd[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bd[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) gs[i] = strides_bytes[i];
  }
  const CUresult r = fn(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gd, gs, bd, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- debug wait
namespace {
__global__ void k_debug_wait(uint32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  // No arrival and no copy is ever issued: the phase never completes.
  mbar_wait(&bar, 0, limit_ns, err);
}
}  // namespace

kvq_status launch_debug_wait(uint64_t limit_ns, cudaStream_t st, const LaunchCtx& ctx) {
  k_debug_wait<<<1, 1, 0, st>>>(ctx.err, limit_ns);
  return launch_status();
}

}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_encode(const kvq_desc* d, const void* x, const kvq_tables* tb, const kvq_packed* out,
                      kvq_stream_t stream) {
  kvq_status s = check_desc(d);
  if (s != KVQ_OK) return s;
  if (!x) return KVQ_ERR_INVALID;
  if (!aligned(x, 16)) return KVQ_ERR_ALIGN;
  if ((s = check_tables(d, tb, static_cast<int64_t>(d->t0) + d->tokens)) != KVQ_OK) return s;
  if ((s = check_packed(d, out)) != KVQ_OK) return s;
  if (d->tokens == 0) return KVQ_OK;
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool listed = tb->sink_pos && d->n_sink > 0;
  kvq_desc dd = *d;
  if (listed) dd.n_sink = 0;  // every slot is coded first; the listed sinks are written after
  switch (dd.rot) {
    case KVQ_ROT_FWHT_GROUP:
      s = launch_encode_group(dd, x, *tb, *out, st, ctx);
      break;
    case KVQ_ROT_ISO_SO4:
    case KVQ_ROT_ISO_SO3:
      s = launch_encode_iso(dd, x, *tb, *out, st, ctx);
      break;
    default:
      s = launch_encode_head(dd, x, *tb, *out, st, ctx);
  }
  if (s != KVQ_OK || !listed) return s;
  return launch_sink_fix_encode(*d, x, *tb, *out, st);
}

kvq_status kvq_decode(const kvq_desc* d, const kvq_packed* in, const kvq_tables* tb, void* x_out,
                      int32_t out_fp32, kvq_stream_t stream) {
  kvq_status s = check_desc(d);
  if (s != KVQ_OK) return s;
  if (!x_out) return KVQ_ERR_INVALID;
  if (!aligned(x_out, 16)) return KVQ_ERR_ALIGN;
  if (out_fp32 != 0 && out_fp32 != 1) return KVQ_ERR_INVALID;
  if ((s = check_tables(d, tb, static_cast<int64_t>(d->t0) + d->tokens)) != KVQ_OK) return s;
  if ((s = check_packed(d, in)) != KVQ_OK) return s;
  if (d->tokens == 0) return KVQ_OK;
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool listed = tb->sink_pos && d->n_sink > 0;
  kvq_desc dd = *d;
  if (listed) dd.n_sink = 0;  // every slot is decoded first; the listed sinks are written after
  switch (dd.rot) {
    case KVQ_ROT_FWHT_GROUP:
      s = launch_decode_group(dd, *in, *tb, x_out, out_fp32, st, ctx);
      break;
    case KVQ_ROT_ISO_SO4:
    case KVQ_ROT_ISO_SO3:
      s = launch_decode_iso(dd, *in, *tb, x_out, out_fp32, st, ctx);
      break;
    default:
      s = launch_decode_head(dd, *in, *tb, x_out, out_fp32, st, ctx);
  }
  if (s != KVQ_OK || !listed) return s;
  return launch_sink_fix_decode(*d, *in, *tb, x_out, out_fp32, st);
}

kvq_status kvq_score(const kvq_desc* d, const void* q, int32_t q_heads, const kvq_packed* cache,
                     const kvq_tables* tb, int32_t n_tokens, float scale, float* scores, kvq_stream_t stream) {
  if (!d) return KVQ_ERR_INVALID;
  kvq_desc dd = *d;
  dd.tokens = 0;
  dd.t0 = 0;
  kvq_status s = check_desc(&dd);
  if (s != KVQ_OK) return s;
  const bool grouped = dd.rot == KVQ_ROT_FWHT_GROUP;
  if (dd.rot != KVQ_ROT_NONE && dd.rot != KVQ_ROT_FWHT_HEAD && !grouped) return KVQ_ERR_UNSUPPORTED;
  if (!q || !scores) return KVQ_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(scores, 16)) return KVQ_ERR_ALIGN;
  if (q_heads <= 0 || q_heads % dd.heads || q_heads / dd.heads > 16) return KVQ_ERR_INVALID;
  if (n_tokens < 0 || n_tokens > dd.t_cap) return KVQ_ERR_INVALID;
  if (grouped) {  // keys with RoPE, no permutation, up to 8 query heads per KV head
    if (!dd.rope || (tb && tb->perm)) return KVQ_ERR_UNSUPPORTED;
    const int gq = q_heads / dd.heads;
    if (gq != 1 && gq != 2 && gq != 4 && gq != 8) return KVQ_ERR_UNSUPPORTED;
  }
  const bool listed = tb && tb->sink_pos && dd.n_sink > 0;
  const int64_t rows = grouped || listed ? n_tokens
                                         : (dd.rope ? (n_tokens < dd.n_sink ? n_tokens : dd.n_sink) : 0);
  if ((s = check_tables(&dd, tb, rows)) != KVQ_OK) return s;
  if ((s = check_packed(&dd, cache)) != KVQ_OK) return s;
  if (n_tokens == 0) return KVQ_OK;
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  kvq_desc dm = dd;
  if (listed) dm.n_sink = 0;  // every slot is scored from its codes first; the listed sinks after
  s = grouped ? launch_score_group(dm, q, q_heads, *cache, *tb, n_tokens, scale, scores, st, ctx)
              : launch_score(dm, q, q_heads, *cache, *tb, n_tokens, scale, scores, st, ctx);
  if (s != KVQ_OK || !listed) return s;
  return launch_sink_fix_score(dd, q, q_heads, *cache, *tb, n_tokens, scale, scores, st);
}

kvq_status kvq_score_literal(const kvq_desc* d, const void* q, int32_t q_heads, const kvq_packed* cache,
                             const kvq_tables* tb, int32_t n_tokens, float scale, float* scores,
                             kvq_stream_t stream) {
  if (!d) return KVQ_ERR_INVALID;
  kvq_desc dd = *d;
  dd.tokens = 0;
  dd.t0 = 0;
  kvq_status s = check_desc(&dd);
  if (s != KVQ_OK) return s;
  if (dd.rot != KVQ_ROT_NONE && dd.rot != KVQ_ROT_FWHT_HEAD) return KVQ_ERR_UNSUPPORTED;
  if (dd.head_dim != 128 || dd.quant != KVQ_Q_MINMAX) return KVQ_ERR_UNSUPPORTED;
  if (!q || !scores) return KVQ_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(scores, 16)) return KVQ_ERR_ALIGN;
  if (q_heads <= 0 || q_heads % dd.heads) return KVQ_ERR_INVALID;
  const int gq = q_heads / dd.heads;
  if (gq != 1 && gq != 2 && gq != 4 && gq != 8) return KVQ_ERR_UNSUPPORTED;
  if (n_tokens < 0 || n_tokens > dd.t_cap) return KVQ_ERR_INVALID;
  const bool listed = tb && tb->sink_pos && dd.n_sink > 0;
  const int64_t rows = listed ? n_tokens : (dd.rope ? (n_tokens < dd.n_sink ? n_tokens : dd.n_sink) : 0);
  if ((s = check_tables(&dd, tb, rows)) != KVQ_OK) return s;
  if ((s = check_packed(&dd, cache)) != KVQ_OK) return s;
  if (n_tokens == 0) return KVQ_OK;
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  kvq_desc dm = dd;
  if (listed) dm.n_sink = 0;  // every slot is scored from its codes first; the listed sinks after
  s = launch_score_literal(dm, q, q_heads, *cache, *tb, n_tokens, scale, scores, st, ctx);
  if (s != KVQ_OK || !listed) return s;
  return launch_sink_fix_score(dd, q, q_heads, *cache, *tb, n_tokens, scale, scores, st);
}

namespace {
// Shapes kvq_attend accepts: dk / dv valid, head-variant (or unrotated) min-max
// caches of the same record shape, head_dim 128, values without RoPE.
kvq_status check_attend(const kvq_desc* dk, const kvq_desc* dv, int32_t q_heads, int32_t n_tokens,
                        kvq_desc* k_out, kvq_desc* v_out) {
  if (!dk || !dv) return KVQ_ERR_INVALID;
  kvq_desc k = *dk, v = *dv;
  k.tokens = v.tokens = 0;
  k.t0 = v.t0 = 0;
  kvq_status s;
  if ((s = check_desc(&k)) != KVQ_OK || (s = check_desc(&v)) != KVQ_OK) return s;
  if (k.rot != KVQ_ROT_NONE && k.rot != KVQ_ROT_FWHT_HEAD) return KVQ_ERR_UNSUPPORTED;
  if (k.quant != KVQ_Q_MINMAX || k.head_dim != 128 || v.rope) return KVQ_ERR_UNSUPPORTED;
  if (k.batch != v.batch || k.heads != v.heads || k.head_dim != v.head_dim || k.t_cap != v.t_cap ||
      k.bits != v.bits || k.group != v.group || k.n_sink != v.n_sink || k.rot != v.rot || k.quant != v.quant)
    return KVQ_ERR_INVALID;
  if (q_heads <= 0 || q_heads % k.heads) return KVQ_ERR_INVALID;
  // the attention kernels put batch x KV head (and batch x query head) on one grid axis
  if (static_cast<int64_t>(k.batch) * q_heads > 65535) return KVQ_ERR_UNSUPPORTED;
  const int gq = q_heads / k.heads;
  if (gq != 1 && gq != 2 && gq != 4 && gq != 8) return KVQ_ERR_UNSUPPORTED;
  if (n_tokens < 1 || n_tokens > k.t_cap) return KVQ_ERR_INVALID;
  *k_out = k;
  *v_out = v;
  return KVQ_OK;
}
}  // namespace

// The tables of an attention call: a sink list goes with both caches (they were
// encoded with it) and needs RoPE rows up to n_tokens for the keys.
static kvq_status check_attend_tables(const kvq_desc& k, const kvq_desc& v, const kvq_tables* tk, const kvq_tables* tv,
                               int32_t n_tokens) {
  if (!tk || !tv) return KVQ_ERR_INVALID;
  const bool listed = k.n_sink > 0 && tk->sink_pos;
  if (k.n_sink > 0 && (!tk->sink_pos != !tv->sink_pos)) return KVQ_ERR_INVALID;
  const int64_t rows = k.rope ? (listed ? n_tokens : (n_tokens < k.n_sink ? n_tokens : k.n_sink)) : 0;
  kvq_status s = check_tables(&k, tk, rows);
  if (s != KVQ_OK) return s;
  return check_tables(&v, tv, 0);
}

size_t kvq_attend_workspace_bytes(const kvq_desc* dk, const kvq_desc* dv, int32_t q_heads, int32_t n_tokens) {
  kvq_desc k, v;
  if (check_attend(dk, dv, q_heads, n_tokens, &k, &v) != KVQ_OK) return 0;
  return attend_workspace_bytes(k, q_heads, n_tokens);
}

kvq_status kvq_attend(const kvq_desc* dk, const kvq_desc* dv, const void* q, int32_t q_heads,
                      const kvq_packed* k_cache, const kvq_tables* tk, const kvq_packed* v_cache,
                      const kvq_tables* tv, int32_t n_tokens, float scale, float* out, void* workspace,
                      size_t workspace_bytes, kvq_stream_t stream) {
  kvq_desc k, v;
  kvq_status s = check_attend(dk, dv, q_heads, n_tokens, &k, &v);
  if (s != KVQ_OK) return s;
  if (!q || !out || !workspace) return KVQ_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256)) return KVQ_ERR_ALIGN;
  if (workspace_bytes < attend_workspace_bytes(k, q_heads, n_tokens)) return KVQ_ERR_INVALID;
  if ((s = check_attend_tables(k, v, tk, tv, n_tokens)) != KVQ_OK) return s;
  if ((s = check_packed(&k, k_cache)) != KVQ_OK || (s = check_packed(&v, v_cache)) != KVQ_OK) return s;
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  return launch_attend(k, v, q, q_heads, *k_cache, *tk, *v_cache, *tv, n_tokens, scale, out, workspace,
                       reinterpret_cast<cudaStream_t>(stream), ctx);
}

kvq_status kvq_attend_noalloc(const kvq_desc* dk, const kvq_desc* dv, const void* q, int32_t q_heads,
                              const kvq_packed* k_cache, const kvq_tables* tk, const kvq_packed* v_cache,
                              const kvq_tables* tv, int32_t n_tokens, float scale, float* out,
                              kvq_stream_t stream) {
  kvq_desc k, v;
  kvq_status s = check_attend(dk, dv, q_heads, n_tokens, &k, &v);
  if (s != KVQ_OK) return s;
  if (!q || !out) return KVQ_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(out, 16)) return KVQ_ERR_ALIGN;
  if (attend_workspace_bytes(k, q_heads, n_tokens) > attend_scratch_bytes()) return KVQ_ERR_UNSUPPORTED;
  if ((s = check_attend_tables(k, v, tk, tv, n_tokens)) != KVQ_OK) return s;
  if ((s = check_packed(&k, k_cache)) != KVQ_OK || (s = check_packed(&v, v_cache)) != KVQ_OK) return s;
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  void* ws = attend_scratch();
  if (!ws) return KVQ_ERR_CUDA;
  return launch_attend(k, v, q, q_heads, *k_cache, *tk, *v_cache, *tv, n_tokens, scale, out, ws,
                       reinterpret_cast<cudaStream_t>(stream), ctx);
}

kvq_status kvq_pair_energy(const kvq_desc* d, const void* x, uint64_t* energy_out, int16_t* rank_out,
                           kvq_stream_t stream) {
  kvq_status s = check_desc(d);
  if (s != KVQ_OK) return s;
  if (!x || !energy_out || !rank_out) return KVQ_ERR_INVALID;
  if (!aligned(x, 16) || !aligned(energy_out, 16) || !aligned(rank_out, 16)) return KVQ_ERR_ALIGN;
  if (static_cast<int64_t>(d->batch) * d->tokens >= (int64_t(1) << 31)) return KVQ_ERR_UNSUPPORTED;
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  return launch_pair_energy(*d, x, energy_out, rank_out, reinterpret_cast<cudaStream_t>(stream));
}

size_t kvq_calibrate_workspace_bytes(const kvq_desc* d) {
  if (check_desc(d) != KVQ_OK || d->rot == KVQ_ROT_ISO_SO4 || d->rot == KVQ_ROT_ISO_SO3) return 0;
  return calibrate_workspace_bytes(*d);
}

kvq_status kvq_calibrate_perm(const kvq_desc* d, const void* x, const kvq_tables* tb, int16_t* perm_out,
                              void* workspace, size_t workspace_bytes, kvq_stream_t stream) {
  kvq_status s = check_desc(d);
  if (s != KVQ_OK) return s;
  if (d->rot == KVQ_ROT_ISO_SO4 || d->rot == KVQ_ROT_ISO_SO3)
    return KVQ_ERR_UNSUPPORTED;  // no permutation in those variants
  if (!x || !perm_out || !workspace || !tb) return KVQ_ERR_INVALID;
  if (!aligned(x, 16) || !aligned(perm_out, 16) || !aligned(workspace, 256)) return KVQ_ERR_ALIGN;
  if (workspace_bytes < calibrate_workspace_bytes(*d)) return KVQ_ERR_INVALID;
  if (calibrate_rope(*d)) {
    if (!tb->rope_cs) return KVQ_ERR_INVALID;
    if (!aligned(tb->rope_cs, 16)) return KVQ_ERR_ALIGN;
    if (tb->rope_rows < static_cast<int64_t>(d->t0) + d->tokens || tb->rope_rows <= 0) return KVQ_ERR_INVALID;
  }
  if (tb->sink_pos && !aligned(tb->sink_pos, 4)) return KVQ_ERR_ALIGN;
  if (static_cast<int64_t>(d->batch) * d->tokens >= (int64_t(1) << 31)) return KVQ_ERR_UNSUPPORTED;
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  return launch_calibrate(*d, x, *tb, perm_out, workspace, reinterpret_cast<cudaStream_t>(stream), ctx.num_sms);
}

size_t kvq_calibrate_codebook_workspace_bytes(const kvq_desc* d) {
  if (check_desc(d) != KVQ_OK || (d->rot != KVQ_ROT_ISO_SO4 && d->rot != KVQ_ROT_ISO_SO3)) return 0;
  return calibrate_codebook_workspace_bytes(*d);
}

kvq_status kvq_calibrate_codebook(const kvq_desc* d, const void* x, const kvq_tables* tb, float* ch_scale_out,
                                  uint32_t* ch_wide_out, void* workspace, size_t workspace_bytes,
                                  kvq_stream_t stream) {
  kvq_status s = check_desc(d);
  if (s != KVQ_OK) return s;
  if (d->rot != KVQ_ROT_ISO_SO4 && d->rot != KVQ_ROT_ISO_SO3) return KVQ_ERR_UNSUPPORTED;
  if (!tb || !ch_scale_out || !ch_wide_out || !workspace || (d->tokens > 0 && !x)) return KVQ_ERR_INVALID;
  if (!tb->qL || (d->rot == KVQ_ROT_ISO_SO4 && !tb->qR)) return KVQ_ERR_INVALID;
  if ((x && !aligned(x, 16)) || !aligned(tb->qL, 16) || (tb->qR && !aligned(tb->qR, 16)) ||
      !aligned(ch_scale_out, 16) || !aligned(ch_wide_out, 4) || !aligned(workspace, 256) ||
      (tb->sink_pos && !aligned(tb->sink_pos, 4)))
    return KVQ_ERR_ALIGN;
  if (workspace_bytes < calibrate_codebook_workspace_bytes(*d)) return KVQ_ERR_INVALID;
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  return launch_calibrate_codebook(*d, x, *tb, ch_scale_out, ch_wide_out, workspace,
                                   reinterpret_cast<cudaStream_t>(stream));
}

size_t kvq_detect_sinks_workspace_bytes(const kvq_desc* d) {
  if (check_desc(d) != KVQ_OK) return 0;
  return detect_sinks_workspace_bytes(*d);
}

kvq_status kvq_detect_sinks(const kvq_desc* d, const void* x, double tau, int32_t max_sinks, int32_t* sink_pos,
                            int32_t* count, void* workspace, size_t workspace_bytes, kvq_stream_t stream) {
  kvq_status s = check_desc(d);
  if (s != KVQ_OK) return s;
  if (!x || !sink_pos || !workspace || d->tokens <= 0) return KVQ_ERR_INVALID;
  if (!isfinite(tau) || max_sinks < 1 || max_sinks > 65536) return KVQ_ERR_INVALID;
  if (!aligned(x, 16) || !aligned(workspace, 16) || !aligned(sink_pos, 4) || (count && !aligned(count, 4)))
    return KVQ_ERR_ALIGN;
  if (workspace_bytes < detect_sinks_workspace_bytes(*d)) return KVQ_ERR_INVALID;
  if (d->batch > 65535) return KVQ_ERR_UNSUPPORTED;  // one CTA per sequence on a grid axis
  LaunchCtx ctx;
  if ((s = get_ctx(&ctx)) != KVQ_OK) return s;
  return launch_detect_sinks(*d, x, tau, max_sinks, sink_pos, count, workspace,
                             reinterpret_cast<cudaStream_t>(stream), ctx.num_sms);
}

size_t kvq_packed_bytes(const kvq_desc* d, int32_t field) {
  if (!d) return 0;
  kvq_desc dd = *d;
  dd.tokens = 0;
  dd.t0 = 0;
  if (check_desc(&dd) != KVQ_OK) return 0;
  const size_t vecs = static_cast<size_t>(d->batch) * d->heads * d->t_cap;
  switch (field) {
    case KVQ_FIELD_CODES:
      return vecs * d->head_dim * d->bits / 8;
    case KVQ_FIELD_SCALE_ZERO:
      return d->quant == KVQ_Q_MINMAX ? vecs * (d->head_dim / d->group) * 4 : 0;
    case KVQ_FIELD_SINK:
      return static_cast<size_t>(d->batch) * d->heads * d->n_sink * d->head_dim * 2;
    case KVQ_FIELD_NORM:
      return (d->rot == KVQ_ROT_ISO_SO4 || d->rot == KVQ_ROT_ISO_SO3) ? vecs * 4 : 0;
    case KVQ_FIELD_EXT:
      return d->quant == KVQ_Q_CODEBOOK_DYN ? vecs * 2 : 0;
    default:
      return 0;
  }
}

kvq_status kvq_rope_table(float* cs_host, int32_t t_max, int32_t head_dim, double base) {
  return kvq_rope_table_ex(cs_host, t_max, head_dim, base, KVQ_ROPE_STANDARD);
}

kvq_status kvq_rope_table_ex(float* cs_host, int32_t t_max, int32_t head_dim, double base, int32_t freq) {
  if (!cs_host || t_max <= 0 || head_dim <= 0 || head_dim % 2 || !(base > 1.0)) return KVQ_ERR_INVALID;
  if (freq != KVQ_ROPE_STANDARD && freq != KVQ_ROPE_FREQ_AWARE) return KVQ_ERR_INVALID;
  if (freq == KVQ_ROPE_FREQ_AWARE && head_dim % 8) return KVQ_ERR_INVALID;
  const int half = head_dim / 2;
  for (int i = 0; i < half; ++i) {
    double theta;
    if (freq == KVQ_ROPE_FREQ_AWARE)  // two samplings: the upper half of the pairs twice as dense
      theta = i < head_dim / 4 ? pow(base, -2.0 * (i + head_dim / 8) / head_dim)
                               : pow(base, -static_cast<double>(i + 3 * head_dim / 4) / head_dim);
    else
      theta = pow(base, -(2.0 * i) / head_dim);
    for (int64_t m = 0; m < t_max; ++m) {
      const double ang = static_cast<double>(m) * theta;
      cs_host[(m * half + i) * 2] = static_cast<float>(cos(ang));
      cs_host[(m * half + i) * 2 + 1] = static_cast<float>(sin(ang));
    }
  }
  return KVQ_OK;
}

kvq_status kvq_lloyd_max_codebook(float* levels_host, int32_t bits, int32_t head_dim) {
  if (!levels_host || bits < 1 || bits > 5 || head_dim <= 0) return KVQ_ERR_INVALID;
  const int n = 1 << bits;
  double lv[32], bd[33];
  for (int k = 0; k < n; ++k) lv[k] = -3.0 + 6.0 * (k + 0.5) / n;
  for (int it = 0; it < 200000; ++it) {
    bd[0] = -INFINITY;
    bd[n] = INFINITY;
    for (int k = 1; k < n; ++k) bd[k] = 0.5 * (lv[k - 1] + lv[k]);
    double moved = 0.0;
    for (int k = 0; k < n; ++k) {
      const double nl = (phi_pdf(bd[k]) - phi_pdf(bd[k + 1])) / cell_mass(bd[k], bd[k + 1]);
      moved = fmax(moved, fabs(nl - lv[k]));
      lv[k] = nl;
    }
    if (moved < 1e-15) break;
  }
  for (int k = 0; k < n; ++k) levels_host[k] = static_cast<float>(lv[k] / sqrt(static_cast<double>(head_dim)));
  return KVQ_OK;
}

kvq_status kvq_check(kvq_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return KVQ_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)) != cudaSuccess) return KVQ_ERR_CUDA;
  if (w) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return KVQ_ERR_CUDA;
    return (w & kErrTimeout) ? KVQ_ERR_TIMEOUT : KVQ_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_debug_expire_wait(uint32_t limit_us, kvq_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return KVQ_ERR_INVALID;
  LaunchCtx ctx;
  kvq_status s = get_ctx(&ctx);
  if (s != KVQ_OK) return s;
  return launch_debug_wait(static_cast<uint64_t>(limit_us) * 1000ull, reinterpret_cast<cudaStream_t>(stream), ctx);
}

const char* kvq_status_str(kvq_status s) {
  switch (s) {
    case KVQ_OK:
      return "ok";
    case KVQ_ERR_INVALID:
      return "invalid argument";
    case KVQ_ERR_UNSUPPORTED:
      return "unsupported parameters";
    case KVQ_ERR_ALIGN:
      return "misaligned pointer";
    case KVQ_ERR_CUDA:
      return "CUDA error";
    case KVQ_ERR_TIMEOUT:
      return "kernel wait timed out";
    default:
      return "unknown status";
  }
}

int32_t kvq_version(void) { return 100; }

}  // extern "C"
