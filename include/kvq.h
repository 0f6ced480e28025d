/*
 * kvq.h -- C ABI of libkvq: rotation + low-bit quantization of an LLM's fp16
 * KV cache on one NVIDIA B200 (sm_100a), its inverse, and the fused
 * decode-step q.K^T score.
 *
 * Pages the operations come from (title, section):
 *   [RoPE-KV]  "RoPE启发的KV缓存压缩技术解析"
 *   [EliteKV]  "EliteKV - RoPE频率选择与低秩投影"
 *   [IsoQuant] "KV缓存压缩技术：IsoQuant在大语言模型中的应用"
 *   [RotateKV] "RotateKV: Accurate and Robust 2-Bit KV Cache Quantization for
 *              LLMs via Outlier-Aware Adaptive Rotations"
 *
 * Conventions for every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller unless a
 *    parameter says "host". The library allocates no device memory, keeps
 *    only a per-device error word (see kvq_check), never synchronises the
 *    stream except in kvq_check, and is safe to call from several threads.
 *  - Arguments are validated on the host before anything is launched; a bad
 *    argument returns a status and launches nothing.
 *  - Layouts are dense and row-major. fp16 is IEEE binary16.
 *  - Inputs holding NaN/Inf, or whose rotated values exceed the fp16 range
 *    (|v| > 65504, so the fp16 zero/scale overflow), give unspecified codes
 *    but never out-of-bounds accesses.
 *  - Output buffers must not overlap inputs.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* kvq_stream_t;

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID = 1,     /* null pointer, bad shape or range */
  KVQ_ERR_UNSUPPORTED = 2, /* valid but not implemented (head_dim, bits, combination) */
  KVQ_ERR_ALIGN = 3,       /* a pointer is not aligned as required below */
  KVQ_ERR_CUDA = 4,        /* a CUDA call or launch failed */
  KVQ_ERR_TIMEOUT = 5      /* a kernel gave up waiting on a copy (from kvq_check) */
} kvq_status;

/* Rotation applied before quantization. */
enum {
  KVQ_ROT_NONE = 0,       /* quantize the (RoPE'd) vector as is */
  KVQ_ROT_FWHT_HEAD = 1,  /* [RotateKV] RoPE -> channel permutation -> normalised FWHT over head_dim */
  KVQ_ROT_FWHT_GROUP = 2, /* [RotateKV] pre-RoPE grouped-head rotation: permutation -> normalised FWHT
                             over group_heads*head_dim channels (the heads of one token concatenated)
                             -> RoPE on each head slice */
  KVQ_ROT_ISO_SO4 = 3,    /* [IsoQuant §2.2, §3.1] norm split rho = ||x||, x/(rho+1e-8), then
                             w = qL (x) v (x) qR on each 4-D block v */
  KVQ_ROT_ISO_SO3 = 4     /* [IsoQuant §2.1, §1] the same norm split, then the 3-D sandwich
                             w = q v q* on each block of 3 channels taken as a pure quaternion; a
                             2-channel tail (head_dim 128: 42 blocks + 2) is turned in its plane by
                             the same sandwich, a 1-channel tail (64, 256) is kept as it is */
};

/* Scalar quantizer. */
enum {
  KVQ_Q_MINMAX = 0,   /* per-token per-group asymmetric min-max, fp16 (scale, zero); with
                         rot in {NONE, FWHT_HEAD, FWHT_GROUP} */
  KVQ_Q_CODEBOOK = 1, /* fixed scalar codebook (Lloyd-Max, [IsoQuant §3.1]); with rot = ISO_SO4
                         or ISO_SO3 */
  KVQ_Q_CODEBOOK_DYN = 2 /* dynamic codebooks ([IsoQuant §4.2]); with rot = ISO_SO4 or ISO_SO3:
                         channel j of head h quantizes against the levels fp32(ch_scale[h][j] * l_k)
                         of the N(0,1) Lloyd-Max design l -- `codebook` (2^bits levels), or
                         `codebook_wide` (2^(bits+1) levels, twice the codebook) for the channels
                         marked in ch_wide -- with fp32 midpoints as boundaries (ties to the lower
                         code). The low `bits` bits of every code go to the record as for
                         KVQ_Q_CODEBOOK; the top bit of each marked channel's code goes to
                         ext[slot], in ascending channel order, LSB first (at most 16 marked
                         channels per head; bits of further ones are dropped). Fill the tables with
                         kvq_calibrate_codebook and kvq_lloyd_max_codebook(.., head_dim = 1). */
};

/* Which packed buffer kvq_packed_bytes sizes. */
enum { KVQ_FIELD_CODES = 0, KVQ_FIELD_SCALE_ZERO = 1, KVQ_FIELD_SINK = 2, KVQ_FIELD_NORM = 3, KVQ_FIELD_EXT = 4 };

typedef struct {
  int32_t batch;       /* B > 0 */
  int32_t heads;       /* H > 0: KV heads */
  int32_t head_dim;    /* D: 64 or 128 (128 only for FWHT_GROUP) */
  int32_t tokens;      /* T >= 0: tokens in this call (T = 0 is a no-op) */
  int32_t t0;          /* first cache slot written/read; also the RoPE position of token 0 */
  int32_t t_cap;       /* cache capacity in slots; t0 + T <= t_cap */
  int32_t bits;        /* 2, 3 or 4 */
  int32_t group;       /* min-max group size in channels: 32, 64 or 128, dividing head_dim
                          (at least head_dim*group_heads/128 channels for FWHT_GROUP) */
  int32_t group_heads; /* FWHT_GROUP: 2, 4 or 8 consecutive heads per rotation, dividing heads */
  int32_t rope;        /* 0: no RoPE (values); 1: RoPE on the interleaved pairs (2i, 2i+1) of the
                          rotation matrix ([EliteKV §2.1]); 2: RoPE on the half-split pairs
                          (i, i + head_dim/2) of the page's apply_rope code ([EliteKV §7.1]);
                          pair i turns by m*theta_i either way, from the same table */
  int32_t n_sink;      /* attention sinks kept verbatim in fp16: positions 0..n_sink-1, or the
                          n_sink entries of kvq_tables.sink_pos when that is given */
  int32_t rot;         /* KVQ_ROT_* */
  int32_t quant;       /* KVQ_Q_* */
} kvq_desc;

/* The compressed cache. Slot s of head (b, h) is record (b*H + h)*t_cap + s.
 *   codes       u8   [B][H][t_cap][head_dim*bits/8]  code j of a record occupies bits
 *                     [bits*j, bits*j+bits) of its little-endian byte stream (LSB first)
 *   scale_zero  half [B][H][t_cap][head_dim/group][2]  (scale S, zero Z); min-max only
 *   sink        half [B][H][n_sink][head_dim]          the sink positions, verbatim (row k: position
 *                                                     k, or the list's entry k)
 *   norm        f32  [B][H][t_cap]                      rho; ISO_SO4 and ISO_SO3 only
 *   ext         u16  [B][H][t_cap]                      KVQ_Q_CODEBOOK_DYN only: the top bits of the
 *                                                     outlier channels' codes
 * Slots of sink positions hold zero codes, zero scale/zero, zero norm and zero ext.
 * Alignment: codes, scale_zero and sink 16 bytes; norm 4 bytes; ext 2 bytes. Unused fields may
 * be NULL. */
typedef struct {
  uint8_t* codes;
  void* scale_zero;
  void* sink;
  float* norm;
  uint16_t* ext;
} kvq_packed;

/* Read-only tables (device pointers).
 *   perm      int16 [H][head_dim] or NULL (identity): the permutation step gathers
 *             p_j = y_perm[h][j] ([RotateKV] channel reordering); must be a permutation
 *   rope_cs   f32 [rope_rows][head_dim/2][2] = (cos, sin) of position m times
 *             theta_i = 10000^(-2i/head_dim) ([EliteKV §2.1]); fill it with kvq_rope_table.
 *             16-byte aligned. Required when rope != 0.
 *   qL, qR    f32 [head_dim/4][4] unit quaternions (real, i, j, k), one pair per 4-D block
 *             (ISO_SO4). ISO_SO3 reads qL only: f32 [ceil(head_dim/3)][4], one unit quaternion
 *             per 3-channel block and, when head_dim mod 3 = 2, one for the 2-channel tail whose
 *             i and j parts must be zero (otherwise the tail's output is not a rotation)
 *   codebook  f32 [1 << bits] ascending levels (kvq_lloyd_max_codebook); for KVQ_Q_CODEBOOK_DYN
 *             the N(0,1) levels (head_dim 1)
 *   codebook_wide  f32 [2 << bits] KVQ_Q_CODEBOOK_DYN: the N(0,1) levels of bits + 1
 *   ch_scale  f32 [H][head_dim] KVQ_Q_CODEBOOK_DYN: per-channel scale (kvq_calibrate_codebook),
 *             16-byte aligned
 *   ch_wide   u32 [H][head_dim/32] KVQ_Q_CODEBOOK_DYN: bit j of word j/32 marks channel j as an
 *             outlier channel (the wide codebook), 4-byte aligned
 *   sink_pos  int32 [B][n_sink] or NULL (the sinks are positions 0..n_sink-1): the list form
 *             of the sink set ([RotateKV] attention sinks found from the activations, e.g. by
 *             kvq_detect_sinks). Entry k of sequence b is the position (cache slot) whose fp16
 *             row is sink row k, or -1 for an unused entry; entries must be distinct. 4-byte
 *             aligned. Read by kvq_encode, kvq_decode, kvq_score, kvq_score_literal,
 *             kvq_calibrate_perm and kvq_attend (which needs it in both caches' tables). With a
 *             list, encode, decode and score run their kernels on every slot and one more small
 *             kernel then writes the sink entries; kvq_score and kvq_attend then need
 *             rope_rows >= n_tokens when rope != 0. */
typedef struct {
  const int16_t* perm;
  const float* rope_cs;
  int32_t rope_rows;
  const float* qL;
  const float* qR;
  const float* codebook;
  const int32_t* sink_pos;
  const float* codebook_wide;
  const float* ch_scale;
  const uint32_t* ch_wide;
} kvq_tables;

/* Encode T tokens into cache slots t0..t0+T-1.
 * x: half [B][H][T][head_dim], 16-byte aligned. Per token-head vector (or per token and head
 * group for FWHT_GROUP): the rotation of d->rot, then the quantizer of d->quant, then bit
 * packing. Min-max ([RotateKV] 2-bit KV quantization; the fp16 rounding reading): per group of
 * `group` consecutive rotated channels, Z = largest fp16 <= min, S = smallest fp16 >=
 * fp32((max - Z)/(2^bits - 1)), code = round-half-even(fp32(p - Z) * fp32(1/S)), so codes lie
 * in [0, 2^bits - 1]. Codebook: code = number of fp32 midpoints 0.5*(l_k + l_{k+1}) below w.
 * Sink positions (< n_sink, or those listed in tb->sink_pos) are copied to `sink` verbatim
 * ([RotateKV] attention sinks). */
kvq_status kvq_encode(const kvq_desc* d, const void* x, const kvq_tables* tb, const kvq_packed* out,
                      kvq_stream_t stream);

/* Decode slots t0..t0+T-1 back to the encoder's input basis (pre-RoPE keys, raw values):
 * dequantize (Z + c*S, or the codebook level), then the inverse rotation in reverse order
 * ([IsoQuant §3.1] step 3: inverse rotation, then restore the norm), then the inverse RoPE.
 * x_out: [B][H][T][head_dim], fp32 if out_fp32 else fp16 (round to nearest), 16-byte
 * aligned. Sink positions come back verbatim. */
kvq_status kvq_decode(const kvq_desc* d, const kvq_packed* in, const kvq_tables* tb, void* x_out,
                      int32_t out_fp32, kvq_stream_t stream);

/* Decode-step attention scores ([EliteKV §2.2]: A_{m,n} = q_m^rot . k_n^rot / sqrt(d)):
 *   scores[b][qh][n] = scale * <q[b][qh], khat[b][qh / (q_heads/H)][n]>,  n in [0, n_tokens)
 * q: half [B][q_heads][head_dim] in attention space (RoPE'd at the query position); q_heads a
 * multiple of H (grouped-query attention). khat_n is the key in attention space: RoPE_n(sink_n)
 * for a sink position n, else slot n decoded without the inverse RoPE. Supported for rot in
 * {NONE, FWHT_HEAD} with min-max codes; the kernel rotates the query once instead of every key
 * (q . P^T H y = (H P q) . y for the orthonormal H and permutation P). Also for FWHT_GROUP
 * (the grouped-head rotation) with rope != 0, no permutation, q_heads/H in {1, 2, 4, 8} and
 * rope_rows >= n_tokens: RoPE comes after the rotation there, so each key is decoded (inverse
 * FWHT over its head group) and turned to its position before the dot product.
 * scores: f32 [B][q_heads][n_tokens]; n_tokens <= t_cap. d->tokens and d->t0 are ignored.
 * Accuracy: the head-variant tensor-core path rounds the rotated query to 16-bit integer digits,
 * so a score's error is bounded by scale * max|H P q| / 64000 * sum_j |y_j| over the stored
 * rotated key y; a key with a massive activation that is neither a sink nor listed spreads it
 * over all rotated channels and can exceed 1e-3 of sum_j |q_j khat_j|. kvq_score_literal has
 * no such term (fp32 throughout). */
kvq_status kvq_score(const kvq_desc* d, const void* q, int32_t q_heads, const kvq_packed* cache,
                     const kvq_tables* tb, int32_t n_tokens, float scale, float* scores,
                     kvq_stream_t stream);

/* Decode-step score in its literal form ([EliteKV §2.2]; [RotateKV] 关键设计: the inverse
 * rotation of the head-variant cache): the same scores as kvq_score, with every key decoded on
 * the fly (unpack, dequantize, inverse FWHT per token) instead of transforming the query once.
 * The channel permutation is applied to the query (sum_i q_i khat_i = sum_j q_perm[j] p_j).
 * fp32 throughout (no integer query digits), so it is the reference form the query-rotation
 * kernel is measured against, at several times its instruction count per element.
 * Arguments, layouts and sinks (prefix or listed) as kvq_score. Supported for rot in
 * {NONE, FWHT_HEAD}, head_dim 128, min-max codes, q_heads/H in {1, 2, 4, 8}; other shapes
 * return KVQ_ERR_UNSUPPORTED. */
kvq_status kvq_score_literal(const kvq_desc* d, const void* q, int32_t q_heads, const kvq_packed* cache,
                             const kvq_tables* tb, int32_t n_tokens, float scale, float* scores,
                             kvq_stream_t stream);

/* Decode-step attention over the compressed cache ([EliteKV §2.2] scores; [EliteKV §7.1] the
 * softmax of the scaled scores weights the values):
 *   out[b][qh] = sum_n p_n vhat[b][h][n],  p = softmax_n(scale * <q[b][qh], khat[b][h][n]>),
 *   n in [0, n_tokens), h = qh / (q_heads/H).
 * khat_n is the kvq_score key (K cache: dk, k_cache, tk); vhat_n is value slot n decoded as by
 * kvq_decode (V cache: dv, v_cache, tv), the sink rows verbatim. dk and dv must agree in batch,
 * heads, head_dim (= 128), t_cap, bits, group, n_sink, rot (NONE or FWHT_HEAD) and quant
 * (MINMAX); dv->rope must be 0 and q_heads/H in {1, 2, 4, 8} (else KVQ_ERR_UNSUPPORTED).
 * The value decode is linear in the dequantized codes y_n, so sum_n p_n vhat_n =
 * P^T H_norm (sum_n p_n y_n): the inverse rotation runs once per output, not per token.
 * q: half [B][q_heads][head_dim] in attention space, 16-byte aligned. out: f32
 * [B][q_heads][head_dim], 16-byte aligned. workspace: caller-owned device memory, 256-byte
 * aligned, at least kvq_attend_workspace_bytes() bytes; it holds per-chunk partial sums (and,
 * outside the fused form, the scores), needs no initialisation and must not be shared by calls
 * in flight at the same time. d->tokens and d->t0 are ignored. With 2- or 4-bit codes and one
 * group per record (group = 128) two kernels run on `stream`: a fused pass over the K and V
 * records (scores, running softmax and value sums on the tensor cores) and a merge launched as
 * its programmatic dependent; other shapes run three (scores, chunked softmax-weighted sums,
 * merge). Results agree with kvq_score's scores through an exact fp64 softmax within
 * 2e-5 * max|vhat|. Sinks given as a list (tk->sink_pos and tv->sink_pos, the list both caches
 * were encoded with; one without the other is KVQ_ERR_INVALID) enter with their exact fp16
 * scores and rows; the fused form masks the listed slots and takes up to 32 entries, longer
 * lists run the three-kernel form. */
kvq_status kvq_attend(const kvq_desc* dk, const kvq_desc* dv, const void* q, int32_t q_heads,
                      const kvq_packed* k_cache, const kvq_tables* tk, const kvq_packed* v_cache,
                      const kvq_tables* tv, int32_t n_tokens, float scale, float* out, void* workspace,
                      size_t workspace_bytes, kvq_stream_t stream);

/* kvq_attend without a workspace argument, for callers that cannot allocate device memory
 * when they call (a fixed-budget serving loop, host code without a device allocator, a caller
 * whose workspace would have to stay put between repeated launches of the same work). The
 * pages have no counterpart: it is a variant of kvq_attend with the same arguments and
 * results, whose workspace (chunk partials, and the scores outside the fused form) lives in a
 * fixed 40 MiB device array of the library (enough for 4 sequences x 32 query heads x 32769
 * cached tokens in either form); it allocates nothing.
 * Returns KVQ_ERR_UNSUPPORTED when kvq_attend_workspace_bytes() exceeds 40 MiB. The array's
 * device address is looked up once per device, by the first call of ANY libkvq entry point that
 * launches work with that device current; with CUDA's lazy module loading (the default) that
 * lookup is also when the driver reserves the array, so make one library call that launches
 * work on each device (an encode, a decode, a score) before the serving loop, and outside any
 * stream capture; a kvq_attend_noalloc that is itself that first call reserves the array then. If the array could not be reserved, this entry point returns KVQ_ERR_CUDA; the
 * others are unaffected. The array is shared by every call on a device: two
 * calls that can run at the same time (different streams, or host threads without ordering)
 * race on it and corrupt each other's results; calls in order on one stream are safe. Nothing
 * in it needs to start at zero. */
kvq_status kvq_attend_noalloc(const kvq_desc* dk, const kvq_desc* dv, const void* q, int32_t q_heads,
                              const kvq_packed* k_cache, const kvq_tables* tk, const kvq_packed* v_cache,
                              const kvq_tables* tv, int32_t n_tokens, float scale, float* out,
                              kvq_stream_t stream);

/* Workspace bytes kvq_attend needs for these arguments; 0 if they are invalid or unsupported. */
size_t kvq_attend_workspace_bytes(const kvq_desc* dk, const kvq_desc* dv, int32_t q_heads, int32_t n_tokens);

/* Channel permutation by abs-max ([RotateKV] outlier-aware rotation: channel reordering before
 * the FWHT). For each head h, a_j = max over the B batches and the positions t0..t0+T-1 that are
 * not sinks (position >= n_sink, or not in tb->sink_pos) of |y_j|, where y is the fp32 input of the permutation step:
 * RoPE_m(x), with kvq_encode's fp32 arithmetic, for rope = 1 and rot NONE or FWHT_HEAD (RoPE comes
 * before the permutation there); x itself otherwise (values; FWHT_GROUP permutes the raw input).
 * perm_out[h] lists the channels by descending a_j, equal a_j in ascending channel order: a table
 * for kvq_tables.perm.
 *   x          half [B][H][T][head_dim], 16-byte aligned (the tensor kvq_encode would take)
 *   tb         rope_cs as for kvq_encode when RoPE applies (other fields unused)
 *   perm_out   int16 [H][head_dim], 16-byte aligned, overwritten
 *   workspace  device memory of at least kvq_calibrate_workspace_bytes(d) bytes (H * head_dim * 4),
 *              256-byte aligned; its contents do not matter (the call zeroes it on the stream first),
 *              the caller owns it
 * The result is integer and exact: it does not depend on scheduling. KVQ_ERR_UNSUPPORTED for
 * ISO_SO4 (no permutation there) and for B*T >= 2^31. */
kvq_status kvq_calibrate_perm(const kvq_desc* d, const void* x, const kvq_tables* tb, int16_t* perm_out,
                              void* workspace, size_t workspace_bytes, kvq_stream_t stream);

/* Workspace bytes kvq_calibrate_perm needs for d; 0 if d is invalid or unsupported. */
size_t kvq_calibrate_workspace_bytes(const kvq_desc* d);

/* Dynamic codebook tables ([IsoQuant §4.2]: the values of each channel are gathered online, the
 * quantization boundaries set by the KL divergence, and outlier channels get a codebook twice the
 * size). For each head h and channel j of the rotated unit vectors w (the quantizer's input of
 * kvq_encode with d->rot, ISO_SO4 or ISO_SO3, over the B batches and the positions t0..t0+T-1
 * that are not sinks):
 *   m2 = mean of w_j^2 (fp64 sums), ch_scale[h][j] = fp32(sqrt(m2)): the sigma of N(0, sigma^2)
 *        nearest to the channel's values in KL divergence (that divergence is
 *        const + log sigma + m2 / (2 sigma^2)); fp32(1/sqrt(head_dim)) when no position counts;
 *   ch_wide[h]: channels with ch_scale > 2 x the lower median of the head's scales, at most
 *        head_dim/8 of them, the largest first, equal scales to the lower channel.
 *   x          half [B][H][T][head_dim], 16-byte aligned
 *   tb         qL (and qR for ISO_SO4) as for kvq_encode; sink_pos optional
 *   ch_scale_out  f32 [H][head_dim], 16-byte aligned;  ch_wide_out  u32 [H][head_dim/32]
 *   workspace  device memory of kvq_calibrate_codebook_workspace_bytes(d) bytes, 256-byte aligned
 * Two kernels: per (sequence, head, 1024-token chunk) sums in a fixed order, then one CTA per head;
 * the result does not depend on scheduling. KVQ_ERR_UNSUPPORTED for other rotations and for
 * B*H > 65535. */
kvq_status kvq_calibrate_codebook(const kvq_desc* d, const void* x, const kvq_tables* tb, float* ch_scale_out,
                                  uint32_t* ch_wide_out, void* workspace, size_t workspace_bytes,
                                  kvq_stream_t stream);

/* Workspace bytes kvq_calibrate_codebook needs for d; 0 if d is invalid or unsupported. */
size_t kvq_calibrate_codebook_workspace_bytes(const kvq_desc* d);

/* Attention sinks by massive activations ([RotateKV] abstract (iii) and 关键设计: the sink
 * tokens carry activations far above the rest and are found from them). Per sequence b of the
 * T tokens x[b][:, t] at positions t0 + t:
 *   a_t  = max over heads and channels of |x[b][h][t][j]| (exact: fp16 magnitudes),
 *   med  = the lower median of a_0 .. a_{T-1} (ascending rank floor((T-1)/2)),
 *   sinks: the tokens with a_t > tau * med, the product and the comparison in fp64; at most
 *          max_sinks of them, the largest a_t first, equal a_t to the earlier token.
 *   x          half [B][H][T][head_dim], 16-byte aligned (only batch, heads, head_dim, tokens, t0
 *              of d are used, but d must be valid as a whole)
 *   sink_pos   int32 [B][max_sinks], overwritten: the sinks' positions ascending, then -1; it is
 *              kvq_tables.sink_pos for a descriptor with n_sink = max_sinks
 *   count      int32 [B] or NULL: how many sinks each sequence has
 *   workspace  device memory of at least kvq_detect_sinks_workspace_bytes(d) bytes, 16-byte
 *              aligned, caller-owned, contents irrelevant
 * tau must be finite, max_sinks in 1..65536, tokens > 0 (else KVQ_ERR_INVALID). Two kernels run
 * on `stream`: one pass over x (the per-token maxima), then one CTA per sequence. NaN inputs
 * give an unspecified list. */
kvq_status kvq_detect_sinks(const kvq_desc* d, const void* x, double tau, int32_t max_sinks, int32_t* sink_pos,
                            int32_t* count, void* workspace, size_t workspace_bytes, kvq_stream_t stream);

/* Workspace bytes kvq_detect_sinks needs for d (2 bytes per token, rounded up to 16); 0 if d is
 * invalid. */
size_t kvq_detect_sinks_workspace_bytes(const kvq_desc* d);

/* Energy of each RoPE frequency pair ([EliteKV] §3.1, frequency energy analysis): per head h,
 *   E[h][i] = sum over the B batches and the T tokens of x[..][2i]^2 + x[..][2i+1]^2,
 * on the keys as given (RoPE rotates each pair without changing its norm), exactly: every fp16
 * square is an integer multiple of 2^-48, and E is returned as an unsigned 128-bit count of 2^-48
 * (energy_out[h][i][0] = low 64 bits, [1] = high 64 bits; E = (lo + hi * 2^64) * 2^-48).
 * rank_out[h] lists the pairs by descending E, equal E in ascending pair order (the elite
 * frequencies are its first entries). Infinite or NaN inputs contribute nothing.
 *   x           half [B][H][T][head_dim], 16-byte aligned (only batch, heads, head_dim, tokens of d
 *               are used)
 *   energy_out  uint64 [H][head_dim/2][2], 16-byte aligned, zeroed and filled by the call
 *   rank_out    int16 [H][head_dim/2], 16-byte aligned
 * The results are integers and exact: they do not depend on scheduling. KVQ_ERR_UNSUPPORTED for
 * B*T >= 2^31. */
kvq_status kvq_pair_energy(const kvq_desc* d, const void* x, uint64_t* energy_out, int16_t* rank_out,
                           kvq_stream_t stream);

/* Bytes of one packed buffer (KVQ_FIELD_*) for this descriptor; 0 if the field is unused or
 * the descriptor is invalid. */
size_t kvq_packed_bytes(const kvq_desc* d, int32_t field);

/* Fill a HOST buffer cs[t_max][head_dim/2][2] with (float)cos(m*theta_i), (float)sin(m*theta_i),
 * theta_i = base^(-2i/head_dim), the angle formed in double ([RoPE-KV §1], [EliteKV §2.1]).
 * The caller copies it to the device. */
kvq_status kvq_rope_table(float* cs_host, int32_t t_max, int32_t head_dim, double base);

/* Frequency tables for kvq_rope_table_ex. Every kernel takes whatever table it is given. */
enum {
  KVQ_ROPE_STANDARD = 0,   /* theta_i = base^(-2i/head_dim): the kvq_rope_table table */
  KVQ_ROPE_FREQ_AWARE = 1  /* [KV-Latent] frequency-aware RoPE: pairs i < head_dim/4 take
                              base^(-2(i + head_dim/8)/head_dim), the others
                              base^(-(i + 3 head_dim/4)/head_dim): the highest frequencies are
                              skipped and the low ones sampled twice as densely */
};

/* kvq_rope_table with a choice of frequencies (KVQ_ROPE_*); head_dim a multiple of 8 for
 * KVQ_ROPE_FREQ_AWARE. Same layout and rounding: (float)cos / (float)sin of the double angle. */
kvq_status kvq_rope_table_ex(float* cs_host, int32_t t_max, int32_t head_dim, double base, int32_t freq);

/* Fill a HOST buffer with the 2^bits Lloyd-Max levels of N(0, 1/head_dim), ascending: Lloyd's
 * iteration on N(0,1) in double, scaled by 1/sqrt(head_dim), rounded to fp32 ([IsoQuant §3.1]).
 * bits 1..5 (5: the wide codebook of 4-bit dynamic codes). */
kvq_status kvq_lloyd_max_codebook(float* levels_host, int32_t bits, int32_t head_dim);

/* Synchronise `stream` and report (then clear) the device error word of the current device:
 * KVQ_ERR_TIMEOUT if a kernel gave up on a bounded wait, KVQ_ERR_CUDA on a CUDA error. */
kvq_status kvq_check(kvq_stream_t stream);

/* Test hook for the bounded-wait path: launches one CTA that waits on a copy that is never
 * issued, with the given limit in microseconds (1..1000000); the wait expires, the kernel sets
 * the error word and returns, and kvq_check then reports KVQ_ERR_TIMEOUT. */
kvq_status kvq_debug_expire_wait(uint32_t limit_us, kvq_stream_t stream);

const char* kvq_status_str(kvq_status s);

/* Library version, major*10000 + minor*100 + patch. */
int32_t kvq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
