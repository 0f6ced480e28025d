#include "kvq_internal.h"
namespace kvq {
kvq_status launch_encode_group(const kvq_desc&, const void*, const kvq_tables&, const kvq_packed&, cudaStream_t, const LaunchCtx&) { return KVQ_ERR_UNSUPPORTED; }
kvq_status launch_decode_group(const kvq_desc&, const kvq_packed&, const kvq_tables&, void*, int, cudaStream_t, const LaunchCtx&) { return KVQ_ERR_UNSUPPORTED; }
kvq_status launch_encode_iso(const kvq_desc&, const void*, const kvq_tables&, const kvq_packed&, cudaStream_t, const LaunchCtx&) { return KVQ_ERR_UNSUPPORTED; }
kvq_status launch_decode_iso(const kvq_desc&, const kvq_packed&, const kvq_tables&, void*, int, cudaStream_t, const LaunchCtx&) { return KVQ_ERR_UNSUPPORTED; }
kvq_status launch_score(const kvq_desc&, const void*, int, const kvq_packed&, const kvq_tables&, int, float, float*, cudaStream_t, const LaunchCtx&) { return KVQ_ERR_UNSUPPORTED; }
}
