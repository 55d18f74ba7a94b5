#include "sana_internal.h"
namespace sana {
sana_status gemm_run(long long, int, int, const void*, long long, const void*, void*, long long, int, cudaStream_t) { return fail(SANA_ERR_UNSUPPORTED, "gemm: not built yet"); }
}
extern "C" size_t sana_hybrid_stack_workspace_size(const sana_shape*, const sana_stack_config*) { return 0; }
extern "C" sana_status sana_hybrid_stack_fwd(const sana_shape*, const sana_stack_config*, const sana_stack_weights*, const sana_rope*, const void*, void*, void*, size_t, sana_stream_t) { return sana::fail(SANA_ERR_UNSUPPORTED, "stack: not built yet"); }
