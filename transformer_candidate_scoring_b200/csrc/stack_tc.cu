// Tensor-core (tcgen05) kernels: placeholder until the fused kernels land.
#include "model.cuh"

namespace tr {
tr_status tc_build(tr_model*) { return TR_OK; }
bool tc_stack_supported(const tr_model*) { return false; }
tr_status tc_score(const tr_model*, const void*, int64_t, const int64_t*, const void* const*, const int32_t*,
                   const int32_t*, int, float*, cudaStream_t) {
  return fail(TR_ERR_UNSUPPORTED, "tensor-core stack not built");
}
bool tc_comp_supported(const tr_model*) { return false; }
tr_status tc_compress(const tr_model*, const void*, int64_t, void*, cudaStream_t) {
  return fail(TR_ERR_UNSUPPORTED, "tensor-core compressor not built");
}
}  // namespace tr
