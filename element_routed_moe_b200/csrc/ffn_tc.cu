// Tensor-core (tcgen05, 3xTF32) grouped expert MLP.  Not built yet: the
// entry points report JANUS_ERR_INVALID_ARG for this mode.
#include "ffn_tc.cuh"

namespace janus {
namespace tc {

size_t workspace_extra() { return 0; }

janus_status expert_ffn_fwd(const float*, const int32_t*, int32_t, int64_t, int32_t, int32_t,
                            const float*, const float*, float*, float*, float*, void*,
                            cudaStream_t) {
  return JANUS_ERR_INVALID_ARG;
}

janus_status expert_ffn_vjp(const float*, const float*, const float*, float*, const int32_t*,
                            int32_t, int64_t, int32_t, int32_t, const float*, const float*,
                            float*, float*, void*, cudaStream_t) {
  return JANUS_ERR_INVALID_ARG;
}

}  // namespace tc
}  // namespace janus
