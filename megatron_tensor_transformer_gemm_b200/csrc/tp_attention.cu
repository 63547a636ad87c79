// Causal attention on each shard's local heads (forward and backward).
#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpi {

tp_status launch_attention_fwd(const tp_plan*, int, int, const PtrArray&, const MutPtrArray&,
                               float* const*, cudaStream_t) {
  return fail(TP_ERR_UNSUPPORTED, "attention forward is not built yet");
}

tp_status launch_attention_bwd(tp_plan*, int, int, const PtrArray&, const PtrArray&,
                               const PtrArray&, const float* const*, const MutPtrArray&,
                               cudaStream_t) {
  return fail(TP_ERR_UNSUPPORTED, "attention backward is not built yet");
}

}  // namespace tpi
