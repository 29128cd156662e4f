// dlm_linear.cu -- fused lm_head + loss (placeholder until the tensor-core
// path is in place: refuses every call).
#include "dlm_host.h"

extern "C" size_t dlm_linear_loss_workspace_size(const dlm_layout_t*, int32_t, int32_t) { return 0; }

extern "C" dlm_status_t dlm_linear_loss_fwd_bwd(const dlm_layout_t*, const uint16_t*, const uint16_t*,
                                                int32_t, int32_t, const int32_t*, const uint8_t*,
                                                const float*, float, float*, float*, uint16_t*,
                                                uint16_t*, void*, size_t, dlm_stream_t) {
    return DLM_ERR_UNSUPPORTED;
}
