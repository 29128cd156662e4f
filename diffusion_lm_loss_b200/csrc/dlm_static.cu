// dlm_static.cu -- dlm_loss_fwd_bwd for callers that cannot allocate device
// memory.
//
// Some callers are not allowed to call cudaMalloc (or any allocating
// routine): code that only receives input and output buffers from a host
// program that owns all device memory -- a plugin or hook inside another
// framework, a process whose memory is carved up by a fixed-budget pool -- and
// so cannot obtain the caller workspace that dlm_loss_fwd_bwd needs.  For them
// the scratch of the loss lives in a fixed array in this library's device
// image instead.  Every GPU that loads the library holds the array until the
// process exits.
//
// The entry point allocates nothing: it finds the array's device address
// (see below) and forwards to dlm_loss_fwd_bwd with that address as the
// workspace.  Everything the loss needs zeroed at the start of
// a call is cleared by the loss itself on every call (its row-plan kernel
// rewrites the header and the completion counter), so the contents a previous
// call left in the array do no harm.
#include "dlm_host.h"

namespace dlm {

// The scratch.  Host code must not use this name as a device address: on the
// host it is only a stand-in for the symbol; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_loss_scratch[DLM_STATIC_SCRATCH_BYTES];

// Device address of g_loss_scratch in the context current on the calling
// thread.  Looked up on every call, not cached: the address belongs to the
// context that loaded this library's device code, and a caller may run under
// a context other than the device's primary one, or reset the device between
// calls, after which a cached address would point at memory that is gone.
// The lookup is a host-side table query and allocates nothing; the first one
// in a context also loads the library's device code into it.
static dlm_status_t scratch_address(void** out) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_loss_scratch);
    if (e != cudaSuccess || !p) {
        cudaGetLastError();
        return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "cudaGetSymbolAddress(scratch)");
    }
    *out = p;
    return DLM_OK;
}

}  // namespace dlm

extern "C" dlm_status_t dlm_loss_fwd_bwd_static(const dlm_layout_t* layout, const uint16_t* logits, int64_t ld,
                                                int32_t vocab, const int32_t* clean_ids,
                                                const uint8_t* corrupted, const float* p, int32_t mode,
                                                int32_t align, const dlm_layout_t* enc_layout,
                                                const uint16_t* enc_logits, int64_t enc_ld, const int32_t* enc_ids,
                                                float enc_ar_weight, float grad_scale, float* loss,
                                                float* unit_loss, uint16_t* dlogits, uint16_t* enc_dlogits,
                                                dlm_stream_t stream) {
    DLM_NVTX("dlm_loss_fwd_bwd_static");
    if (!dlm::layout_ok(layout)) return DLM_ERR_INVALID_ARGUMENT;
    if (enc_logits && !dlm::layout_ok(enc_layout)) return DLM_ERR_INVALID_ARGUMENT;
    const size_t need = dlm_loss_workspace_size(layout, enc_logits ? enc_layout : nullptr);
    if (need > size_t(DLM_STATIC_SCRATCH_BYTES)) return DLM_ERR_WORKSPACE_TOO_SMALL;
    dlm_status_t st = dlm::check_device();
    if (st != DLM_OK) return st;
    void* ws = nullptr;
    if ((st = dlm::scratch_address(&ws)) != DLM_OK) return st;
    return dlm_loss_fwd_bwd(layout, logits, ld, vocab, clean_ids, corrupted, p, mode, align, enc_layout,
                            enc_logits, enc_ld, enc_ids, enc_ar_weight, grad_scale, loss, unit_loss, dlogits,
                            enc_dlogits, ws, size_t(DLM_STATIC_SCRATCH_BYTES), stream);
}
