// dlm_host.h -- host-side helpers shared by the entry points: argument
// checks, the device capability check, launch-error mapping.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/dlm.h"

namespace dlm {

constexpr size_t kWsAlign = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The library is built for sm_100a only: refuse anything else up front.
dlm_status_t check_device();

// Remember the text of a CUDA error for dlm_last_cuda_error().
void record_cuda_error(cudaError_t e, const char* where);

inline dlm_status_t cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return DLM_OK;
    record_cuda_error(e, where);
    return DLM_ERR_CUDA;
}

inline dlm_status_t last_launch_status(const char* where = "kernel launch") {
    return cuda_status(cudaGetLastError(), where);
}

// Layout sanity that the host can see (the device checks cu_seqlens itself).
inline bool layout_ok(const dlm_layout_t* L) {
    if (!L) return false;
    if (L->n_units < 0 || L->n_tokens < 0) return false;
    if (L->n_units >= (1 << 24)) return false;
    if (L->n_tokens >= (int64_t(1) << 31)) return false;
    if (!L->cu_seqlens) {
        if (L->seq_len < 0) return false;
        if (int64_t(L->n_units) * L->seq_len != L->n_tokens) return false;
    } else if (L->n_units == 0 && L->n_tokens != 0) {
        return false;
    }
    return true;
}

// Number of logits rows described by a layout (one per token).
inline int64_t layout_rows(const dlm_layout_t* L) { return L ? L->n_tokens : 0; }

}  // namespace dlm
