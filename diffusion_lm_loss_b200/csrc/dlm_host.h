// dlm_host.h -- host-side helpers shared by the entry points: argument
// checks, the device capability check, launch-error mapping.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "../../include/dlm.h"

namespace dlm {

// NVTX range around an entry point, so a profiler's timeline shows each
// library call by name (header-only NVTX: a no-op unless a tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
#define DLM_NVTX(name) ::dlm::NvtxRange dlm_nvtx_range_(name)

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

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream is still running; it must call
// pdl_wait() before reading that kernel's results.
template <typename... KArgs, typename... Args>
inline dlm_status_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                               const char* what, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (e != cudaSuccess) cudaGetLastError();
    return cuda_status(e, what);
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

// Header of a loss workspace (first 256 bytes), written by the row-plan
// kernel and read by the kernels after it.
struct WsHeader {
    uint32_t status;      // DLM_DEV_* bits of this call
    int32_t n_scored;     // scored rows, both terms
    int32_t n_rows;       // rows, both terms
    int32_t n_nonpad;     // N of the diffusion layout
    int32_t n_scored_a;   // scored diffusion rows
    int32_t n_scored_b;   // scored encoder rows
    uint32_t ticket;      // completion counter of the unit reduction (zeroed by the plan)
    uint32_t next_s;      // CE row tickets: next scored / unscored list entry (zeroed by the plan)
    uint32_t next_u;
};
static_assert(sizeof(WsHeader) <= kWsAlign, "header");

// Objective options of the uniform-noise canvas term (see
// dlm_loss_fwd_bwd_ex); unit_cnt: [n_units] int32 scratch for the
// per-example mean.
struct ObjOpts {
    int time_weighting = DLM_TIME_WEIGHT_NONE;
    float weight_clip = 0.f;
    int reduction = DLM_REDUCE_TOKEN_MEAN;
    int32_t* unit_cnt = nullptr;
    int keep_unscored_rows = 0;   // unscored dlogits rows are not written
};

// Row plan (one cluster of CTAs): classifies every row of `a` (and of the
// encoder layout `b`, rows after a's), writes list[] = {row, target, weight
// bits, unit} with the scored rows first in row order, and fills *hdr.
dlm_status_t launch_plan(const dlm_layout_t* a, const int32_t* clean, const uint8_t* corrupted,
                         const float* p, int mode, int align, const dlm_layout_t* b,
                         const int32_t* ids_b, float lam, int vocab, WsHeader* hdr, int4* list,
                         cudaStream_t s, const ObjOpts& opts = ObjOpts());

// Per-unit sums of row_loss over a's rows (and b's rows, indexed after a's)
// and their total, in a fixed order.  Uses hdr->ticket (zeroed by the plan).
dlm_status_t launch_reduce(const dlm_layout_t* a, const dlm_layout_t* b, const float* row_loss,
                           double* unit_acc, float* unit_loss, float* loss, WsHeader* hdr,
                           cudaStream_t s);

// Number of logits rows described by a layout (one per token).
inline int64_t layout_rows(const dlm_layout_t* L) { return L ? L->n_tokens : 0; }

}  // namespace dlm
