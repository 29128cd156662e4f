// dlm_noise.cu -- time draw and seeded corruption.
//
// "LLaDA-8B-MDLM-LoRA", Training table, row "Objective": t ~ U(0,1) per
// sequence, mask probability p = (1 - 1e-3) t + 1e-3, masked tokens replaced
// by the mask id.  "diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning
// notes: t ~ U(eps, 1) per example, canvas tokens replaced by uniform-random
// vocabulary ids.  "Native diffusion language-model training", Packed
// training: positions restart at document boundaries, so a document's noise
// does not depend on where it was packed.
//
// Both kernels are integer/ALU work over a few KB to a few MB: one thread per
// unit or per token, 128-bit-free, launched on the caller's stream.
#include "dlm_device.cuh"
#include "dlm_host.h"

namespace dlm {

__global__ void k_sample_t(uint64_t seed, int n_units, int mode, float eps,
                           float* __restrict__ t, float* __restrict__ p) {
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    pdl_wait();   // earlier kernels may still read t / p
    pdl_launch_dependents();
    if (u >= n_units) return;
    const uint32_t k = uint32_t(splitmix64_at(seed, rng_counter(0, uint32_t(u), 0)) >> 40);
    const float x = float(k) * (1.0f / 16777216.0f);            // exact
    const float c1 = __fsub_rn(1.0f, eps);
    const float v = __fadd_rn(__fmul_rn(c1, x), eps);           // no contraction
    if (mode == DLM_ABSORBING) { t[u] = x; p[u] = v; }
    else                       { t[u] = v; p[u] = v; }
}

// One thread per token.  Packed layouts: the unit comes from a binary search
// of cu_seqlens; thread u < n_units also checks that cu_seqlens is
// consistent and flags the status word if not.
__global__ void k_corrupt(int n_units, int seq_len, const int32_t* __restrict__ cu,
                          const uint8_t* __restrict__ pad, int64_t n_tokens,
                          const int32_t* __restrict__ clean, const float* __restrict__ p,
                          int mode, int32_t mask_id, uint32_t vocab, uint64_t seed,
                          int32_t* __restrict__ noisy, uint8_t* __restrict__ corrupted,
                          uint32_t* __restrict__ status) {
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    pdl_wait();   // p comes from the previous kernel; outputs may still be read by earlier ones
    pdl_launch_dependents();
    if (cu && i <= n_units && status) {
        const int32_t c = cu[i];
        bool bad = (i == 0 && c != 0) || (i == n_units && int64_t(c) != n_tokens);
        if (i > 0) bad |= cu[i - 1] > c;
        if (bad) atomicOr(status, DLM_DEV_BAD_LAYOUT);
    }
    if (i >= n_tokens) return;
    int u;
    int64_t pos;
    if (cu) {
        u = find_unit(cu, n_units, i);
        pos = i - __ldg(cu + u);
    } else {
        u = int(i / seq_len);
        pos = i - int64_t(u) * seq_len;
    }
    const int32_t c = clean[i];
    if (pad && pad[i]) { noisy[i] = c; corrupted[i] = 0; return; }
    const uint64_t h1 = splitmix64_at(seed, rng_counter(1, uint32_t(u), uint32_t(pos)));
    const float thr = __fmul_rn(__ldg(p + u), 16777216.0f);
    const bool hit = float(uint32_t(h1 >> 40)) < thr;
    corrupted[i] = hit ? 1 : 0;
    if (!hit) { noisy[i] = c; return; }
    if (mode == DLM_ABSORBING) {
        noisy[i] = mask_id;
    } else {
        const uint64_t h2 = splitmix64_at(seed, rng_counter(2, uint32_t(u), uint32_t(pos)));
        noisy[i] = int32_t(((h2 >> 32) * uint64_t(vocab)) >> 32);
    }
}

}  // namespace dlm

using namespace dlm;

extern "C" dlm_status_t dlm_sample_t(uint64_t seed, int32_t n_units, int32_t mode, float eps,
                                     float* t, float* p, dlm_stream_t stream) {
    DLM_NVTX("dlm_sample_t");
    if (n_units < 0 || n_units >= (1 << 24)) return DLM_ERR_INVALID_ARGUMENT;
    if (mode != DLM_ABSORBING && mode != DLM_UNIFORM) return DLM_ERR_INVALID_ARGUMENT;
    if (!(eps >= 0.0f && eps < 1.0f)) return DLM_ERR_INVALID_ARGUMENT;
    if (n_units == 0) return DLM_OK;
    if (!t || !p) return DLM_ERR_INVALID_ARGUMENT;
    dlm_status_t s = check_device();
    if (s != DLM_OK) return s;
    const int threads = 128;
    return launch_pdl(k_sample_t, dim3((n_units + threads - 1) / threads), dim3(threads), 0,
                      (cudaStream_t)stream, "k_sample_t launch", seed, n_units, mode, eps, t, p);
}

extern "C" dlm_status_t dlm_corrupt(const dlm_layout_t* layout, const int32_t* clean_ids,
                                    const float* p, int32_t mode, int32_t mask_id, int32_t vocab,
                                    uint64_t seed, int32_t* noisy_ids, uint8_t* corrupted,
                                    uint32_t* dev_status, dlm_stream_t stream) {
    DLM_NVTX("dlm_corrupt");
    if (!layout_ok(layout)) return DLM_ERR_INVALID_ARGUMENT;
    if (mode != DLM_ABSORBING && mode != DLM_UNIFORM) return DLM_ERR_INVALID_ARGUMENT;
    if (mode == DLM_UNIFORM && vocab <= 0) return DLM_ERR_INVALID_ARGUMENT;
    const int64_t n = layout->n_tokens;
    if (n == 0 && !(layout->cu_seqlens && dev_status)) return DLM_OK;
    if (n > 0 && (!clean_ids || !p || !noisy_ids || !corrupted)) return DLM_ERR_INVALID_ARGUMENT;
    if (!layout->cu_seqlens && layout->seq_len == 0 && n > 0) return DLM_ERR_INVALID_ARGUMENT;
    dlm_status_t s = check_device();
    if (s != DLM_OK) return s;
    const int threads = 256;
    const int64_t work = n > layout->n_units + 1 ? n : int64_t(layout->n_units) + 1;
    const int64_t blocks = (work + threads - 1) / threads;
    return launch_pdl(k_corrupt, dim3(unsigned(blocks)), dim3(threads), 0, (cudaStream_t)stream,
                      "k_corrupt launch", layout->n_units, layout->seq_len, layout->cu_seqlens,
                      layout->pad_mask, n, clean_ids, p, mode, mask_id, uint32_t(vocab), seed, noisy_ids,
                      corrupted, dev_status);
}
