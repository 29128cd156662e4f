// dlm_scale.cu -- multiply a bf16 gradient in place by a scalar that lives
// on the device (the upstream gradient of a scalar loss, handed over by an
// autograd engine after the loss call has already written its gradient).
//
// Every CTA first reads the scalar and returns at once when it is exactly
// 1, the usual case (loss.backward() on the loss itself): then the call
// costs one launch and no memory traffic, and the host never has to read
// the scalar (no synchronisation).  Otherwise it is one HBM pass over the
// tensor (2 bytes read + 2 written per element), grid-stride, 16-byte
// vectors where the row stride and the pointer allow.
#include "dlm_device.cuh"
#include "dlm_host.h"

namespace dlm {

constexpr int kScaleThreads = 256;

__global__ void __launch_bounds__(kScaleThreads) k_scale_bf16(uint16_t* __restrict__ x, int64_t rows,
                                                              int64_t cols, int64_t ld,
                                                              const float* __restrict__ scale, int vec) {
    pdl_wait();                        // the gradient comes from the previous kernel
    const float g = *scale;
    if (g == 1.0f) return;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    const int64_t t0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (vec) {
        const int64_t per_row = cols / 8;
        const int64_t n = rows * per_row;
        for (int64_t i = t0; i < n; i += stride) {
            const int64_t r = i / per_row, c = (i - r * per_row) * 8;
            uint4* p = reinterpret_cast<uint4*>(x + r * ld + c);
            uint4 v = *p;
            uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            #pragma unroll
            for (int k = 0; k < 4; ++k) w4[k] = pack_bf16x2(bf16lo(w4[k]) * g, bf16hi(w4[k]) * g);
            *p = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        return;
    }
    const int64_t n = rows * cols;
    for (int64_t i = t0; i < n; i += stride) {
        const int64_t r = i / cols, c = i - r * cols;
        uint16_t* p = x + r * ld + c;
        *p = __bfloat16_as_ushort(__float2bfloat16_rn(bf16_bits_to_float(*p) * g));
    }
}

}  // namespace dlm

using namespace dlm;

extern "C" dlm_status_t dlm_scale_bf16(uint16_t* x, int64_t rows, int64_t cols, int64_t ld, const float* scale,
                                       dlm_stream_t stream) {
    DLM_NVTX("dlm_scale_bf16");
    if (rows < 0 || cols < 0 || ld < cols || !scale) return DLM_ERR_INVALID_ARGUMENT;
    if (rows == 0 || cols == 0) return DLM_OK;
    if (!x) return DLM_ERR_INVALID_ARGUMENT;
    dlm_status_t st = check_device();
    if (st != DLM_OK) return st;
    const int vec = (cols % 8 == 0) && (ld % 8 == 0) && aligned16(x);
    const int64_t work = vec ? rows * (cols / 8) : rows * cols;
    int64_t blocks = (work + kScaleThreads - 1) / kScaleThreads;
    if (blocks > 148 * 8) blocks = 148 * 8;
    return launch_pdl(k_scale_bf16, dim3(unsigned(blocks)), dim3(kScaleThreads), 0, (cudaStream_t)stream,
                      "k_scale_bf16 launch", x, rows, cols, ld, scale, vec);
}
