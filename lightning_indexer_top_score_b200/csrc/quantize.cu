// quantize.cu -- per-row FP8 (E4M3) quantisation for the FP8 indexer (lsa_quantize_fp8).
//
// Paper: Sec. 2.2 ("Why Lightning": the indexer may compute in FP8) and Sec. 1 (DSA
// lowers the indexer's cost by FP8 quantisation).  The pages fix no scheme; the one used here:
// one fp32 scale per row (a key row = one token's d_I values, a query row = one (token, head)
// vector), scale = amax / 448, code = E4M3(x / scale) rounded to nearest even and saturated to
// +-448, both quotients in IEEE fp32 (so the codes are a function of the bf16 inputs alone).
#include <cuda_fp8.h>

#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kRowsPerBlock = 8;  // one warp per row

__global__ void __launch_bounds__(32 * kRowsPerBlock)
    quantize_e4m3_kernel(const __nv_bfloat16 *x, int64_t x_stride, int64_t rows, int D,
                         uint8_t *codes, int64_t codes_stride, float *scales,
                         int64_t scales_stride, int32_t *err) {
    const int64_t r = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const __nv_bfloat16 *xr = x + r * x_stride;
    float amax = 0.f;
    bool bad = false;
    for (int i = lane; i < D; i += 32) {
        const float v = __bfloat162float(xr[i]);
        bad |= !isfinite(v);
        amax = fmaxf(amax, fabsf(v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) raise_error(err, LSA_DEVERR_NONFINITE);
    const float scale = __fdiv_rn(amax, 448.0f);
    if (lane == 0) scales[r * scales_stride] = scale;
    uint8_t *cr = codes + r * codes_stride;
    for (int i = 2 * lane; i < D; i += 64) {
        float2 y = make_float2(0.f, 0.f);
        if (scale > 0.f)
            y = make_float2(__fdiv_rn(__bfloat162float(xr[i]), scale),
                            __fdiv_rn(__bfloat162float(xr[i + 1]), scale));
        // .x lands in the lower byte, i.e. at cr[i]
        *reinterpret_cast<__nv_fp8x2_storage_t *>(cr + i) =
            __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
    }
}

}  // namespace
}  // namespace lsa

extern "C" lsa_status lsa_quantize_fp8(const void *x, int64_t x_stride, int64_t rows, int D,
                                       uint8_t *codes, int64_t codes_stride, float *scales,
                                       int64_t scales_stride, int32_t *device_error,
                                       void *stream) {
    if (!x || !codes || !scales || rows < 0 || D < 2 || D % 2 || D > 4096)
        return LSA_ERR_INVALID_ARG;
    if (x_stride < D || codes_stride < D || codes_stride % 2 || scales_stride < 1)
        return LSA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(codes) % 2) return LSA_ERR_INVALID_ARG;
    if (rows == 0) return LSA_OK;
    const int64_t blocks = (rows + lsa::kRowsPerBlock - 1) / lsa::kRowsPerBlock;
    if (blocks > 0x7FFFFFFF) return LSA_ERR_INVALID_ARG;
    lsa::quantize_e4m3_kernel<<<(unsigned)blocks, 32 * lsa::kRowsPerBlock, 0,
                                static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(x), x_stride, rows, D, codes, codes_stride, scales,
        scales_stride, device_error);
    return lsa::launched() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}
