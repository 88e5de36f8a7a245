// FP8 latent cache rows: quantisation of bf16 cache rows.
//
// A quantised latent cache is named by the pages as a further compression of the MLA cache
// ("02 - Multi-Latent Attention (MLA)", "Lo que esta fase NO cubre") and as an engine's own
// cache format ("Multi-head Latent Attention (MLA) si arhitectura DeepSeekMoE", "Exemplul 1");
// neither gives a format.  Here each token's latent c (d_c = 512 values) becomes FP8 E4M3
// codes with one fp32 scale per token, s = max_i |c_i| / 448 (s = 1 for an all-zero c), and
// code_i = e4m3(c_i / s) (nearest even, saturating at 448); the rotary key stays bf16.  Every
// decision is taken in fp32: the bf16 inputs are exact in fp32, s is one correctly rounded
// division, c_i / s another, and the E4M3 rounding is the hardware conversion.
//
// Row layout (kF8RowBytes = 656 bytes): codes [0, 512), k_r as 64 bf16 [512, 640), the scale
// as fp32 [640, 644), zeros [644, 656).
#include "common.cuh"
#include "decode_tc.cuh"
#include "fp8.cuh"
#include "tc_common.cuh"

namespace mla {
namespace tc {

namespace {

// two fp32 -> two E4M3 codes, `lo` in the low byte (nearest even, saturating to +-448)
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// One warp per row: lane l holds latent columns 16 l .. 16 l + 15.
__global__ void __launch_bounds__(256)
quantize_rows_kernel(const __nv_bfloat16* __restrict__ rows, const int64_t* __restrict__ slot, int n,
                     uint8_t* __restrict__ cache, long long capacity, int* err_code, long long* err_detail) {
    const int lane = threadIdx.x & 31;
    const long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long i = w; i < n; i += nw) {
        const long long dst = slot ? slot[i] : i;
        if (dst < 0 || dst >= capacity) {
            if (lane == 0) latch(DevErr{err_code, err_detail}, kErrOutOfRange, i);
            continue;
        }
        const __nv_bfloat16* r = rows + i * kRow;
        const uint4 a = ((const uint4*)r)[2 * lane], b = ((const uint4*)r)[2 * lane + 1];
        const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float c[16];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            c[2 * k] = __uint_as_float(wv[k] << 16);
            c[2 * k + 1] = __uint_as_float(wv[k] & 0xFFFF0000u);
        }
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(c[k]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        uint32_t q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            q[k] = e4m3x2(__fdiv_rn(c[4 * k], s), __fdiv_rn(c[4 * k + 1], s)) |
                   (e4m3x2(__fdiv_rn(c[4 * k + 2], s), __fdiv_rn(c[4 * k + 3], s)) << 16);
        uint8_t* out = cache + dst * kF8RowBytes;
        ((uint4*)out)[lane] = make_uint4(q[0], q[1], q[2], q[3]);
        if (lane < 8) ((uint4*)(out + 512))[lane] = ((const uint4*)(r + kDc))[lane];
        if (lane == 8) ((uint4*)(out + kF8ScaleOffset))[0] = make_uint4(__float_as_uint(s), 0u, 0u, 0u);
    }
}

}  // namespace

cudaError_t quantize_rows_fp8(const __nv_bfloat16* rows, const int64_t* slot, int n, uint8_t* cache,
                              long long capacity, int* err_code, long long* err_detail, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const long long blocks = ((long long)n * 32 + 255) / 256;
    quantize_rows_kernel<<<(int)(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(rows, slot, n, cache, capacity,
                                                                              err_code, err_detail);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace mla
