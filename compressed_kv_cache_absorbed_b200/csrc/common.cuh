// Shared device helpers and the internal launcher interface of the MLA library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

// ------------------------------------------------------------------ storage types

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// ------------------------------------------------------------------------ RoPE

// The rotation of one RoPE pair (x0, x1) by the angle whose cosine and sine are (c, s):
//     (x0 c - x1 s, x0 s + x1 c)
// in double, every product and sum rounded on its own (no fused multiply-add), then rounded
// to float.  Every kernel that rotates uses this, so an IEEE double restatement on the CPU
// with the same inputs gives the same bits.
__device__ __forceinline__ void rope_rotate(float& x0, float& x1, double c, double s) {
    const double a = (double)x0, b = (double)x1;
    const double r0 = __dsub_rn(__dmul_rn(a, c), __dmul_rn(b, s));
    const double r1 = __dadd_rn(__dmul_rn(a, s), __dmul_rn(b, c));
    x0 = __double2float_rn(r0);
    x1 = __double2float_rn(r1);
}

// ------------------------------------------------------------ device error word

// Kernels that meet bad device-side data (a slot outside the cache, decreasing offsets)
// or a wait that gave up latch the first such event here; the host reads and clears it.
struct DevErr {
    int* code;
    long long* detail;
};

__device__ __forceinline__ void latch(DevErr e, int code, long long detail) {
    if (atomicCAS(e.code, 0, code) == 0) *e.detail = detail;
}

// status codes mirrored from mla.h (kept numeric here so device code needs no C header)
constexpr int kErrOutOfRange = 6;
constexpr int kErrTimeout = 5;

// ---------------------------------------------------------------- launch helpers

// Programmatic dependent launch: a kernel launched with launch_pdl may start while the
// previous kernel in the stream is still running; it must call pdl_wait() before touching
// anything that kernel (or any earlier one) writes or reads.  pdl_trigger() lets the next
// kernel start its own independent prologue.  Both are no-ops without the launch attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
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
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// per-kernel event timing (profile.cu); no-ops unless mla_profile_enable(1)
void prof_begin(cudaStream_t s, const char* name);
void prof_end(cudaStream_t s);
struct ProfScope {
    cudaStream_t s;
    ProfScope(cudaStream_t st, const char* name) : s(st) { prof_begin(st, name); }
    ~ProfScope() { prof_end(s); }
};

template <typename T> struct Dt;
template <> struct Dt<float> { static constexpr int id = 0; };
template <> struct Dt<__nv_bfloat16> { static constexpr int id = 1; };

inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// ------------------------------------------------------------- SIMT launchers
// (defined in simt.cu; all return cudaError_t of the launch)

// out[dst(i), j] = sum_k A[i,k] W[j,k] for j < N, W = rows of W1 for j < n1 else W2[j-n1];
// columns with (j % period) >= rope_start are rotated in pairs at pos[i] (or i % pos_mod
// when pos == nullptr); dst(i) = slot[i] (checked against capacity) or i.
template <typename T>
cudaError_t launch_proj_rope(const T* A, int M, int K, const T* W1, int n1, const T* W2, int N,
                             int period, int rope_start, int d_rope, const int32_t* pos,
                             int pos_mod, float theta, const int64_t* slot, long long capacity,
                             T* out, long long ld_out, DevErr err, cudaStream_t s);

// C[z][m][n] = sum_k A[z][m][k] B[z][n][k], element strides given per dimension.
template <typename TA, typename TB, typename TC>
cudaError_t launch_gemm_nt(int Z, int M, int N, int K, const TA* A, long long sAz, long long sAm,
                           long long sAk, const TB* B, long long sBz, long long sBn, long long sBk,
                           TC* C, long long sCz, long long sCm, long long sCn, cudaStream_t s);

// split-KV decode on CUDA cores; q_lat fp32 [B,H,d_c]; q_rope rows at q_rope + b*sQb + h*sQh
template <typename T>
cudaError_t launch_decode_split_simt(const float* q_lat, const T* q_rope, long long sQb,
                                     long long sQh, const T* cache, long long cache_rows,
                                     const int32_t* offsets, int B, int H, int d_c, int d_hR,
                                     float scale, int nsplit, float* part_o, float* part_ml,
                                     DevErr err, cudaStream_t s);

// merge nsplit partials (O unnormalised, m, l) -> o_lat fp32 [B,H,d_c]
cudaError_t launch_combine(const float* part_o, const float* part_ml, int nsplit, int B, int H,
                           int d_c, float* o_lat, cudaStream_t s);

// causal prefill attention on CUDA cores
template <typename T>
cudaError_t launch_prefill_attn_simt(const T* q, const T* k_nope, const T* cache, const T* v,
                                     int B, int S, int H, int qk_nope, int d_hR, int d_c,
                                     int v_head, float scale, T* out, cudaStream_t s);

// per-head transpose: dst[h][c][r] = src[h][r][c]; head h of src starts at h * src_head_stride
// elements (R * C when negative), dst is [Hn, C, R]
template <typename T>
cudaError_t launch_transpose_heads(const T* src, T* dst, int Hn, int R, int C, cudaStream_t s,
                                   long long src_head_stride = -1);

}  // namespace mla
