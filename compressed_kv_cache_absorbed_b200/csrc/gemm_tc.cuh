// Batched bf16 GEMM on the tcgen05 tensor cores (TMA-fed, fp32 accumulation in TMEM).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace mla {
namespace tc {

// Where and how the fp32 accumulator tile is written: element (z, m, n) goes to
// C + z*sz + m*sm + row(n)*sn, as bf16 (f32 == 0) or fp32 (f32 == 1), where row(n) = n, or
// slot[n] when slot is set (a slot outside [0, cap) is skipped and latched as out of range).
// Rotary post-processing (period > 0): output rows m with (m % period) >= rope_start come in
// pairs (m, m + 1) that are rotated by the angle pos(n) * theta^(-2i/d_rope), i the pair
// index within the rotary block, pos(n) = pos ? pos[n] : n % pos_mod; with rope_tab set the
// (cos, sin) of that angle are read from rope_tab[n * d_rope / 2 + i] instead of computed.
// Rotation is done in double precision and the result rounded once.
// f16 (with f32 == 0) stores fp16 instead of bf16: every column, or with period > 0 only the
// columns m with (m % period) < rope_start (the rotary columns stay bf16).  fp16 stores
// saturate at +-65504.  in_f16: the operands A and B hold fp16, not bf16 (both the same).
struct GemmOut {
    void* C;
    long long sz, sm, sn;
    int f32;
    int f16 = 0;
    const int64_t* slot = nullptr;
    long long cap = 0;
    int period = 0, rope_start = 0, d_rope = 0;
    const int32_t* pos = nullptr;
    int pos_mod = 1;
    float theta = 10000.f;
    const double2* rope_tab = nullptr;
    int in_f16 = 0;
};

// rope_tab[n * d_rope / 2 + i] = (cos, sin)(pos(n) * theta^(-2i/d_rope)), computed in double.
cudaError_t rope_table(const int32_t* pos, int pos_mod, int N, int d_rope, float theta, double2* tab,
                       cudaStream_t s);

// C[z][m][n] = sum_k A[z][m][k] * B[z][n][k] for z < Z, m < M, n < N.
// A rows are K-contiguous with element strides (sAz, sAm); B rows likewise (sBz, sBn);
// sBz = 0 shares one B among all z, and sAz = 0 (Z > 1) one A.  From 1024 tokens (N) on,
// with bf16 output, unit m stride and 16-byte aligned rows, the tile is computed token-major
// (a thread per token, 16-byte stores); otherwise weights-major.  The grid is persistent:
// min(tiles, SMs) CTAs.
// Row strides must be multiples of 8 elements (16 bytes) and the bases 16-byte aligned.
// The launch uses programmatic dependent launch.  A (read before waiting for the previous
// kernel) must not be written by it.  chain_head: wait for all earlier work before letting
// the next kernel launch.
cudaError_t gemm_bf16_tc(int Z, int M, int N, int K, const __nv_bfloat16* A, long long sAz, long long sAm,
                         const __nv_bfloat16* B, long long sBz, long long sBn, const GemmOut& out,
                         int* err_code, long long* err_detail, cudaStream_t s, bool chain_head = false);

// y = each pair (x[2i], x[2i+1]) rotated by (cos, sin) = cs[i] with the arithmetic every
// rotating epilogue uses (rope_rotate).
cudaError_t rope_apply(const float* x, const double2* cs, long long pairs, float* y, cudaStream_t s);

// Sets the polls a bounded wait of the GEMM kernel makes before giving up (current device).
cudaError_t set_wait_limit_gemm(uint32_t polls);

// Failure-detection test hook: while on, the GEMM's loader issues no loads, so its MMA and
// epilogue waits run out and the launch latches a timeout with nothing in flight
// (current device).
cudaError_t set_starve_gemm(int on);

}  // namespace tc
}  // namespace mla
