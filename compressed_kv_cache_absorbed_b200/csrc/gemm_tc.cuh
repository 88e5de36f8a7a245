// Batched bf16 GEMM on the tcgen05 tensor cores (TMA-fed, fp32 accumulation in TMEM).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace mla {
namespace tc {

// Where and how the fp32 accumulator tile is written: element (z, m, n) goes to
// C + z*sz + m*sm + n*sn, as bf16 (f32 == 0) or fp32 (f32 == 1).
struct GemmOut {
    void* C;
    long long sz, sm, sn;
    int f32;
};

// C[z][m][n] = sum_k A[z][m][k] * B[z][n][k] for z < Z, m < M, n < N.
// A rows are K-contiguous with element strides (sAz, sAm); B rows likewise (sBz, sBn).
// Row strides must be multiples of 8 elements (16 bytes) and the bases 16-byte aligned.
// The launch uses programmatic dependent launch.  A (read before waiting for the previous
// kernel) must not be written by it.  chain_head: wait for all earlier work before letting
// the next kernel launch.
cudaError_t gemm_bf16_tc(int Z, int M, int N, int K, const __nv_bfloat16* A, long long sAz, long long sAm,
                         const __nv_bfloat16* B, long long sBz, long long sBn, const GemmOut& out,
                         int* err_code, long long* err_detail, cudaStream_t s, bool chain_head = false);

}  // namespace tc
}  // namespace mla
