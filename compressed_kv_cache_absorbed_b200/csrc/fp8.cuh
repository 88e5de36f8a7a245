// FP8 latent cache rows (layout: decode_tc.cuh, kF8RowBytes).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {
namespace tc {

// cache[slot[i]] (or cache[i] when slot is null) = the FP8 row of bf16 row i of `rows`
// ([n, 576]) for i < n; a slot outside [0, capacity) is skipped and latched as out of range.
cudaError_t quantize_rows_fp8(const __nv_bfloat16* rows, const int64_t* slot, int n, uint8_t* cache,
                              long long capacity, int* err_code, long long* err_detail, cudaStream_t s);

}  // namespace tc
}  // namespace mla
