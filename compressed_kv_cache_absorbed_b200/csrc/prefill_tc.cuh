// Causal prefill attention on the tcgen05 tensor cores (K and V materialised), for the
// DeepSeek-V2/V3 head shape: q [B*S, H, 192] (128 content columns in fp16, then 64 rotary
// columns in bf16, rotated), k_nope [B*S, H, 128] fp16, cache rows [B*S, 576] bf16 (k_r in
// columns 512 .. 575), v [B*S, H, 128] fp16, out [B*S, H, 128] bf16; fp32 accumulation.
// The materialised intermediates are fp16 because their magnitudes (about 1) sit well inside
// fp16's range, where it rounds 8 times finer than bf16.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace mla {
namespace tc {

cudaError_t prefill_attn_tc(const void* q, const void* k_nope, const __nv_bfloat16* cache,
                            const void* v, int B, int S, int H, float scale, __nv_bfloat16* out,
                            int* err_code, long long* err_detail, cudaStream_t s);

// Sets the polls a bounded wait of the prefill kernel makes before giving up (current device).
cudaError_t set_wait_limit_prefill(uint32_t polls);

}  // namespace tc
}  // namespace mla
