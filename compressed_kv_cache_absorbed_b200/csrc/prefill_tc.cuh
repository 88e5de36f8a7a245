// Causal prefill attention on the tcgen05 tensor cores (K and V materialised), for the
// DeepSeek-V2/V3 head shape: q [B*S, H, 192] (128 content + 64 rotary, rotated),
// k_nope [B*S, H, 128], cache rows [B*S, 576] (k_r in columns 512 .. 575), v [B*S, H, 128],
// out [B*S, H, 128]; bf16 storage, fp32 accumulation.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace mla {
namespace tc {

cudaError_t prefill_attn_tc(const __nv_bfloat16* q, const __nv_bfloat16* k_nope, const __nv_bfloat16* cache,
                            const __nv_bfloat16* v, int B, int S, int H, float scale, __nv_bfloat16* out,
                            int* err_code, long long* err_detail, cudaStream_t s);

}  // namespace tc
}  // namespace mla
