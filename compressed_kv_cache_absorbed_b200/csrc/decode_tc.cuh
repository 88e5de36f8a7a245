// Tensor-core (tcgen05 / TMEM / TMA) absorbed decode for the DeepSeek-V2/V3 head shape:
// H = 128 heads, latent d_c = 512, rotary key d_hR = 64, bf16 storage, fp32 accumulation.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mla {
namespace tc {

constexpr int kH = 128;
constexpr int kDc = 512;
constexpr int kDr = 64;
constexpr int kRow = kDc + kDr;  // 576 cache elements per token
constexpr bool kEnabled = true;

// Workspace pieces of the tensor-core decode (all device memory, carved by the caller).
struct DecodeWs {
    __nv_bfloat16* q_lat;   // [B, H, d_c] absorbed query, bf16
    __nv_bfloat16* q_cat;   // unused
    float* part_o;          // [max_parts, d_c, H] un-normalised partial o_lat
    float* part_ml;         // [max_parts, H, 2] running max (log2 domain) and sum
    int32_t* work;          // split plan: totals, first tile and first partial slot per sequence
    __nv_bfloat16* o_lat;   // [B, H, d_c] merged, normalised o_lat (bf16, W_UV operand)
    int max_parts;
};

size_t decode_ws_bytes(int B, int num_sms);
DecodeWs carve_decode_ws(char* base, int B, int num_sms);

// q_nope rows at qn + b*sQn_b + h*sQn_h (qk_nope = 128), q_rope rows at qr + b*sQr_b + h*sQr_h.
// W_UKT [H, d_c, qk_nope]; W_UV [H, v_head = 128, d_c]; out o [B, H, 128] bf16.
cudaError_t decode_absorbed_tc(const __nv_bfloat16* qn, long long sQn_b, long long sQn_h,
                               const __nv_bfloat16* qr, long long sQr_b, long long sQr_h,
                               const __nv_bfloat16* W_UKT, const __nv_bfloat16* W_UV,
                               const __nv_bfloat16* cache, long long cache_rows, const int32_t* offsets,
                               int B, float scale, __nv_bfloat16* o, const DecodeWs& ws, int num_sms,
                               int* err_code, long long* err_detail, cudaStream_t s);

}  // namespace tc
}  // namespace mla
