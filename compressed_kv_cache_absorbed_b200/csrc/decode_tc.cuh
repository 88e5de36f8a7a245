// Tensor-core (tcgen05 / TMEM / TMA) absorbed decode for the DeepSeek-V2/V3 head shape:
// H = 128 heads, latent d_c = 512, rotary key d_hR = 64, bf16 storage, fp32 accumulation.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mla {
namespace tc {

constexpr int kH = 128;
constexpr int kDc = 512;
constexpr int kDr = 64;
constexpr int kRow = kDc + kDr;  // 576 cache elements per token
constexpr int kPageTokens = 64;  // tokens per page of a paged cache (one decode tile)
constexpr bool kEnabled = true;

// An FP8 cache row: the latent c as d_c = 512 FP8 E4M3 codes (bytes 0 .. 511), the rotary key
// as 64 bf16 (bytes 512 .. 639), the token's scale as fp32 (bytes 640 .. 643) and 12 bytes
// of zero padding, so that rows stay 16-byte aligned: c = code x scale.
constexpr int kF8RowBytes = 656;
constexpr int kF8ScaleOffset = 640;

// Workspace pieces of the tensor-core decode (all device memory, carved by the caller).
struct DecodeWs {
    __nv_bfloat16* q_lat;   // [B, H, d_c] absorbed query, bf16
    __half* part_o;         // [max_parts, H, d_c] a piece's normalised partial o_lat (fp16)
    float* part_ml;         // [max_parts, H, 2] running max (log2 domain) and sum
    int max_parts;
};

size_t decode_ws_bytes(int B, int num_sms);
DecodeWs carve_decode_ws(char* base, int B, int num_sms);

// Bytes of one tiled weight tensor (W_UK^T or W_UV) for the tensor-core kernels.
constexpr size_t kTiledWeightBytes = (size_t)kH * kDc * 128 * 2;

// The weights laid out as the shared-memory operand images of the q-absorb and merge
// kernels, so that a CTA loads a head's matrix with contiguous bulk copies: per head, 8
// chunks of 128 rows x 64 columns (16 KB), each row 128 bytes with its 16-byte units in the
// 128-byte-swizzle order (unit u of row r at u ^ (r % 8)).
//   ukt: chunk (t, k) = rows 128t .. +127 of W_UK^T[h] (latent index), columns 64k .. +63 (qk_nope)
//   uv:  chunk k      = rows 0 .. 127 of W_UV[h] (v_head), columns 64k .. +63 (latent), in
//        fp16 (saturated at +-65504): the merge's W_UV product takes o_lat in fp16
// W_UKT [H, d_c, qk_nope] and W_UV [H, v_head, d_c] are the plain layouts.
cudaError_t tile_weights_tc(const __nv_bfloat16* W_UKT, const __nv_bfloat16* W_UV, __nv_bfloat16* ukt,
                            __nv_bfloat16* uv, cudaStream_t s);

// Q queries per sequence (Q = 1: decode; Q > 1: the last Q rows of each sequence are new
// tokens and query v = b Q + t attends to the first len(b) - (Q - 1 - t) rows).
// q_nope rows at qn + v*sQn_b + h*sQn_h (qk_nope = 128), q_rope rows at qr + v*sQr_b + h*sQr_h.
// ukt / uv: the tiled weights written by tile_weights_tc; out o [B * Q, H, 128] bf16.
// Sequence b's cache rows are [offsets[b], offsets[b+1]) when block_table is null; with a
// block table (paged cache, 64-token pages) sequence b has seq_lens[b] tokens and its tile j
// is page block_table[b * bt_stride + j] (rows 64 page .. 64 page + 63).
// stream_once: the call reads each cache tile once (loads carry an L2 evict-first hint);
// pass false when other queries of the call read the same tiles.  1 <= Q <= the cluster
// count; the workspace is that of B * Q queries.
// fp8: the cache holds FP8 rows (kF8RowBytes each) instead of bf16 rows.
// folded: q_lat is already in ws.q_lat (the absorbed query projection wrote it; qn and ukt
// are not read) and the output is o_lat itself, o [B * Q, H, 512] in fp16 (saturated),
// without W_UV (uv is not read); o may be ws.q_lat.
cudaError_t decode_absorbed_tc(const __nv_bfloat16* qn, long long sQn_b, long long sQn_h,
                               const __nv_bfloat16* qr, long long sQr_b, long long sQr_h,
                               const __nv_bfloat16* ukt, const __nv_bfloat16* uv,
                               const void* cache, bool fp8, long long cache_rows, const int32_t* offsets,
                               const int32_t* seq_lens, const int32_t* block_table, int bt_stride,
                               int B, int Q, bool stream_once, float scale, __nv_bfloat16* o, const DecodeWs& ws,
                               int num_sms, int* err_code, long long* err_detail, cudaStream_t s,
                               bool folded = false);

// Clusters of the decode kernel on this device (sibling groups are formed from these).
int decode_clusters(int num_sms);

// Sets the polls a bounded wait of this file's kernels makes before giving up (current device).
cudaError_t set_wait_limit_decode(uint32_t polls);

}  // namespace tc
}  // namespace mla
