/*
 * mla.h -- C ABI of the B200 (sm_100a) Multi-head Latent Attention library.
 *
 * The library computes decode-time attention over the compressed MLA cache (each token
 * stores only its latent c_kv and a small decoupled RoPE key), with W_UK absorbed into
 * the query and W_UV applied after the softmax-weighted sum, so per-head K and V are never
 * formed; plus the cache append and a materialised-K/V causal prefill.
 *
 * Sources, by page title and section:
 *   [L1] "02 - Multi-Latent Attention (MLA)" (lynx-cortex, phase 36): "La compresion de
 *        MLA" (c_t = W_DKV h_t; k_t = W_UK c_t; v_t = W_UV c_t), "Truco de codificacion
 *        posicional" (decoupled rotary key k^rope, width d_hR, cached as is), "Coste de
 *        computo" (re-associating the matmuls so attention runs on c directly).
 *   [L2] "Multi-head latent attention" (aiunderstanding.org), "Informacion tecnica":
 *        the up-projections are absorbed into the query and output projections.
 *   [L4] "Multi-head Latent Attention (MLA) si arhitectura DeepSeekMoE" (dexblog.ro),
 *        opening section: (d_c + d_hR) cached elements per token per layer.
 *   [L5] "DeepSeek MLA" (llm-engineer cards): score = content + positional; decode reads
 *        the whole cache every step.
 *
 * Conventions shared by every call
 *   - Every tensor pointer is a DEVICE pointer unless stated; tensors are dense row-major.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Argument errors are detected on the host and returned before anything is launched;
 *     outputs are then untouched.  Errors found on the device (a slot outside the cache,
 *     decreasing offsets, a sequence past the cache) skip the offending work and latch a
 *     device error word that mla_get_device_error() reads.  No call traps, aborts or throws.
 *   - The caller owns every tensor (cache, inputs, outputs, workspace).  The only
 *     library-owned object is an mla_weights handle (device memory it allocates once).
 *   - Storage type: all float tensors of one call share `dims->dtype` (fp32 or bf16);
 *     accumulation is always fp32.  Index arrays are int32 (offsets, positions) or
 *     int64 (slots); row arithmetic is done in 64 bits.
 *   - Cache layout [L4]: row r of the cache is (d_c + d_hR) elements, the latent c in
 *     columns [0, d_c) and the rotated key k_rope in [d_c, d_c + d_hR).
 *   - RoPE: pairs (2i, 2i+1) rotated by pos * theta^(-2i/d_hR); one rotary key per token,
 *     shared by all heads.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* mla_stream_t; /* cudaStream_t */

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,    /* a pointer, size or dimension is invalid */
    MLA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. odd d_hR) */
    MLA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than *_workspace_size() */
    MLA_ERR_CUDA = 4,           /* a CUDA runtime call failed (message: mla_last_cuda_error) */
    MLA_ERR_DEVICE_TIMEOUT = 5, /* a device-side wait gave up (reported by mla_get_device_error) */
    MLA_ERR_OUT_OF_RANGE = 6,   /* device-side: a slot/offset outside the cache */
    MLA_ERR_NO_MEMORY = 7       /* allocation of an mla_weights handle failed */
} mla_status;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype;

/* Layer dimensions.  softmax_scale <= 0 selects 1/sqrt(qk_nope + d_hR); rope_theta <= 0
 * selects 10000.  d_model may be 0 for calls that never touch the hidden size. */
typedef struct {
    int32_t H;          /* attention heads */
    int32_t d_model;    /* hidden size */
    int32_t d_c;        /* latent width (kv_lora_rank) */
    int32_t d_hR;       /* decoupled RoPE key width (even) */
    int32_t qk_nope;    /* per-head content query/key width */
    int32_t v_head;     /* per-head value width */
    float softmax_scale;
    float rope_theta;
    int32_t dtype;      /* mla_dtype */
} mla_dims;

typedef struct mla_weights_s* mla_weights;

/* ---------------------------------------------------------------- host-only helpers */

/* Human-readable name of a status code (static string). */
const char* mla_status_string(mla_status s);

/* Message of the last failed CUDA runtime call in this process (static buffer). */
const char* mla_last_cuda_error(void);

/* Elements one token adds to the cache per layer: d_c + d_hR [L4].  -1 if dims invalid. */
int64_t mla_cache_row_elems(const mla_dims* dims);

/* Bytes one token adds to the cache over `layers` layers: (d_c + d_hR) * layers * elem. */
int64_t mla_cache_bytes_per_token(const mla_dims* dims, int32_t layers);

/* Which decode kernel family a call with these dims would use: 1 = tcgen05/TMEM
 * split-KV kernel (bf16, H = 128, d_c = 512, d_hR = 64), 0 = CUDA-core kernel,
 * -1 = invalid dims.  Host-only; used by tests to assert the fast path is taken. */
int32_t mla_decode_path(const mla_dims* dims);

/* ------------------------------------------------------------------------- weights */

/* Pack the per-head up-projections for the kernels [L1 "Coste de computo"; L2].
 *   W_UK [H, qk_nope, d_c]   (k_nope = W_UK[h] c)          -- copied and re-laid out
 *   W_UV [H, v_head, d_c]    (v = W_UV[h] c)               -- copied
 *   W_Q  [H*(qk_nope+d_hR), d_model] or NULL               -- borrowed (not copied)
 *   W_O  [d_model, H*v_head] or NULL                       -- borrowed (not copied)
 * W_Q rows are head-major, the qk_nope content rows of a head before its d_hR rotary rows.
 * Borrowed tensors must stay valid until mla_weights_destroy.  The handle owns device
 * memory allocated here (the only allocation the library makes).  Stream-ordered: the
 * packing kernels run on `stream`.
 *
 * fold = 1 also precomputes the matrix products the up-projections can be folded into
 * [L1 "Coste de computo": precomputed products], per head h (fp32 sums, one rounding; W_QUK
 * in bf16, W_OUV in fp16 as it meets the merged latent output kept in fp16):
 *   W_QUK [H*d_c, d_model]:  W_QUK[h*d_c + c, :] = sum_j W_UK[h, j, c] W_Q[h*(qk_nope+d_hR) + j, :]
 *   W_OUV [d_model, H*d_c]:  W_OUV[:, h*d_c + c] = sum_v W_O[:, h*v_head + v] W_UV[h, v, c]
 * and a copy of W_Q's rotary rows.  mla_decode_absorbed from hidden states then computes
 * q_lat = W_QUK h directly (no q_nope, no absorption kernel) and out = W_OUV o_lat (no W_UV
 * product): the same attention, with different rounding points.  At V2/V3 sizes the two
 * products take ~0.94 GB each, and a decode step reads them all, ~3x the projection bytes
 * and flops of fold = 0.  Requires W_Q and W_O (else MLA_ERR_INVALID_ARG) and the bf16
 * tensor-core shape (else MLA_ERR_UNSUPPORTED); temporary device memory is allocated and
 * freed stream-ordered.  Other entry points ignore the folded products. */
mla_status mla_absorb_weights(const mla_dims* dims, const void* W_UK, const void* W_UV,
                              const void* W_Q, const void* W_O, int32_t fold, mla_weights* out,
                              mla_stream_t stream);

/* Free a handle (synchronises the device first).  NULL is accepted. */
mla_status mla_weights_destroy(mla_weights w);

/* ------------------------------------------------------------------- cache append */

/* KV down-projection, RoPE and cache write [L1 "La compresion de MLA", "Truco de
 * codificacion posicional"; L4]: for token i < n,
 *     c = W_DKV h_i,   k_r = RoPE(W_KR h_i, pos[i]),   cache[slot[i]] = [c | k_r]
 * (fp32 accumulation, one rounding to the storage type).
 *   h [n, d_model]; W_DKV [d_c, d_model]; W_KR [d_hR, d_model]; pos int32 [n];
 *   slot int64 [n]; cache [capacity, d_c + d_hR].
 * Only the rows slot[i] are written.  A slot outside [0, capacity) is skipped and latches
 * MLA_ERR_OUT_OF_RANGE in the device error word.  Duplicate slots race (last writer wins).
 * n = 0 is a no-op. */
mla_status mla_append_cache(const mla_dims* dims, const void* h, const void* W_DKV,
                            const void* W_KR, const int32_t* pos, const int64_t* slot,
                            int32_t n, void* cache, int64_t capacity, mla_stream_t stream);

/* --------------------------------------------------------------- absorbed decode */

/* Bytes of workspace mla_decode_absorbed needs for B sequences on the current device. */
size_t mla_decode_workspace_size(const mla_dims* dims, int32_t B);

/* Absorbed decode attention over the latent cache, one query token per sequence
 * [L1 "Coste de computo"; L2; L5]:
 *     q_lat[b,h]  = W_UK[h]^T q_nope[b,h]                         (d_c)
 *     s[b,h,t]    = scale * (q_lat[b,h] . c_t + q_rope[b,h] . k_r,t)
 *     o_lat[b,h]  = sum_t softmax_t(s[b,h,:]) c_t                 (d_c, fp32)
 *     o[b,h]      = W_UV[h] o_lat[b,h]                            (v_head)
 *     out[b]      = W_O concat_h o[b,h]        (only when the handle holds W_O)
 * Sequence b attends over cache rows [offsets[b], offsets[b+1]) (int32 [B+1], ragged) of a
 * cache of cache_rows rows (1 <= cache_rows < 2^31).  A sequence whose rows are not inside
 * the cache (offsets[b] < 0, offsets[b+1] < offsets[b] or offsets[b+1] > cache_rows) latches
 * MLA_ERR_OUT_OF_RANGE on the device and decodes to zeros; the other sequences of the call
 * are computed as usual.
 * An empty sequence gives o = 0.  The query comes either from (q_nope [B,H,qk_nope],
 * q_rope [B,H,d_hR], q_rope already rotated) or, when both are NULL, from the hidden
 * state h [B, d_model] through the handle's W_Q with RoPE at q_pos int32 [B].
 * out is [B, H, v_head], or [B, d_model] when the handle holds W_O.
 * workspace: device, >= mla_decode_workspace_size(dims, B) bytes, 256-byte aligned;
 * its contents on entry do not matter. */
mla_status mla_decode_absorbed(const mla_dims* dims, mla_weights w, const void* q_nope,
                               const void* q_rope, const void* h, const int32_t* q_pos,
                               const void* cache, int64_t cache_rows, const int32_t* offsets,
                               int32_t B, void* out, void* workspace, size_t ws_bytes,
                               mla_stream_t stream);

/* mla_decode_absorbed over a PAGED latent cache: the cache is num_pages pages of 64 tokens
 * ([num_pages, 64, d_c + d_hR] rows, the row layout of mla_decode_absorbed); sequence b has
 * seq_lens[b] tokens (int32 [B], device) and its j-th 64-token block is page
 * block_table[b * max_blocks + j] (int32 [B, max_blocks], device).  The result is that of
 * mla_decode_absorbed on the same rows laid out contiguously.  The pages describe a paged
 * cache as a layer orthogonal to MLA ["DeepSeek MLA", the PagedAttention comparison].
 * Queries from q_nope/q_rope only; the tensor-core shape only (bf16, H = 128, d_c = 512,
 * d_hR = 64, qk_nope = v_head = 128) and handles without W_O, else MLA_ERR_UNSUPPORTED.
 * A sequence needing more than max_blocks pages (or with seq_lens[b] < 0) latches
 * MLA_ERR_OUT_OF_RANGE on the device and decodes to zeros; a page outside [0, num_pages)
 * latches the same error and its tile is read as zeros (that sequence's output is then
 * meaningless; the others are unaffected).  Workspace: mla_decode_workspace_size(dims, B). */
mla_status mla_decode_absorbed_paged(const mla_dims* dims, mla_weights w, const void* q_nope,
                                     const void* q_rope, const void* cache, int64_t num_pages,
                                     const int32_t* block_table, int32_t max_blocks,
                                     const int32_t* seq_lens, int32_t B, void* out, void* workspace,
                                     size_t ws_bytes, mla_stream_t stream);

/* Multi-token decode over a PAGED latent cache: q_len >= 1 new tokens per sequence in one
 * call (the verification of draft tokens in speculative decoding; the DeepSeek pages name
 * the multi-token-prediction module's use for it ["Multi-head Latent Attention (MLA) si
 * arhitectura DeepSeekMoE", "Concepte cheie"]).  The new tokens' cache rows must already be
 * appended: sequence b holds seq_lens[b] tokens (int32 [B], device), the last q_len of them
 * the new ones, in the pages of block_table (int32 [B, max_blocks], device), laid out as for
 * mla_decode_absorbed_paged.  New token t (0 <= t < q_len) of sequence b sits at position
 * seq_lens[b] - q_len + t and attends to the sequence's first seq_lens[b] - q_len + t + 1
 * tokens: causal inside the window, the rule of causal attention ["02 - Multi-Latent
 * Attention (MLA)", "La compresion de MLA"].
 *   q_nope [B, q_len, H, qk_nope], q_rope [B, q_len, H, d_hR] (rotated at the tokens'
 *   positions), out [B, q_len, H, v_head]: device, storage type, contiguous.
 * The result for token (b, t) is that of mla_decode_absorbed_paged on a sequence of
 * seq_lens[b] - q_len + t + 1 tokens; a token with no key (seq_lens[b] < q_len - t) gets
 * zeros.  Tensor-core shape only and handles without W_O, else MLA_ERR_UNSUPPORTED; a page
 * outside [0, num_pages) or more than max_blocks blocks latch MLA_ERR_OUT_OF_RANGE on the
 * device, as for mla_decode_absorbed_paged.
 * Up to 8 new tokens per sequence run on sibling groups of clusters that walk the same cache
 * tiles at the same time, so the cache streams from HBM once per call (the siblings' reads
 * are served by L2); longer chunks (chunked prefill) make every new token a query sequence
 * of its own, and the prefix tiles, read by neighbouring clusters at the same time, are
 * served from L2 after their first read.
 * Workspace: device, >= mla_decode_multi_workspace_size(dims, B, q_len, max_blocks) bytes,
 * 256-byte aligned, contents on entry do not matter. */
mla_status mla_decode_absorbed_paged_multi(const mla_dims* dims, mla_weights w, const void* q_nope,
                                           const void* q_rope, const void* cache, int64_t num_pages,
                                           const int32_t* block_table, int32_t max_blocks,
                                           const int32_t* seq_lens, int32_t B, int32_t q_len, void* out,
                                           void* workspace, size_t ws_bytes, mla_stream_t stream);

/* Workspace bytes of mla_decode_absorbed_paged_multi; 0 for shapes it does not support or
 * sizes out of range (q_len < 1, max_blocks < 1, B * q_len * max_blocks >= 2^31). */
size_t mla_decode_multi_workspace_size(const mla_dims* dims, int32_t B, int32_t q_len, int32_t max_blocks);

/* mla_decode_absorbed with the queries and the output in HOST memory: the call copies
 * q_nope [B,H,qk_nope] and q_rope [B,H,d_hR] (storage type, rotated) host->device into the
 * workspace, runs the same decode on the stream, and copies o [B,H,v_head] device->host.
 * Everything is enqueued on `stream` and the call returns at once; out_host is valid after
 * the stream has been synchronised.  Host buffers should be page-locked (cudaHostAlloc or
 * cudaHostRegister) for the copies to be asynchronous; pageable memory works but the copies
 * then block the calling thread.  The workspace is the one of mla_decode_absorbed.
 * Handles holding W_O are not accepted here (MLA_ERR_UNSUPPORTED): use mla_decode_absorbed.
 * The pages have no counterpart to this call; it is the end-to-end path of a server that
 * keeps the cache on the GPU and exchanges only the step's queries and outputs. */
mla_status mla_decode_absorbed_host(const mla_dims* dims, mla_weights w, const void* q_nope_host,
                                    const void* q_rope_host, const void* cache, int64_t cache_rows,
                                    const int32_t* offsets, int32_t B, void* out_host, void* workspace,
                                    size_t ws_bytes, mla_stream_t stream);

/* Size of the fixed device scratch used by mla_decode_absorbed_noalloc (64 MiB). */
#define MLA_NOALLOC_SCRATCH_BYTES (64u << 20)

/* mla_decode_absorbed without a workspace argument, for callers that cannot allocate
 * device memory (an engine that gives all GPU memory to its own pool at start-up, code
 * in a region where allocation is forbidden, a plugin host without an allocation hook).
 * The source pages have no counterpart to this call; it exists for those callers.
 * Arguments, layouts and results are those of mla_decode_absorbed.  The scratch comes
 * from one fixed device array of MLA_NOALLOC_SCRATCH_BYTES inside the library, which
 * every GPU that loads the library holds until the process exits; this call itself
 * allocates nothing (no cudaMalloc, no cudaFree).
 *   - A call whose scratch need (mla_decode_workspace_size(dims, B)) exceeds
 *     MLA_NOALLOC_SCRATCH_BYTES returns MLA_ERR_WORKSPACE before launching anything
 *     (compare the two to know in advance whether a batch fits).
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     with that device current; make that first call before any stream capture.  The
 *     address is kept for the life of the process: a cudaDeviceReset in the same process
 *     destroys the array with the rest of the library's device state, and the library must
 *     not be called on that device afterwards.
 *   - All calls share the one array and it keeps the previous call's contents (nothing
 *     in it needs to start at zero).  Calls that overlap on the GPU (other streams,
 *     other host threads, without ordering between them) race on it and give wrong
 *     results; order them on one stream or with events. */
mla_status mla_decode_absorbed_noalloc(const mla_dims* dims, mla_weights w, const void* q_nope,
                                       const void* q_rope, const void* h, const int32_t* q_pos,
                                       const void* cache, int64_t cache_rows,
                                       const int32_t* offsets, int32_t B, void* out,
                                       mla_stream_t stream);

/* -------------------------------------------------------------- FP8 latent cache */

/* A quantised latent cache, which the pages name as a further compression ["02 - Multi-
 * Latent Attention (MLA)", "Lo que esta fase NO cubre"] and as an engine's own cache format
 * ["Multi-head Latent Attention (MLA) si arhitectura DeepSeekMoE", "Exemplul 1"], without
 * giving a format.  An FP8 cache row holds one token: the latent c as d_c FP8 E4M3 codes
 * (bytes [0, d_c)), the rotary key as d_hR bf16 values (bytes [d_c, d_c + 2 d_hR)), the
 * token's scale s as fp32 (next 4 bytes), then zeros up to mla_fp8_row_bytes() (a multiple
 * of 16); c_i = code_i * s.  Quantisation: s = max_i |c_i| / 448 (1 for an all-zero c) and
 * code_i = e4m3(c_i / s), nearest even, every decision in fp32 from the bf16 row.  Half the
 * bytes of a bf16 row per token (656 against 1152 for the V2/V3 shape).
 * Tensor-core shape only (bf16, H = 128, d_c = 512, d_hR = 64, qk_nope = v_head = 128);
 * other dims get -1 / 0 / MLA_ERR_UNSUPPORTED. */

/* Bytes of one FP8 cache row (656 for the supported shape), or -1. */
int64_t mla_fp8_row_bytes(const mla_dims* dims);

/* FP8 rows of n bf16 cache rows (rows [n, d_c + d_hR], device, 16-byte aligned):
 * cache_fp8[slot[i]] for i < n (slot int64 [n], device; NULL writes rows 0 .. n-1).
 * cache_fp8: device, [capacity, mla_fp8_row_bytes()] bytes, 16-byte aligned.  A slot outside
 * [0, capacity) is skipped and latches MLA_ERR_OUT_OF_RANGE.  n = 0 is a no-op. */
mla_status mla_quantize_cache_fp8(const mla_dims* dims, const void* rows, const int64_t* slot, int32_t n,
                                  void* cache_fp8, int64_t capacity, mla_stream_t stream);

/* Workspace bytes of mla_append_cache_fp8 for n tokens (their bf16 rows), 0 if unsupported. */
size_t mla_append_fp8_workspace_size(const mla_dims* dims, int32_t n);

/* mla_append_cache into an FP8 cache: the same down-projection and RoPE give each token's
 * bf16 row (in the workspace), which is quantised into cache_fp8[slot[i]] as by
 * mla_quantize_cache_fp8.  workspace: device, >= mla_append_fp8_workspace_size(dims, n)
 * bytes, 256-byte aligned. */
mla_status mla_append_cache_fp8(const mla_dims* dims, const void* h, const void* W_DKV, const void* W_KR,
                                const int32_t* pos, const int64_t* slot, int32_t n, void* cache_fp8,
                                int64_t capacity, void* workspace, size_t ws_bytes, mla_stream_t stream);

/* mla_decode_absorbed over an FP8 cache: the result of the decode on the dequantised rows
 * [code * s | k_r].  Queries from q_nope/q_rope only, handles without W_O; cache_fp8
 * [cache_rows, mla_fp8_row_bytes()] bytes, 16-byte aligned; offsets, invalid sequences and
 * the workspace (mla_decode_workspace_size) as for mla_decode_absorbed.  The kernel
 * dequantises each tile in shared memory to fp16 (code x s) and runs the latent products on
 * fp16 operands (the absorbed query and the probabilities in fp16 too), the rotary ones in
 * bf16, all accumulating in fp32. */
mla_status mla_decode_absorbed_fp8(const mla_dims* dims, mla_weights w, const void* q_nope,
                                   const void* q_rope, const void* cache_fp8, int64_t cache_rows,
                                   const int32_t* offsets, int32_t B, void* out, void* workspace,
                                   size_t ws_bytes, mla_stream_t stream);

/* ---------------------------------------------------------------- causal prefill */

/* Bytes of workspace mla_prefill_causal needs for B sequences of S tokens. */
size_t mla_prefill_workspace_size(const mla_dims* dims, int32_t B, int32_t S);

/* Causal prefill with K and V materialised from the latent [L1 "La compresion de MLA"]:
 * appends every token (as mla_append_cache, position t, cache row b*S + t), then per head
 *     K_t = [W_UK[h] c_t | k_r,t],   V_t = W_UV[h] c_t,
 *     q = W_Q h_t (rotary part rotated at t),
 *     out[b,t,h] = sum_{tau <= t} softmax(scale * q . K_tau) V_tau.
 *   h [B, S, d_model]; W_DKV [d_c, d_model]; W_KR [d_hR, d_model];
 *   cache [B*S, d_c + d_hR] (written); out [B, S, H, v_head].
 * The handle must hold W_Q.  workspace >= mla_prefill_workspace_size(dims, B, S). */
mla_status mla_prefill_causal(const mla_dims* dims, mla_weights w, const void* h,
                              const void* W_DKV, const void* W_KR, void* cache, void* out,
                              int32_t B, int32_t S, void* workspace, size_t ws_bytes,
                              mla_stream_t stream);

/* ------------------------------------------------------------------- diagnostics */

/* Synchronise `stream`, then read and clear the device error word of the current device.
 * Returns MLA_OK if no device-side error was latched since the last call, else the
 * latched code (MLA_ERR_OUT_OF_RANGE, MLA_ERR_DEVICE_TIMEOUT); *detail (nullable)
 * receives a kernel-specific detail value. */
mla_status mla_get_device_error(mla_stream_t stream, int64_t* detail);

/* The rotary step alone, for checking its arithmetic: y[2i], y[2i+1] = the pair (x[2i],
 * x[2i+1]) rotated by the angle whose (cos, sin) are cos_sin[2i], cos_sin[2i+1] ["02 -
 * Multi-Latent Attention (MLA)", "Truco de codificacion posicional": the decoupled key
 * carries the rotary position].  The rotation is the one every rotating kernel of the
 * library applies (the cache append's k_r and the query projection's rotary part): in
 * double, each product and sum rounded on its own, then rounded to float.  x, y: float
 * [2 pairs], cos_sin: double [2 pairs] (16-byte aligned); device pointers. */
mla_status mla_rope_apply(const float* x, const double* cos_sin, int64_t pairs, float* y, mla_stream_t stream);

/* Failure-detection test hooks.  Leave both at their defaults outside tests.
 *
 * mla_set_wait_limit: on the current device, the number of polls each bounded wait in the
 * library's tensor-core kernels (a kernel waiting for its own loads, MMAs or sibling warps)
 * makes before it gives up, latches MLA_ERR_DEVICE_TIMEOUT, drains what it issued, frees its
 * tensor memory and returns.  0 restores the default (2^22 polls, seconds).  Synchronous
 * (cudaMemcpyToSymbol); call it with no library kernel running.
 *
 * mla_test_starve_projection: while on != 0, the loader warp of the tensor-core projection
 * GEMM (the kernel behind mla_append_cache on bf16, the query projection and W_O) issues no
 * loads, so its MMA and epilogue waits run out: such a call writes no output and latches
 * MLA_ERR_DEVICE_TIMEOUT, with no copy and no MMA in flight, and the next call works.  It is
 * how the timeout path is tested without faulting or hanging the GPU.  Current device,
 * synchronous. */
mla_status mla_set_wait_limit(uint32_t polls);
mla_status mla_test_starve_projection(int32_t on);

/* Per-kernel device timing of this library's own launches (a diagnostic, off by default).
 * While enabled, each launch is bracketed by two CUDA events recorded on its stream. */
void mla_profile_enable(int32_t on);

/* Writes one line "kernel_name launches total_ms" per kernel timed since the last reset
 * into buf (nullable; truncated to cap), waiting for the recorded events.  Returns the
 * number of kernels; reset != 0 clears the totals. */
int32_t mla_profile_report(char* buf, size_t cap, int32_t reset);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
