// The C ABI (include/mla.h): argument validation, workspace carving, kernel dispatch.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "decode_tc.cuh"
#include "fp8.cuh"
#include "gemm_tc.cuh"
#include "multi.cuh"
#include "prefill_tc.cuh"
#include "mla.h"

using mla::DevErr;
using bf16 = __nv_bfloat16;

// ------------------------------------------------------------------ error plumbing

static __device__ int g_err_code;
static __device__ long long g_err_detail;
static char g_cuda_msg[256] = "no CUDA error";

static mla_status cuda_fail(cudaError_t e, const char* where) {
    snprintf(g_cuda_msg, sizeof g_cuda_msg, "%s: %s", where, cudaGetErrorString(e));
    return MLA_ERR_CUDA;
}
#define MLA_CUDA(call)                                    \
    do {                                                  \
        cudaError_t e_ = (call);                          \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
    } while (0)

static mla_status dev_err(DevErr* out) {
    static std::mutex mu;
    static DevErr cache[64];
    static bool have[64];
    int dev = 0;
    MLA_CUDA(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> g(mu);
    if (dev < 64 && have[dev]) {
        *out = cache[dev];
        return MLA_OK;
    }
    DevErr e;
    MLA_CUDA(cudaGetSymbolAddress((void**)&e.code, g_err_code));
    MLA_CUDA(cudaGetSymbolAddress((void**)&e.detail, g_err_detail));
    if (dev < 64) {
        cache[dev] = e;
        have[dev] = true;
    }
    *out = e;
    return MLA_OK;
}

// ---------------------------------------------------------------------- handle

struct mla_weights_s {
    mla_dims dims;
    int device;
    void* W_UK;    // [H, qk_nope, d_c]   copy, storage type
    void* W_UKT;   // [H, d_c, qk_nope]   per-head transpose (K-major for the q absorption)
    void* W_UV;    // [H, v_head, d_c]    copy
    void* ukt_tiled;   // W_UKT and W_UV as the tensor-core kernels' shared-memory images
    void* uv_tiled;    //   (bf16 V2/V3 head shape only; else null)
    const void* W_Q;
    const void* W_O;
    // fold = 1 (bf16): W_UK folded into W_Q, W_UV into W_O, and W_Q's rotary rows
    void* W_QUK = nullptr;   // [H*d_c, d_model]
    void* W_OUV = nullptr;   // [d_model, H*d_c], fp16
    void* W_QR = nullptr;    // [H*d_hR, d_model]
};

// ------------------------------------------------------------------- validation

static size_t esize(const mla_dims* d) { return d->dtype == MLA_BF16 ? 2 : 4; }
static float scale_of(const mla_dims* d) {
    return d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / sqrtf((float)(d->qk_nope + d->d_hR));
}
static float theta_of(const mla_dims* d) { return d->rope_theta > 0.f ? d->rope_theta : 10000.f; }

static bool dims_ok(const mla_dims* d) {
    if (!d) return false;
    if (d->H <= 0 || d->d_c <= 0 || d->d_hR <= 0 || d->qk_nope <= 0 || d->v_head <= 0) return false;
    if (d->d_model < 0) return false;
    if (d->dtype != MLA_F32 && d->dtype != MLA_BF16) return false;
    return true;
}
// Shapes the kernels implement: rotary pairs must not straddle the content/rotary border.
static mla_status dims_supported(const mla_dims* d) {
    if (!dims_ok(d)) return MLA_ERR_INVALID_ARG;
    if ((d->d_hR & 1) || (d->d_c & 1) || (d->qk_nope & 1)) return MLA_ERR_UNSUPPORTED;
    if (d->d_c > 512 || d->v_head > 128 || d->qk_nope + d->d_hR > 256) return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

static int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// KV splits of the CUDA-core decode: about two waves of blocks.
static int simt_splits(int B, int H) {
    const int groups = (H + 7) / 8;
    int ns = (2 * num_sms() + B * groups - 1) / (B * groups > 0 ? B * groups : 1);
    return ns < 1 ? 1 : (ns > 32 ? 32 : ns);
}

// Bump allocator over the caller's workspace (256-byte aligned pieces).
struct Carve {
    char* base;
    size_t used = 0;
    explicit Carve(void* b) : base((char*)b) {}
    void* take(size_t bytes) {
        void* p = base ? base + used : nullptr;
        used += (bytes + 255) & ~(size_t)255;
        return p;
    }
};

// ---------------------------------------------------------------- host helpers

extern "C" const char* mla_status_string(mla_status s) {
    switch (s) {
        case MLA_OK: return "MLA_OK";
        case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: invalid pointer, size or dimension";
        case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: shape not implemented";
        case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace missing or too small";
        case MLA_ERR_CUDA: return "MLA_ERR_CUDA: CUDA runtime call failed";
        case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT: device-side wait gave up";
        case MLA_ERR_OUT_OF_RANGE: return "MLA_ERR_OUT_OF_RANGE: slot or offset outside the cache";
        case MLA_ERR_NO_MEMORY: return "MLA_ERR_NO_MEMORY: device allocation failed";
    }
    return "unknown mla_status";
}

extern "C" const char* mla_last_cuda_error(void) { return g_cuda_msg; }

extern "C" int64_t mla_cache_row_elems(const mla_dims* d) {
    if (!dims_ok(d)) return -1;
    return (int64_t)d->d_c + d->d_hR;
}

extern "C" int64_t mla_cache_bytes_per_token(const mla_dims* d, int32_t layers) {
    if (!dims_ok(d) || layers < 0) return -1;
    return ((int64_t)d->d_c + d->d_hR) * layers * (int64_t)esize(d);
}

static bool tc_decode_ok(const mla_dims* d) {
    return mla::tc::kEnabled && d->dtype == MLA_BF16 && d->H == mla::tc::kH &&
           d->d_c == mla::tc::kDc && d->d_hR == mla::tc::kDr && d->qk_nope == 128 &&
           d->v_head == 128;
}

// The projections (append, query, W_O, prefill K/V) run on the tcgen05 GEMM for bf16 when
// every row stride is a multiple of 16 bytes and the operands are 16-byte aligned (TMA);
// otherwise on the CUDA-core kernels.
static bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }
static bool tc_proj_ok(const mla_dims* d) {
    return d->dtype == MLA_BF16 && d->d_model % 8 == 0 && d->d_c % 8 == 0 && (d->d_c + d->d_hR) % 8 == 0 &&
           (d->H * (d->qk_nope + d->d_hR)) % 8 == 0 && (d->H * d->v_head) % 8 == 0 && d->d_hR % 2 == 0 &&
           (d->qk_nope + d->d_hR) % 2 == 0 && d->qk_nope % 2 == 0;
}

extern "C" int32_t mla_decode_path(const mla_dims* d) {
    if (dims_supported(d) != MLA_OK) return -1;
    return tc_decode_ok(d) ? 1 : 0;
}

// ---------------------------------------------------------------------- weights

// The folded products [L1 "Coste de computo"], per head h (fp32 sums on the tensor cores, one
// rounding):  W_QUK[h*d_c + c, :] = sum_j W_UKT[h, c, j] W_Q[h*qh + j, :] in bf16 (it meets
// the bf16 hidden states) and W_OUV[:, h*d_c + c] = sum_v W_O[:, h*v_head + v] W_UV[h, v, c]
// in fp16 (it meets o_lat, which the merge keeps in fp16); and W_Q's rotary rows.
static cudaError_t fold_weights(const mla_dims* d, mla_weights w, DevErr err, cudaStream_t s) {
    const int H = d->H, dc = d->d_c, qk = d->qk_nope, dR = d->d_hR, vh = d->v_head, dm = d->d_model;
    const int qh = qk + dR;
    const size_t nQUK = (size_t)H * dc * dm, nQR = (size_t)H * dR * dm;
    cudaError_t e = cudaSuccess;
    if (cudaMalloc(&w->W_QUK, nQUK * 2) != cudaSuccess || cudaMalloc(&w->W_OUV, nQUK * 2) != cudaSuccess ||
        cudaMalloc(&w->W_QR, nQR * 2) != cudaSuccess)
        return cudaErrorMemoryAllocation;
    void* qnT = nullptr;   // [H, d_model, qk_nope]: W_Q's content rows, transposed per head
    void* uvT = nullptr;   // [H, d_c, v_head]
    if ((e = cudaMallocAsync(&qnT, (size_t)H * dm * qk * 2, s)) != cudaSuccess) return e;
    if ((e = cudaMallocAsync(&uvT, (size_t)H * dc * vh * 2, s)) != cudaSuccess) {
        cudaFreeAsync(qnT, s);
        return e;
    }
    e = mla::launch_transpose_heads((const bf16*)w->W_Q, (bf16*)qnT, H, qk, dm, s, (long long)qh * dm);
    if (e == cudaSuccess) e = mla::launch_transpose_heads((const bf16*)w->W_UV, (bf16*)uvT, H, vh, dc, s);
    if (e == cudaSuccess) {
        // C[h][c][j] = sum_k W_UKT[h][c][k] qnT[h][j][k]  ->  W_QUK[h*dc + c][j]
        mla::tc::GemmOut o{w->W_QUK, (long long)dc * dm, dm, 1, 0};
        e = mla::tc::gemm_bf16_tc(H, dc, dm, qk, (const bf16*)w->W_UKT, (long long)dc * qk, qk, (const bf16*)qnT,
                                  (long long)dm * qk, qk, o, err.code, err.detail, s);
    }
    if (e == cudaSuccess) {
        // C[h][i][c] = sum_v W_O[i][h*vh + v] uvT[h][c][v]  ->  W_OUV[i][h*dc + c]
        mla::tc::GemmOut o{w->W_OUV, dc, (long long)H * dc, 1, 0};
        o.f16 = 1;
        e = mla::tc::gemm_bf16_tc(H, dm, dc, vh, (const bf16*)w->W_O, vh, (long long)H * vh, (const bf16*)uvT,
                                  (long long)dc * vh, vh, o, err.code, err.detail, s);
    }
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(w->W_QR, (size_t)dR * dm * 2, (const bf16*)w->W_Q + (size_t)qk * dm, (size_t)qh * dm * 2,
                              (size_t)dR * dm * 2, H, cudaMemcpyDeviceToDevice, s);
    const cudaError_t f1 = cudaFreeAsync(qnT, s), f2 = cudaFreeAsync(uvT, s);
    return e != cudaSuccess ? e : f1 != cudaSuccess ? f1 : f2;
}

static void free_weights(mla_weights w) {
    cudaFree(w->W_UK);
    cudaFree(w->W_UKT);
    cudaFree(w->W_UV);
    cudaFree(w->ukt_tiled);
    cudaFree(w->uv_tiled);
    cudaFree(w->W_QUK);
    cudaFree(w->W_OUV);
    cudaFree(w->W_QR);
    delete w;
}

extern "C" mla_status mla_absorb_weights(const mla_dims* d, const void* W_UK, const void* W_UV,
                                         const void* W_Q, const void* W_O, int32_t fold, mla_weights* out,
                                         mla_stream_t stream) {
    if (!out) return MLA_ERR_INVALID_ARG;
    *out = nullptr;
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (!W_UK || !W_UV) return MLA_ERR_INVALID_ARG;
    if ((W_Q || W_O) && d->d_model <= 0) return MLA_ERR_INVALID_ARG;
    if (fold != 0 && fold != 1) return MLA_ERR_INVALID_ARG;
    if (fold && (!W_Q || !W_O)) return MLA_ERR_INVALID_ARG;
    if (fold && (!tc_decode_ok(d) || !tc_proj_ok(d) || !aligned16(W_Q) || !aligned16(W_O)))
        return MLA_ERR_UNSUPPORTED;
    DevErr fold_err;
    if (fold && (st = dev_err(&fold_err)) != MLA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t es = esize(d);
    const size_t nk = (size_t)d->H * d->qk_nope * d->d_c, nv = (size_t)d->H * d->v_head * d->d_c;
    int device = 0;
    MLA_CUDA(cudaGetDevice(&device));
    mla_weights w = new mla_weights_s();
    w->dims = *d;
    w->device = device;
    w->W_Q = W_Q;
    w->W_O = W_O;
    if (cudaMalloc(&w->W_UK, nk * es) != cudaSuccess || cudaMalloc(&w->W_UKT, nk * es) != cudaSuccess ||
        cudaMalloc(&w->W_UV, nv * es) != cudaSuccess) {
        cudaFree(w->W_UK);
        cudaFree(w->W_UKT);
        cudaFree(w->W_UV);
        delete w;
        cudaGetLastError();
        return MLA_ERR_NO_MEMORY;
    }
    cudaError_t e = cudaMemcpyAsync(w->W_UK, W_UK, nk * es, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w->W_UV, W_UV, nv * es, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
        e = d->dtype == MLA_BF16
                ? mla::launch_transpose_heads((const bf16*)W_UK, (bf16*)w->W_UKT, d->H, d->qk_nope, d->d_c, s)
                : mla::launch_transpose_heads((const float*)W_UK, (float*)w->W_UKT, d->H, d->qk_nope, d->d_c, s);
    if (e == cudaSuccess && tc_decode_ok(d)) {
        if (cudaMalloc(&w->ukt_tiled, mla::tc::kTiledWeightBytes) != cudaSuccess ||
            cudaMalloc(&w->uv_tiled, mla::tc::kTiledWeightBytes) != cudaSuccess) {
            cudaGetLastError();
            cudaFree(w->ukt_tiled);
            cudaFree(w->W_UK);
            cudaFree(w->W_UKT);
            cudaFree(w->W_UV);
            delete w;
            return MLA_ERR_NO_MEMORY;
        }
        e = mla::tc::tile_weights_tc((const bf16*)w->W_UKT, (const bf16*)w->W_UV, (bf16*)w->ukt_tiled,
                                     (bf16*)w->uv_tiled, s);
    }
    if (e == cudaSuccess && fold) {
        e = fold_weights(d, w, fold_err, s);
        if (e == cudaErrorMemoryAllocation) {
            cudaGetLastError();
            cudaStreamSynchronize(s);
            free_weights(w);
            return MLA_ERR_NO_MEMORY;
        }
    }
    if (e != cudaSuccess) {
        cudaStreamSynchronize(s);
        free_weights(w);
        return cuda_fail(e, "mla_absorb_weights");
    }
    *out = w;
    return MLA_OK;
}

extern "C" mla_status mla_weights_destroy(mla_weights w) {
    if (!w) return MLA_OK;
    cudaDeviceSynchronize();
    free_weights(w);
    return MLA_OK;
}

// ------------------------------------------------------------------------ append

// [c | k_r] = h [W_DKV; W_KR]^T on the tensor cores: two GEMMs whose epilogues write the
// cache rows (slot scatter) and rotate the k_r columns [L1 "La compresion de MLA",
// "Truco de codificacion posicional"]
static cudaError_t append_tc(const mla_dims* d, const void* h, const void* W_DKV, const void* W_KR,
                             const int32_t* pos, int pos_mod, const int64_t* slot, int n, void* cache,
                             long long capacity, DevErr err, cudaStream_t s) {
    const int row = d->d_c + d->d_hR;
    mla::ProfScope ps(s, "tc_append_proj_rope");
    mla::tc::GemmOut oc{cache, 0, 1, row, 0};
    oc.slot = slot;
    oc.cap = capacity;
    cudaError_t e = mla::tc::gemm_bf16_tc(1, d->d_c, n, d->d_model, (const bf16*)W_DKV, 0, d->d_model,
                                          (const bf16*)h, 0, d->d_model, oc, err.code, err.detail, s);
    if (e != cudaSuccess) return e;
    mla::tc::GemmOut orope{(bf16*)cache + d->d_c, 0, 1, row, 0};
    orope.slot = slot;
    orope.cap = capacity;
    orope.period = d->d_hR;
    orope.rope_start = 0;
    orope.d_rope = d->d_hR;
    orope.pos = pos;
    orope.pos_mod = pos_mod;
    orope.theta = theta_of(d);
    return mla::tc::gemm_bf16_tc(1, d->d_hR, n, d->d_model, (const bf16*)W_KR, 0, d->d_model, (const bf16*)h,
                                 0, d->d_model, orope, err.code, err.detail, s);
}

template <typename T>
static cudaError_t append_impl(const mla_dims* d, const void* h, const void* W_DKV, const void* W_KR,
                               const int32_t* pos, int pos_mod, const int64_t* slot, int n,
                               void* cache, long long capacity, DevErr err, cudaStream_t s) {
    if (tc_proj_ok(d) && aligned16(h) && aligned16(W_DKV) && aligned16(W_KR) && aligned16(cache))
        return append_tc(d, h, W_DKV, W_KR, pos, pos_mod, slot, n, cache, capacity, err, s);
    const int row = d->d_c + d->d_hR;
    mla::ProfScope ps(s, "simt_append_proj_rope");
    return mla::launch_proj_rope<T>((const T*)h, n, d->d_model, (const T*)W_DKV, d->d_c,
                                    (const T*)W_KR, row, row, d->d_c, d->d_hR, pos, pos_mod,
                                    theta_of(d), slot, capacity, (T*)cache, row, err, s);
}

extern "C" mla_status mla_append_cache(const mla_dims* d, const void* h, const void* W_DKV,
                                       const void* W_KR, const int32_t* pos, const int64_t* slot,
                                       int32_t n, void* cache, int64_t capacity,
                                       mla_stream_t stream) {
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (n < 0 || capacity < 0 || d->d_model <= 0) return MLA_ERR_INVALID_ARG;
    if (n == 0) return MLA_OK;
    if (!h || !W_DKV || !W_KR || !pos || !slot || !cache) return MLA_ERR_INVALID_ARG;
    DevErr err;
    if ((st = dev_err(&err)) != MLA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = d->dtype == MLA_BF16
                        ? append_impl<bf16>(d, h, W_DKV, W_KR, pos, 1, slot, n, cache, capacity, err, s)
                        : append_impl<float>(d, h, W_DKV, W_KR, pos, 1, slot, n, cache, capacity, err, s);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_append_cache");
}

// ------------------------------------------------------------------------ decode

struct DecodeWs {
    void* q_buf;     // [B, H, qk_nope + d_hR] query projected from h (storage type)
    float* q_lat;    // [B, H, d_c] fp32 (CUDA-core path)
    float* part_o;   // [nsplit, B, H, d_c]
    float* part_ml;  // [nsplit, B, H, 2]
    float* o_lat;    // [B, H, d_c]
    void* o_buf;     // [B, H, v_head] (storage type) when W_O follows
    double2* rope_tab;   // [B, d_hR / 2] (cos, sin) of the query rotation (tensor-core projection)
    mla::tc::DecodeWs tc;  // tcgen05 path
    size_t bytes;
};

static DecodeWs carve_decode(const mla_dims* d, int B, void* base, bool tc_path) {
    Carve c(base);
    DecodeWs w{};
    const size_t es = esize(d), BH = (size_t)B * d->H;
    w.q_buf = c.take(BH * (d->qk_nope + d->d_hR) * es);
    w.o_buf = c.take(BH * d->v_head * es);
    w.rope_tab = (double2*)c.take((size_t)B * (d->d_hR / 2) * sizeof(double2));
    if (tc_path) {
        w.tc = mla::tc::carve_decode_ws(c.base ? c.base + c.used : nullptr, B, num_sms());
        c.used += mla::tc::decode_ws_bytes(B, num_sms());
    } else {
        const int ns = simt_splits(B, d->H);
        w.q_lat = (float*)c.take(BH * d->d_c * 4);
        w.part_o = (float*)c.take((size_t)ns * BH * d->d_c * 4);
        w.part_ml = (float*)c.take((size_t)ns * BH * 2 * 4);
        w.o_lat = (float*)c.take(BH * d->d_c * 4);
    }
    w.bytes = c.used;
    return w;
}

extern "C" size_t mla_decode_workspace_size(const mla_dims* d, int32_t B) {
    if (dims_supported(d) != MLA_OK || B < 0) return 0;
    return carve_decode(d, B, nullptr, tc_decode_ok(d)).bytes;
}

template <typename T>
static cudaError_t decode_simt(const mla_dims* d, mla_weights w, const T* qn, long long sQn_b,
                               long long sQn_h, const T* qr, long long sQr_b, long long sQr_h,
                               const T* cache, long long cache_rows, const int32_t* offsets, int B, T* o_dst,
                               const DecodeWs& ws, DevErr err, cudaStream_t s) {
    const int H = d->H, dc = d->d_c, qk = d->qk_nope, vh = d->v_head;
    const int ns = simt_splits(B, H);
    cudaError_t e;
    // q_lat[b,h] = W_UK[h]^T q_nope[b,h]
    { mla::ProfScope ps(s, "simt_q_absorb");
    e = mla::launch_gemm_nt<T, T, float>(H, B, dc, qk, qn, sQn_h, sQn_b, 1, (const T*)w->W_UKT,
                                         (long long)dc * qk, qk, 1, ws.q_lat, dc, (long long)H * dc, 1, s); }
    if (e != cudaSuccess) return e;
    { mla::ProfScope ps(s, "simt_decode_split");
    e = mla::launch_decode_split_simt<T>(ws.q_lat, qr, sQr_b, sQr_h, cache, cache_rows, offsets, B, H, dc,
                                         d->d_hR, scale_of(d), ns, ws.part_o, ws.part_ml, err, s); }
    if (e != cudaSuccess) return e;
    { mla::ProfScope ps(s, "simt_combine");
    e = mla::launch_combine(ws.part_o, ws.part_ml, ns, B, H, dc, ws.o_lat, s); }
    if (e != cudaSuccess) return e;
    // o[b,h] = W_UV[h] o_lat[b,h]
    mla::ProfScope ps(s, "simt_w_uv");
    return mla::launch_gemm_nt<float, T, T>(H, B, vh, dc, ws.o_lat, dc, (long long)H * dc, 1,
                                            (const T*)w->W_UV, (long long)vh * dc, dc, 1, o_dst, vh,
                                            (long long)H * vh, 1, s);
}

template <typename T>
static cudaError_t decode_impl(const mla_dims* d, mla_weights w, const void* q_nope,
                               const void* q_rope, const void* h, const int32_t* q_pos,
                               const void* cache, long long cache_rows, const int32_t* offsets, int B, void* out,
                               const DecodeWs& ws, bool tc_path, DevErr err, cudaStream_t s) {
    const int H = d->H, qk = d->qk_nope, dR = d->d_hR, vh = d->v_head;
    const T* qn = (const T*)q_nope;
    const T* qr = (const T*)q_rope;
    long long sQn_b = (long long)H * qk, sQn_h = qk, sQr_b = (long long)H * dR, sQr_h = dR;
    cudaError_t e;
    const bool tc_proj = tc_proj_ok(d) && (q_nope || aligned16(h)) && (q_nope || aligned16(w->W_Q)) &&
                         (!w->W_O || (aligned16(w->W_O) && aligned16(out)));
    if (!q_nope && tc_proj && tc_path && w->W_QUK) {
        // folded weights [L1 "Coste de computo": precomputed products]:
        //   q_lat[b] = W_QUK h[b],  q_rope[b] = RoPE(W_QR h[b]),  attention on the latent cache,
        //   o_lat = the merged latent output,  out[b] = W_OUV o_lat[b]
        const int dc = d->d_c, dm = d->d_model;
        {
            mla::ProfScope ps(s, "tc_q_lat_folded");
            mla::tc::GemmOut oq{ws.tc.q_lat, 0, 1, (long long)H * dc, 0};
            e = mla::tc::gemm_bf16_tc(1, H * dc, B, dm, (const bf16*)w->W_QUK, 0, dm, (const bf16*)h, 0, dm, oq,
                                      err.code, err.detail, s, true);
            if (e != cudaSuccess) return e;
        }
        {
            mla::ProfScope ps(s, "tc_q_rope_folded");
            e = mla::tc::rope_table(q_pos, 1, B, dR, theta_of(d), ws.rope_tab, s);
            if (e != cudaSuccess) return e;
            mla::tc::GemmOut oq{ws.q_buf, 0, 1, (long long)H * dR, 0};
            oq.period = dR;
            oq.rope_start = 0;
            oq.d_rope = dR;
            oq.rope_tab = ws.rope_tab;
            e = mla::tc::gemm_bf16_tc(1, H * dR, B, dm, (const bf16*)w->W_QR, 0, dm, (const bf16*)h, 0, dm, oq,
                                      err.code, err.detail, s);
            if (e != cudaSuccess) return e;
        }
        // o_lat overwrites q_lat: the merge writes it only after the decode kernel has finished
        e = mla::tc::decode_absorbed_tc(nullptr, 0, 0, (const bf16*)ws.q_buf, (long long)H * dR, dR, nullptr, nullptr,
                                        cache, false, cache_rows, offsets, nullptr, nullptr, 0, B, 1, true,
                                        scale_of(d), ws.tc.q_lat, ws.tc, num_sms(), err.code, err.detail, s,
                                        true);
        if (e != cudaSuccess) return e;
        mla::ProfScope ps(s, "tc_w_o_folded");
        mla::tc::GemmOut oo{out, 0, 1, dm, 0};
        oo.in_f16 = 1;   // W_OUV and o_lat in fp16
        return mla::tc::gemm_bf16_tc(1, dm, B, H * dc, (const bf16*)w->W_OUV, 0, (long long)H * dc,
                                     (const bf16*)ws.tc.q_lat, 0, (long long)H * dc, oo, err.code, err.detail, s);
    }
    if (!q_nope && tc_proj) {
        // q = W_Q h with RoPE on each head's rotary part at q_pos [L1 "Multi-head attention estandar"]
        const int qh = qk + dR;
        mla::ProfScope ps(s, "tc_q_proj_rope");
        e = mla::tc::rope_table(q_pos, 1, B, dR, theta_of(d), ws.rope_tab, s);
        if (e != cudaSuccess) return e;
        mla::tc::GemmOut oq{ws.q_buf, 0, 1, (long long)H * qh, 0};
        oq.period = qh;
        oq.rope_start = qk;
        oq.d_rope = dR;
        oq.rope_tab = ws.rope_tab;
        e = mla::tc::gemm_bf16_tc(1, H * qh, B, d->d_model, (const bf16*)w->W_Q, 0, d->d_model, (const bf16*)h, 0,
                                  d->d_model, oq, err.code, err.detail, s);
        if (e != cudaSuccess) return e;
        qn = (const T*)ws.q_buf;
        qr = (const T*)ws.q_buf + qk;
        sQn_b = sQr_b = (long long)H * qh;
        sQn_h = sQr_h = qh;
    } else if (!q_nope) {
        // q = W_Q h with RoPE on each head's rotary part [L1 "Multi-head attention estandar"]
        const int qh = qk + dR;
        mla::ProfScope ps(s, "simt_q_proj_rope");
        e = mla::launch_proj_rope<T>((const T*)h, B, d->d_model, (const T*)w->W_Q, H * qh, nullptr,
                                     H * qh, qh, qk, dR, q_pos, 1, theta_of(d), nullptr, 0,
                                     (T*)ws.q_buf, (long long)H * qh, err, s);
        if (e != cudaSuccess) return e;
        qn = (const T*)ws.q_buf;
        qr = (const T*)ws.q_buf + qk;
        sQn_b = sQr_b = (long long)H * qh;
        sQn_h = sQr_h = qh;
    }
    T* o_dst = w->W_O ? (T*)ws.o_buf : (T*)out;
    if (tc_path) {
        e = mla::tc::decode_absorbed_tc((const bf16*)qn, sQn_b, sQn_h, (const bf16*)qr, sQr_b, sQr_h,
                                        (const bf16*)w->ukt_tiled, (const bf16*)w->uv_tiled,
                                        cache, false, cache_rows, offsets, nullptr, nullptr, 0, B, 1, true,
                                        scale_of(d), (bf16*)o_dst,
                                        ws.tc, num_sms(), err.code, err.detail, s);
    } else {
        e = decode_simt<T>(d, w, qn, sQn_b, sQn_h, qr, sQr_b, sQr_h, (const T*)cache, cache_rows, offsets, B,
                           o_dst, ws, err, s);
    }
    if (e != cudaSuccess) return e;
    if (w->W_O && tc_proj) {
        // out[b] = W_O concat_h o[b,h] [L2 "Informacion tecnica": output projection]
        const int Hv = H * vh;
        mla::ProfScope ps(s, "tc_w_o");
        mla::tc::GemmOut oo{out, 0, 1, d->d_model, 0};
        e = mla::tc::gemm_bf16_tc(1, d->d_model, B, Hv, (const bf16*)w->W_O, 0, Hv, (const bf16*)ws.o_buf, 0, Hv,
                                  oo, err.code, err.detail, s);
    } else if (w->W_O) {
        // out[b] = W_O concat_h o[b,h] [L2 "Informacion tecnica": output projection]
        const int Hv = H * vh;
        mla::ProfScope ps(s, "simt_w_o");
        e = mla::launch_gemm_nt<T, T, T>(1, B, d->d_model, Hv, (const T*)ws.o_buf, 0, Hv, 1,
                                         (const T*)w->W_O, 0, Hv, 1, (T*)out, 0, d->d_model, 1, s);
    }
    return e;
}

extern "C" mla_status mla_decode_absorbed(const mla_dims* d, mla_weights w, const void* q_nope,
                                          const void* q_rope, const void* h, const int32_t* q_pos,
                                          const void* cache, int64_t cache_rows, const int32_t* offsets,
                                          int32_t B, void* out, void* workspace, size_t ws_bytes,
                                          mla_stream_t stream) {
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (!w || B < 0) return MLA_ERR_INVALID_ARG;
    if (memcmp(&w->dims, d, sizeof(mla_dims)) != 0) return MLA_ERR_INVALID_ARG;
    if (B == 0) return MLA_OK;
    if (!cache || !offsets || !out || cache_rows <= 0 || cache_rows > 0x7FFFFFFFLL) return MLA_ERR_INVALID_ARG;
    const bool from_q = q_nope || q_rope;
    if (from_q && (!q_nope || !q_rope)) return MLA_ERR_INVALID_ARG;
    if (!from_q && (!h || !q_pos || !w->W_Q)) return MLA_ERR_INVALID_ARG;
    const bool tc_path = tc_decode_ok(d);
    DecodeWs ws = carve_decode(d, B, workspace, tc_path);
    if (!workspace || ws_bytes < ws.bytes || ((uintptr_t)workspace & 255)) return MLA_ERR_WORKSPACE;
    DevErr err;
    if ((st = dev_err(&err)) != MLA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = d->dtype == MLA_BF16
                        ? decode_impl<bf16>(d, w, q_nope, q_rope, h, q_pos, cache, cache_rows, offsets, B, out, ws, tc_path, err, s)
                        : decode_impl<float>(d, w, q_nope, q_rope, h, q_pos, cache, cache_rows, offsets, B, out, ws, false, err, s);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_decode_absorbed");
}

extern "C" mla_status mla_decode_absorbed_host(const mla_dims* d, mla_weights w, const void* q_nope_host,
                                               const void* q_rope_host, const void* cache, int64_t cache_rows,
                                               const int32_t* offsets, int32_t B, void* out_host, void* workspace,
                                               size_t ws_bytes, mla_stream_t stream) {
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (!w || B < 0) return MLA_ERR_INVALID_ARG;
    if (memcmp(&w->dims, d, sizeof(mla_dims)) != 0) return MLA_ERR_INVALID_ARG;
    if (w->W_O) return MLA_ERR_UNSUPPORTED;
    if (B == 0) return MLA_OK;
    if (!q_nope_host || !q_rope_host || !out_host) return MLA_ERR_INVALID_ARG;
    if (!cache || !offsets || cache_rows <= 0 || cache_rows > 0x7FFFFFFFLL) return MLA_ERR_INVALID_ARG;
    const bool tc_path = tc_decode_ok(d);
    DecodeWs ws = carve_decode(d, B, workspace, tc_path);
    if (!workspace || ws_bytes < ws.bytes || ((uintptr_t)workspace & 255)) return MLA_ERR_WORKSPACE;
    DevErr err;
    if ((st = dev_err(&err)) != MLA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // the query staging area (q_buf, [B*H*(qk + dR)] elements) holds q_nope then q_rope,
    // each in its plain [B, H, .] layout; o goes through o_buf ([B, H, v_head])
    const size_t es = esize(d), BH = (size_t)B * d->H;
    char* qn = (char*)ws.q_buf;
    char* qr = qn + BH * d->qk_nope * es;
    cudaError_t e = cudaMemcpyAsync(qn, q_nope_host, BH * d->qk_nope * es, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(qr, q_rope_host, BH * d->d_hR * es, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "mla_decode_absorbed_host");
    e = d->dtype == MLA_BF16
            ? decode_impl<bf16>(d, w, qn, qr, nullptr, nullptr, cache, cache_rows, offsets, B, ws.o_buf, ws, tc_path, err, s)
            : decode_impl<float>(d, w, qn, qr, nullptr, nullptr, cache, cache_rows, offsets, B, ws.o_buf, ws, false, err, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(out_host, ws.o_buf, BH * d->v_head * es, cudaMemcpyDeviceToHost, s);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_decode_absorbed_host");
}

extern "C" mla_status mla_decode_absorbed_paged(const mla_dims* d, mla_weights w, const void* q_nope,
                                                const void* q_rope, const void* cache, int64_t num_pages,
                                                const int32_t* block_table, int32_t max_blocks,
                                                const int32_t* seq_lens, int32_t B, void* out, void* workspace,
                                                size_t ws_bytes, mla_stream_t stream) {
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (!w || B < 0) return MLA_ERR_INVALID_ARG;
    if (memcmp(&w->dims, d, sizeof(mla_dims)) != 0) return MLA_ERR_INVALID_ARG;
    if (!tc_decode_ok(d) || w->W_O) return MLA_ERR_UNSUPPORTED;
    if (B == 0) return MLA_OK;
    if (!q_nope || !q_rope || !cache || !block_table || !seq_lens || !out || max_blocks <= 0 || num_pages <= 0)
        return MLA_ERR_INVALID_ARG;
    const long long rows = (long long)num_pages * mla::tc::kPageTokens;
    if (rows > 0x7FFFFFFFLL) return MLA_ERR_UNSUPPORTED;
    DecodeWs ws = carve_decode(d, B, workspace, true);
    if (!workspace || ws_bytes < ws.bytes || ((uintptr_t)workspace & 255)) return MLA_ERR_WORKSPACE;
    DevErr err;
    if ((st = dev_err(&err)) != MLA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const long long H = d->H;
    cudaError_t e = mla::tc::decode_absorbed_tc(
        (const bf16*)q_nope, H * d->qk_nope, d->qk_nope, (const bf16*)q_rope, H * d->d_hR, d->d_hR,
        (const bf16*)w->ukt_tiled, (const bf16*)w->uv_tiled, cache, false, rows, nullptr, seq_lens,
        block_table, max_blocks, B, 1, true, scale_of(d), (bf16*)out, ws.tc, num_sms(), err.code, err.detail, s);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_decode_absorbed_paged");
}

// ---------------------------------------------------------- multi-token decode

// The decode workspace for B * q_len sequences, then the per-token block table and lengths.
struct MultiWs {
    DecodeWs dec;
    int32_t* vbt;    // [B * q_len, max_blocks]
    int32_t* vlen;   // [B * q_len]
    size_t bytes;
};

static MultiWs carve_multi(const mla_dims* d, int B, int q_len, int max_blocks, void* base) {
    MultiWs m{};
    m.dec = carve_decode(d, B * q_len, base, true);
    const size_t head = (m.dec.bytes + 255) & ~(size_t)255;
    Carve c(base ? (char*)base + head : nullptr);
    m.vbt = (int32_t*)c.take((size_t)B * q_len * max_blocks * sizeof(int32_t));
    m.vlen = (int32_t*)c.take((size_t)B * q_len * sizeof(int32_t));
    m.bytes = head + c.used;
    return m;
}

// Sibling clusters for a few new tokens per sequence, while at least two cost ranges remain;
// longer chunks expand into per-token sequences.
static bool multi_siblings(int q_len) {
    return q_len <= 8 && mla::tc::decode_clusters(num_sms()) / q_len >= 2;
}

static bool multi_sizes_ok(int32_t B, int32_t q_len, int32_t max_blocks) {
    return B >= 0 && q_len >= 1 && max_blocks >= 1 && (long long)B * q_len <= 0x7FFFFFFFLL &&
           (long long)B * q_len * max_blocks <= 0x7FFFFFFFLL;
}

extern "C" size_t mla_decode_multi_workspace_size(const mla_dims* d, int32_t B, int32_t q_len,
                                                  int32_t max_blocks) {
    if (dims_supported(d) != MLA_OK || !tc_decode_ok(d) || !multi_sizes_ok(B, q_len, max_blocks)) return 0;
    return carve_multi(d, B, q_len, max_blocks, nullptr).bytes;
}

extern "C" mla_status mla_decode_absorbed_paged_multi(const mla_dims* d, mla_weights w, const void* q_nope,
                                                      const void* q_rope, const void* cache, int64_t num_pages,
                                                      const int32_t* block_table, int32_t max_blocks,
                                                      const int32_t* seq_lens, int32_t B, int32_t q_len,
                                                      void* out, void* workspace, size_t ws_bytes,
                                                      mla_stream_t stream) {
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (!w || B < 0 || q_len < 1) return MLA_ERR_INVALID_ARG;
    if (memcmp(&w->dims, d, sizeof(mla_dims)) != 0) return MLA_ERR_INVALID_ARG;
    if (!tc_decode_ok(d) || w->W_O) return MLA_ERR_UNSUPPORTED;
    if (B == 0) return MLA_OK;
    if (!q_nope || !q_rope || !cache || !block_table || !seq_lens || !out || max_blocks <= 0 || num_pages <= 0)
        return MLA_ERR_INVALID_ARG;
    if (!multi_sizes_ok(B, q_len, max_blocks)) return MLA_ERR_UNSUPPORTED;
    const long long rows = (long long)num_pages * mla::tc::kPageTokens;
    if (rows > 0x7FFFFFFFLL) return MLA_ERR_UNSUPPORTED;
    MultiWs ws = carve_multi(d, B, q_len, max_blocks, workspace);
    if (!workspace || ws_bytes < ws.bytes || ((uintptr_t)workspace & 255)) return MLA_ERR_WORKSPACE;
    DevErr err;
    if ((st = dev_err(&err)) != MLA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    const long long H = d->H;
    if (multi_siblings(q_len)) {
        // a few new tokens per sequence (draft verification): the q_len queries of a sequence
        // run on sibling clusters that walk the same tiles together, so each cache tile
        // streams from HBM once
        e = mla::tc::decode_absorbed_tc((const bf16*)q_nope, H * d->qk_nope, d->qk_nope, (const bf16*)q_rope,
                                        H * d->d_hR, d->d_hR, (const bf16*)w->ukt_tiled, (const bf16*)w->uv_tiled,
                                        cache, false, rows, nullptr, seq_lens, block_table, max_blocks, B,
                                        q_len, false, scale_of(d), (bf16*)out, ws.dec.tc, num_sms(), err.code,
                                        err.detail, s);
        return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_decode_absorbed_paged_multi");
    }
    // a long chunk of new tokens (chunked prefill): every token becomes a query sequence of
    // its own on its parent's pages, cut at its own row; consecutive tokens of a sequence run
    // on neighbouring clusters at the same time, and the prefix stays in L2 (loads without the
    // evict-first hint)
    {
        mla::ProfScope ps(s, "multi_token_views");
        e = mla::expand_multi_token(block_table, seq_lens, B, q_len, max_blocks, ws.vbt, ws.vlen, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "mla_decode_absorbed_paged_multi");
    e = mla::tc::decode_absorbed_tc((const bf16*)q_nope, H * d->qk_nope, d->qk_nope, (const bf16*)q_rope,
                                    H * d->d_hR, d->d_hR, (const bf16*)w->ukt_tiled, (const bf16*)w->uv_tiled,
                                    cache, false, rows, nullptr, ws.vlen, ws.vbt, max_blocks, B * q_len, 1,
                                    false, scale_of(d), (bf16*)out, ws.dec.tc, num_sms(), err.code, err.detail, s);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_decode_absorbed_paged_multi");
}

// -------------------------------------------------------------- FP8 latent cache

extern "C" int64_t mla_fp8_row_bytes(const mla_dims* d) {
    if (dims_supported(d) != MLA_OK || !tc_decode_ok(d)) return -1;
    return mla::tc::kF8RowBytes;
}

extern "C" mla_status mla_quantize_cache_fp8(const mla_dims* d, const void* rows, const int64_t* slot, int32_t n,
                                             void* cache_fp8, int64_t capacity, mla_stream_t stream) {
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (!tc_decode_ok(d)) return MLA_ERR_UNSUPPORTED;
    if (n < 0 || capacity < 0) return MLA_ERR_INVALID_ARG;
    if (n == 0) return MLA_OK;
    if (!rows || !cache_fp8 || !aligned16(rows) || !aligned16(cache_fp8)) return MLA_ERR_INVALID_ARG;
    DevErr err;
    if ((st = dev_err(&err)) != MLA_OK) return st;
    cudaError_t e = mla::tc::quantize_rows_fp8((const bf16*)rows, slot, n, (uint8_t*)cache_fp8, capacity, err.code,
                                               err.detail, (cudaStream_t)stream);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_quantize_cache_fp8");
}

extern "C" size_t mla_append_fp8_workspace_size(const mla_dims* d, int32_t n) {
    if (dims_supported(d) != MLA_OK || !tc_decode_ok(d) || n < 0) return 0;
    return ((size_t)n * (d->d_c + d->d_hR) * 2 + 255) & ~(size_t)255;
}

extern "C" mla_status mla_append_cache_fp8(const mla_dims* d, const void* h, const void* W_DKV, const void* W_KR,
                                           const int32_t* pos, const int64_t* slot, int32_t n, void* cache_fp8,
                                           int64_t capacity, void* workspace, size_t ws_bytes, mla_stream_t stream) {
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (!tc_decode_ok(d)) return MLA_ERR_UNSUPPORTED;
    if (n < 0 || capacity < 0 || d->d_model <= 0) return MLA_ERR_INVALID_ARG;
    if (n == 0) return MLA_OK;
    if (!h || !W_DKV || !W_KR || !pos || !slot || !cache_fp8 || !aligned16(cache_fp8)) return MLA_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < mla_append_fp8_workspace_size(d, n) || ((uintptr_t)workspace & 255))
        return MLA_ERR_WORKSPACE;
    DevErr err;
    if ((st = dev_err(&err)) != MLA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // the bf16 rows of the n tokens into the workspace (rows 0 .. n-1, no slot scatter), then
    // quantised into their slots
    cudaError_t e = append_impl<bf16>(d, h, W_DKV, W_KR, pos, 1, nullptr, n, workspace, n, err, s);
    if (e == cudaSuccess) {
        mla::ProfScope ps(s, "fp8_quantize_rows");
        e = mla::tc::quantize_rows_fp8((const bf16*)workspace, slot, n, (uint8_t*)cache_fp8, capacity, err.code,
                                       err.detail, s);
    }
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_append_cache_fp8");
}

extern "C" mla_status mla_decode_absorbed_fp8(const mla_dims* d, mla_weights w, const void* q_nope,
                                              const void* q_rope, const void* cache_fp8, int64_t cache_rows,
                                              const int32_t* offsets, int32_t B, void* out, void* workspace,
                                              size_t ws_bytes, mla_stream_t stream) {
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (!w || B < 0) return MLA_ERR_INVALID_ARG;
    if (memcmp(&w->dims, d, sizeof(mla_dims)) != 0) return MLA_ERR_INVALID_ARG;
    if (!tc_decode_ok(d) || w->W_O) return MLA_ERR_UNSUPPORTED;
    if (B == 0) return MLA_OK;
    if (!q_nope || !q_rope || !cache_fp8 || !offsets || !out || cache_rows <= 0 || cache_rows > 0x7FFFFFFFLL ||
        !aligned16(cache_fp8))
        return MLA_ERR_INVALID_ARG;
    DecodeWs ws = carve_decode(d, B, workspace, true);
    if (!workspace || ws_bytes < ws.bytes || ((uintptr_t)workspace & 255)) return MLA_ERR_WORKSPACE;
    DevErr err;
    if ((st = dev_err(&err)) != MLA_OK) return st;
    const long long H = d->H;
    cudaError_t e = mla::tc::decode_absorbed_tc(
        (const bf16*)q_nope, H * d->qk_nope, d->qk_nope, (const bf16*)q_rope, H * d->d_hR, d->d_hR,
        (const bf16*)w->ukt_tiled, (const bf16*)w->uv_tiled, cache_fp8, true, cache_rows, offsets, nullptr, nullptr, 0,
        B, 1, true, scale_of(d), (bf16*)out, ws.tc, num_sms(), err.code, err.detail, (cudaStream_t)stream);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_decode_absorbed_fp8");
}

// ----------------------------------------------------------------------- prefill

struct PrefillWs {
    void* q_buf;   // [B*S, H, qk_nope + d_hR]
    void* k_buf;   // [B*S, H, qk_nope]
    void* v_buf;   // [B*S, H, v_head]
    double2* rope_tab;   // [B*S, d_hR / 2] (cos, sin) of the query rotation (tensor-core projection)
    size_t bytes;
};

static PrefillWs carve_prefill(const mla_dims* d, int B, int S, void* base) {
    Carve c(base);
    PrefillWs w{};
    const size_t es = esize(d), nH = (size_t)B * S * d->H;
    w.q_buf = c.take(nH * (d->qk_nope + d->d_hR) * es);
    w.k_buf = c.take(nH * d->qk_nope * es);
    w.v_buf = c.take(nH * d->v_head * es);
    w.rope_tab = (double2*)c.take((size_t)B * S * (d->d_hR / 2) * sizeof(double2));
    w.bytes = c.used;
    return w;
}

extern "C" size_t mla_prefill_workspace_size(const mla_dims* d, int32_t B, int32_t S) {
    if (dims_supported(d) != MLA_OK || B < 0 || S < 0) return 0;
    return carve_prefill(d, B, S, nullptr).bytes;
}

template <typename T>
static cudaError_t prefill_impl(const mla_dims* d, mla_weights w, const void* h, const void* W_DKV,
                                const void* W_KR, void* cache, void* out, int B, int S,
                                const PrefillWs& ws, DevErr err, cudaStream_t s) {
    const int H = d->H, dc = d->d_c, dR = d->d_hR, qk = d->qk_nope, vh = d->v_head;
    const int n = B * S, row = dc + dR, qh = qk + dR;
    cudaError_t e;
    // 1. cache rows for every token, position t = i % S, row b*S + t
    e = append_impl<T>(d, h, W_DKV, W_KR, nullptr, S, nullptr, n, cache, n, err, s);
    if (e != cudaSuccess) return e;
    const bool tc_proj = tc_proj_ok(d) && aligned16(h) && aligned16(w->W_Q) && aligned16(cache) &&
                         aligned16(w->W_UK) && aligned16(w->W_UV);
    if (tc_proj) {
        // The tensor-core attention reads the content parts of q and K and all of V as fp16
        // (more precise than bf16 for these magnitudes, same MMA rate); the rotary columns stay
        // bf16, as the cache's k_r is.  Other shapes keep every intermediate in bf16.
        const bool tc_attn = qk == 128 && dR == 64 && vh == 128 && dc == 512 && aligned16(out);
        // 2. queries with RoPE at t = i % S
        { mla::ProfScope ps(s, "tc_q_proj_rope");
        e = mla::tc::rope_table(nullptr, S, n, dR, theta_of(d), ws.rope_tab, s);
        if (e != cudaSuccess) return e;
        mla::tc::GemmOut oq{ws.q_buf, 0, 1, (long long)H * qh, 0};
        oq.period = qh;
        oq.rope_start = qk;
        oq.d_rope = dR;
        oq.rope_tab = ws.rope_tab;
        oq.f16 = tc_attn;
        e = mla::tc::gemm_bf16_tc(1, H * qh, n, d->d_model, (const bf16*)w->W_Q, 0, d->d_model, (const bf16*)h, 0,
                                  d->d_model, oq, err.code, err.detail, s); }
        if (e != cudaSuccess) return e;
        // 3. K_nope[t, h] = W_UK[h] c_t and V[t, h] = W_UV[h] c_t: one B (the cache rows) for all heads
        { mla::ProfScope ps(s, "tc_k_materialise");
        // all heads in one product: W_UK as [H * qk, d_c] rows, K_nope[t] = [H * qk] wide
        mla::tc::GemmOut okb{ws.k_buf, 0, 1, (long long)H * qk, 0};
        okb.f16 = tc_attn;
        e = mla::tc::gemm_bf16_tc(1, H * qk, n, dc, (const bf16*)w->W_UK, 0, dc, (const bf16*)cache, 0, row, okb,
                                  err.code, err.detail, s); }
        if (e != cudaSuccess) return e;
        { mla::ProfScope ps(s, "tc_v_materialise");
        mla::tc::GemmOut ovb{ws.v_buf, 0, 1, (long long)H * vh, 0};
        ovb.f16 = tc_attn;
        e = mla::tc::gemm_bf16_tc(1, H * vh, n, dc, (const bf16*)w->W_UV, 0, dc, (const bf16*)cache, 0, row, ovb,
                                  err.code, err.detail, s); }
        if (e != cudaSuccess) return e;
        if (tc_attn) {
            // 4. causal attention on the tensor cores
            mla::ProfScope ps(s, "tc_prefill_attn");
            return mla::tc::prefill_attn_tc(ws.q_buf, ws.k_buf, (const bf16*)cache, ws.v_buf, B, S, H, scale_of(d),
                                            (bf16*)out, err.code, err.detail, s);
        }
        mla::ProfScope ps(s, "simt_prefill_attn");
        return mla::launch_prefill_attn_simt<T>((const T*)ws.q_buf, (const T*)ws.k_buf, (const T*)cache,
                                                (const T*)ws.v_buf, B, S, H, qk, dR, dc, vh, scale_of(d),
                                                (T*)out, s);
    }
    // 2. queries with RoPE at t
    { mla::ProfScope ps(s, "simt_q_proj_rope");
    e = mla::launch_proj_rope<T>((const T*)h, n, d->d_model, (const T*)w->W_Q, H * qh, nullptr, H * qh,
                                 qh, qk, dR, nullptr, S, theta_of(d), nullptr, 0, (T*)ws.q_buf,
                                 (long long)H * qh, err, s); }
    if (e != cudaSuccess) return e;
    // 3. K_nope = W_UK[h] c and V = W_UV[h] c, materialised [L1 "La compresion de MLA"]
    { mla::ProfScope ps(s, "simt_k_materialise");
    e = mla::launch_gemm_nt<T, T, T>(H, n, qk, dc, (const T*)cache, 0, row, 1, (const T*)w->W_UK,
                                     (long long)qk * dc, dc, 1, (T*)ws.k_buf, qk, (long long)H * qk, 1, s); }
    if (e != cudaSuccess) return e;
    { mla::ProfScope ps(s, "simt_v_materialise");
    e = mla::launch_gemm_nt<T, T, T>(H, n, vh, dc, (const T*)cache, 0, row, 1, (const T*)w->W_UV,
                                     (long long)vh * dc, dc, 1, (T*)ws.v_buf, vh, (long long)H * vh, 1, s); }
    if (e != cudaSuccess) return e;
    // 4. causal attention
    mla::ProfScope ps(s, "simt_prefill_attn");
    return mla::launch_prefill_attn_simt<T>((const T*)ws.q_buf, (const T*)ws.k_buf, (const T*)cache,
                                            (const T*)ws.v_buf, B, S, H, qk, dR, dc, vh, scale_of(d),
                                            (T*)out, s);
}

extern "C" mla_status mla_prefill_causal(const mla_dims* d, mla_weights w, const void* h,
                                         const void* W_DKV, const void* W_KR, void* cache, void* out,
                                         int32_t B, int32_t S, void* workspace, size_t ws_bytes,
                                         mla_stream_t stream) {
    mla_status st = dims_supported(d);
    if (st != MLA_OK) return st;
    if (!w || B < 0 || S < 0 || d->d_model <= 0) return MLA_ERR_INVALID_ARG;
    if (memcmp(&w->dims, d, sizeof(mla_dims)) != 0) return MLA_ERR_INVALID_ARG;
    if ((long long)B * S > (1LL << 31) - 1) return MLA_ERR_UNSUPPORTED;
    if (B == 0 || S == 0) return MLA_OK;
    if (!h || !W_DKV || !W_KR || !cache || !out || !w->W_Q) return MLA_ERR_INVALID_ARG;
    PrefillWs ws = carve_prefill(d, B, S, workspace);
    if (!workspace || ws_bytes < ws.bytes || ((uintptr_t)workspace & 255)) return MLA_ERR_WORKSPACE;
    DevErr err;
    if ((st = dev_err(&err)) != MLA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = d->dtype == MLA_BF16
                        ? prefill_impl<bf16>(d, w, h, W_DKV, W_KR, cache, out, B, S, ws, err, s)
                        : prefill_impl<float>(d, w, h, W_DKV, W_KR, cache, out, B, S, ws, err, s);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_prefill_causal");
}

// ------------------------------------------------------------------- diagnostics

extern "C" mla_status mla_rope_apply(const float* x, const double* cos_sin, int64_t pairs, float* y,
                                     mla_stream_t stream) {
    if (pairs < 0) return MLA_ERR_INVALID_ARG;
    if (pairs == 0) return MLA_OK;
    if (!x || !cos_sin || !y || ((uintptr_t)cos_sin & 15)) return MLA_ERR_INVALID_ARG;
    cudaError_t e = mla::tc::rope_apply(x, (const double2*)cos_sin, pairs, y, (cudaStream_t)stream);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "mla_rope_apply");
}

extern "C" mla_status mla_set_wait_limit(uint32_t polls) {
    const uint32_t p = polls ? polls : 1u << 22;
    MLA_CUDA(mla::tc::set_wait_limit_decode(p));
    MLA_CUDA(mla::tc::set_wait_limit_gemm(p));
    MLA_CUDA(mla::tc::set_wait_limit_prefill(p));
    return MLA_OK;
}

extern "C" mla_status mla_test_starve_projection(int32_t on) {
    MLA_CUDA(mla::tc::set_starve_gemm(on ? 1 : 0));
    return MLA_OK;
}

extern "C" mla_status mla_get_device_error(mla_stream_t stream, int64_t* detail) {
    MLA_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
    int code = 0;
    long long det = 0;
    MLA_CUDA(cudaMemcpyFromSymbol(&code, g_err_code, sizeof code));
    MLA_CUDA(cudaMemcpyFromSymbol(&det, g_err_detail, sizeof det));
    const int zero = 0;
    const long long zero64 = 0;
    MLA_CUDA(cudaMemcpyToSymbol(g_err_code, &zero, sizeof zero));
    MLA_CUDA(cudaMemcpyToSymbol(g_err_detail, &zero64, sizeof zero64));
    if (detail) *detail = det;
    return (mla_status)code;
}
