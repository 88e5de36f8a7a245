// Causal prefill attention with K and V materialised, on the tcgen05 tensor cores, for the
// DeepSeek-V2/V3 head shape (qk_nope = 128, d_hR = 64, v_head = 128): bf16 cache and output,
// the materialised content parts of q and K, and V, in fp16 (see prefill_tc.cuh), P in fp16.
//
// For sequence b, head h and query position t (keys t' <= t of the same sequence):
//     s[t, t'] = scale * (q_nope[t] . k_nope[t'] + q_rope[t] . k_r[t'])     (192-long)
//     o[t]     = sum_t' softmax_t'(s[t, :]) v[t']                              (128 wide)
// with q = [q_nope | q_rope] from the query projection, k_nope and v materialised per head,
// and k_r the (shared) rotary key of the cache row.
//
// One CTA per (block of 128 queries, head, sequence), the longest blocks first.  The query
// block stays in shared memory; key/value blocks of 128 tokens stream through a 2-stage ring
// (K: two 64-column boxes of k_nope and the 64 rotary columns of the cache rows; V: two
// 64-column boxes), each with its own ring.  Per key block: S = Q K^T (M = 128, N = 128, K = 192: 12 MMAs, both
// operands in shared memory) into TMEM, the online softmax in registers (base-2, lazy
// rescale), P (fp16) back to TMEM in one of two buffers, O += P V (M = 128, N = 128,
// K = 128: 8 MMAs with A = P from TMEM and B = V from shared memory).  The diagonal block is
// masked causally; positions at or past the sequence end are masked too.  K and V have
// rings of their own: a K stage is refilled as soon as its Q K^T product completes, and K
// runs one block ahead of V.
// Warp roles (320 threads): warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps
// 2-9 softmax and epilogue: the two warps of a TMEM lane quarter split each score row into
// key halves (and the output into column halves) and exchange their row maxima through
// shared memory.  With two P buffers the softmax of block i + 1 waits for the P V product
// of block i only when it has to rescale O.  Every wait is bounded; a timeout latches an
// error and the kernel drains and returns (the warp pairs leave their loop together).
#include <math.h>

#include "common.cuh"
#include "prefill_tc.cuh"
#include "tc_common.cuh"

namespace mla {
namespace tc {

namespace {

constexpr int kQ = 128, kKB = 128;          // queries per CTA, keys per block
constexpr int kBox = 128 * 128;             // one 128-row x 64-column box of 2-byte values (16 KB)
constexpr int kQBytes = 3 * kBox;           // Q: nope 0-63, nope 64-127, rope
constexpr int kKBytes = 3 * kBox;           // K: the same three column groups
constexpr int kVBytes = 2 * kBox;           // V: columns 0-63, 64-127
constexpr int kRedBytes = 4096;             // row-max / row-sum exchange between warp pairs
constexpr int kPfSmem = kQBytes + 2 * (kKBytes + kVBytes) + 1024 + 256 + kRedBytes;
static_assert(kPfSmem <= 232448, "prefill kernel shared memory over the 227 KB limit");
constexpr uint32_t kColS = 0, kColP = 128, kColO = 256, kPfTmem = 512;   // P: two 64-column buffers
constexpr int kPfThreads = 320;
constexpr float kPfRescale = 8.0f;          // log2 units

__device__ __forceinline__ float ex2f_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(kPfThreads, 1)
prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_v, int S,
                       int H, float scale_log2, __nv_bfloat16* __restrict__ out, int* err_code,
                       long long* err_detail) {
    extern __shared__ uint8_t pf_smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)pf_smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sQ = smem;
    uint8_t* sK = smem + kQBytes;          // [2] K stages (3 boxes)
    uint8_t* sV = sK + 2 * kKBytes;        // [2] V stages (2 boxes)
    uint64_t* bars = (uint64_t*)(sV + 2 * kVBytes);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;     // [2]
    uint64_t* k_empty = bars + 3;    // [2]
    uint64_t* v_full = bars + 5;     // [2]
    uint64_t* v_empty = bars + 7;    // [2]
    uint64_t* s_full = bars + 9;
    uint64_t* s_free = bars + 10;
    uint64_t* p_ready = bars + 11;   // [2] per P buffer
    uint64_t* o_done = bars + 13;    // [2] per P buffer
    uint64_t* drain = bars + 15;
    uint32_t* tmem_slot = (uint32_t*)(bars + 16);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
    float* red_max = (float*)((uint8_t*)bars + 256);   // [2 parity][2 half][128 rows]
    float* red_sum = red_max + 512;                    // [2 half][128 rows]
    volatile int* red_ok = (volatile int*)(red_sum + 256);   // [2 parity][2 half][4 quarters]
    volatile int* fin_ok = red_ok + 16;                      // [2 half][4 quarters]

    // longest query blocks (most key blocks) first, so the short ones fill the tail
    const int qb = gridDim.x - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = qb * kQ;                      // first query position in the sequence
    const long long tok0 = (long long)b * S;     // first token row of the sequence
    const int nkb = qb + 1;                      // key blocks 0 .. qb (causal)

    if (threadIdx.x == 0) {
        ptx::mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&k_full[i], 1);
            ptx::mbar_init(&k_empty[i], 1);
            ptx::mbar_init(&v_full[i], 1);
            ptx::mbar_init(&v_empty[i], 1);
            ptx::mbar_init(&p_ready[i], 256);
            ptx::mbar_init(&o_done[i], 1);
        }
        ptx::mbar_init(s_full, 1);
        ptx::mbar_init(s_free, 256);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, kPfTmem);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) pdl_trigger();

    auto fail = [&](int where) {
        latch(DevErr{err_code, err_detail}, kErrTimeout, 9000000 + where);
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            pdl_wait();   // q, k_nope, v and the cache come from the kernels before
            ptx::tma_prefetch(&tm_q);
            ptx::tma_prefetch(&tm_k);
            ptx::tma_prefetch(&tm_kr);
            ptx::tma_prefetch(&tm_v);
            const int qrow = (int)(tok0 + q0);
            ptx::mbar_expect_tx(q_full, kQBytes);
            ptx::tma_load_3d(sQ, &tm_q, q_full, 0, h, qrow);
            ptx::tma_load_3d(sQ + kBox, &tm_q, q_full, 64, h, qrow);
            ptx::tma_load_3d(sQ + 2 * kBox, &tm_q, q_full, 128, h, qrow);
            // K(i) is issued before V(i - 1): K is needed one product earlier
            int nk_issued = 0, nv_issued = 0;
            for (int i = 0; i <= nkb; ++i) {
                if (i < nkb) {
                    const int st = i & 1;
                    if (i >= 2 && !ptx::mbar_wait(&k_empty[st], ((i >> 1) - 1) & 1, abort_flag)) {
                        fail(1);
                        break;
                    }
                    uint8_t* dst = sK + st * kKBytes;
                    const int krow = (int)(tok0 + (long long)i * kKB);
                    ptx::mbar_expect_tx(&k_full[st], kKBytes);
                    ptx::tma_load_3d(dst, &tm_k, &k_full[st], 0, h, krow);
                    ptx::tma_load_3d(dst + kBox, &tm_k, &k_full[st], 64, h, krow);
                    ptx::tma_load_2d(dst + 2 * kBox, &tm_kr, &k_full[st], 512, krow);
                    ++nk_issued;
                }
                if (i >= 1) {
                    const int j = i - 1, st = j & 1;
                    if (j >= 2 && !ptx::mbar_wait(&v_empty[st], ((j >> 1) - 1) & 1, abort_flag)) {
                        fail(5);
                        break;
                    }
                    uint8_t* dst = sV + st * kVBytes;
                    const int vrow = (int)(tok0 + (long long)j * kKB);
                    ptx::mbar_expect_tx(&v_full[st], kVBytes);
                    ptx::tma_load_3d(dst, &tm_v, &v_full[st], 0, h, vrow);
                    ptx::tma_load_3d(dst + kBox, &tm_v, &v_full[st], 64, h, vrow);
                    ++nv_issued;
                }
            }
            // loads in flight complete before the CTA leaves
            ptx::mbar_wait(q_full, 0, nullptr);
            for (int k = (nk_issued >= 2 ? nk_issued - 2 : 0); k < nk_issued; ++k)
                ptx::mbar_wait(&k_full[k & 1], (k >> 1) & 1, nullptr);
            for (int k = (nv_issued >= 2 ? nv_issued - 2 : 0); k < nv_issued; ++k)
                ptx::mbar_wait(&v_full[k & 1], (k >> 1) & 1, nullptr);
        }
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            // content columns (q_nope, k_nope) and P, V are fp16; the rotary columns bf16
            constexpr uint32_t idesc_s_nope = ptx::idesc_f16_f32(128, kKB, 0, 0);
            constexpr uint32_t idesc_s_rope = ptx::idesc_bf16_f32(128, kKB, 0, 0);
            constexpr uint32_t idesc_o = ptx::idesc_f16_f32(128, 128, 0, 1);   // B = V (MN-major)
            bool ok = ptx::mbar_wait(q_full, 0, abort_flag);
            const uint32_t qa = ptx::smem_u32(sQ);
            auto issue_s = [&](int i) -> bool {
                if (!ptx::mbar_wait(&k_full[i & 1], (i >> 1) & 1, abort_flag)) return false;
                if (i > 0 && !ptx::mbar_wait(s_free, (i - 1) & 1, abort_flag)) return false;
                ptx::tc_fence_after();
                const uint32_t ka = ptx::smem_u32(sK + (i & 1) * kKBytes);
#pragma unroll
                for (int ks = 0; ks < 12; ++ks)   // 3 column groups x 4 K-steps of 16
                    ptx::mma_ss(tmem + kColS, ptx::desc_kmajor_sw128(qa + (ks >> 2) * kBox + (ks & 3) * 32),
                                ptx::desc_kmajor_sw128(ka + (ks >> 2) * kBox + (ks & 3) * 32),
                                ks < 8 ? idesc_s_nope : idesc_s_rope, ks != 0);
                ptx::mma_commit(s_full);
                ptx::mma_commit(&k_empty[i & 1]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int i = 0; ok && i < nkb; ++i) {
                if (i + 1 < nkb && !issue_s(i + 1)) {
                    ok = false;
                    break;
                }
                const int pb = i & 1;
                if (!ptx::mbar_wait(&v_full[i & 1], (i >> 1) & 1, abort_flag) ||
                    !ptx::mbar_wait(&p_ready[pb], (i >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t va = ptx::smem_u32(sV + (i & 1) * kVBytes);
#pragma unroll
                for (int k = 0; k < kKB / 16; ++k)
                    ptx::mma_ts(tmem + kColO, tmem + kColP + pb * 64 + 8 * k,
                                ptx::desc_mnmajor_sw128(va + 2048 * k, kBox), idesc_o, i > 0 || k > 0);
                ptx::mma_commit(&o_done[pb]);
                ptx::mma_commit(&v_empty[i & 1]);
            }
            if (!ok) fail(2);
            ptx::mma_commit(drain);
            if (!ptx::mbar_wait(drain, 0, nullptr)) fail(3);
        }
    } else {
        // ------------------------------------------------ softmax and epilogue
        const int q4 = warp & 3;                     // TMEM lane quarter of this warp
        const int hf = (warp - 2) >> 2;              // key half of S, column half of O
        const int r = q4 * 32 + lane;                // query row in the block
        const int tq = q0 + r;                       // query position
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        const uint32_t pair_bar = 1 + q4;            // the two warps of this lane quarter
        auto uwait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort_flag));
        };
        auto mark_bad = [&](bool& bad) {
            if (!bad && lane == 0) fail(4);
            bad = true;
        };
        float m_run = -INFINITY, l_run = 0.f;
        bool bad = false;
        for (int i = 0; i < nkb; ++i) {
            const int par = i & 1;
            float sc[64];
            float mt = -INFINITY;
            if (!bad && uwait(s_full, i & 1)) {
                ptx::tc_fence_after();
#pragma unroll
                for (int c = 0; c < 64; c += 32) {
                    uint32_t v[32];
                    ptx::tmem_ld32(lane_addr + kColS + hf * 64 + c, v);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) sc[c + j] = __uint_as_float(v[j]);
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(s_free);
                // causal mask on the diagonal block; keys at or past the sequence end
                const int lim = min(tq, S - 1) - (i * kKB + hf * 64);   // last allowed key offset
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    sc[j] = j <= lim ? sc[j] : -INFINITY;
                    mt = fmaxf(mt, sc[j]);
                }
            } else {
                mark_bad(bad);
            }
            // exchange the half-row maxima (and whether both warps may go on)
            red_max[(par * 2 + hf) * 128 + r] = mt;
            if (lane == 0) red_ok[(par * 2 + hf) * 4 + q4] = bad ? 0 : 1;
            ptx::named_barrier_sync(pair_bar, 64);
            if (!red_ok[(par * 2) * 4 + q4] || !red_ok[(par * 2 + 1) * 4 + q4]) {
                bad = true;
                break;
            }
            mt = fmaxf(mt, red_max[(par * 2 + (hf ^ 1)) * 128 + r]);
            float alpha = 1.f;
            const bool first = (i == 0);
            if (mt != -INFINITY && mt * scale_log2 > m_run + kPfRescale) {
                const float m_new = mt * scale_log2;
                alpha = first ? 0.f : ex2f_ftz(m_run - m_new);
                m_run = m_new;
            }
            if (__any_sync(0xffffffffu, !first && alpha != 1.f)) {
                // O of the previous block is complete before it is rescaled
                if (!uwait(&o_done[(i - 1) & 1], ((i - 1) >> 1) & 1)) {
                    mark_bad(bad);
                    continue;
                }
                ptx::tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 64; c += 32) {
                    uint32_t v[32];
                    ptx::tmem_ld32(lane_addr + kColO + hf * 64 + c, v);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
                    ptx::tmem_st32(lane_addr + kColO + hf * 64 + c, v);
                }
            }
            // P buffer `par` is free once the P V product of block i - 2 has completed
            if (i >= 2) {
                if (!uwait(&o_done[par], ((i >> 1) - 1) & 1)) {
                    mark_bad(bad);
                    continue;
                }
                ptx::tc_fence_after();
            }
            // P = 2^(s scale_log2 - m) as fp16 pairs (p <= 2^8 under the lazy rescale), 32
            // keys (16 TMEM columns) at a time
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 64; c += 32) {
                uint32_t pw[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float p0 = ex2f_ftz(fmaf(sc[c + j], scale_log2, -m_run));
                    const float p1 = ex2f_ftz(fmaf(sc[c + j + 1], scale_log2, -m_run));
                    sum += p0 + p1;
                    pw[j / 2] = ptx::pack_f16(p0, p1);
                }
                ptx::tmem_st16(lane_addr + kColP + par * 64 + hf * 32 + c / 2, pw);
            }
            l_run = l_run * alpha + sum;
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&p_ready[par]);
        }
        // the two half-row sums add up
        red_sum[hf * 128 + r] = l_run;
        if (lane == 0) fin_ok[hf * 4 + q4] = bad ? 0 : 1;
        ptx::named_barrier_sync(pair_bar, 64);
        bool ok = fin_ok[q4] && fin_ok[4 + q4];
        const float l_tot = l_run + red_sum[(hf ^ 1) * 128 + r];
        // epilogue: o = O / l for the queries inside the sequence, this warp's 64 columns
        if (ok) ok = uwait(&o_done[(nkb - 1) & 1], ((nkb - 1) >> 1) & 1);
        if (ok) {
            ptx::tc_fence_after();
            const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
            __nv_bfloat16* dst = out + ((tok0 + tq) * H + h) * 128 + hf * 64;
#pragma unroll 1
            for (int c = 0; c < 64; c += 32) {
                uint32_t v[32];
                ptx::tmem_ld32(lane_addr + kColO + hf * 64 + c, v);
                ptx::tmem_wait_ld();
                if (tq < S) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8)
                        *(uint4*)(dst + c + j) = make_uint4(
                            ptx::pack_bf16(__uint_as_float(v[j]) * inv, __uint_as_float(v[j + 1]) * inv),
                            ptx::pack_bf16(__uint_as_float(v[j + 2]) * inv, __uint_as_float(v[j + 3]) * inv),
                            ptx::pack_bf16(__uint_as_float(v[j + 4]) * inv, __uint_as_float(v[j + 5]) * inv),
                            ptx::pack_bf16(__uint_as_float(v[j + 6]) * inv, __uint_as_float(v[j + 7]) * inv));
                }
            }
        } else {
            mark_bad(bad);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, kPfTmem);
}

}  // namespace

cudaError_t set_wait_limit_prefill(uint32_t polls) { return ptx::set_wait_limit_of_this_file(polls); }

cudaError_t prefill_attn_tc(const void* q, const void* k_nope, const __nv_bfloat16* cache,
                            const void* v, int B, int S, int H, float scale, __nv_bfloat16* out,
                            int* err_code, long long* err_detail, cudaStream_t s) {
    if (B <= 0 || S <= 0) return cudaSuccess;
    const uint64_t n = (uint64_t)B * S;
    CUtensorMap mq, mk, mkr, mv;
    const uint64_t dq[3] = {192, (uint64_t)H, n};
    const uint64_t sq[2] = {192 * 2, (uint64_t)H * 192 * 2};
    const uint64_t dk[3] = {128, (uint64_t)H, n};
    const uint64_t sk[2] = {128 * 2, (uint64_t)H * 128 * 2};
    const uint32_t box3[3] = {64, 1, 128};
    const uint64_t dr[2] = {576, n};
    const uint64_t sr[1] = {576 * 2};
    const uint32_t box2[2] = {64, 128};
    if (!make_tmap_bf16(&mq, q, 3, dq, sq, box3) || !make_tmap_bf16(&mk, k_nope, 3, dk, sk, box3) ||
        !make_tmap_bf16(&mkr, cache, 2, dr, sr, box2) || !make_tmap_bf16(&mv, v, 3, dk, sk, box3))
        return cudaErrorInvalidValue;
    static const cudaError_t attr =
        cudaFuncSetAttribute(prefill_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfSmem);
    if (attr != cudaSuccess) return attr;
    dim3 grid((S + kQ - 1) / kQ, H, B);
    return launch_pdl(prefill_attn_tc_kernel, grid, dim3(kPfThreads), kPfSmem, s, mq, mk, mkr, mv, S, H,
                      scale * 1.4426950408889634f, out, err_code, err_detail);
}

}  // namespace tc
}  // namespace mla
