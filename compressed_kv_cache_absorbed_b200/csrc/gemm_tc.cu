// Batched bf16 GEMM on the tcgen05 tensor cores.
//
// One 128 x BN output tile per CTA.  Warp 0 streams 128x64 A and BNx64 B tiles (128-byte
// swizzled) into a ring of shared-memory stages with TMA; warp 1 allocates TMEM and issues
// tcgen05.mma (M = 128, N = BN, K = 16) into a fp32 TMEM accumulator, releasing each stage
// with tcgen05.commit; warps 2-5 read the accumulator back with tcgen05.ld (one TMEM lane
// = one output row per thread) and store it.  Every wait is bounded: on a timeout the
// kernel latches an error, drains the MMAs it issued, frees TMEM and returns.
#include "common.cuh"
#include "gemm_tc.cuh"
#include "tc_common.cuh"

namespace mla {
namespace tc {

namespace {

constexpr int kBM = 128, kBK = 64;

template <int BN>
struct GemmCfg {
    static constexpr int A_BYTES = kBM * kBK * 2;
    static constexpr int B_BYTES = BN * kBK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int MAX_STAGES = (196608 / STAGE) > 8 ? 8 : (196608 / STAGE);
    static constexpr int TMEM_COLS = BN < 32 ? 32 : BN;
    static constexpr int smem(int stages) { return stages * STAGE + 1024 + 256; }
};

__device__ __forceinline__ void fail(int* code, long long* detail, volatile int* abort_flag, int where) {
    latch(DevErr{code, detail}, kErrTimeout, (long long)where * 1000000 + blockIdx.x * 1000 + blockIdx.y);
    *abort_flag = 1;
}

template <int BN>
__global__ void __launch_bounds__(192, 1)
gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M,
                    int N, int K, int stages, GemmOut out, int chain_head, int b_bcast, int* err_code,
                    long long* err_detail) {
    using C = GemmCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = (uint64_t*)(smem + stages * C::STAGE);
    uint64_t* empty = full + stages;
    uint64_t* accum = empty + stages;
    uint32_t* tmem_slot = (uint32_t*)(accum + 1);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * BN, z = blockIdx.z;
    const int nk = (K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(accum, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Dependents may launch once every CTA got here.  As the first kernel of a chain this
    // waits for all earlier work first, so that later kernels of the chain may read the
    // chain's inputs without waiting.
    if (threadIdx.x == 64) {
        if (chain_head) pdl_wait();
        pdl_trigger();
    }

    if (warp == 0) {
        if (lane == 0) {
            ptx::tma_prefetch(&tmA);
            ptx::tma_prefetch(&tmB);
            // A (the weights) of the first stages does not depend on earlier kernels: start it
            // before waiting for them; B and the output do.
            const int pre = nk < stages ? nk : stages;
            for (int kb = 0; kb < pre; ++kb) {
                ptx::mbar_expect_tx(&full[kb], C::STAGE);
                ptx::tma_load_3d(smem + kb * C::STAGE, &tmA, &full[kb], kb * kBK, m0, z);
            }
            pdl_wait();
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % stages;
                const uint32_t ph = (kb / stages) & 1;
                uint8_t* a = smem + s * C::STAGE;
                if (kb >= pre) {
                    if (!ptx::mbar_wait(&empty[s], ph ^ 1, abort_flag)) {
                        fail(err_code, err_detail, abort_flag, 1);
                        break;
                    }
                    ptx::mbar_expect_tx(&full[s], C::STAGE);
                    ptx::tma_load_3d(a, &tmA, &full[s], kb * kBK, m0, z);
                }
                if (b_bcast)
                    ptx::tma_load_2d(a + C::A_BYTES, &tmB, &full[s], kb * kBK, n0);
                else
                    ptx::tma_load_3d(a + C::A_BYTES, &tmB, &full[s], kb * kBK, n0, z);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(kBM, BN, 0, 0);
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % stages;
                const uint32_t ph = (kb / stages) & 1;
                if (!ptx::mbar_wait(&full[s], ph, abort_flag)) {
                    fail(err_code, err_detail, abort_flag, 2);
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t a = ptx::smem_u32(smem + s * C::STAGE);
                const uint32_t b = a + C::A_BYTES;
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k)
                    ptx::mma_ss(tmem, ptx::desc_kmajor_sw128(a + 32 * k), ptx::desc_kmajor_sw128(b + 32 * k),
                                idesc, (kb | k) != 0);
                ptx::mma_commit(&empty[s]);
            }
            // completes once every MMA issued above has finished (also after an abort)
            ptx::mma_commit(accum);
        }
    } else {
        const int sub = warp & 3;
        pdl_wait();   // the output may still be read by an earlier kernel
        const bool ok = ptx::mbar_wait(accum, 0, nullptr);
        if (!ok) fail(err_code, err_detail, abort_flag, 3);
        ptx::tc_fence_after();
        const int row = m0 + sub * 32 + lane;
        const int within = out.period > 0 ? row % out.period : -1;
        const bool rope_row = out.period > 0 && within >= out.rope_start;
        if (ok && !*abort_flag && nk > 0) {
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t r[32];
                ptx::tmem_ld32(tmem + ((uint32_t)(sub * 32) << 16) + c0, r);
                ptx::tmem_wait_ld();
                char* base = (char*)out.C;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int n = n0 + c0 + j;   // the same for the whole warp
                    if (n >= N) continue;
                    float v = __uint_as_float(r[j]);
                    if (out.period > 0) {
                        // rows m and m ^ 1 are adjacent lanes: the pair (even, odd) is rotated
                        const float partner = __shfl_xor_sync(0xffffffffu, v, 1);
                        if (rope_row) {
                            const int pi = (within - out.rope_start) >> 1;
                            double cs, sn;
                            if (out.rope_tab) {
                                const double2 t = out.rope_tab[(long long)n * (out.d_rope >> 1) + pi];
                                cs = t.x;
                                sn = t.y;
                            } else {
                                const int p = out.pos ? out.pos[n] : n % out.pos_mod;
                                const double inv = pow((double)out.theta, -2.0 * (double)pi / (double)out.d_rope);
                                sincos((double)p * inv, &sn, &cs);
                            }
                            v = (row & 1) ? (float)((double)partner * sn + (double)v * cs)
                                          : (float)((double)v * cs - (double)partner * sn);
                        }
                    }
                    if (row >= M) continue;
                    long long orow = n;
                    if (out.slot) {
                        orow = out.slot[n];
                        if (orow < 0 || orow >= out.cap) {
                            if (lane == 0) latch(DevErr{err_code, err_detail}, kErrOutOfRange, n);
                            continue;
                        }
                    }
                    const long long idx = (long long)z * out.sz + (long long)row * out.sm + orow * out.sn;
                    if (out.f32)
                        ((float*)base)[idx] = v;
                    else
                        ((__nv_bfloat16*)base)[idx] = __float2bfloat16_rn(v);
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int BN>
cudaError_t launch(int Z, int M, int N, int K, const CUtensorMap& ma, const CUtensorMap& mb, const GemmOut& out,
                   bool chain_head, bool b_bcast, int* err_code, long long* err_detail, cudaStream_t s) {
    using C = GemmCfg<BN>;
    static bool attr_set = false;   // the attribute is per function; set it once
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::smem(C::MAX_STAGES));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int nk = (K + kBK - 1) / kBK;
    const int stages = nk < C::MAX_STAGES ? (nk < 2 ? 2 : nk) : C::MAX_STAGES;
    dim3 grid((N + BN - 1) / BN, (M + kBM - 1) / kBM, Z);
    return launch_pdl(gemm_bf16_tc_kernel<BN>, grid, dim3(192), C::smem(stages), s, ma, mb, M, N, K, stages, out,
                      (int)chain_head, (int)b_bcast, err_code, err_detail);
}

__global__ void __launch_bounds__(256)
rope_table_kernel(const int32_t* __restrict__ pos, int pos_mod, int N, int half, float theta, double2* __restrict__ tab) {
    const long long total = (long long)N * half;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
        const int n = (int)(i / half), pi = (int)(i % half);
        const int p = pos ? pos[n] : n % pos_mod;
        const double inv = pow((double)theta, -2.0 * (double)pi / (double)(2 * half));
        double sn, cs;
        sincos((double)p * inv, &sn, &cs);
        tab[i] = make_double2(cs, sn);
    }
}

}  // namespace

cudaError_t rope_table(const int32_t* pos, int pos_mod, int N, int d_rope, float theta, double2* tab,
                       cudaStream_t s) {
    if (N <= 0) return cudaSuccess;
    const long long total = (long long)N * (d_rope / 2);
    const int blocks = (int)min(4096LL, (total + 255) / 256);
    rope_table_kernel<<<blocks, 256, 0, s>>>(pos, pos_mod, N, d_rope / 2, theta, tab);
    return cudaGetLastError();
}

cudaError_t gemm_bf16_tc(int Z, int M, int N, int K, const __nv_bfloat16* A, long long sAz, long long sAm,
                         const __nv_bfloat16* B, long long sBz, long long sBn, const GemmOut& out,
                         int* err_code, long long* err_detail, cudaStream_t s, bool chain_head) {
    if (Z <= 0 || M <= 0 || N <= 0 || K <= 0) return cudaSuccess;
    // the narrowest tile that covers N, narrowed further while the grid has fewer CTAs than a
    // quarter of the SMs (very skinny weight-streaming GEMMs: A is then re-read from L2)
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    }
    int BN = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
    const long long mtiles = (long long)Z * ((M + 127) / 128);
    while (BN > 32 && mtiles * ((N + BN - 1) / BN) < sms / 4) BN >>= 1;
    const bool b_bcast = sBz == 0;   // one B for every z: a 2-D map
    if (Z == 1) {
        sAz = (long long)M * sAm;
        sBz = (long long)N * sBn;
    }
    CUtensorMap ma, mb;
    const uint64_t da[3] = {(uint64_t)K, (uint64_t)M, (uint64_t)Z};
    const uint64_t sa[2] = {(uint64_t)sAm * 2, (uint64_t)sAz * 2};
    const uint32_t ba[3] = {(uint32_t)kBK, (uint32_t)kBM, 1};
    const uint64_t db[3] = {(uint64_t)K, (uint64_t)N, (uint64_t)Z};
    const uint64_t sb[2] = {(uint64_t)sBn * 2, (uint64_t)sBz * 2};
    const uint32_t bb[3] = {(uint32_t)kBK, (uint32_t)BN, 1};
    if (!make_tmap_bf16(&ma, A, 3, da, sa, ba) || !make_tmap_bf16(&mb, B, b_bcast ? 2 : 3, db, sb, bb))
        return cudaErrorInvalidValue;
    switch (BN) {
        case 32: return launch<32>(Z, M, N, K, ma, mb, out, chain_head, b_bcast, err_code, err_detail, s);
        case 64: return launch<64>(Z, M, N, K, ma, mb, out, chain_head, b_bcast, err_code, err_detail, s);
        case 128: return launch<128>(Z, M, N, K, ma, mb, out, chain_head, b_bcast, err_code, err_detail, s);
        default: return launch<256>(Z, M, N, K, ma, mb, out, chain_head, b_bcast, err_code, err_detail, s);
    }
}

}  // namespace tc
}  // namespace mla
