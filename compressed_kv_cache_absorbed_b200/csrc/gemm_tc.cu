// Batched bf16 GEMM on the tcgen05 tensor cores.
//
// Persistent: one CTA per SM walks the output tiles (128 x BN) in a grouped order (16
// row-tiles by all column-tiles, so that both operands of the tiles in flight stay in L2).
// Warp 0 streams 128x64 X and BNx64 Y tiles (128-byte swizzled) into a ring of
// shared-memory stages with TMA, across tile boundaries; warp 1 allocates TMEM and issues
// tcgen05.mma (M = 128, N = BN, K = 16) into one of two fp32 TMEM accumulators, releasing
// each stage with tcgen05.commit; warps 2-5 read a finished accumulator back with
// tcgen05.ld (one TMEM lane = one output row of the tile per thread) and store it while the
// next tile accumulates into the other one.  Every wait is bounded: on a timeout the kernel
// latches an error, drains the MMAs it issued and the loads in flight, frees TMEM and
// returns.
//
// Two orientations of the same product C = A B^T:
//  - weights-major (X = A, Y = B): a thread owns an output feature m and writes it for BN
//    tokens n (a warp writes 32 consecutive features of one token at a time).  Used for
//    few tokens, where the weights stream from HBM and more row-tiles mean more CTAs.
//  - token-major (X = B, Y = A): a thread owns a token n and writes 32 consecutive features
//    of it as four 16-byte stores; rotary pairs are adjacent columns of one thread.
#include "common.cuh"
#include "gemm_tc.cuh"
#include "tc_common.cuh"

namespace mla {
namespace tc {

namespace {

// A k-block is kSub TMA boxes of 64 columns (one 128-byte swizzle atom) per operand, so each
// operand row is read in kSub * 128 contiguous bytes per stage: 2 boxes up to BN = 128 (the
// weight-streaming shapes, where longer runs per row read DRAM better), 1 box for BN = 256
// (whose stages would otherwise drop to two).
constexpr int kBM = 128, kBox = 64, kGroupRows = 16;
constexpr int kSwapMinTokens = 1024;   // token-major from this many tokens on

template <int BN>
struct GemmCfg {
    static constexpr int kSub = BN >= 256 ? 1 : 2;
    static constexpr int kBK = kBox * kSub;
    static constexpr int X_BYTES = kBM * kBK * 2;
    static constexpr int Y_BYTES = BN * kBK * 2;
    static constexpr int STAGE = X_BYTES + Y_BYTES;
    static constexpr int STAGES = (196608 / STAGE) > 8 ? 8 : (196608 / STAGE);
    static constexpr int ACC_COLS = BN < 32 ? 32 : BN;   // one accumulator; two are allocated
    static constexpr int SMEM = STAGES * STAGE + 1024 + 256;
};

// Test hook for the failure-detection path (set only by mla_test_starve_projection): when
// nonzero the loader warp issues no loads, so the MMA issuer's and the epilogue's bounded
// waits run out and latch a timeout while no copy and no MMA is in flight.
__device__ int g_starve_loads = 0;

// fp16 store of an fp32 value, saturated to the finite range
__device__ __forceinline__ __half to_half_sat(float v) { return __float2half_rn(fminf(fmaxf(v, -65504.f), 65504.f)); }
__device__ __forceinline__ uint32_t pack_half_sat(float lo, float hi) {
    __half2 h = __halves2half2(to_half_sat(lo), to_half_sat(hi));
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void fail(int* code, long long* detail, volatile int* abort_flag, int where) {
    latch(DevErr{code, detail}, kErrTimeout, (long long)where * 1000000 + blockIdx.x);
    *abort_flag = 1;
}

struct Tile {
    int z, i0, j0;   // batch, first X row, first Y row
};

// tile t -> (z, X row-tile, Y row-tile): groups of kGroupRows X row-tiles, Y fastest-varying
// across the group's columns
__device__ __forceinline__ Tile tile_of(int t, int tiles_x, int tiles_y, int BN) {
    const int per = tiles_x * tiles_y;
    const int z = t / per, r = t % per;
    const int g = r / (kGroupRows * tiles_y);
    const int first = g * kGroupRows;
    const int gs = min(kGroupRows, tiles_x - first);
    const int w = r - g * kGroupRows * tiles_y;
    return Tile{z, (first + w % gs) * kBM, (w / gs) * BN};
}

// (cos, sin) of the rotary angle of pair pi at token n
__device__ __noinline__ double2 rope_cs(const double2* tab, int d_rope, const int32_t* pos, int pos_mod, float theta,
                                       int n, int pi) {
    if (tab) return tab[(long long)n * (d_rope >> 1) + pi];
    const int p = pos ? pos[n] : n % pos_mod;
    const double inv = pow((double)theta, -2.0 * (double)pi / (double)d_rope);
    double sn, cs;
    sincos((double)p * inv, &sn, &cs);
    return make_double2(cs, sn);
}

template <int BN>
__global__ void __launch_bounds__(192, 1)
gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY, int Mx,
                    int Ny, int K, int Z, GemmOut out, int chain_head, int x_2d, int y_2d, int swap,
                    int* err_code, long long* err_detail) {
    using C = GemmCfg<BN>;
    constexpr int kSub = C::kSub, kBK = C::kBK;
    constexpr int stages = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = (uint64_t*)(smem + stages * C::STAGE);
    uint64_t* empty = full + stages;
    uint64_t* acc_full = empty + stages;   // [2]
    uint64_t* acc_empty = acc_full + 2;    // [2]
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = (K + kBK - 1) / kBK;
    const int tiles_x = (Mx + kBM - 1) / kBM, tiles_y = (Ny + BN - 1) / BN;
    const int tiles = Z * tiles_x * tiles_y;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&acc_full[b], 1);
            ptx::mbar_init(&acc_empty[b], 128);
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 2 * C::ACC_COLS);
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
        if (lane == 0 && !g_starve_loads) {
            ptx::tma_prefetch(&tmX);
            ptx::tma_prefetch(&tmY);
            auto load_x = [&](uint8_t* st, uint64_t* bar, int kb, const Tile& tl) {
#pragma unroll
                for (int b = 0; b < kSub; ++b) {
                    if (x_2d)
                        ptx::tma_load_2d(st + b * kBM * 128, &tmX, bar, kb * kBK + b * kBox, tl.i0);
                    else
                        ptx::tma_load_3d(st + b * kBM * 128, &tmX, bar, kb * kBK + b * kBox, tl.i0, tl.z);
                }
            };
            auto load_y = [&](uint8_t* st, uint64_t* bar, int kb, const Tile& tl) {
#pragma unroll
                for (int b = 0; b < kSub; ++b) {
                    if (y_2d)
                        ptx::tma_load_2d(st + C::X_BYTES + b * BN * 128, &tmY, bar, kb * kBK + b * kBox, tl.j0);
                    else
                        ptx::tma_load_3d(st + C::X_BYTES + b * BN * 128, &tmY, bar, kb * kBK + b * kBox, tl.j0, tl.z);
                }
            };
            // The weights (X weights-major, Y token-major) of the first stages do not depend
            // on earlier kernels: start them before waiting for those; the activations do.
            int pre = 0;
            if ((int)blockIdx.x < tiles) {
                const Tile tl = tile_of(blockIdx.x, tiles_x, tiles_y, BN);
                pre = nk < stages ? nk : stages;
                for (int kb = 0; kb < pre; ++kb) {
                    ptx::mbar_expect_tx(&full[kb], C::STAGE);
                    if (swap)
                        load_y(smem + kb * C::STAGE, &full[kb], kb, tl);
                    else
                        load_x(smem + kb * C::STAGE, &full[kb], kb, tl);
                }
            }
            pdl_wait();
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
                const Tile tl = tile_of(t, tiles_x, tiles_y, BN);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % stages;
                    uint8_t* st = smem + s * C::STAGE;
                    if (it >= pre) {
                        if (it >= stages && !ptx::mbar_wait(&empty[s], ((it / stages) & 1) ^ 1, abort_flag)) {
                            fail(err_code, err_detail, abort_flag, 1);
                            ok = false;
                            break;
                        }
                        ptx::mbar_expect_tx(&full[s], C::STAGE);
                        if (swap)
                            load_y(st, &full[s], kb, tl);
                        else
                            load_x(st, &full[s], kb, tl);
                    }
                    if (swap)
                        load_x(st, &full[s], kb, tl);
                    else
                        load_y(st, &full[s], kb, tl);
                }
            }
            // the loads in flight land before the CTA leaves
            for (int k = (it > stages ? it - stages : 0); k < it; ++k)
                ptx::mbar_wait(&full[k % stages], (k / stages) & 1, nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = out.in_f16 ? ptx::idesc_f16_f32(kBM, BN, 0, 0) : ptx::idesc_bf16_f32(kBM, BN, 0, 0);
            int it = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
                const int buf = lt & 1;
                if (lt >= 2 && !ptx::mbar_wait(&acc_empty[buf], ((lt >> 1) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d = tmem + buf * C::ACC_COLS;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % stages;
                    if (!ptx::mbar_wait(&full[s], (it / stages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a = ptx::smem_u32(smem + s * C::STAGE);
                    const uint32_t b = a + C::X_BYTES;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)   // box k / 4, K-step k % 4 within it
                        ptx::mma_ss(d, ptx::desc_kmajor_sw128(a + (k >> 2) * kBM * 128 + 32 * (k & 3)),
                                    ptx::desc_kmajor_sw128(b + (k >> 2) * BN * 128 + 32 * (k & 3)), idesc,
                                    (kb | k) != 0);
                    ptx::mma_commit(&empty[s]);
                }
                if (ok) ptx::mma_commit(&acc_full[buf]);
            }
            if (!ok) fail(err_code, err_detail, abort_flag, 2);
            // completes once every MMA issued above has finished (also after an abort)
            ptx::mma_commit(drain);
            if (!ptx::mbar_wait(drain, 0, nullptr)) fail(err_code, err_detail, abort_flag, 3);
        }
    } else {
        const int sub = warp & 3;
        pdl_wait();   // the output may still be read by an earlier kernel
        int lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            const int buf = lt & 1;
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(&acc_full[buf], (lt >> 1) & 1, abort_flag));
            if (!ok) break;
            ptx::tc_fence_after();
            const Tile tl = tile_of(t, tiles_x, tiles_y, BN);
            const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + buf * C::ACC_COLS;
            const int xr = tl.i0 + sub * 32 + lane;   // this thread's X row
            char* base = (char*)out.C;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t r[32];
                ptx::tmem_ld32(taddr + c0, r);
                ptx::tmem_wait_ld();
                if (c0 + 32 >= BN) {   // the accumulator may be reused from here on
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(&acc_empty[buf]);
                }
                if (*abort_flag) continue;
                if (swap) {
                    // token xr, features f0 .. f0 + 31 (Ny % 32 == 0: all or none in range)
                    const int f0 = tl.j0 + c0;
                    if (xr >= Mx || f0 >= Ny) continue;
                    long long orow = xr;
                    if (out.slot) {
                        orow = out.slot[xr];
                        if (orow < 0 || orow >= out.cap) {
                            latch(DevErr{err_code, err_detail}, kErrOutOfRange, xr);
                            continue;
                        }
                    }
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
                    if (out.period > 0) {
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const int within = (f0 + j) % out.period;
                            if (within < out.rope_start) continue;
                            const double2 t = rope_cs(out.rope_tab, out.d_rope, out.pos, out.pos_mod, out.theta, xr, (within - out.rope_start) >> 1);
                            rope_rotate(v[j], v[j + 1], t.x, t.y);
                        }
                    }
                    uint4* dst = (uint4*)((__nv_bfloat16*)base + (long long)tl.z * out.sz + f0 + orow * out.sn);
                    // 32 columns from a multiple of 32: all fp16 or all bf16 (rope_start % 32 == 0)
                    const bool half_out = out.f16 && (out.period == 0 || f0 % out.period < out.rope_start);
                    if (half_out) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(pack_half_sat(v[8 * q], v[8 * q + 1]), pack_half_sat(v[8 * q + 2], v[8 * q + 3]),
                                                pack_half_sat(v[8 * q + 4], v[8 * q + 5]),
                                                pack_half_sat(v[8 * q + 6], v[8 * q + 7]));
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(ptx::pack_bf16(v[8 * q], v[8 * q + 1]), ptx::pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                                ptx::pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                                                ptx::pack_bf16(v[8 * q + 6], v[8 * q + 7]));
                    }
                    continue;
                }
                // weights-major: feature row xr, tokens n0 + c0 .. + 31
                const int row = xr;
                const int within = out.period > 0 ? row % out.period : -1;
                const bool rope_row = out.period > 0 && within >= out.rope_start;
                const bool half_row = out.f16 && !rope_row;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int n = tl.j0 + c0 + j;   // the same for the whole warp
                    if (n >= Ny) continue;
                    float v = __uint_as_float(r[j]);
                    if (out.period > 0) {
                        // rows m and m ^ 1 are adjacent lanes: the pair (even, odd) is rotated
                        const float partner = __shfl_xor_sync(0xffffffffu, v, 1);
                        if (rope_row) {
                            const double2 t = rope_cs(out.rope_tab, out.d_rope, out.pos, out.pos_mod, out.theta, n, (within - out.rope_start) >> 1);
                            float x0 = (row & 1) ? partner : v, x1 = (row & 1) ? v : partner;
                            rope_rotate(x0, x1, t.x, t.y);
                            v = (row & 1) ? x1 : x0;
                        }
                    }
                    if (row >= Mx) continue;
                    long long orow = n;
                    if (out.slot) {
                        orow = out.slot[n];
                        if (orow < 0 || orow >= out.cap) {
                            if (lane == 0) latch(DevErr{err_code, err_detail}, kErrOutOfRange, n);
                            continue;
                        }
                    }
                    const long long idx = (long long)tl.z * out.sz + (long long)row * out.sm + orow * out.sn;
                    if (out.f32)
                        ((float*)base)[idx] = v;
                    else if (half_row)
                        ((__half*)base)[idx] = to_half_sat(v);
                    else
                        ((__nv_bfloat16*)base)[idx] = __float2bfloat16_rn(v);
                }
            }
        }
        if (!ok && lane == 0) fail(err_code, err_detail, abort_flag, 4);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, 2 * C::ACC_COLS);
}

template <int BN>
cudaError_t launch(int Z, int Mx, int Ny, int K, const CUtensorMap& mx, const CUtensorMap& my, const GemmOut& out,
                   bool chain_head, bool x_2d, bool y_2d, bool swap, int sms, int* err_code,
                   long long* err_detail, cudaStream_t s) {
    using C = GemmCfg<BN>;
    static bool attr_set = false;   // the attribute is per function; set it once
    if (!attr_set) {
        cudaError_t e =
            cudaFuncSetAttribute(gemm_bf16_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const long long tiles = (long long)Z * ((Mx + kBM - 1) / kBM) * ((Ny + BN - 1) / BN);
    if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int grid = (int)(tiles < sms ? tiles : sms);
    return launch_pdl(gemm_bf16_tc_kernel<BN>, dim3(grid), dim3(192), C::SMEM, s, mx, my, Mx, Ny, K, Z, out,
                      (int)chain_head, (int)x_2d, (int)y_2d, (int)swap, err_code, err_detail);
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

namespace {
__global__ void __launch_bounds__(256)
rope_apply_kernel(const float* __restrict__ x, const double2* __restrict__ cs, long long pairs, float* __restrict__ y) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < pairs; i += (long long)gridDim.x * blockDim.x) {
        float x0 = x[2 * i], x1 = x[2 * i + 1];
        rope_rotate(x0, x1, cs[i].x, cs[i].y);
        y[2 * i] = x0;
        y[2 * i + 1] = x1;
    }
}
}  // namespace

cudaError_t rope_apply(const float* x, const double2* cs, long long pairs, float* y, cudaStream_t s) {
    if (pairs <= 0) return cudaSuccess;
    const long long want = (pairs + 255) / 256;
    rope_apply_kernel<<<(int)(want < 4096 ? want : 4096), 256, 0, s>>>(x, cs, pairs, y);
    return cudaGetLastError();
}

cudaError_t set_wait_limit_gemm(uint32_t polls) { return ptx::set_wait_limit_of_this_file(polls); }

cudaError_t set_starve_gemm(int on) { return cudaMemcpyToSymbol(g_starve_loads, &on, sizeof on); }

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
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    }
    // token-major for many tokens when the output rows take 16-byte stores
    const bool swap = N >= kSwapMinTokens && !out.f32 && out.sm == 1 && M % 32 == 0 && out.sz % 8 == 0 &&
                      out.sn % 8 == 0 && ((uintptr_t)out.C & 15) == 0 &&
                      (out.period == 0 || (out.period % 2 == 0 && out.rope_start % 2 == 0)) &&
                      (!out.f16 || out.period == 0 || (out.period % 32 == 0 && out.rope_start % 32 == 0));
    const int Mx = swap ? N : M, Ny = swap ? M : N;   // MMA rows (128-tiles) and columns (BN-tiles)
    // the narrowest tile that covers Ny, narrowed to 64 while there are fewer tiles than two
    // waves of CTAs, and further to 32 while fewer than a quarter of the SMs (skinny
    // weight-streaming GEMMs: more CTAs stream the weights, the operand re-reads come from L2)
    int BN = Ny <= 32 ? 32 : Ny <= 64 ? 64 : Ny <= 128 ? 128 : 256;
    const long long xtiles = (long long)Z * ((Mx + 127) / 128);
    while (BN > 64 && xtiles * ((Ny + BN - 1) / BN) < 2 * sms) BN >>= 1;
    while (BN > 32 && xtiles * ((Ny + BN - 1) / BN) < sms / 4) BN >>= 1;
    const bool b_bcast = sBz == 0;   // one B for every z: a 2-D map
    const bool a_bcast = sAz == 0 && Z > 1;
    if (Z == 1) {
        sAz = (long long)M * sAm;
        sBz = (long long)N * sBn;
    }
    CUtensorMap ma, mb;
    const uint64_t da[3] = {(uint64_t)K, (uint64_t)M, (uint64_t)Z};
    const uint64_t sa[2] = {(uint64_t)sAm * 2, (uint64_t)sAz * 2};
    const uint64_t db[3] = {(uint64_t)K, (uint64_t)N, (uint64_t)Z};
    const uint64_t sb[2] = {(uint64_t)sBn * 2, (uint64_t)sBz * 2};
    const uint32_t bx[3] = {(uint32_t)kBox, (uint32_t)kBM, 1};   // the 128-row operand
    const uint32_t by[3] = {(uint32_t)kBox, (uint32_t)BN, 1};    // the BN-row operand
    const CUtensorMapDataType dt = out.in_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_tmap(&ma, dt, 2, A, a_bcast ? 2 : 3, da, sa, swap ? by : bx, 128) ||
        !make_tmap(&mb, dt, 2, B, b_bcast ? 2 : 3, db, sb, swap ? bx : by, 128))
        return cudaErrorInvalidValue;
    const CUtensorMap& mx = swap ? mb : ma;
    const CUtensorMap& my = swap ? ma : mb;
    const bool x_2d = swap ? b_bcast : a_bcast, y_2d = swap ? a_bcast : b_bcast;
    switch (BN) {
        case 32: return launch<32>(Z, Mx, Ny, K, mx, my, out, chain_head, x_2d, y_2d, swap, sms, err_code, err_detail, s);
        case 64: return launch<64>(Z, Mx, Ny, K, mx, my, out, chain_head, x_2d, y_2d, swap, sms, err_code, err_detail, s);
        case 128:
            return launch<128>(Z, Mx, Ny, K, mx, my, out, chain_head, x_2d, y_2d, swap, sms, err_code, err_detail, s);
        default:
            return launch<256>(Z, Mx, Ny, K, mx, my, out, chain_head, x_2d, y_2d, swap, sms, err_code, err_detail, s);
    }
}

}  // namespace tc
}  // namespace mla
