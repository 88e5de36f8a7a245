// CUDA-core (FFMA) kernels: the fp32 path and the general-shape path of every MLA step.
// fp32 storage needs ~1e-5 relative accuracy, which tensor-core tf32 cannot give, so the
// fp32 layer runs here; bf16 layers whose dims the tcgen05 kernels do not cover run here too.
#include <math.h>

#include "common.cuh"

namespace mla {

namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// ----------------------------------------------------------- projection + RoPE
// A 32 x 64 output tile per block; each thread owns 2 rows x 4 columns (two RoPE pairs),
// so the rotation of a pair happens in the registers that accumulated it.
template <typename T>
__global__ void __launch_bounds__(256)
proj_rope_kernel(const T* __restrict__ A, int M, int K, const T* __restrict__ W1, int n1,
                 const T* __restrict__ W2, int N, int period, int rope_start, int d_rope,
                 const int32_t* __restrict__ pos, int pos_mod, float theta,
                 const int64_t* __restrict__ slot, long long capacity, T* __restrict__ out,
                 long long ld_out, DevErr err) {
    constexpr int TM = 32, TN = 64, TK = 32;
    __shared__ float As[TM][TK + 1];
    __shared__ float Ws[TN][TK + 1];
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    const int tr = tid / 16, tc = tid % 16;
    float acc[2][4] = {};
    for (int k0 = 0; k0 < K; k0 += TK) {
        for (int e = tid; e < TM * TK; e += 256) {
            int r = e / TK, c = e % TK, gm = m0 + r, gk = k0 + c;
            As[r][c] = (gm < M && gk < K) ? to_f(A[(long long)gm * K + gk]) : 0.f;
        }
        for (int e = tid; e < TN * TK; e += 256) {
            int r = e / TK, c = e % TK, gn = n0 + r, gk = k0 + c;
            float v = 0.f;
            if (gn < N && gk < K) {
                const T* wr = gn < n1 ? W1 + (long long)gn * K : W2 + (long long)(gn - n1) * K;
                v = to_f(wr[gk]);
            }
            Ws[r][c] = v;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < TK; ++kk) {
            float a0 = As[tr * 2][kk], a1 = As[tr * 2 + 1][kk];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float w = Ws[tc * 4 + j][kk];
                acc[0][j] = fmaf(a0, w, acc[0][j]);
                acc[1][j] = fmaf(a1, w, acc[1][j]);
            }
        }
        __syncthreads();
    }
    for (int i = 0; i < 2; ++i) {
        const int gm = m0 + tr * 2 + i;
        if (gm >= M) continue;
        long long dst = gm;
        if (slot) {
            dst = slot[gm];
            if (dst < 0 || dst >= capacity) {
                if (blockIdx.x == 0 && tc == 0) latch(err, kErrOutOfRange, gm);
                continue;
            }
        }
        const int p = pos ? pos[gm] : (gm % pos_mod);
#pragma unroll
        for (int jp = 0; jp < 4; jp += 2) {
            const int gn = n0 + tc * 4 + jp;
            if (gn >= N) continue;
            float v0 = acc[i][jp], v1 = acc[i][jp + 1];
            const int within = gn % period;
            if (within >= rope_start) {
                // pair index within the rotary block; angle = pos * theta^(-2i/d), in double
                const int pi = (within - rope_start) / 2;
                const double inv = pow((double)theta, -2.0 * (double)pi / (double)d_rope);
                double sn, cs;
                sincos((double)p * inv, &sn, &cs);
                rope_rotate(v0, v1, cs, sn);
            }
            T* o = out + dst * ld_out + gn;
            o[0] = from_f<T>(v0);
            if (gn + 1 < N) o[1] = from_f<T>(v1);
        }
    }
}

// ------------------------------------------------------------ strided batched GEMM
template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256)
gemm_nt_kernel(int M, int N, int K, const TA* __restrict__ A, long long sAz, long long sAm,
               long long sAk, const TB* __restrict__ B, long long sBz, long long sBn,
               long long sBk, TC* __restrict__ C, long long sCz, long long sCm, long long sCn) {
    constexpr int TM = 32, TN = 64, TK = 32;
    __shared__ float As[TM][TK + 1];
    __shared__ float Bs[TN][TK + 1];
    const int tid = threadIdx.x, z = blockIdx.z;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    const int tr = tid / 16, tc = tid % 16;
    A += z * sAz;
    B += z * sBz;
    C += z * sCz;
    const bool a_kfast = (sAk == 1), b_kfast = (sBk == 1);
    float acc[2][4] = {};
    for (int k0 = 0; k0 < K; k0 += TK) {
        for (int e = tid; e < TM * TK; e += 256) {
            int r = a_kfast ? e / TK : e % TM, c = a_kfast ? e % TK : e / TM;
            int gm = m0 + r, gk = k0 + c;
            As[r][c] = (gm < M && gk < K) ? to_f(A[gm * sAm + gk * sAk]) : 0.f;
        }
        for (int e = tid; e < TN * TK; e += 256) {
            int r = b_kfast ? e / TK : e % TN, c = b_kfast ? e % TK : e / TN;
            int gn = n0 + r, gk = k0 + c;
            Bs[r][c] = (gn < N && gk < K) ? to_f(B[gn * sBn + gk * sBk]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < TK; ++kk) {
            float a0 = As[tr * 2][kk], a1 = As[tr * 2 + 1][kk];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float w = Bs[tc * 4 + j][kk];
                acc[0][j] = fmaf(a0, w, acc[0][j]);
                acc[1][j] = fmaf(a1, w, acc[1][j]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int gm = m0 + tr * 2 + i;
        if (gm >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int gn = n0 + tc * 4 + j;
            if (gn < N) C[gm * sCm + gn * sCn] = from_f<TC>(acc[i][j]);
        }
    }
}

// --------------------------------------------------------- split-KV decode (SIMT)
// Block = (split, sequence, group of 8 heads); one warp per head.  32 cache rows are
// staged in shared memory (fp32, row stride padded by one to spread banks); lane t scores
// token t, the warp runs the online softmax and accumulates o_lat (d_c / 32 per lane).
constexpr int kDecTT = 32;
constexpr int kDecHPB = 8;

template <typename T>
__global__ void __launch_bounds__(256)
decode_split_simt_kernel(const float* __restrict__ q_lat, const T* __restrict__ q_rope,
                         long long sQb, long long sQh, const T* __restrict__ cache,
                         long long cache_rows, const int32_t* __restrict__ offsets, int B, int H,
                         int d_c, int d_hR, float scale, int nsplit, float* __restrict__ part_o,
                         float* __restrict__ part_ml, DevErr err) {
    extern __shared__ float sm[];
    const int row = d_c + d_hR, rs = row + 1;
    float* tile = sm;
    float* qs = sm + kDecTT * rs;
    const int split = blockIdx.x, b = blockIdx.y, hg = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int h = hg * kDecHPB + warp;
    long long r0 = offsets[b], r1 = offsets[b + 1];
    if (r1 < r0 || r0 < 0 || r1 > cache_rows) {
        if (threadIdx.x == 0 && split == 0 && hg == 0) latch(err, kErrOutOfRange, b);
        r0 = r1 = 0;
    }
    const long long Tn = r1 - r0;
    const long long chunk = (Tn + nsplit - 1) / nsplit;
    const long long t0 = min(Tn, (long long)split * chunk), t1 = min(Tn, t0 + chunk);
    for (int e = threadIdx.x; e < kDecHPB * row; e += blockDim.x) {
        const int hh = e / row, c = e % row, gh = hg * kDecHPB + hh;
        float v = 0.f;
        if (gh < H)
            v = c < d_c ? q_lat[((long long)b * H + gh) * d_c + c]
                        : to_f(q_rope[b * sQb + gh * sQh + (c - d_c)]);
        qs[e] = v;
    }
    float m = -INFINITY, l = 0.f;
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    for (long long tb = t0; tb < t1; tb += kDecTT) {
        const int nt = (int)min((long long)kDecTT, t1 - tb);
        __syncthreads();
        for (int e = threadIdx.x; e < nt * row; e += blockDim.x) {
            const int r = e / row, c = e % row;
            tile[r * rs + c] = to_f(cache[(r0 + tb + r) * row + c]);
        }
        __syncthreads();
        if (h < H) {
            float s = -INFINITY;
            if (lane < nt) {
                const float* kr = tile + lane * rs;
                const float* q = qs + warp * row;
                float a = 0.f;
                for (int c = 0; c < row; ++c) a = fmaf(q[c], kr[c], a);
                s = a * scale;
            }
            const float mn = fmaxf(m, warp_max(s));   // finite: lane 0 holds a real token
            const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
            const float p = (lane < nt) ? expf(s - mn) : 0.f;
            l = l * alpha + warp_sum(p);
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] *= alpha;
            for (int tt = 0; tt < nt; ++tt) {
                const float pt = __shfl_sync(kFull, p, tt);
                const float* kr = tile + tt * rs;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int c = lane + 32 * j;
                    if (c < d_c) acc[j] = fmaf(pt, kr[c], acc[j]);
                }
            }
            m = mn;
        }
    }
    if (h < H) {
        const long long pidx = ((long long)split * B + b) * H + h;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int c = lane + 32 * j;
            if (c < d_c) part_o[pidx * d_c + c] = acc[j];
        }
        if (lane == 0) {
            part_ml[pidx * 2] = m;
            part_ml[pidx * 2 + 1] = l;
        }
    }
}

// ------------------------------------------------------------- log-sum-exp merge
__global__ void combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                               int nsplit, int B, int H, int d_c, float* __restrict__ o_lat) {
    const int h = blockIdx.x, b = blockIdx.y;
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, part_ml[(((long long)s * B + b) * H + h) * 2]);
    float L = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        const long long p = ((long long)s * B + b) * H + h;
        const float ms = part_ml[p * 2];
        if (ms != -INFINITY) L += expf(ms - M) * part_ml[p * 2 + 1];
    }
    for (int c = threadIdx.x; c < d_c; c += blockDim.x) {
        float v = 0.f;
        for (int s = 0; s < nsplit; ++s) {
            const long long p = ((long long)s * B + b) * H + h;
            const float ms = part_ml[p * 2];
            if (ms != -INFINITY) v += expf(ms - M) * part_o[p * d_c + c];
        }
        o_lat[((long long)b * H + h) * d_c + c] = L > 0.f ? v / L : 0.f;
    }
}

// ------------------------------------------------------ causal prefill (SIMT)
// Block = (64 queries, head, sequence); keys in blocks of 64 up to the diagonal.  Each
// thread owns 4 query rows: 4 score columns and 8 output columns of them; the 16 threads
// sharing a row reduce with shuffles inside their half-warp.
constexpr int kPfB = 64;

template <typename T>
__global__ void __launch_bounds__(256)
prefill_attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k_nope,
                         const T* __restrict__ cache, const T* __restrict__ v, int S, int H,
                         int qk, int dR, int d_c, int vh, float scale, T* __restrict__ out) {
    extern __shared__ float sm[];
    const int dq = qk + dR, qs_ld = dq + 1, vs_ld = vh + 1, ps_ld = kPfB + 1;
    float* Qs = sm;
    float* Ks = Qs + kPfB * qs_ld;
    float* Vs = Ks + kPfB * qs_ld;
    float* Ps = Vs + kPfB * vs_ld;
    const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, tr = tid / 16, tc = tid % 16;
    const long long base = (long long)b * S;
    const int q0 = qb * kPfB;
    const int row = d_c + dR;
    for (int e = tid; e < kPfB * dq; e += 256) {
        const int r = e / dq, c = e % dq, t = q0 + r;
        Qs[r * qs_ld + c] = t < S ? to_f(q[((base + t) * H + h) * dq + c]) : 0.f;
    }
    float m[4], l[4], o[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) o[i][c] = 0.f;
    }
    for (int kb = 0; kb <= qb; ++kb) {
        __syncthreads();
        for (int e = tid; e < kPfB * dq; e += 256) {
            const int r = e / dq, c = e % dq, t = kb * kPfB + r;
            float x = 0.f;
            if (t < S)
                x = c < qk ? to_f(k_nope[((base + t) * H + h) * qk + c])
                           : to_f(cache[(base + t) * row + d_c + (c - qk)]);
            Ks[r * qs_ld + c] = x;
        }
        for (int e = tid; e < kPfB * vh; e += 256) {
            const int r = e / vh, c = e % vh, t = kb * kPfB + r;
            Vs[r * vs_ld + c] = t < S ? to_f(v[((base + t) * H + h) * vh + c]) : 0.f;
        }
        __syncthreads();
        float s[4][4] = {};
        for (int d = 0; d < dq; ++d) {
            float a[4], kk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = Qs[(tr * 4 + i) * qs_ld + d];
#pragma unroll
            for (int j = 0; j < 4; ++j) kk[j] = Ks[(tc * 4 + j) * qs_ld + d];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) s[i][j] = fmaf(a[i], kk[j], s[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int qi = q0 + tr * 4 + i;
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int kj = kb * kPfB + tc * 4 + j;
                s[i][j] = (kj <= qi && kj < S) ? s[i][j] * scale : -INFINITY;
                mt = fmaxf(mt, s[i][j]);
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, off));
            const float mn = fmaxf(m[i], mt);
            float alpha = 1.f, rs = 0.f;
            if (mn != -INFINITY) alpha = (m[i] == -INFINITY) ? 0.f : expf(m[i] - mn);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float p = (s[i][j] == -INFINITY) ? 0.f : expf(s[i][j] - mn);
                Ps[(tr * 4 + i) * ps_ld + tc * 4 + j] = p;
                rs += p;
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) rs += __shfl_xor_sync(kFull, rs, off);
            l[i] = l[i] * alpha + rs;
#pragma unroll
            for (int c = 0; c < 8; ++c) o[i][c] *= alpha;
            m[i] = mn;
        }
        __syncthreads();
        for (int k = 0; k < kPfB; ++k) {
            float p[4], vv[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) p[i] = Ps[(tr * 4 + i) * ps_ld + k];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int cc = tc * 8 + c;
                vv[c] = cc < vh ? Vs[k * vs_ld + cc] : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 8; ++c) o[i][c] = fmaf(p[i], vv[c], o[i][c]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = q0 + tr * 4 + i;
        if (t >= S) continue;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int cc = tc * 8 + c;
            if (cc < vh) out[((base + t) * H + h) * vh + cc] = from_f<T>(l[i] > 0.f ? o[i][c] / l[i] : 0.f);
        }
    }
}

template <typename T>
__global__ void transpose_heads_kernel(const T* __restrict__ src, T* __restrict__ dst, int R, int C,
                                       long long src_head_stride) {
    __shared__ T tile[32][33];
    const int h = blockIdx.z;
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    const T* s = src + (long long)h * src_head_stride;
    T* d = dst + (long long)h * R * C;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < R && c < C) tile[i][threadIdx.x] = s[(long long)r * C + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (r < R && c < C) d[(long long)c * R + r] = tile[threadIdx.x][i];
    }
}

}  // namespace

// ------------------------------------------------------------------- launchers

template <typename T>
cudaError_t launch_proj_rope(const T* A, int M, int K, const T* W1, int n1, const T* W2, int N,
                             int period, int rope_start, int d_rope, const int32_t* pos,
                             int pos_mod, float theta, const int64_t* slot, long long capacity,
                             T* out, long long ld_out, DevErr err, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    dim3 grid(ceil_div(N, 64), ceil_div(M, 32));
    proj_rope_kernel<T><<<grid, 256, 0, s>>>(A, M, K, W1, n1, W2, N, period, rope_start, d_rope,
                                             pos, pos_mod, theta, slot, capacity, out, ld_out, err);
    return cudaGetLastError();
}

template <typename TA, typename TB, typename TC>
cudaError_t launch_gemm_nt(int Z, int M, int N, int K, const TA* A, long long sAz, long long sAm,
                           long long sAk, const TB* B, long long sBz, long long sBn, long long sBk,
                           TC* C, long long sCz, long long sCm, long long sCn, cudaStream_t s) {
    if (Z == 0 || M == 0 || N == 0) return cudaSuccess;
    dim3 grid(ceil_div(N, 64), ceil_div(M, 32), Z);
    gemm_nt_kernel<TA, TB, TC><<<grid, 256, 0, s>>>(M, N, K, A, sAz, sAm, sAk, B, sBz, sBn, sBk,
                                                    C, sCz, sCm, sCn);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_decode_split_simt(const float* q_lat, const T* q_rope, long long sQb,
                                     long long sQh, const T* cache, long long cache_rows,
                                     const int32_t* offsets, int B, int H, int d_c, int d_hR,
                                     float scale, int nsplit, float* part_o, float* part_ml,
                                     DevErr err, cudaStream_t s) {
    if (B == 0) return cudaSuccess;
    const int row = d_c + d_hR;
    const size_t smem = sizeof(float) * ((size_t)kDecTT * (row + 1) + (size_t)kDecHPB * row);
    cudaError_t e = cudaFuncSetAttribute(decode_split_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(nsplit, B, ceil_div(H, kDecHPB));
    decode_split_simt_kernel<T><<<grid, 256, smem, s>>>(q_lat, q_rope, sQb, sQh, cache, cache_rows, offsets, B,
                                                        H, d_c, d_hR, scale, nsplit, part_o,
                                                        part_ml, err);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float* part_o, const float* part_ml, int nsplit, int B, int H,
                           int d_c, float* o_lat, cudaStream_t s) {
    if (B == 0) return cudaSuccess;
    combine_kernel<<<dim3(H, B), 128, 0, s>>>(part_o, part_ml, nsplit, B, H, d_c, o_lat);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_prefill_attn_simt(const T* q, const T* k_nope, const T* cache, const T* v,
                                     int B, int S, int H, int qk_nope, int d_hR, int d_c,
                                     int v_head, float scale, T* out, cudaStream_t s) {
    if (B == 0 || S == 0) return cudaSuccess;
    const int dq = qk_nope + d_hR;
    const size_t smem = sizeof(float) * ((size_t)2 * kPfB * (dq + 1) + (size_t)kPfB * (v_head + 1) +
                                         (size_t)kPfB * (kPfB + 1));
    cudaError_t e = cudaFuncSetAttribute(prefill_attn_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(S, kPfB), H, B);
    prefill_attn_simt_kernel<T><<<grid, 256, smem, s>>>(q, k_nope, cache, v, S, H, qk_nope, d_hR,
                                                        d_c, v_head, scale, out);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_transpose_heads(const T* src, T* dst, int Hn, int R, int C, cudaStream_t s,
                                   long long src_head_stride) {
    dim3 grid(ceil_div(C, 32), ceil_div(R, 32), Hn);
    transpose_heads_kernel<T><<<grid, dim3(32, 8), 0, s>>>(src, dst, R, C,
                                                           src_head_stride < 0 ? (long long)R * C : src_head_stride);
    return cudaGetLastError();
}

// ----------------------------------------------------------- instantiations
using bf16 = __nv_bfloat16;
#define MLA_INST_T(T)                                                                         \
    template cudaError_t launch_proj_rope<T>(const T*, int, int, const T*, int, const T*, int,  \
                                             int, int, int, const int32_t*, int, float,         \
                                             const int64_t*, long long, T*, long long, DevErr,  \
                                             cudaStream_t);                                     \
    template cudaError_t launch_decode_split_simt<T>(const float*, const T*, long long,         \
                                                     long long, const T*, long long,            \
                                                     const int32_t*, int, int, int, int, float, \
                                                     int, float*, float*, DevErr, cudaStream_t);\
    template cudaError_t launch_prefill_attn_simt<T>(const T*, const T*, const T*, const T*,    \
                                                     int, int, int, int, int, int, int, float,  \
                                                     T*, cudaStream_t);                         \
    template cudaError_t launch_transpose_heads<T>(const T*, T*, int, int, int, cudaStream_t, long long);
MLA_INST_T(float)
MLA_INST_T(bf16)

#define MLA_INST_G(TA, TB, TC)                                                                   \
    template cudaError_t launch_gemm_nt<TA, TB, TC>(int, int, int, int, const TA*, long long,     \
                                                    long long, long long, const TB*, long long,   \
                                                    long long, long long, TC*, long long,         \
                                                    long long, long long, cudaStream_t);
MLA_INST_G(float, float, float)
MLA_INST_G(bf16, bf16, float)
MLA_INST_G(bf16, bf16, bf16)
MLA_INST_G(float, bf16, bf16)
MLA_INST_G(float, float, bf16)

}  // namespace mla
