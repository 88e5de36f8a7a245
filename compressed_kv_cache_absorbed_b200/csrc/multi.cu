// Multi-token decode over a paged latent cache, for long chunks of new tokens (an absorbed
// chunked prefill over a cached prefix): per-token views of the pages.  Each new token
// becomes a sequence of its own that shares its parent's pages and stops at the token's own
// row, so the paged absorbed decode runs on them unchanged.  (A few new tokens per sequence,
// as in draft verification, run on sibling clusters instead, without these views.)
#include "multi.cuh"

namespace mla {

namespace {

__global__ void __launch_bounds__(256)
expand_multi_token_kernel(const int32_t* __restrict__ bt, const int32_t* __restrict__ lens, int q_len,
                          int max_blocks, long long n, int32_t* __restrict__ vbt, int32_t* __restrict__ vlen) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const long long v = i / max_blocks;            // new-token sequence
        const int j = (int)(i - v * max_blocks);       // block of it
        const long long b = v / q_len;                 // parent sequence
        vbt[i] = bt[b * max_blocks + j];
        if (j == 0) {
            const int L = lens[b] - (q_len - 1 - (int)(v - b * q_len));
            vlen[v] = L > 0 ? L : 0;   // a token with no key decodes to zeros
        }
    }
}

}  // namespace

cudaError_t expand_multi_token(const int32_t* block_table, const int32_t* seq_lens, int B, int q_len,
                               int max_blocks, int32_t* vbt, int32_t* vlen, cudaStream_t s) {
    if (B <= 0 || q_len <= 0 || max_blocks <= 0) return cudaSuccess;
    const long long n = (long long)B * q_len * max_blocks;
    const long long want = (n + 255) / 256;
    const int blocks = (int)(want < 4096 ? want : 4096);
    expand_multi_token_kernel<<<blocks, 256, 0, s>>>(block_table, seq_lens, q_len, max_blocks, n, vbt, vlen);
    return cudaGetLastError();
}

}  // namespace mla
