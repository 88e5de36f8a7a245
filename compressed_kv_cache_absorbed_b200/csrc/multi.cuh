// Multi-token decode over a paged latent cache: per-token views of the pages.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

// q_len new tokens per sequence, their cache rows already appended: sequence b holds
// seq_lens[b] tokens in the pages block_table[b * max_blocks + j].  New token t of sequence
// b attends to the first seq_lens[b] - q_len + t + 1 of them (causal inside the window), so
// it is a sequence of its own, v = b * q_len + t, on the same pages:
//     vbt[v * max_blocks + j] = block_table[b * max_blocks + j]
//     vlen[v]                 = max(0, seq_lens[b] - (q_len - 1 - t))
// B * q_len * max_blocks must fit in 63 bits; all pointers are device memory.
cudaError_t expand_multi_token(const int32_t* block_table, const int32_t* seq_lens, int B, int q_len,
                               int max_blocks, int32_t* vbt, int32_t* vlen, cudaStream_t s);

}  // namespace mla
