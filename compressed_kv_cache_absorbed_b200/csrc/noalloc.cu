// Absorbed decode for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: an inference engine that hands every byte
// of the GPU to its own pool allocator at start-up, code running inside a region where
// allocation is forbidden (a stream being captured, a real-time loop that must not block
// on the driver's allocator), or a plugin host that gives its plugins no allocation
// callback.  mla_decode_absorbed needs a caller-provided workspace for its scratch (the
// absorbed queries, the split-KV partial results and the merged latent outputs); this
// entry point instead carves that scratch out of one fixed device array compiled into
// the library, so the caller passes only inputs and outputs.
#include <mutex>

#include "common.cuh"
#include "mla.h"

namespace {

// The fixed scratch.  Every GPU that loads this module holds it until the process exits.
__device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_scratch_addr[64];  // device address of g_noalloc_scratch, per device ordinal

// The array's name in host code is only a host-side stand-in; its device address is
// looked up once per device, with that device current.
mla_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (dev < 0 || dev >= 64) return MLA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MLA_OK;
}

}  // namespace

extern "C" mla_status mla_decode_absorbed_noalloc(const mla_dims* dims, mla_weights w,
                                                  const void* q_nope, const void* q_rope,
                                                  const void* h, const int32_t* q_pos,
                                                  const void* cache, int64_t cache_rows,
                                                  const int32_t* offsets, int32_t B, void* out,
                                                  mla_stream_t stream) {
    const size_t need = mla_decode_workspace_size(dims, B);
    if (need == 0 && B != 0) return mla_decode_absorbed(dims, w, q_nope, q_rope, h, q_pos, cache,
                                                        cache_rows, offsets, B, out, nullptr, 0, stream);
    if (need > (size_t)MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
    void* scratch = nullptr;
    mla_status st = scratch_address(&scratch);
    if (st != MLA_OK) return st;
    return mla_decode_absorbed(dims, w, q_nope, q_rope, h, q_pos, cache, cache_rows, offsets, B, out, scratch,
                               (size_t)MLA_NOALLOC_SCRATCH_BYTES, stream);
}
