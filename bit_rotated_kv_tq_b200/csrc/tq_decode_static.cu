// tq_decode_static.cu -- decode attention for callers that cannot allocate
// device memory.
//
// tq_decode_attention needs a caller-provided workspace for the partial
// results of its context splits.  Some callers have no way to provide one:
// a plugin or operator hosted by another runtime typically receives only the
// tensors of the call, and the host runtime owns every other byte of device
// memory (its own pool, no stray cudaMalloc allowed, or allocation is simply
// not reachable from that code).  This file gives them the same computation
// with the workspace taken from a fixed array compiled into the library.
//
// The array lives in device memory of every GPU that loads the library, for
// the life of the process, so it is kept small (kScratchBytes).  Its host-side
// name is only a stand-in for the symbol; the device address is looked up
// once per device with cudaGetSymbolAddress and cached.
#include <stdio.h>

#include <mutex>
#include <vector>

#include "tq_kernels.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;  // 8 MiB of split partials

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// Device address of g_decode_scratch on the current device (nullptr on error).
void* scratch_on_current_device(cudaError_t* err) {
    static std::mutex mu;
    static std::vector<void*> addr;
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if ((int)addr.size() <= dev) addr.resize(dev + 1, nullptr);
    if (!addr[dev]) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

TQ_API size_t tq_decode_static_scratch_bytes(void) { return kScratchBytes; }

TQ_API int tq_decode_attention_static(const void* q, const tq_cache_t* cache,
                                      const uint16_t* k_tables, const int32_t* block_tables,
                                      int max_blocks, const int32_t* seq_lens, int B, int H_q,
                                      int max_seq_len, float scale, float* out, int num_splits,
                                      int32_t* status, void* stream) {
    if (!cache || B < 0 || H_q <= 0 || num_splits < 0) {
        // let the full checks of tq_decode_attention report the problem
        return tq_decode_attention(q, cache, k_tables, block_tables, max_blocks, seq_lens, B, H_q,
                                   max_seq_len, scale, out, nullptr, 0, num_splits, status, stream);
    }
    const size_t need = tq_decode_workspace_bytes(B, H_q, cache->head_dim, num_splits);
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "tq_decode_attention_static: num_splits %d may need %zu bytes of partials, more "
                 "than the library's fixed %zu-byte scratch; pass 0 or fewer splits, or use "
                 "tq_decode_attention",
                 num_splits, need, kScratchBytes);
        return tq::set_last_error(TQ_ERR_WORKSPACE, msg);
    }
    cudaError_t e = cudaSuccess;
    void* ws = scratch_on_current_device(&e);
    if (!ws) {
        char msg[256];
        snprintf(msg, sizeof msg, "tq_decode_attention_static: scratch address lookup failed: %s",
                 cudaGetErrorString(e));
        return tq::set_last_error(TQ_ERR_CUDA, msg);
    }
    // Every partial slot is written by the split kernel before the combine reads
    // it, so nothing in the scratch has to start at zero; the bound above covers
    // the plan tq_decode_attention makes from the same num_splits.
    return tq_decode_attention(q, cache, k_tables, block_tables, max_blocks, seq_lens, B, H_q,
                               max_seq_len, scale, out, ws, kScratchBytes, num_splits, status,
                               stream);
}

}  // extern "C"
