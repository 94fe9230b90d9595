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
// once per device with cudaGetSymbolAddress and cached.  A device reset
// (cudaDeviceReset, or anything else that destroys the primary context)
// unloads the module and leaves that cached address stale: a process that
// resets a device must not call tq_decode_attention_static on it afterwards.
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
    // every check of tq_decode_attention first, so a bad argument gets its own code
    tq::DecodeArgs a;
    size_t need = 0;
    const int err = tq::decode_prepare(q, cache, k_tables, block_tables, max_blocks, seq_lens, B,
                                       H_q, max_seq_len, scale, out, num_splits, status, a, need);
    if (err != TQ_OK || B == 0) return err;
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "tq_decode_attention_static: this split plan (num_splits %d) needs %zu bytes of "
                 "partials, more than the library's fixed %zu-byte scratch; pass fewer splits "
                 "(1 needs none) or use tq_decode_attention",
                 num_splits, need, kScratchBytes);
        return tq::set_last_error(TQ_ERR_WORKSPACE, msg);
    }
    void* ws = nullptr;
    if (need) {
        cudaError_t e = cudaSuccess;
        ws = scratch_on_current_device(&e);
        if (!ws) {
            char msg[256];
            snprintf(msg, sizeof msg, "tq_decode_attention_static: scratch address lookup failed: %s",
                     cudaGetErrorString(e));
            return tq::set_last_error(TQ_ERR_CUDA, msg);
        }
    }
    // Every partial slot the plan uses is written by the split kernel before the
    // combine reads it, so nothing in the scratch has to start at zero.
    return tq::decode_launch(a, cache->head_dim, ws, stream);
}

}  // extern "C"
