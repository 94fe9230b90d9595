// tq_kernels.cuh -- argument blocks and launchers of the TQ4/4 kernels
// (internal to the library; the public interface is include/tq.h).
#pragma once

#include "tq_common.cuh"

namespace tq {

struct AppendArgs {
    const uint16_t* K;          // bf16 [T][Hkv][D]
    const uint16_t* V;          // bf16 [T][Hkv][D]
    const int32_t* block_table; // [num_seqs][max_blocks] or null
    int num_seqs, max_blocks;
    const int32_t* slots;       // [T]
    int T;
    unsigned char* cache;
    int num_blocks, Hkv;
    const uint16_t* k_tables;   // fp16 [Hkv][16] or null
    uint16_t default_table[16]; // fp16
    int32_t* status;
    uint64_t div_hkv, div_cap;  // fast-division multipliers (set by the launcher)
};

struct DecodeArgs {
    const uint16_t* q;           // bf16 [B][Hq][D]
    const unsigned char* cache;  // [num_blocks][Hkv][record]
    int num_blocks, Hkv, Hq, B;
    const uint16_t* k_tables;    // fp16 [Hkv][16] or null
    uint16_t default_table[16];  // fp16
    const int32_t* block_tables; // [B][max_blocks]
    int max_blocks;
    const int32_t* seq_lens;     // [B]
    float scale_log2;            // scale * log2(e)
    float* out;                  // [B][Hq][D]
    float* ws_o;                 // [ranges][2][4][D] partial outputs (unnormalised)
    float2* ws_ml;               // [ranges][2][4] (running max in log2 units, sum)
    int num_splits;              // 0: even cut over the grid; S: ranges of nmax/S blocks
    int max_seq_len;
    int32_t* status;
    // set by decode_plan
    int quads;            // groups of four query heads per kv head
    int items;            // B * Hkv * quads
    int nmax;             // blocks of the longest sequence (>= 1)
    int vrec;             // virtual records items x nmax (< 2^30)
    int R;                // records per range
    int nranges;
    uint64_t div_nmax, div_hkv, div_quads;  // fast_div multipliers
    uint32_t smem_bytes;  // dynamic shared memory of the split kernel
};

struct DequantArgs {
    const unsigned char* cache;
    int num_blocks, Hkv;
    const uint16_t* k_tables;   // fp16 [Hkv][16] or null
    uint16_t default_table[16];
    const int32_t* block_tables;
    int max_blocks;
    const int32_t* seq_lens;
    int B, max_len;
    float* K_hat;  // [B][max_len][Hkv][D]
    float* V_hat;
    int32_t* status;
};

size_t append_smem_bytes(int Hkv);
int set_last_error(int code, const char* msg);
cudaError_t launch_append(const AppendArgs& a, int head_dim, int num_sms, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, int head_dim, int num_sms, cudaStream_t stream);
uint32_t decode_smem_bytes(int head_dim);  // dynamic shared memory of the split kernel
bool decode_plan(DecodeArgs& a, int num_sms);            // ranges; false: too many
bool decode_needs_combine(const DecodeArgs& a);          // some item is cut by a range
size_t decode_workspace_for(const DecodeArgs& a, int head_dim);  // partials, bytes
cudaError_t launch_dequant(const DequantArgs& a, int head_dim, int num_sms, cudaStream_t stream);

}  // namespace tq
