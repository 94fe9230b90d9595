// tq_kernels.cuh -- argument blocks and launchers of the TQ4/4 kernels
// (internal to the library; the public interface is include/tq.h).
#pragma once

#include <math.h>

#include "tq_common.cuh"

namespace tq {

// ---- key binning of the append: uniform bins over y in [-1, 1] (a unit
// vector's rotated coordinates), width 1/64, bin = (int)(64 y + 64) in [0, 128]
constexpr int kBins = 129;
constexpr float kBinScale = 64.0f;
// Absolute margin, in rotated unit-vector units, inside which an fp32
// centroid decision is re-taken in fp64.  The fp32 butterfly of a bf16 key
// followed by one scaling is accurate to ~1.3e-6 in the worst case
// (7 stages, rsqrt within 2 ulp); typical errors are ~1e-7.
constexpr float kKeyMargin = 3.0e-6f;

struct HeadBins {
    float c[16];  // the head's table
    int dense;    // 1: some bin holds more than one midpoint -> exact count path
    int pad;      // keeps the BinEntry array that follows 8-byte aligned
};
struct __align__(8) BinEntry {
    float mid;  // the one midpoint inside the bin (with margins), or +inf
    int k_lo;   // number of midpoints strictly below the bin
};

// One bin of a strictly ascending 16-entry table c: the midpoints below the
// bin's range widened by 2 kKeyMargin on each side are counted by a binary
// search (the midpoints ascend too), and the one or more inside it follow.
// Returns true when more than one midpoint falls inside (the exact count path).
// The host (default table) and the device (per-head tables) both use it; the
// margins make the result insensitive to their float contraction differing.
__host__ __device__ inline bool bin_entry(const float* c, int bin, BinEntry& e) {
    const float delta = 2.0f * kKeyMargin;
    const float w = 1.0f / kBinScale;
    const float ext_lo = -1.0f + bin * w - delta;
    const float ext_hi = -1.0f + (bin + 1) * w + delta;
    int below = 0;  // #{k < 15 : m_k < ext_lo}, m_k = (c_k + c_k+1) / 2 (exact: fp16 values)
    for (int step = 8; step >= 1; step >>= 1) {
        const int k = below + step - 1;
        if (k < 15 && 0.5f * (c[k] + c[k + 1]) < ext_lo) below += step;
    }
    int inside = 0;
    float m_in = INFINITY;
    for (int k = below; k < 15; k++) {
        const float m = 0.5f * (c[k] + c[k + 1]);
        if (m > ext_hi) break;
        inside++;
        m_in = m;
    }
    e.mid = m_in;
    e.k_lo = below;
    return inside > 1;
}

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
    HeadBins default_hb;        // bins of default_table (set by the launcher)
    BinEntry default_bins[kBins];
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
