// tq_kernels.cuh -- argument blocks and launchers of the TQ4/4 kernels
// (internal to the library; the public interface is include/tq.h).
#pragma once

#include <math.h>

#include "tq_common.cuh"

namespace tq {

// ---- key binning of the append.  A rotated unit-vector coordinate y in
// [-1, 1] is mapped to x = S y + S + 1 (S = kBinScale) and rounded to 1/8 by
// one fma against kBinMagic = 2^20 + S + 1 (floats in [2^20, 2^21) are spaced
// 1/8 apart); bits 3-9 of the result are then bin * 8 with bin = floor(x) mod
// 128, in [0, 127] for |y| <= 1.  Bin b is taken to cover x in
// [b - 1/8, b + 1 + 1/8] (the rounding to 1/8 and the fp32 error of x stay
// inside that slack), widened further by 2 kKeyMargin in y.
constexpr int kBins = 128;
constexpr float kBinScale = 63.0f;
constexpr float kBinMagic = 1048576.0f + kBinScale + 1.0f;
// Absolute margin, in rotated unit-vector units, inside which an fp32
// centroid decision is re-taken exactly.  The fp32 butterfly of a bf16 key
// (L <= 7 rounding stages; stage s adds rounding errors of 2-norm at most
// 2^-24 of its output, and the later stages scale them with the vector)
// errs by at most L 2^-24 in unit-vector units, and the normalisation by at
// most 10 ulp of |y| <= 1, so the fast path's y is within 17 ulp (1.0e-6) of
// the exact one; the margin is twice that.
constexpr float kKeyMargin = 2.0e-6f;

struct HeadBins {
    float c[16];  // the head's table
    int dense;    // 1: some bin holds more than one midpoint -> exact count path
    int pad;
};
struct __align__(8) BinEntry {
    float mid;  // the one midpoint inside the bin (with margins), or +inf
    int k_lo;   // the number of midpoints strictly below the bin (the code below its midpoint)
};

// One bin of a strictly ascending 16-entry table c: the midpoints below the
// bin's widened range are counted by a binary search (the midpoints ascend
// too), and the one or more inside it follow.  Returns true when more than
// one midpoint falls inside (the exact count path).  The host (default table)
// and the device (per-head tables) both use it; the margins make the result
// insensitive to their float contraction differing.
__host__ __device__ inline bool bin_entry(const float* c, int bin, BinEntry& e) {
    const float delta = 2.0f * kKeyMargin;
    const float ext_lo = ((float)bin - 1.125f - kBinScale) / kBinScale - delta;
    const float ext_hi = ((float)bin + 0.125f - kBinScale) / kBinScale + delta;
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
    int rotate;                 // 1: keys rotated (the TQ4/4 format); 0: TQ_CACHE_UNROTATED
    Div32 dv_hkv, dv_cap;       // division by H_kv and by max_blocks * 16 (set by the launcher)
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
    int rotate;                  // 0: TQ_CACHE_UNROTATED (the query is not rotated)
    int bf16;                    // 1: a TQ_CACHE_BF16 cache (the bf16 kernels and plan)
    int bf_splits, bf_hgroups;   // bf16 plan: ranges per item, items of <= 8 heads per kv head
    // set by decode_plan
    int qpi;              // groups of four query heads per item (1, or 2 at d = 64 with G > 4)
    int quads;            // items per kv head
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
    int rotate;    // 0: TQ_CACHE_UNROTATED (no inverse rotation)
};

// Host checks and split plan of a decode call (the checks of tq_decode_attention
// except the workspace ones); on TQ_OK with B > 0, `need` is the plan's workspace.
int decode_prepare(const void* q, const tq_cache_t* cache, const uint16_t* k_tables,
                   const int32_t* block_tables, int max_blocks, const int32_t* seq_lens, int B,
                   int H_q, int max_seq_len, float scale, float* out, int num_splits,
                   int32_t* status, DecodeArgs& a, size_t& need);
int decode_launch(DecodeArgs& a, int head_dim, void* workspace, void* stream);
size_t append_smem_bytes(int ntab, int head_dim);  // ntab bin tables (1, or H_kv per-head tables)
int set_last_error(int code, const char* msg);
cudaError_t launch_append(const AppendArgs& a, int head_dim, int num_sms, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, int head_dim, int num_sms, cudaStream_t stream);
uint32_t decode_smem_bytes(int head_dim);  // dynamic shared memory of the split kernel
bool decode_plan(DecodeArgs& a, int head_dim, int num_sms);  // ranges; false: too many
bool decode_needs_combine(const DecodeArgs& a);          // some item is cut by a range
size_t decode_workspace_for(const DecodeArgs& a, int head_dim);  // partials, bytes
cudaError_t launch_dequant(const DequantArgs& a, int head_dim, int num_sms, cudaStream_t stream);
// the full-precision (TQ_CACHE_BF16) cache
cudaError_t launch_bf16_append(const AppendArgs& a, int head_dim, int num_sms, cudaStream_t stream);
cudaError_t launch_bf16_decode(const DecodeArgs& a, int head_dim, cudaStream_t stream);
cudaError_t launch_bf16_dequant(const DequantArgs& a, int head_dim, int num_sms, cudaStream_t stream);
cudaError_t launch_prefill(const void* q, const unsigned char* cache, int num_blocks, int Hkv, int Hq, int B,
                           const uint16_t* k_tables, const uint16_t* default_table,
                           const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                           const int32_t* q_start, int T, int max_q_len, float scale, float* out,
                           int32_t* status, int head_dim, int rotate, cudaStream_t stream);
size_t prefill_smem_bytes(int head_dim);

}  // namespace tq
