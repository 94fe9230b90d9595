// tq_bf16.cu -- the full-precision cache of the layers a model keeps unquantised:
// bf16 keys and values in 16-token blocks ("TurboQuant 在 AMD GPU 上把長上下文延遲壓下來",
// section 3: full-attention models leave the first and last layers unquantised,
// the layers most sensitive to KV quantisation).  The append, decode and
// dequantise calls of a TQ_CACHE_BF16 cache run here.
//
// Record of one (physical block, kv head): the 16 tokens' bf16 key rows [16][D],
// then their bf16 value rows [16][D] (64 D bytes: 8192 at D = 128, 4096 at D = 64),
// row r = token for keys, 16 + token for values.  Within a row the 16-byte chunks
// are stored swizzled: chunk j (elements 8j .. 8j+7) sits at chunk position
// j ^ (r mod 8).  A record then moves to shared memory with one bulk copy, and the
// 8-row ldmatrix reads of the decode (eight rows, one logical chunk) still hit
// eight different 16-byte bank groups.
//
// Decode (split-K flash decoding).  A CTA of four warps takes one item (sequence,
// kv head, group of up to eight query heads) and one of S ranges of the item's
// blocks; warp w takes the range's blocks w, w + 4, ...  A block's record comes
// in with one bulk copy into a stage of the warp's ring (swizzled as in the
// cache).  Per block, on mma.sync m16n8k16 with bf16 operands:
//   scores  S[token][head] = K q^T: A = key rows (ldmatrix), B = q (exact bf16,
//           one column per head);
//   output  O^T[dim][head] += V^T p^T: A = value rows transposed
//           (ldmatrix.trans), B = p in two bf16 parts, high and the remainder
//           (two mma into one accumulator: p to ~2^-16 relative).
// The softmax is online in base 2.  The four warps merge in shared memory; with
// S > 1 the CTA writes a partial (max, sum, unnormalised output) per query head
// and a combine kernel merges the S partials.
#include <mutex>

#include "tq_kernels.cuh"

namespace tq {
namespace {

constexpr int kBfWarps = 4;   // warps per CTA
constexpr int kBfStages = 3;  // blocks in flight per warp
constexpr int kBfHeads = 8;   // query heads per item (the mma's columns)

template <int D>
struct BfGeo {
    static constexpr uint32_t kRow = 2 * D;                          // stage row (as in the cache)
    static constexpr uint32_t kStage = 32 * kRow;                    // 16 key + 16 value rows
    static constexpr uint32_t kRec = 64 * D;                         // record bytes in the cache
    static constexpr uint32_t kRing = kBfWarps * kBfStages * kStage;
    static constexpr uint32_t kSmem = kRing + kBfWarps * kBfStages * 8;  // + one mbarrier per stage
    static constexpr int kMergeFloats = D / 4 + 4;                   // a lane's state: O, m, l
    static_assert(3u * 32u * kMergeFloats * 4u <= kRing, "merge buffer must fit in the ring");
};

__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(phase)
        : "memory");
    return ok != 0;
}
// Wait for a phase, giving up after ~2^31 clocks (about a second).
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t phase) {
    if (bar_try(bar, phase)) return true;
    const long long t0 = clock64();
    while (!bar_try(bar, phase))
        if (clock64() - t0 > (1LL << 31)) return false;
    return true;
}

__device__ __forceinline__ float ex2f(float x) {  // 2^x; -inf gives 0
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t a, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t bf2u(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

// ------------------------------------------------------------------ append
// One warp per (token, kv head): lanes 0 .. 2D/16 - 1 copy the key row, lanes 16 ..
// the value row, 16 bytes each.  Slots as for the TQ4/4 append.
template <int D>
__global__ void __launch_bounds__(256) bf16_append_kernel(AppendArgs a) {
    constexpr int LPR = 2 * D / 16;  // lanes per row
    const int lane = threadIdx.x & 31;
    const long long total = (long long)a.T * a.Hkv;
    const long long nwarps = (long long)gridDim.x * (blockDim.x / 32);
    for (long long v = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; v < total; v += nwarps) {
        const int t = (int)(v / a.Hkv), h = (int)(v % a.Hkv);
        const int slot = __ldg(a.slots + t);
        if (slot < 0) continue;
        int blk = -1;
        if (a.block_table) {
            const long long cap = (long long)a.max_blocks * kBlock;
            const long long seq = slot / cap, pos = slot % cap;
            if (seq >= a.num_seqs) {
                if (lane == 0) flag_status(a.status, TQ_STATUS_BAD_SLOT);
                continue;
            }
            const int pb = __ldg(a.block_table + seq * a.max_blocks + pos / kBlock);
            if (pb < 0 || pb >= a.num_blocks) {
                if (lane == 0) flag_status(a.status, TQ_STATUS_BAD_BLOCK);
                continue;
            }
            blk = pb;
        } else {
            if (slot / kBlock >= a.num_blocks) {
                if (lane == 0) flag_status(a.status, TQ_STATUS_BAD_SLOT);
                continue;
            }
            blk = slot / kBlock;
        }
        const int off = slot & (kBlock - 1);
        const int r = lane & 15;  // the 16-byte chunk this lane copies
        if (r < LPR) {
            const uint16_t* src = (lane < 16 ? a.K : a.V) + (size_t)v * D + 8 * r;
            // rows off and 16 + off share off mod 8, the chunks' swizzle
            unsigned char* dst = a.cache + ((size_t)blk * a.Hkv + h) * BfGeo<D>::kRec +
                                 (size_t)((lane < 16 ? 0 : kBlock) + off) * (2 * D) + 16 * (r ^ (off & 7));
            *reinterpret_cast<uint4*>(dst) = ld_stream_u4(src);
        }
    }
}

// ------------------------------------------------------------------ decode
template <int D>
__global__ void __launch_bounds__(kBfWarps * 32) bf16_decode_kernel(DecodeArgs a) {
    using Gm = BfGeo<D>;
    constexpr int KS = D / 16;  // k-steps of the scores = m-tiles of the output
    extern __shared__ __align__(128) unsigned char bsm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int S = a.bf_splits;
    const int s = (int)(blockIdx.x % (unsigned)S);
    const int item = (int)(blockIdx.x / (unsigned)S);
    const int hg = item % a.bf_hgroups, bk = item / a.bf_hgroups;
    const int kv = bk % a.Hkv, b = bk / a.Hkv;
    const int G = a.Hq / a.Hkv;
    const int h0 = kv * G + hg * kBfHeads;         // first query head of the item
    const int nh = min(kBfHeads, G - hg * kBfHeads);
    const bool reporter = threadIdx.x == 0 && s == 0 && kv == 0 && hg == 0;
    int L = a.seq_lens[b];
    if (L < 0 || L > a.max_blocks * kBlock) {
        if (reporter) flag_status(a.status, TQ_STATUS_BAD_LEN);
        L = 0;
    } else if (L > a.max_seq_len) {
        if (reporter) flag_status(a.status, TQ_STATUS_BAD_LEN);
        L = a.max_seq_len;
    }
    const int nblk = (L + kBlock - 1) / kBlock;
    const int j0 = (int)((long long)s * nblk / S), j1 = (int)((long long)(s + 1) * nblk / S);
    const int cnt = j1 - j0 > warp ? (j1 - j0 - warp + kBfWarps - 1) / kBfWarps : 0;

    const uint32_t ring = saddr(bsm) + (uint32_t)warp * kBfStages * Gm::kStage;
    const uint32_t bar0 = saddr(bsm) + Gm::kRing + (uint32_t)warp * kBfStages * 8;
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < kBfStages; i++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8 * i) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    const int32_t* bt = a.block_tables + (size_t)b * a.max_blocks;
    const unsigned char* kvbase = a.cache + (size_t)kv * Gm::kRec;
    const size_t blk_stride = (size_t)a.Hkv * Gm::kRec;
    // Copy this warp's k-th block's record into stage k % kBfStages (one bulk copy);
    // a block id outside the cache brings nothing, and the consumer counts it empty.
    auto issue = [&](int k) {
        if (k >= cnt) return;
        const int pb = __ldg(bt + j0 + warp + kBfWarps * k);
        const bool ok = (uint32_t)pb < (uint32_t)a.num_blocks;
        const uint32_t st = ring + (uint32_t)(k % kBfStages) * Gm::kStage;
        const uint32_t bar = bar0 + 8u * (uint32_t)(k % kBfStages);
        if (lane == 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            if (ok)
                asm volatile(
                    "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n"
                    "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%2], [%3], %1, [%0];"
                    ::"r"(bar), "r"(Gm::kRec), "r"(st), "l"(kvbase + (size_t)pb * blk_stride)
                    : "memory");
            else
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
        }
    };
#pragma unroll 1
    for (int k = 0; k < kBfStages; k++) issue(k);

    // q as the B operand of the scores: column g is head h0 + g (zero past the
    // item's heads); k-step ks takes dims 16 ks + 2c, +1 and 16 ks + 2c + 8, +9
    uint32_t qb[KS][2];
    {
        const bool hv = g < nh;
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(a.q + ((size_t)b * a.Hq + h0 + (hv ? g : 0)) * D);
#pragma unroll
        for (int ks = 0; ks < KS; ks++) {
            qb[ks][0] = hv ? __ldg(qrow + 8 * ks + c) : 0u;
            qb[ks][1] = hv ? __ldg(qrow + 8 * ks + c + 4) : 0u;
        }
    }
    const float sl = a.scale_log2;
    // per lane: heads 2c, 2c + 1 (the mma's columns); O[m] rows = dims 16 m + g, + 8
    float O[KS][4];
#pragma unroll
    for (int m = 0; m < KS; m++) O[m][0] = O[m][1] = O[m][2] = O[m][3] = 0.f;
    float mrun0 = -INFINITY, mrun1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    // weight sources of the p.V operand: tokens 2c (+8) and 2c + 1 (+9) of head g
    const int sA = 8 * c + (g >> 1), sB = sA + 4;
    const bool odd = g & 1;
    // ldmatrix rows of this lane: key row lane % 16, logical chunk 2 ks + lane / 16;
    // value row 16 + lane % 8 + 8 (lane / 16), logical chunk 2 m + (lane / 8) % 2;
    // a chunk's position is its index xor (row mod 8), and row mod 8 = lane mod 8
    const uint32_t krow = (uint32_t)(lane & 15) * Gm::kRow, kx = (uint32_t)(lane & 7), kh = (uint32_t)(lane >> 4);
    const uint32_t vrow = (uint32_t)(16 + (lane & 7) + 8 * (lane >> 4)) * Gm::kRow, vh = (uint32_t)((lane >> 3) & 1);

    int k = 0, issued = min(cnt, kBfStages);
    bool aborted = false;
#pragma unroll 1
    for (; k < cnt; k++) {
        const uint32_t bar = bar0 + 8u * (uint32_t)(k % kBfStages);
        if (!__all_sync(kFull, bar_wait(bar, (uint32_t)(k / kBfStages) & 1u))) {
            if (lane == 0) flag_status(a.status, TQ_STATUS_TIMEOUT);
            aborted = true;
            break;
        }
        const int j = j0 + warp + kBfWarps * k;
        const int pb = __ldg(bt + j);
        const bool ok = (uint32_t)pb < (uint32_t)a.num_blocks;
        if (!ok && lane == 0) flag_status(a.status, TQ_STATUS_BAD_BLOCK);
        const int n = ok ? min(kBlock, L - kBlock * j) : 0;
        if (n > 0) {
            const uint32_t st = ring + (uint32_t)(k % kBfStages) * Gm::kStage;
            if (n < kBlock) {
                // a sequence's last block: its value rows past the length hold whatever
                // the cache held there (a NaN times a zero weight is still NaN), so
                // they are zeroed; the scores of those rows are masked below
                constexpr int C16 = 2 * D / 16;
                for (int i = lane; i < (kBlock - n) * C16; i += 32)
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(
                                     st + (uint32_t)(kBlock + n + i / C16) * Gm::kRow + 16u * (i % C16)),
                                 "r"(0u)
                                 : "memory");
                __syncwarp();
            }
            // -------- scores of tokens g, g + 8 for heads 2c, 2c + 1
            float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < KS; ks++) {
                uint32_t af[4];
                ldsm_x4(st + krow + 16u * (((uint32_t)(2 * ks) + kh) ^ kx), af);
                mma_bf16(sc, af, qb[ks][0], qb[ks][1]);
            }
            const bool va = g < n, vb = g + 8 < n;
            const float x0 = va ? sc[0] * sl : -INFINITY, x1 = va ? sc[1] * sl : -INFINITY;
            const float x2 = vb ? sc[2] * sl : -INFINITY, x3 = vb ? sc[3] * sl : -INFINITY;
            float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
            for (int m = 4; m < 32; m <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, m));
                mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, m));
            }
            // token 0 of the block is valid, so the new maxima are finite
            const float mn0 = fmaxf(mrun0, mx0), mn1 = fmaxf(mrun1, mx1);
            const float c0 = ex2f(mrun0 - mn0), c1 = ex2f(mrun1 - mn1);
            mrun0 = mn0;
            mrun1 = mn1;
#pragma unroll
            for (int m = 0; m < KS; m++) {
                O[m][0] *= c0;
                O[m][2] *= c0;
                O[m][1] *= c1;
                O[m][3] *= c1;
            }
            const float p0 = ex2f(x0 - mn0), p1 = ex2f(x1 - mn1), p2 = ex2f(x2 - mn0), p3 = ex2f(x3 - mn1);
            l0 = fmaf(l0, c0, p0 + p2);
            l1 = fmaf(l1, c1, p1 + p3);
            // -------- the p.V operand: head g at tokens 2c, 2c + 1 | 2c + 8, 2c + 9
            const float e0 = __shfl_sync(kFull, p0, sA), o0 = __shfl_sync(kFull, p1, sA);
            const float e1 = __shfl_sync(kFull, p0, sB), o1 = __shfl_sync(kFull, p1, sB);
            const float e2 = __shfl_sync(kFull, p2, sA), o2 = __shfl_sync(kFull, p3, sA);
            const float e3 = __shfl_sync(kFull, p2, sB), o3 = __shfl_sync(kFull, p3, sB);
            const float t0 = odd ? o0 : e0, t1 = odd ? o1 : e1, t2 = odd ? o2 : e2, t3 = odd ? o3 : e3;
            const __nv_bfloat162 h01 = __floats2bfloat162_rn(t0, t1), h23 = __floats2bfloat162_rn(t2, t3);
            const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
            const uint32_t bh0 = bf2u(h01), bh1 = bf2u(h23);
            const uint32_t bl0 = bf2u(__floats2bfloat162_rn(t0 - f01.x, t1 - f01.y));
            const uint32_t bl1 = bf2u(__floats2bfloat162_rn(t2 - f23.x, t3 - f23.y));
            // -------- output += V^T p^T
#pragma unroll
            for (int m = 0; m < KS; m++) {
                uint32_t af[4];
                ldsm_x4_t(st + vrow + 16u * (((uint32_t)(2 * m) + vh) ^ kx), af);
                mma_bf16(O[m], af, bh0, bh1);
                mma_bf16(O[m], af, bl0, bl1);
            }
        }
        __syncwarp();
        issue(k + kBfStages);
        if (k + kBfStages < cnt) issued++;
    }
    if (aborted) {  // give the copies still in flight a bounded chance to land
#pragma unroll 1
        for (int i = k; i < issued; i++)
            bar_wait(bar0 + 8u * (uint32_t)(i % kBfStages), (uint32_t)(i / kBfStages) & 1u);
    }
    // sums of weights over the 16 token rows of the fragments
#pragma unroll
    for (int m = 4; m < 32; m <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, m);
        l1 += __shfl_xor_sync(kFull, l1, m);
    }

    // ---- merge the four warps (their rings are free now) in warp 0
    __syncthreads();
    float* mb = reinterpret_cast<float*>(bsm);
    constexpr int MF = Gm::kMergeFloats;
    if (warp > 0) {
        float* p = mb + ((warp - 1) * 32 + lane) * MF;
#pragma unroll
        for (int m = 0; m < KS; m++)
#pragma unroll
            for (int i = 0; i < 4; i++) p[4 * m + i] = O[m][i];
        p[4 * KS] = mrun0;
        p[4 * KS + 1] = mrun1;
        p[4 * KS + 2] = l0;
        p[4 * KS + 3] = l1;
    }
    __syncthreads();
    if (warp != 0) return;
#pragma unroll 1
    for (int w = 0; w < kBfWarps - 1; w++) {
        const float* p = mb + (w * 32 + lane) * MF;
        const float pm0 = p[4 * KS], pm1 = p[4 * KS + 1];
        const float M0 = fmaxf(mrun0, pm0), M1 = fmaxf(mrun1, pm1);
        // a side that saw no token (maximum -inf) contributes nothing
        const float fa0 = mrun0 == -INFINITY ? 0.f : ex2f(mrun0 - M0);
        const float fb0 = pm0 == -INFINITY ? 0.f : ex2f(pm0 - M0);
        const float fa1 = mrun1 == -INFINITY ? 0.f : ex2f(mrun1 - M1);
        const float fb1 = pm1 == -INFINITY ? 0.f : ex2f(pm1 - M1);
#pragma unroll
        for (int m = 0; m < KS; m++) {
            O[m][0] = fmaf(fb0, p[4 * m], fa0 * O[m][0]);
            O[m][2] = fmaf(fb0, p[4 * m + 2], fa0 * O[m][2]);
            O[m][1] = fmaf(fb1, p[4 * m + 1], fa1 * O[m][1]);
            O[m][3] = fmaf(fb1, p[4 * m + 3], fa1 * O[m][3]);
        }
        l0 = fmaf(fb0, p[4 * KS + 2], fa0 * l0);
        l1 = fmaf(fb1, p[4 * KS + 3], fa1 * l1);
        mrun0 = M0;
        mrun1 = M1;
    }
    // ---- the output (one range) or this range's partial, heads 2c and 2c + 1
#pragma unroll
    for (int e = 0; e < 2; e++) {
        const int hq = 2 * c + e;
        if (hq >= nh) continue;
        const int hh = h0 + hq;
        const float l = e ? l1 : l0, mr = e ? mrun1 : mrun0;
        if (S == 1) {
            float* dst = a.out + ((size_t)b * a.Hq + hh) * D + g;
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int m = 0; m < KS; m++) {
                dst[16 * m] = O[m][e] * inv;
                dst[16 * m + 8] = O[m][2 + e] * inv;
            }
        } else {
            const size_t pr = ((size_t)b * a.Hq + hh) * S + s;
            float* dst = a.ws_o + pr * D + g;
#pragma unroll
            for (int m = 0; m < KS; m++) {
                dst[16 * m] = O[m][e];
                dst[16 * m + 8] = O[m][2 + e];
            }
            if (g == 0) a.ws_ml[pr] = make_float2(mr, l);
        }
    }
}

// Merge the S partials of each (sequence, query head): one warp each.
template <int D>
__global__ void __launch_bounds__(32) bf16_combine_kernel(DecodeArgs a) {
    constexpr int DPL = D / 32;
    const int lane = threadIdx.x;
    const int S = a.bf_splits;
#pragma unroll 1
    for (int bh = blockIdx.x; bh < a.B * a.Hq; bh += gridDim.x) {
        float M = -INFINITY, l = 0.f, o[DPL];
#pragma unroll
        for (int j = 0; j < DPL; j++) o[j] = 0.f;
#pragma unroll 1
        for (int s = 0; s < S; s++) {
            const size_t pr = (size_t)bh * S + s;
            const float2 ml = a.ws_ml[pr];
            if (ml.x == -INFINITY) continue;  // the range saw no token
            const float Mn = fmaxf(M, ml.x);
            const float f0 = M == -INFINITY ? 0.f : ex2f(M - Mn), f1 = ex2f(ml.x - Mn);
#pragma unroll
            for (int j = 0; j < DPL; j++) o[j] = fmaf(f1, a.ws_o[pr * D + j * 32 + lane], f0 * o[j]);
            l = fmaf(f1, ml.y, f0 * l);
            M = Mn;
        }
#pragma unroll
        for (int j = 0; j < DPL; j++) a.out[(size_t)bh * D + j * 32 + lane] = l > 0.f ? o[j] / l : 0.f;
    }
}

// ------------------------------------------------------------------ dequantise
// The rows as fp32 [B][max_len][Hkv][D]; rows at or past a length are 0.
template <int D>
__global__ void __launch_bounds__(256) bf16_dequant_kernel(DequantArgs a) {
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long total = (long long)a.B * a.max_len * a.Hkv;
    const long long nwarps = (long long)gridDim.x * (blockDim.x / 32);
    for (long long v = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; v < total; v += nwarps) {
        const int h = (int)(v % a.Hkv);
        const long long bt = v / a.Hkv;
        const int t = (int)(bt % a.max_len), b = (int)(bt / a.max_len);
        int L = a.seq_lens[b];
        if (L < 0 || L > a.max_blocks * kBlock) {
            if (lane == 0 && t == 0 && h == 0) flag_status(a.status, TQ_STATUS_BAD_LEN);
            L = 0;
        }
        const unsigned char* rec = nullptr;
        if (t < L) {
            const int pb = a.block_tables[(size_t)b * a.max_blocks + t / kBlock];
            if (pb >= 0 && pb < a.num_blocks)
                rec = a.cache + ((size_t)pb * a.Hkv + h) * BfGeo<D>::kRec;
            else if (lane == 0)
                flag_status(a.status, TQ_STATUS_BAD_BLOCK);
        }
        float* kd = a.K_hat + (size_t)v * D + lane * EPL;
        float* vd = a.V_hat + (size_t)v * D + lane * EPL;
#pragma unroll
        for (int e = 0; e < EPL; e++) {
            float kx = 0.f, vx = 0.f;
            if (rec) {
                const int i = lane * EPL + e, pos = (((i >> 3) ^ (t & 7)) << 3) | (i & 7);  // swizzled chunk
                const uint16_t* kr = reinterpret_cast<const uint16_t*>(rec) + (t % kBlock) * D;
                const uint16_t* vr = kr + kBlock * D;
                kx = __uint_as_float((uint32_t)kr[pos] << 16);
                vx = __uint_as_float((uint32_t)vr[pos] << 16);
            }
            kd[e] = kx;
            vd[e] = vx;
        }
    }
}

template <int D>
cudaError_t launch_d(const DecodeArgs& a, cudaStream_t stream) {
    static std::mutex mu;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (dev < 0 || dev >= 64 || !configured[dev]) {
            e = cudaFuncSetAttribute(bf16_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)BfGeo<D>::kSmem);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) configured[dev] = true;
        }
    }
    const long long grid = (long long)a.B * a.Hkv * a.bf_hgroups * a.bf_splits;
    bf16_decode_kernel<D><<<(unsigned)grid, kBfWarps * 32, BfGeo<D>::kSmem, stream>>>(a);
    if (a.bf_splits > 1) bf16_combine_kernel<D><<<a.B * a.Hq, 32, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bf16_append(const AppendArgs& a, int head_dim, int num_sms, cudaStream_t stream) {
    const long long warps = (long long)a.T * a.Hkv;
    long long blocks = (warps + 7) / 8;
    if (blocks > (long long)num_sms * 8) blocks = (long long)num_sms * 8;
    if (blocks < 1) blocks = 1;
    if (head_dim == 128)
        bf16_append_kernel<128><<<(unsigned)blocks, 256, 0, stream>>>(a);
    else
        bf16_append_kernel<64><<<(unsigned)blocks, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_bf16_decode(const DecodeArgs& a, int head_dim, cudaStream_t stream) {
    return head_dim == 128 ? launch_d<128>(a, stream) : launch_d<64>(a, stream);
}

cudaError_t launch_bf16_dequant(const DequantArgs& a, int head_dim, int num_sms, cudaStream_t stream) {
    const long long warps = (long long)a.B * a.max_len * a.Hkv;
    long long blocks = (warps + 7) / 8;
    if (blocks > (long long)num_sms * 8) blocks = (long long)num_sms * 8;
    if (blocks < 1) blocks = 1;
    if (head_dim == 128)
        bf16_dequant_kernel<128><<<(unsigned)blocks, 256, 0, stream>>>(a);
    else
        bf16_dequant_kernel<64><<<(unsigned)blocks, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace tq
