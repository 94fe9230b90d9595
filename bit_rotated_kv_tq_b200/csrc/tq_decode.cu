// tq_decode.cu -- split-K decode attention over the TQ4/4 cache and the
// log-sum-exp combine of the splits.
//
// Scores: H is symmetric and orthogonal, so <q, k_hat_t> = n_t <H q, C[idx_t]>.
// The query is rotated once (q~ = H q) and every score is formed in the
// rotated domain against the stored centroids; keys are never un-rotated.
// Values: v_hat = code * s + z per group of 32, so
//   o = sum_t p_t v_hat_t = sum_t (p_t s_t,g) code_t + sum_t p_t z_t,g.
//
// Work: one CTA per (split, kv head, sequence); 8 warps take the split's
// 16-token blocks round-robin.  Each warp streams its blocks' records (2336
// bytes at d=128, 1184 at d=64) through a private ring of shared-memory
// stages with bulk asynchronous copies (cp.async.bulk + mbarrier).  Per block
// every product runs on the tensor cores (mma.sync m16n8k16, fp32 accumulate):
//   q.K  A = 16 tokens x 16 dims of fp16 centroids, fetched two at a time
//        from a 256-entry byte -> (C[lo], C[hi]) table held once per lane
//        (conflict-free); B = q~ as fp16 high and low parts in adjacent
//        columns of the same head, so scores carry q~ to ~22 bits;
//   p.V  A = 16 dims x 16 tokens of value codes made exact fp16 integers by
//        a mask-and-bias nibble trick; B = p_t s_t,g as exact fp16 two-part
//        products (an fma two-product of the fp16 halves of p and the fp16
//        scale);
//   p.z  A = the fp16 zero points (exact), B = p as fp16 high and low parts.
// Softmax runs online in base 2 (scale * log2 e is folded into q~) and the
// accumulators are rescaled only when a running maximum moves.  Each split
// leaves an unnormalised partial (o, m, l) that the combine kernel merges; a
// single split writes the output directly.
#include "tq_kernels.cuh"

namespace tq {
namespace {

constexpr int kNW = 8;      // warps per CTA
constexpr int kStages = 3;  // records in flight per warp
constexpr int kLutWords = 256 * 32;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(phase)
        : "memory");
    return ok != 0;
}
// Wait for a phase of the barrier, giving up after ~2^31 clocks (about a second).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase) {
    if (mbar_try_wait(bar, phase)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, phase))
        if (clock64() - t0 > (1LL << 31)) return false;
    return true;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2^x for x <= 0 (softmax weights); the hardware approximation is accurate to
// ~2 ulp and flushes results below 2^-126 to zero.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// fp16 pair (x0 in the low half) and its rounding remainder as a second pair
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(x0, x1);
    const float2 f = __half22float2(h);
    hi = h2u(h);
    lo = h2u(__floats2half2_rn(x0 - f.x, x1 - f.y));
}

// (ph + pl) * s as a high part and a low part, all fp16 pairs:
//   hi = fl(ph * s); r = ph * s - hi is exact (fma two-product);
//   lo = fl(r + pl * s).  hi + lo equals p * s to ~2^-21 relative.
__device__ __forceinline__ void scaled_pair(uint32_t ph, uint32_t pl, uint32_t s, uint32_t& hi,
                                            uint32_t& lo) {
    const __half2 h = __hmul2(u2h(ph), u2h(s));
    const __half2 r = __hfma2(u2h(ph), u2h(s), __hneg2(h));
    hi = h2u(h);
    lo = h2u(__hfma2(u2h(pl), u2h(s), r));
}

// X holds the code bytes of two tokens in bytes 0 and 2.  Low nibbles ->
// exact fp16 pair (n0, n1); high nibbles -> exact fp16 pair (n0', n1').
// 0x6400 | n is the fp16 value 1024 + n; 0x6400 | (n << 4) is 1024 + 16 n.
__device__ __forceinline__ void value_pair(uint32_t X, uint32_t& lo_nib, uint32_t& hi_nib) {
    const uint32_t a = (X & 0x000F000Fu) | 0x64006400u;
    const uint32_t b = (X & 0x00F000F0u) | 0x64006400u;
    lo_nib = h2u(__hsub2(u2h(a), u2h(0x64006400u)));                    // - 1024
    hi_nib = h2u(__hfma2(u2h(b), u2h(0x2C002C00u), u2h(0xD400D400u)));  // / 16 - 64
}

// Table addresses (word indices (byte << 5) | lane) of the two low bytes of x.
__device__ __forceinline__ void lut_idx2(uint32_t x, uint32_t lane2, uint32_t& i0, uint32_t& i1) {
    const uint32_t t = __byte_perm(x, 0u, 0x4140u) * 32u + lane2;  // (b0, b1) in 16-bit halves
    i0 = t & 0xffffu;
    i1 = t >> 16;
}

template <int D, int GP>
__global__ void __launch_bounds__(kNW * 32, 2) decode_split_kernel(DecodeArgs a) {
    constexpr int KS = D / 16;   // k-steps of q.K
    constexpr int MT = D / 16;   // m-tiles of p.V
    constexpr int NG = D / 32;   // value groups
    constexpr int BPL = D / 8;   // key-code bytes per lane per token
    constexpr int VPL = D / 16;  // value-code bytes per lane per token
    constexpr int NT = GP / 4;   // n-tiles: 4 heads x (hi, lo) per tile
    constexpr int KW = BPL / 4;  // key-code words per lane per token
    constexpr int VW = VPL / 4;  // value-code words per lane per token
    constexpr int REC = Rec<D>::kBytes;
    using R = Rec<D>;

    __shared__ uint32_t lut[kLutWords];
    __shared__ float ctab[16];
    extern __shared__ __align__(128) unsigned char dsm[];
    constexpr size_t kRing = (size_t)kNW * kStages * REC;
    constexpr size_t kMerge = (size_t)kNW * GP * D * 4 + 2 * kNW * GP * 4;
    unsigned char* ring = dsm;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(dsm + (kRing > kMerge ? kRing : kMerge));
    float* qs = reinterpret_cast<float*>(mbar + kNW * kStages);  // [GP][D]
    float* ps = qs + GP * D;                                      // [NW][16][GP]
    float* pc = ps + kNW * 16 * GP;                               // [NW][GP]
    float* zs = pc + kNW * GP;                                    // [NW][NG][GP]

    const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int G = a.Hq / a.Hkv;

    int L = a.seq_lens[b];
    if (L < 0 || L > a.max_blocks * kBlock) {
        if (tid == 0 && split == 0 && kv == 0) flag_status(a.status, TQ_STATUS_BAD_LEN);
        L = 0;
    }
    if (L > a.num_splits * a.blocks_per_split * kBlock) {
        if (tid == 0 && split == 0 && kv == 0) flag_status(a.status, TQ_STATUS_BAD_LEN);
        L = a.num_splits * a.blocks_per_split * kBlock;
    }
    const int nblk = (L + kBlock - 1) / kBlock;
    const int jb = split * a.blocks_per_split;
    const int je = min(jb + a.blocks_per_split, nblk);
    const int nk = je - jb - warp > 0 ? (je - jb - warp + kNW - 1) / kNW : 0;

    // ---- per-warp copy ring
    const uint32_t bar0 = smem_u32(mbar + warp * kStages);
    const uint32_t ring0 = smem_u32(ring + (size_t)warp * kStages * REC);
    if (lane == 0) {
        for (int s = 0; s < kStages; s++) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();
    const int32_t* bt_row = a.block_tables + (size_t)b * a.max_blocks;
    auto load_id = [&](int k) { return k < nk ? bt_row[jb + warp + kNW * k] : -1; };
    int idA = load_id(lane), idB = load_id(32 + lane), kA = 0;
    auto get_id = [&](int k) {
        const int r = k - kA;
        const int x = __shfl_sync(kFull, idA, r & 31);
        const int y = __shfl_sync(kFull, idB, r & 31);
        return r < 32 ? x : y;
    };
    const unsigned char* cache_kv = a.cache + (size_t)kv * REC;
    auto issue = [&](int k, int id) {  // lane 0 only
        const uint32_t bar = bar0 + 8 * (k % kStages);
        if (id >= 0 && id < a.num_blocks) {
            fence_proxy_async();
            mbar_expect_tx(bar, REC);
            bulk_g2s(ring0 + (k % kStages) * REC, cache_kv + (size_t)id * a.Hkv * REC, REC, bar);
        } else {
            mbar_arrive(bar);
        }
    };
    for (int k = 0; k < kStages && k < nk; k++) {
        const int id = get_id(k);
        if (lane == 0) issue(k, id);
    }

    // ---- centroid table of this head
    const uint16_t* tab = a.k_tables ? a.k_tables + kv * 16 : a.default_table;
    if (tid < 16) ctab[tid] = half_bits_to_float(tab[tid]);
    // ---- rotate the queries of this kv head (heads >= G stay zero)
    {
        constexpr int EPL = D / 32;
        const float sc = a.scale_log2 * rsqrtf((float)D);
        for (int h = warp; h < GP; h += kNW) {
            float x[EPL];
            if (h < G) {
                const uint16_t* src = a.q + ((size_t)b * a.Hq + kv * G + h) * D + lane * EPL;
#pragma unroll
                for (int e = 0; e < EPL; e++) x[e] = __uint_as_float((uint32_t)src[e] << 16);
            } else {
#pragma unroll
                for (int e = 0; e < EPL; e++) x[e] = 0.f;
            }
#pragma unroll
            for (int m = 1; m < EPL; m <<= 1)
#pragma unroll
                for (int e = 0; e < EPL; e++)
                    if (!(e & m)) {
                        const float u = x[e], v = x[e | m];
                        x[e] = u + v;
                        x[e | m] = u - v;
                    }
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const bool upper = lane & m;
#pragma unroll
                for (int e = 0; e < EPL; e++) {
                    const float p = __shfl_xor_sync(kFull, x[e], m);
                    x[e] = upper ? p - x[e] : x[e] + p;
                }
            }
#pragma unroll
            for (int e = 0; e < EPL; e++) qs[h * D + lane * EPL + e] = x[e] * sc;
        }
    }
    __syncthreads();
    // ---- centroid pair table, one copy per lane: lut[(byte << 5) | lane]
    for (int e = tid; e < kLutWords; e += kNW * 32) {
        const int v = e >> 5;
        lut[e] = h2u(__floats2half2_rn(ctab[v & 15], ctab[v >> 4]));
    }

    // ---- query fragments (B of q.K).  Column n of tile t is head 4t + n/2,
    // its high fp16 part for even n and its low part for odd n; this lane
    // supplies column g.
    const bool hi_role = (g & 1) == 0;
    uint32_t bq[NT][KS][2];
#pragma unroll
    for (int t = 0; t < NT; t++) {
        const int h = 4 * t + (g >> 1);
#pragma unroll
        for (int ks = 0; ks < KS; ks++)
#pragma unroll
            for (int r = 0; r < 2; r++) {
                const int j = c * BPL + 2 * ks + r;  // key-code byte -> dims 2j, 2j+1
                uint32_t hi, lo;
                split_pair(qs[h * D + 2 * j], qs[h * D + 2 * j + 1], hi, lo);
                bq[t][ks][r] = hi_role ? hi : lo;
            }
    }
    __syncthreads();  // lut complete

    // ---- per-lane state.  Score / output layout: lane (g, c) holds head
    // 4t + c of tile t, tokens g and g + 8 (dims 2(8m + g), +1 of m-tile m).
    float mrun[NT], lrun[NT];
    float O[MT][NT][4];
    float Z[NT][4];  // p.z accumulator: rows = value groups (g < NG), head 4t + c
#pragma unroll
    for (int t = 0; t < NT; t++) {
        mrun[t] = -INFINITY;
        lrun[t] = 0.f;
#pragma unroll
        for (int i = 0; i < 4; i++) Z[t][i] = 0.f;
#pragma unroll
        for (int m = 0; m < MT; m++)
#pragma unroll
            for (int i = 0; i < 4; i++) O[m][t][i] = 0.f;
    }
    float* wps = ps + warp * 16 * GP;
    float* wpc = pc + warp * GP;
    const uint32_t lane2 = (uint32_t)lane | ((uint32_t)lane << 16);
    const int ph_head = g >> 1;  // this lane's B-fragment head within each tile
    bool aborted = false;
    int stage = 0;
    uint32_t phase = 0;

    for (int k = 0; k < nk; k++) {
        if (k - kA == 32) {  // next batch of block ids
            idA = idB;
            kA += 32;
            idB = load_id(kA + 32 + lane);
        }
        const int id = get_id(k);
        const bool ok = mbar_wait(bar0 + 8 * stage, phase);
        if (!__all_sync(kFull, ok)) {
            if (lane == 0) flag_status(a.status, TQ_STATUS_TIMEOUT);
            aborted = true;
            break;
        }
        if (id < 0 || id >= a.num_blocks) {
            if (lane == 0) flag_status(a.status, TQ_STATUS_BAD_BLOCK);
        } else {
            const unsigned char* rec = ring + (size_t)(warp * kStages + stage) * REC;
            const int nvalid = min(kBlock, L - (jb + warp + kNW * k) * kBlock);

            // -------- q.K: tokens g and g+8, this lane's BPL key-code bytes
            uint32_t kw0[KW], kw1[KW];
            {
                const unsigned char* krow0 = rec + R::kKCodes + g * (D / 2) + c * BPL;
                const unsigned char* krow1 = krow0 + 8 * (D / 2);
#pragma unroll
                for (int w = 0; w < KW; w += 2) {
                    const uint2 u0 = *reinterpret_cast<const uint2*>(krow0 + 4 * w);
                    const uint2 u1 = *reinterpret_cast<const uint2*>(krow1 + 4 * w);
                    kw0[w] = u0.x;
                    kw0[w + 1] = u0.y;
                    kw1[w] = u1.x;
                    kw1[w + 1] = u1.y;
                }
            }
            float acc[NT][4];
#pragma unroll
            for (int t = 0; t < NT; t++)
#pragma unroll
                for (int i = 0; i < 4; i++) acc[t][i] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ks++) {
                const int wi = ks >> 1, sh = (ks & 1) * 16;  // bytes 2ks, 2ks+1 of the chunk
                uint32_t i0, i2, i1, i3;
                lut_idx2(kw0[wi] >> sh, lane2, i0, i2);
                lut_idx2(kw1[wi] >> sh, lane2, i1, i3);
                const uint32_t a0 = lut[i0], a1 = lut[i1], a2 = lut[i2], a3 = lut[i3];
#pragma unroll
                for (int t = 0; t < NT; t++) mma16816(acc[t], a0, a1, a2, a3, bq[t][ks][0], bq[t][ks][1]);
            }
            const float n_a =
                half_bits_to_float(*reinterpret_cast<const uint16_t*>(rec + R::kKNorm + 2 * g));
            const float n_b = half_bits_to_float(
                *reinterpret_cast<const uint16_t*>(rec + R::kKNorm + 2 * (g + 8)));
            float sa[NT], sb[NT];  // scores of tokens g, g+8 for head 4t + c
#pragma unroll
            for (int t = 0; t < NT; t++) {
                sa[t] = (acc[t][0] + acc[t][1]) * n_a;
                sb[t] = (acc[t][2] + acc[t][3]) * n_b;
            }
            const bool partial = nvalid < kBlock;  // the last block of a sequence
            if (partial) {
#pragma unroll
                for (int t = 0; t < NT; t++) {
                    sa[t] = g < nvalid ? sa[t] : -INFINITY;
                    sb[t] = g + 8 < nvalid ? sb[t] : -INFINITY;
                }
            }

            // -------- online softmax
            bool grew = false;
            float corr[NT];
#pragma unroll
            for (int t = 0; t < NT; t++) {
                float x = fmaxf(sa[t], sb[t]);
#pragma unroll
                for (int m = 4; m < 32; m <<= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, m));
                const float mn = fmaxf(mrun[t], x);
                grew |= mn > mrun[t];
                corr[t] = ex2(mrun[t] - mn);
                mrun[t] = mn;
                sa[t] = ex2(sa[t] - mn);
                sb[t] = ex2(sb[t] - mn);
                lrun[t] = fmaf(lrun[t], corr[t], sa[t] + sb[t]);
            }
            if (__any_sync(kFull, grew)) {
#pragma unroll
                for (int t = 0; t < NT; t++) {
#pragma unroll
                    for (int i = 0; i < 4; i++) Z[t][i] *= corr[t];
#pragma unroll
                    for (int m = 0; m < MT; m++)
#pragma unroll
                        for (int i = 0; i < 4; i++) O[m][t][i] *= corr[t];
                }
            }
#pragma unroll
            for (int t = 0; t < NT; t++) {
                wps[g * GP + 4 * t + c] = sa[t];
                wps[(g + 8) * GP + 4 * t + c] = sb[t];
            }
            __syncwarp();

            // -------- B fragments of p (this lane: column g -> head 4t + g/2,
            // tokens 2c, 2c+1 and 2c+8, 2c+9), fp16 high and low parts
            const int t0 = 2 * c, t2 = 2 * c + 8;
            uint32_t bph[NT][2], bpl[NT][2];
#pragma unroll
            for (int t = 0; t < NT; t++) {
                const int h = 4 * t + ph_head;
                split_pair(wps[t0 * GP + h], wps[(t0 + 1) * GP + h], bph[t][0], bpl[t][0]);
                split_pair(wps[t2 * GP + h], wps[(t2 + 1) * GP + h], bph[t][1], bpl[t][1]);
            }
            // value groups (s, z) of tokens t0, t0+1, t2, t2+1; masked for a partial block
            const unsigned char* vg = rec + R::kVGroups;
            uint32_t sz[4][NG];
#pragma unroll
            for (int w = 0; w < NG; w += 2) {
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int tok = (u < 2 ? t0 : t2) + (u & 1);
                    const uint2 q2 = *reinterpret_cast<const uint2*>(vg + tok * NG * 4 + 4 * w);
                    sz[u][w] = q2.x;
                    sz[u][w + 1] = q2.y;
                }
            }
            if (partial) {
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const bool v = (u < 2 ? t0 : t2) + (u & 1) < nvalid;
#pragma unroll
                    for (int w = 0; w < NG; w++) sz[u][w] = v ? sz[u][w] : 0u;
                }
            }
            // -------- p.z: A rows = value groups (row g < NG), tokens as columns
            {
                uint32_t za0 = 0u, za2 = 0u;
#pragma unroll
                for (int w = 0; w < NG; w++)
                    if (g == w) {
                        za0 = __byte_perm(sz[0][w], sz[1][w], 0x7632u);  // (z_t0, z_t0+1)
                        za2 = __byte_perm(sz[2][w], sz[3][w], 0x7632u);
                    }
#pragma unroll
                for (int t = 0; t < NT; t++) {
                    mma16816(Z[t], za0, 0u, za2, 0u, hi_role ? bph[t][0] : bpl[t][0],
                             hi_role ? bph[t][1] : bpl[t][1]);
                }
            }
            // -------- p.V
            const unsigned char* vrow = rec + R::kVCodes + g * VPL;
            uint32_t cw[4][VW];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int tok = (u < 2 ? t0 : t2) + (u & 1);
#pragma unroll
                for (int w = 0; w < VW; w++)
                    cw[u][w] = *reinterpret_cast<const uint32_t*>(vrow + tok * (D / 2) + 4 * w);
            }
#pragma unroll
            for (int G_ = 0; G_ < NG; G_++) {
                const uint32_t s01 = __byte_perm(sz[0][G_], sz[1][G_], 0x5410u);  // (s_t0, s_t0+1)
                const uint32_t s23 = __byte_perm(sz[2][G_], sz[3][G_], 0x5410u);
                uint32_t b0[NT], b1[NT];
#pragma unroll
                for (int t = 0; t < NT; t++) {
                    uint32_t h0, l0, h1, l1;
                    scaled_pair(bph[t][0], bpl[t][0], s01, h0, l0);
                    scaled_pair(bph[t][1], bpl[t][1], s23, h1, l1);
                    b0[t] = hi_role ? h0 : l0;
                    b1[t] = hi_role ? h1 : l1;
                }
#pragma unroll
                for (int mm = 0; mm < 2; mm++) {
                    const int m = 2 * G_ + mm;
                    const int wi = m >> 2;
                    const uint32_t sel = (uint32_t)(m & 3) | ((uint32_t)(4 + (m & 3)) << 8);
                    uint32_t a0, a1, a2, a3;
                    value_pair(__byte_perm(cw[0][wi], cw[1][wi], sel), a0, a1);
                    value_pair(__byte_perm(cw[2][wi], cw[3][wi], sel), a2, a3);
#pragma unroll
                    for (int t = 0; t < NT; t++) mma16816(O[m][t], a0, a1, a2, a3, b0[t], b1[t]);
                }
            }
        }
        __syncwarp();
        const int kn = k + kStages;
        if (kn < nk) {
            const int idn = get_id(kn);
            if (lane == 0) issue(kn, idn);
        }
        if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
        }
    }
    if (aborted) {  // give copies still in flight a bounded chance to land
        for (int s = 0; s < kStages; s++) {
            mbar_wait(bar0 + 8 * s, 0);
            mbar_wait(bar0 + 8 * s, 1);
        }
    }

    // ---- finish this warp: l over tokens; z terms to shared memory
#pragma unroll
    for (int t = 0; t < NT; t++) {
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) lrun[t] += __shfl_xor_sync(kFull, lrun[t], m);
    }
    float* wzs = zs + warp * NG * GP;
    if (g < NG) {
#pragma unroll
        for (int t = 0; t < NT; t++) wzs[g * GP + 4 * t + c] = Z[t][0] + Z[t][1];
    }
    __syncthreads();  // every warp is done with its ring; zs is written

    float* red_o = reinterpret_cast<float*>(ring);  // [NW][GP][D]
    float* red_m = red_o + kNW * GP * D;            // [NW][GP]
    float* red_l = red_m + kNW * GP;                // [NW][GP]
#pragma unroll
    for (int t = 0; t < NT; t++) {
        const int h = 4 * t + c;
        if (g == 0) {
            red_m[warp * GP + h] = mrun[t];
            red_l[warp * GP + h] = lrun[t];
        }
#pragma unroll
        for (int m = 0; m < MT; m++) {
            const int dA = 2 * (8 * m + g);
            const float z = wzs[(m >> 1) * GP + h];
            red_o[(warp * GP + h) * D + dA] = O[m][t][0] + O[m][t][1] + z;
            red_o[(warp * GP + h) * D + dA + 1] = O[m][t][2] + O[m][t][3] + z;
        }
    }
    __syncthreads();

    // ---- merge the warps and write the split's partial (or the output)
    for (int idx = tid; idx < G * D; idx += kNW * 32) {
        const int h = idx / D, i = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kNW; w++) M = fmaxf(M, red_m[w * GP + h]);
        float o = 0.f, l = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kNW; w++) {
                const float f = ex2(red_m[w * GP + h] - M);
                o = fmaf(f, red_o[(w * GP + h) * D + i], o);
                l = fmaf(f, red_l[w * GP + h], l);
            }
        }
        const int hh = kv * G + h;
        if (a.num_splits == 1) {
            a.out[((size_t)b * a.Hq + hh) * D + i] = l > 0.f ? o / l : 0.f;
        } else {
            const size_t row = ((size_t)b * a.Hq + hh) * a.num_splits + split;
            a.ws_o[row * D + i] = o;
            if (i == 0) a.ws_ml[row] = make_float2(M, l);
        }
    }
}

// out[b][h] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s, M = max_s m_s.
template <int D>
__global__ void __launch_bounds__(D) combine_kernel(DecodeArgs a) {
    const int bh = blockIdx.x;
    const int i = threadIdx.x;
    const size_t row0 = (size_t)bh * a.num_splits;
    float M = -INFINITY;
    for (int s = 0; s < a.num_splits; s++) M = fmaxf(M, a.ws_ml[row0 + s].x);
    float o = 0.f, l = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < a.num_splits; s++) {
            const float2 ml = a.ws_ml[row0 + s];
            const float f = ex2(ml.x - M);
            o = fmaf(f, a.ws_o[(row0 + s) * D + i], o);
            l = fmaf(f, ml.y, l);
        }
    }
    a.out[(size_t)bh * D + i] = l > 0.f ? o / l : 0.f;
}

template <int D, int GP>
constexpr size_t decode_smem_bytes() {
    constexpr size_t ring = (size_t)kNW * kStages * Rec<D>::kBytes;
    constexpr size_t merge = (size_t)kNW * GP * D * 4 + 2 * kNW * GP * 4;
    return (ring > merge ? ring : merge) + kNW * kStages * 8 + GP * D * 4 + kNW * 16 * GP * 4 +
           kNW * GP * 4 + kNW * GP * (D / 32) * 4;
}

template <int D, int GP>
cudaError_t launch_dg(const DecodeArgs& a, cudaStream_t stream) {
    constexpr size_t smem = decode_smem_bytes<D, GP>();
    static bool configured = false;  // per instantiation; setting it twice is harmless
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, GP>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    dim3 grid(a.num_splits, a.Hkv, a.B);
    decode_split_kernel<D, GP><<<grid, kNW * 32, smem, stream>>>(a);
    if (a.num_splits > 1) combine_kernel<D><<<a.B * a.Hq, D, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, int head_dim, cudaStream_t stream) {
    const int G = a.Hq / a.Hkv;
    if (head_dim == 128) return G <= 4 ? launch_dg<128, 4>(a, stream) : launch_dg<128, 8>(a, stream);
    return G <= 4 ? launch_dg<64, 4>(a, stream) : launch_dg<64, 8>(a, stream);
}

}  // namespace tq
