// tq_append.cu -- the TQ4/4 write path: rotate, quantise and pack new tokens
// into the paged cache.
//
// Keys ("TurboQuant 在 AMD GPU 上把長上下文延遲壓下來", sections 2 and 4;
// "UltraQuant：4-bit KV 快取加速長代理", 「方法怎麼做，白話講」):
//   n = ||k||, stored as fp16;  y = H_d k / n with H_d the normalised
//   Sylvester-Hadamard matrix;  idx_i = nearest entry of the 16-level table
//   (ties to the lower index);  two 4-bit indices per byte.
// Values (section 2, uniform quantisation), per group of 32:
//   z = fp16 rounded down from min, s = fp16 rounded up from (max - z)/15,
//   q = round-half-even((v - z)/s) in [0, 15].
//
// Work split: one vector (token, kv head) is spread over D/32 lanes holding 32
// consecutive elements each (one value group per lane), so a warp pass covers
// 16 (D=64) or 8 (D=128) vectors, 2 KB of keys and 2 KB of values.  The grid
// is persistent (one CTA per SM); each CTA takes an even share of the passes
// and deals them to its warps, and each warp streams its passes' keys and
// values through a private ring of shared-memory stages filled by bulk copies
// (one mbarrier per stage).  The rotation is an in-register butterfly over the
// 5 element bits inside a lane plus xor-shuffles over the lane bits.  Decisions
// inside their error margin are flagged per element pair in the main loop and
// taken again afterwards by short loops over the flagged pairs only (the code
// of the main loop stays small enough for the instruction cache).
//
// Nearest centroid: x = 63 y + 64 is rounded to 1/8 by one fma against a
// 2^20 magic constant, whose low mantissa bits then address a 128-entry bin
// table in shared memory (1 KB per table).  A bin holds at most one midpoint
// of the default tables; its entry gives that midpoint and the count of
// midpoints below, and the code is that count plus one fp32 comparison.
// Tables with closer midpoints take an exact count over all 15 midpoints.
//
// Exactness: the fast path runs in fp32.  Every decision it takes is
// re-taken exactly whenever the fp32 input lies inside the fp32 error bound
// of the decision threshold: the fp16 rounding of the norm and the nearest
// centroid in fp64 from the bf16 inputs (exact +-1 Hadamard sums, compared
// against midpoint * n * sqrt(D)), the value codes by comparing v - z with
// (k + 1/2) s in fp64, and the fp16 rounding up of the scale by an exact fp32
// comparison of 15 s with max - z (fp64 when max - z is inexact in fp32).  The
// stored codes are therefore those of the exact-arithmetic definition except
// within ~1e-15 (relative) of a key threshold.
#include <mutex>

#include "tq_kernels.cuh"

namespace tq {

// Relative margin on the norm before its fp16 rounding: twice the error bound
// of the fast path's norm (fp32 sum of exact squares along a tree of depth
// <= 8, then ss * rsqrt with one Newton step: <= 9 ulp).
constexpr float kNormMargin = 1.1e-6f;
// Margin, in value-code units, around the .5 rounding points of (v - z)/s:
// the fp32 residual v - z - t s errs by at most 16 ulp of s (v - z rounded
// once, the fused residual once), far inside 2^-16.
constexpr float kValueMargin = 1.0f / 65536.0f;

// Bin tables in shared memory (called by the whole CTA): the tables sit at
// the start of the dynamic shared memory, 1 KB each, the HeadBins after them.
// Without per-head tables every head uses the default table, whose bins the
// launcher computed once on the host: they are copied, and every head
// indexes them as head 0.  Per-head tables are binned here.
__device__ void build_bins(HeadBins* hb, BinEntry* bins, const AppendArgs& a) {
    if (!a.k_tables) {
        for (int e = threadIdx.x; e < kBins; e += blockDim.x) bins[e] = a.default_bins[e];
        if (threadIdx.x == 0) hb[0] = a.default_hb;
        __syncthreads();
        return;
    }
    for (int h = threadIdx.x; h < a.Hkv; h += blockDim.x) {
        for (int k = 0; k < 16; k++) hb[h].c[k] = half_bits_to_float(a.k_tables[16 * h + k]);
        hb[h].dense = 0;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.Hkv * kBins; e += blockDim.x) {
        const int h = e / kBins, bin = e % kBins;
        if (bin_entry(hb[h].c, bin, bins[e])) hb[h].dense = 1;  // benign race: all store 1
    }
    __syncthreads();
}

__device__ __forceinline__ float rsqrt_approx(float x) {  // x normal and positive
    float y;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {  // x normal
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// four bytes (the low byte of each argument) into one word
__device__ __forceinline__ uint32_t pack4(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// 1/15 rounded down to fp32
__device__ __forceinline__ float inv15_dn() { return __uint_as_float(0x3d888888u); }

constexpr int kAppWarps = 16;   // warps per CTA (one persistent CTA per SM)
constexpr int kAppStages = 3;   // passes in flight per warp

template <int D>
struct Geo {
    static constexpr int LPV = D / 32;    // lanes per vector (one value group each)
    static constexpr int VPW = 32 / LPV;  // vectors per warp pass
    static constexpr uint32_t kPass = VPW * D * 2;  // bytes of one pass's keys (or values)
    static constexpr uint32_t kStage = 2 * kPass;   // a ring stage: keys, then values
};

// ---- shared-memory helpers of the input ring
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
// the 32 bf16 elements (16 words) at a stage address
__device__ __forceinline__ void lds_32(uint32_t a, uint32_t (&w)[16]) {
#pragma unroll
    for (int c = 0; c < 4; c++) {
        const uint4 t = lds_u4(a + 16 * c);
        w[4 * c] = t.x;
        w[4 * c + 1] = t.y;
        w[4 * c + 2] = t.z;
        w[4 * c + 3] = t.w;
    }
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t phase) {
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
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t phase) {
    if (mbar_try(bar, phase)) return true;
    const long long t0 = clock64();
    while (!mbar_try(bar, phase))
        if (clock64() - t0 > (1LL << 31)) return false;
    return true;
}

// The pass-level bookkeeping of one warp pass (its inputs sit in a ring stage).
struct Pass {
    int slot;      // slot_mapping entry of the token (-1: skip)
    int pb;        // physical block read from the block table (when one is given)
    uint32_t vec;  // this lane's vector (token * H_kv + head)
    bool in;       // the vector exists
};

template <int D>
__device__ __forceinline__ void pass_slot(const AppendArgs& a, uint32_t p, uint32_t total, int grp,
                                          Pass& L) {
    L.vec = p * Geo<D>::VPW + grp;
    L.in = L.vec < total;
    L.slot = L.in ? __ldg(a.slots + fast_div32(L.vec, a.dv_hkv)) : -1;
    L.pb = -1;
}

// With a block table, fetch the physical block of the pass's slot (issued at
// the top of the pass, used by its stores at the end).
__device__ __forceinline__ void fetch_block(const AppendArgs& a, Pass& L) {
    if (a.block_table && L.in && L.slot >= 0) {
        const uint32_t s = (uint32_t)L.slot;
        const uint32_t seq = fast_div32(s, a.dv_cap);
        const uint32_t pos = s - seq * (uint32_t)(a.max_blocks * kBlock);
        L.pb = seq < (uint32_t)a.num_seqs
                   ? __ldg(a.block_table + (size_t)seq * a.max_blocks + pos / kBlock)
                   : -2;  // -2: the logical slot is outside the table
    }
}

// f32x2 helpers (B200 packed fp32 pipe)
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    return __ffma2_rn(b, make_float2(-1.f, -1.f), a);  // a - b, one rounding
}
__device__ __forceinline__ __nv_bfloat162 as_bf2(uint32_t w) {
    return *reinterpret_cast<const __nv_bfloat162*>(&w);
}
__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 v) {
    return *reinterpret_cast<const uint32_t*>(&v);
}

// 1.5 * 2^23: x + kRound rounds x (0 <= x < 2^22) to the nearest integer,
// ties to even, and leaves that integer in the low mantissa bits.
constexpr float kRound = 12582912.0f;

// Shared memory: the bin tables (ntab tables of kBins entries, then the
// HeadBins), then each warp's ring of kAppStages stages (a pass's keys and
// values, 128-byte aligned), then one mbarrier per stage.
template <int D>
struct AppPlan {
    uint32_t rings, bars, end;
    __host__ __device__ explicit AppPlan(int ntab) {
        const uint32_t tab = (uint32_t)ntab * (kBins * sizeof(BinEntry) + sizeof(HeadBins));
        rings = (tab + 127) & ~127u;
        bars = rings + kAppWarps * kAppStages * Geo<D>::kStage;
        end = bars + kAppWarps * kAppStages * 8;
    }
};

// ROT = false: keys quantised without the rotation (an unrotated cache).
template <int D, bool ROT>
__global__ void __launch_bounds__(kAppWarps * 32, 1) append_kernel(AppendArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    constexpr int LPV = Geo<D>::LPV;
    constexpr int VPW = Geo<D>::VPW;
    constexpr uint32_t PB = Geo<D>::kPass;
    using R = Rec<D>;
    const int ntab = a.k_tables ? a.Hkv : 1;
    BinEntry* bins = reinterpret_cast<BinEntry*>(smem);
    HeadBins* hb = reinterpret_cast<HeadBins*>(smem + (size_t)ntab * kBins * sizeof(BinEntry));
    const AppPlan<D> P(ntab);

    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int sub = lane % LPV;  // the lane's 32 elements: 32 sub .. 32 sub + 31
    const int grp = lane / LPV;  // the lane's vector within the pass
    const uint32_t total = (uint32_t)a.T * (uint32_t)a.Hkv;
    const uint32_t npass = (total + VPW - 1) / VPW;
    const float inv_sqrt_d = D == 128 ? 0.08838834764831845f : 0.125f;  // fp32 of 1/sqrt(D)

    // ---- the CTA's passes are an even share [p0, p1) of all of them (so every SM
    // has the same work); warp wid takes p0 + wid, p0 + wid + kAppWarps, ...,
    // and their keys and values stream through the warp's ring (one bulk copy
    // each, one mbarrier per stage)
    const uint32_t p0 = (uint32_t)(((unsigned long long)blockIdx.x * npass) / gridDim.x);
    const uint32_t p1 = (uint32_t)(((unsigned long long)(blockIdx.x + 1) * npass) / gridDim.x);
    const uint32_t gw = p0 + (uint32_t)wid;
    const int cnt = gw < p1 ? (int)((p1 - 1 - gw) / kAppWarps) + 1 : 0;
    const uint32_t ring = smem_addr(smem) + P.rings + wid * kAppStages * Geo<D>::kStage;
    const uint32_t bar0 = smem_addr(smem) + P.bars + wid * kAppStages * 8;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kAppStages; s++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8 * s) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    // Copy pass k of this warp into stage k % kAppStages (lane 0; nothing past the end).
    auto issue = [&](int k) {
        if (k >= cnt || lane != 0) return;
        const uint32_t p = gw + (uint32_t)k * kAppWarps;
        const uint32_t v0 = p * VPW;
        const uint32_t bytes = min((uint32_t)VPW, total - v0) * D * 2;
        const uint32_t st = ring + (uint32_t)(k % kAppStages) * Geo<D>::kStage;
        const uint32_t bar = bar0 + 8 * (uint32_t)(k % kAppStages);
        asm volatile(
            "fence.proxy.async.shared::cta;\n"
            "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n"
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%2], [%3], %4, [%0];\n"
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%5], [%6], %4, [%0];\n"
            ::"r"(bar), "r"(2 * bytes), "r"(st), "l"(a.K + (size_t)v0 * D), "r"(bytes), "r"(st + PB),
            "l"(a.V + (size_t)v0 * D)
            : "memory");
    };
#pragma unroll 1
    for (int k = 0; k < kAppStages; k++) issue(k);
    Pass cur, nxt;
    if (cnt > 0) pass_slot<D>(a, gw, total, grp, cur);
    build_bins(hb, bins, a);

    int issued = min(cnt, kAppStages), k = 0;
    bool aborted = false;
#pragma unroll 1
    for (; k < cnt; k++) {
        const uint32_t pass = gw + (uint32_t)k * kAppWarps;
        fetch_block(a, cur);  // its slot was loaded a pass ago
        if (k + 1 < cnt) pass_slot<D>(a, pass + kAppWarps, total, grp, nxt);
        const uint32_t t = fast_div32(cur.vec, a.dv_hkv);
        const int h = cur.in ? (int)(cur.vec - t * (uint32_t)a.Hkv) : 0;
        const uint32_t stage = ring + (uint32_t)(k % kAppStages) * Geo<D>::kStage;
        if (!__all_sync(kFull, mbar_wait_bounded(bar0 + 8 * (uint32_t)(k % kAppStages),
                                                 (uint32_t)(k / kAppStages) & 1u))) {
            if (lane == 0) flag_status(a.status, TQ_STATUS_TIMEOUT);
            aborted = true;
            break;
        }
        // the lane's elements in the stage (a lane past the pass's last vector reads
        // stale stage bytes; it stores nothing)
        const uint32_t eoff = (uint32_t)(grp * D + sub * 32) * 2;

        // ---- values: the lane's 32 elements are one group
        uint32_t vwd[16];
        lds_32(stage + PB + eoff, vwd);
        __nv_bfloat162 mn2 = as_bf2(vwd[0]), mx2 = mn2;
#pragma unroll
        for (int j = 1; j < 16; j++) {
            mn2 = __hmin2(mn2, as_bf2(vwd[j]));
            mx2 = __hmax2_nan(mx2, as_bf2(vwd[j]));  // a NaN reaches the scale and flags the group
        }
        const uint32_t mnw = bf2_bits(mn2);
        const float mn = fminf(bf16_lo(mnw), bf16_hi(mnw));
        // the maximum of the two halves keeps a NaN (fmaxf would drop it)
        const float mx = __bfloat162float(__hmax_nan(__low2bfloat16(mx2), __high2bfloat16(mx2)));
        // z = fp16 rounded down from the minimum (exact when it lies in fp16's normal range)
        const __half zh = __float2half_rd(mn);
        const float zf = __half2float(zh);
        uint16_t s16;
        {
            // s = fp16 rounded up from D / 15, D = max - z.  c, the smallest fp16 at or
            // above a lower bound of D / 15 within one fp16 step of it, is s unless
            // 15 c < D, and then s is the next fp16.  15 c is exact in fp32, and so is
            // D when its two directed roundings agree (otherwise fp64 decides).
            // (+0 in round-to-nearest turns the -0 that max - max gives toward -inf into +0)
            const float Dd = __fsub_rd(mx, zf), Du = __fsub_ru(mx, zf);
            const float lo = __fadd_rn(__fmul_rd(Dd, inv15_dn()), 0.0f);
            const uint16_t c16 = __half_as_ushort(__float2half_ru(lo));
            if (Dd == Du)
                s16 = (uint16_t)(c16 + (half_bits_to_float(c16) * 15.f < Dd ? 1u : 0u));
            else
                s16 = double_to_half_up_nonneg(((double)mx - (double)zf) / 15.0);
        }
        const float sf = half_bits_to_float(s16);
        const bool vbad = !isfinite(sf) || !isfinite(zf);
        // sv[r]: the record's 16-bit chunk r of this lane, the code bytes of its
        // element pairs r (low byte) and 8 + r (high byte)
        uint32_t sv[8];
#pragma unroll
        for (int r = 0; r < 8; r++) sv[r] = 0;
        if (sf > 0.f) {
            // 1/s to ~1 ulp (approximation and one Newton step): it only picks the
            // candidate code, whose exact residual is checked below
            const float is0 = rcp_approx(sf);
            const float is = fmaf(is0, fmaf(-sf, is0, 1.0f), is0);
            const float2 z2 = make_float2(zf, zf), is2 = make_float2(is, is), s2 = make_float2(sf, sf);
            const float2 rnd = make_float2(kRound, kRound);
            // |v - z - t s| >= s / 2 (less the fp32 error of v - z, <= 16 ulp of s)
            // marks an exact .5 tie, or a quotient whose fp32 rounding may be on the
            // wrong side of a .5 point: such pairs are flagged in vpm
            const float thr = (0.5f - kValueMargin) * sf;
            uint32_t vpm = 0;
            uint32_t by[16];
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const float2 vz = sub2(make_float2(bf16_lo(vwd[j]), bf16_hi(vwd[j])), z2);
                const float2 tr = __ffma2_rn(vz, is2, rnd);  // kRound + round-half-even(r)
                const float2 nti = sub2(rnd, tr);            // minus that integer t, exact
                const float2 e = __ffma2_rn(nti, s2, vz);    // v - z - t s
                if (fmaxf(fabsf(e.x), fabsf(e.y)) >= thr) vpm |= 1u << j;
                // the codes are the low bytes of tr
                by[j] = __float_as_uint(tr.x) + (__float_as_uint(tr.y) << 4);
            }
#pragma unroll
            for (int r = 0; r < 8; r++) sv[r] = __byte_perm(by[r], by[8 + r], 0x0040);
            // a flagged pair's elements are decided exactly: v - z against (k + 1/2) s
            // in fp64, k the integer below, ties to even (its word is read again from
            // the stage)
#pragma unroll 1
            while (vpm) {
                const int j = __ffs(vpm) - 1;
                vpm &= vpm - 1u;
                const uint32_t wv = lds_u32(stage + PB + eoff + 4 * j);
                uint32_t pb = 0;
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    const float vf = hh ? bf16_hi(wv) : bf16_lo(wv);
                    const float vz = vf - zf;
                    const float tr = fmaf(vz, is, kRound);
                    uint32_t c = __float_as_uint(tr) & 15u;
                    if (fabsf(fmaf(kRound - tr, sf, vz)) >= thr) {
                        const float kf = floorf(vz * is);
                        const double v = (double)vf - (double)zf;
                        const double bnd = ((double)kf + 0.5) * (double)sf;
                        const int ki = (int)kf;
                        const int q = v > bnd ? ki + 1 : (v < bnd ? ki : ki + (ki & 1));
                        c = (uint32_t)min(max(q, 0), 15);
                    }
                    pb |= c << (4 * hh);
                }
                // pair j is byte j / 8 of chunk j % 8
                const int sh = 8 * (j >> 3);
                const uint32_t jr = (uint32_t)j & 7u, cm = ~(0xffu << sh), cv = pb << sh;
#pragma unroll
                for (int r = 0; r < 8; r++) sv[r] = jr == (uint32_t)r ? (sv[r] & cm) | cv : sv[r];
            }
        }

        // ---- key: norm and in-lane butterfly over element bits 0-4.  Q[j]
        // holds elements (2j, 2j+1) of the lane's 32.
        float2 Q[16];
        float ss;
        {
            uint32_t kwd[16];
            lds_32(stage + eoff, kwd);
            float2 s4[4];
#pragma unroll
            for (int i = 0; i < 4; i++) s4[i] = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const float2 P = make_float2(bf16_lo(kwd[j]), bf16_hi(kwd[j]));
                s4[j & 3] = __ffma2_rn(P, P, s4[j & 3]);
                Q[j] = ROT ? make_float2(P.x + P.y, P.x - P.y) : P;
            }
            const float2 s2 = add2(add2(s4[0], s4[1]), add2(s4[2], s4[3]));
            ss = s2.x + s2.y;
        }
#pragma unroll
        for (int m = 1; m < LPV; m <<= 1) ss += __shfl_xor_sync(kFull, ss, m);
#pragma unroll
        for (int b = 1; b < (ROT ? 16 : 1); b <<= 1) {
#pragma unroll
            for (int j = 0; j < 16; j++)
                if (!(j & b)) {
                    const float2 x = Q[j], y = Q[j | b];
                    Q[j] = add2(x, y);
                    Q[j | b] = sub2(x, y);
                }
        }
        // ---- key: butterfly over the lane bits (upper half: partner - own)
#pragma unroll
        for (int m = 1; m < (ROT ? LPV : 1); m <<= 1) {
            const float sg = (sub & m) ? -1.f : 1.f;
            const float2 sg2 = make_float2(sg, sg);
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const float2 pr = make_float2(__shfl_xor_sync(kFull, Q[j].x, m),
                                              __shfl_xor_sync(kFull, Q[j].y, m));
                Q[j] = __ffma2_rn(sg2, Q[j], pr);
            }
        }
        // ---- key: norm (fp16) and the scale to unit-vector coordinates: rsqrt
        // refined by one Newton step (relative error ~4 ulp whatever the
        // approximation's), so n errs by <= 9 ulp and 1 / (n sqrt(D)) by <= 10 ulp
        const float ssc = fmaxf(ss, 1.17549435e-38f);
        const float rs0 = rsqrt_approx(ssc);
        const float rs = rs0 * fmaf(-0.5f * ssc * rs0, rs0, 1.5f);
        const float n = ss * rs;
        uint16_t n16 = __half_as_ushort(__float2half_rn(n));
        const bool nnorm = __half_as_ushort(__float2half_rn(n * (1.0f - kNormMargin))) !=
                           __half_as_ushort(__float2half_rn(n * (1.0f + kNormMargin)));
        // squares that leave the normal fp32 range (or a non-finite key) lose the
        // fp32 error bound: every decision is re-taken.  An all-zero key stays here;
        // whether any element is nonzero is asked of the whole vector, since one
        // lane's 32 elements may all be zero while the others' are not.
        const bool small = !(ss >= 1e-30f && ss <= 1e30f);
        bool wild = false;
        if (__any_sync(kFull, small)) {
            uint32_t kor = 0;
#pragma unroll
            for (int c = 0; c < 4; c++) {
                const uint4 t4 = lds_u4(stage + eoff + 16 * c);
                kor |= t4.x | t4.y | t4.z | t4.w;
            }
#pragma unroll
            for (int m = 1; m < LPV; m <<= 1) kor |= __shfl_xor_sync(kFull, kor, m);
            wild = small && (kor & 0x7fff7fffu) != 0u;
        }
        // y = Q / (n sqrt(D)) after the +-1 butterfly, Q / n without it
        const float inv = ROT ? rs * inv_sqrt_d : rs;
        const float A = ROT ? rs * (inv_sqrt_d * kBinScale) : rs * kBinScale;

        // ---- key: nearest centroid.  kc[i] holds the codes of elements 8i .. 8i+7;
        // kpm flags the pairs with a decision inside the margin.
        const int hs = a.k_tables ? h : 0;  // whose table
        const HeadBins& B = hb[hs];
        const unsigned char* tab = smem + (size_t)hs * (kBins * sizeof(BinEntry));
        uint32_t kc[4] = {0u, 0u, 0u, 0u};
        uint32_t kpm = 0;
        if (!B.dense) {
            const float2 A2 = make_float2(A, A), M2 = make_float2(kBinMagic, kBinMagic);
            uint32_t by[16];
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const float2 x = __ffma2_rn(Q[j], A2, M2);
                const BinEntry e0 = *reinterpret_cast<const BinEntry*>(tab + (__float_as_uint(x.x) & 0x3f8u));
                const BinEntry e1 = *reinterpret_cast<const BinEntry*>(tab + (__float_as_uint(x.y) & 0x3f8u));
                // mid - y with one rounding: its sign is the decision (y == mid gives
                // +0 and the lower code, and is near anyway)
                const float d0 = fmaf(-Q[j].x, inv, e0.mid);
                const float d1 = fmaf(-Q[j].y, inv, e1.mid);
                if (fminf(fabsf(d0), fabsf(d1)) < kKeyMargin) kpm |= 1u << j;
                // k_lo + 1 where y > mid (the sign bit of mid - y)
                const uint32_t c0 = (uint32_t)e0.k_lo + (__float_as_uint(d0) >> 31);
                const uint32_t c1 = (uint32_t)e1.k_lo + (__float_as_uint(d1) >> 31);
                by[j] = c0 | (c1 << 4);
            }
#pragma unroll
            for (int i = 0; i < 4; i++) kc[i] = pack4(by[4 * i], by[4 * i + 1], by[4 * i + 2], by[4 * i + 3]);
        } else {  // midpoints closer than a bin: count them all
#pragma unroll
            for (int j = 0; j < 16; j++) {
                uint32_t pc = 0;
                bool nr = false;
#pragma unroll 1
                for (int k = 0; k < 15; k++) {
                    const float m = 0.5f * (B.c[k] + B.c[k + 1]);
                    const float dx = Q[j].x * inv - m, dy = Q[j].y * inv - m;
                    pc += (dx > 0.f ? 1u : 0u) + (dy > 0.f ? 16u : 0u);
                    nr |= fminf(fabsf(dx), fabsf(dy)) < kKeyMargin;
                }
                if (nr) kpm |= 1u << j;
                kc[j >> 2] |= pc << (8 * (j & 3));
            }
        }
        const bool live = cur.in && cur.slot >= 0;
        const bool near = live && (wild || kpm != 0 || nnorm);

        // ---- key: exact decisions when any decision of the warp is close
        if (__any_sync(kFull, near)) {
            // the pairs to decide again (all of them when the fp32 scale is unusable)
            uint32_t nm = near ? (wild ? 0xffffu : kpm) : 0u;
            // the exact norm from the fp64 sum of squares of this lane's keys (still
            // in the stage)
            double ssd = 0.0;
            {
                uint32_t w[16];
                lds_32(stage + eoff, w);
                double s0 = 0.0, s1 = 0.0;
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    const double x = (double)bf16_lo(w[j]), y = (double)bf16_hi(w[j]);
                    s0 = fma(x, x, s0);
                    s1 = fma(y, y, s1);
                }
                ssd = s0 + s1;
            }
#pragma unroll
            for (int m = 1; m < LPV; m <<= 1) ssd += __shfl_xor_sync(kFull, ssd, m);
            const double nd = sqrt(ssd);
            const double denom = ROT ? nd * sqrt((double)D) : nd;  // y_e = (H k)_e / denom, or k_e / denom
            if (near) n16 = __half_as_ushort(__double2half(nd));
            if (near && ssd == 0.0) {
                // an all-zero key: y = 0 exactly, every element takes the code of 0
                uint32_t c0 = 0;
                const BinEntry be = *reinterpret_cast<const BinEntry*>(tab + (__float_as_uint(kBinMagic) & 0x3f8u));
                if (!B.dense) c0 = (uint32_t)be.k_lo + (0.f > be.mid ? 1u : 0u);
                else
                    for (int k = 0; k < 15; k++) c0 += 0.f > 0.5f * (B.c[k] + B.c[k + 1]) ? 1u : 0u;
#pragma unroll
                for (int i = 0; i < 4; i++) kc[i] = c0 * 0x11111111u;
                nm = 0;
            }
            // 1 / denom, only to pick a bin: the fast path's fp32 scale, or from the
            // exact norm when that scale is unusable
            float rden = inv;
            if (wild) rden = ssd > 0.0 ? (float)(1.0 / denom) : 0.f;
            // Pair pj's two decisions from their exact numerators (y times denom):
            // each against midpoint * denom, then the pair's byte of kc
            auto decide_pair = [&](int pj, double part0, double part1) {
                uint32_t pc = 0;
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    const double part = hh ? part1 : part0;
                    uint32_t idx = 0;
                    if (!B.dense) {
                        const float x = fmaf((float)part * rden, kBinScale, kBinMagic);
                        const BinEntry be = *reinterpret_cast<const BinEntry*>(tab + (__float_as_uint(x) & 0x3f8u));
                        idx = (uint32_t)be.k_lo + (part > (double)be.mid * denom ? 1u : 0u);
                    } else {
#pragma unroll 1
                        for (int k = 0; k < 15; k++)
                            idx += part > 0.5 * ((double)B.c[k] + (double)B.c[k + 1]) * denom ? 1u : 0u;
                    }
                    pc |= idx << (4 * hh);
                }
                // pair pj is byte pj % 4 of word pj / 4
                const int sh = 8 * (pj & 3);
                const uint32_t wi = (uint32_t)pj >> 2, cm = ~(0xffu << sh), cv = pc << sh;
#pragma unroll
                for (int i = 0; i < 4; i++) kc[i] = wi == (uint32_t)i ? (kc[i] & cm) | cv : kc[i];
            };
            if constexpr (ROT) {
                // one flagged pair per vector per round.  Its rows 2p and 2p + 1 of
                // the Hadamard sum share their signs on each element pair (row 2p + 1
                // flips the odd elements), so the sums over the even and the odd
                // elements, exact in fp64, give both: E + O and E - O.
                const uint32_t gmask = ((1u << LPV) - 1u) << (grp * LPV);
#pragma unroll 1
                while (__any_sync(kFull, nm != 0)) {
                    const uint32_t pend = __ballot_sync(kFull, nm != 0) & gmask;
                    const int owner = pend ? __ffs(pend) - 1 : lane;
                    const int mine = nm ? __ffs(nm) - 1 : 0;
                    const uint32_t pr = (uint32_t)__shfl_sync(kFull, 16 * sub + mine, owner);  // pair of the vector
                    double pe = 0.0, po = 0.0;
#pragma unroll 4
                    for (int j = 0; j < 16; j++) {
                        const uint32_t wv = lds_u32(stage + eoff + 4 * j);
                        const double x0 = (double)bf16_lo(wv), x1 = (double)bf16_hi(wv);
                        const bool neg = __popc((pr & 15u) & (uint32_t)j) & 1;
                        pe += neg ? -x0 : x0;
                        po += neg ? -x1 : x1;
                    }
                    if (__popc((pr >> 4) & (uint32_t)sub) & 1) {
                        pe = -pe;
                        po = -po;
                    }
#pragma unroll
                    for (int m = 1; m < LPV; m <<= 1) {
                        pe += __shfl_xor_sync(kFull, pe, m);
                        po += __shfl_xor_sync(kFull, po, m);
                    }
                    if (pend && lane == owner) {
                        decide_pair(mine, pe + po, pe - po);
                        nm &= nm - 1u;
                    }
                }
            } else {
                // unrotated: a coordinate's numerator is the key element itself
#pragma unroll 1
                while (nm) {
                    const int pj = __ffs(nm) - 1;
                    nm &= nm - 1u;
                    const uint32_t wv = lds_u32(stage + eoff + 4 * pj);
                    decide_pair(pj, (double)bf16_lo(wv), (double)bf16_hi(wv));
                }
            }
        }

        // the stage is read: refill it with the pass kAppStages ahead
        __syncwarp();
        issue(k + kAppStages);
        if (k + kAppStages < cnt) issued++;

        // ---- where this vector goes (the block-table read was issued at the top)
        int blk = -1;
        const int off = cur.slot & (kBlock - 1);  // table rows span whole blocks
        if (cur.in && cur.slot >= 0) {
            if (a.block_table) {
                if (cur.pb >= 0 && cur.pb < a.num_blocks) {
                    blk = cur.pb;
                } else if (sub == 0) {
                    flag_status(a.status, cur.pb == -2 ? TQ_STATUS_BAD_SLOT : TQ_STATUS_BAD_BLOCK);
                }
            } else if (cur.slot / kBlock < a.num_blocks) {
                blk = cur.slot / kBlock;
            } else if (sub == 0) {
                flag_status(a.status, TQ_STATUS_BAD_SLOT);
            }
        }
        if (blk >= 0) {
            unsigned char* rec = a.cache + ((size_t)blk * a.Hkv + h) * (size_t)R::kBytes;
            *reinterpret_cast<uint4*>(rec + R::kKCodes + off * R::kCodeRow + sub * 16) =
                make_uint4(kc[0], kc[1], kc[2], kc[3]);
            // code bytes 16 sub + r (m = 2 sub) and 16 sub + 8 + r (m = 2 sub + 1) of
            // this token sit side by side in the chunk of r, its pair's chunks rotated
            // by 2 (off / 2): chunks r and r + 1 (r even) stay adjacent
            unsigned char* vdst = rec + R::kVCodes + R::vcode_pos(off, 16 * sub);  // chunk of r = 0
            const int rot = (off >> 1) & 3;  // the rotation in chunk pairs
#pragma unroll
            for (int r = 0; r < 8; r += 2) {
                unsigned char* cp = vdst + (((r >> 1) + rot) & 3) * (2 * R::kPairChunk) - 2 * rot * R::kPairChunk;
                *reinterpret_cast<uint16_t*>(cp) = (uint16_t)sv[r];
                *reinterpret_cast<uint16_t*>(cp + R::kPairChunk) = (uint16_t)sv[r + 1];
            }
            if (sub == 0) *reinterpret_cast<uint16_t*>(rec + R::kKNorm + off * 2) = n16;
            const int gp = R::group_pos(off, sub);
            *reinterpret_cast<uint16_t*>(rec + R::kVScale + gp) = s16;
            *reinterpret_cast<uint16_t*>(rec + R::kVZero + gp) = __half_as_ushort(zh);
            const bool bad = vbad || (sub == 0 && !isfinite(half_bits_to_float(n16)));
            if (bad) flag_status(a.status, TQ_STATUS_RANGE);
        }

        cur = nxt;
    }
    if (aborted) {  // give the copies still in flight a bounded chance to land
#pragma unroll 1
        for (int j = k; j < issued; j++)
            mbar_wait_bounded(bar0 + 8 * (uint32_t)(j % kAppStages), (uint32_t)(j / kAppStages) & 1u);
    }
}

size_t append_smem_bytes(int ntab, int head_dim) {
    return head_dim == 128 ? AppPlan<128>(ntab).end : AppPlan<64>(ntab).end;
}

// The bins of the default table of head_dim d, computed once per process
// (every caller waits until they are complete).
static void default_bins(int d, const uint16_t* table16, HeadBins& hb, BinEntry* bins) {
    static std::once_flag once[2];
    static HeadBins cached_hb[2];
    static BinEntry cached[2][kBins];
    const int key = d == 128 ? 1 : 0;
    std::call_once(once[key], [&] {
        HeadBins& h = cached_hb[key];
        for (int k = 0; k < 16; k++) h.c[k] = __half2float(__ushort_as_half(table16[k]));
        h.dense = 0;
        h.pad = 0;
        for (int b = 0; b < kBins; b++)
            if (bin_entry(h.c, b, cached[key][b])) h.dense = 1;
    });
    hb = cached_hb[key];
    memcpy(bins, cached[key], sizeof cached[key]);
}

template <int D, bool ROT>
static cudaError_t launch_a(const AppendArgs& a, int num_sms, cudaStream_t stream) {
    // the largest shared-memory size, set once per device (under a lock: the
    // library may be called from several host threads)
    static std::mutex mu;
    static bool configured[64] = {};
    static const size_t max_smem = AppPlan<D>(32).end;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (dev < 0 || dev >= 64 || !configured[dev]) {
            e = cudaFuncSetAttribute(append_kernel<D, ROT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)max_smem);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) configured[dev] = true;
        }
    }
    const long long vectors = (long long)a.T * a.Hkv;
    const long long passes = (vectors + Geo<D>::VPW - 1) / Geo<D>::VPW;
    // one persistent wave over every SM (each CTA takes an even share of the passes,
    // so a small append spreads over the whole GPU rather than filling a few SMs)
    long long blocks = passes;
    if (blocks > num_sms) blocks = num_sms;
    if (blocks < 1) blocks = 1;
    const size_t smem = AppPlan<D>(a.k_tables ? a.Hkv : 1).end;
    append_kernel<D, ROT><<<(unsigned)blocks, kAppWarps * 32, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs& args, int head_dim, int num_sms, cudaStream_t stream) {
    AppendArgs a = args;
    if (!a.k_tables) default_bins(head_dim, a.default_table, a.default_hb, a.default_bins);
    a.dv_hkv = div32_magic((uint32_t)a.Hkv);
    a.dv_cap = div32_magic((uint32_t)(a.max_blocks > 0 ? a.max_blocks * kBlock : 1));
    if (head_dim == 128) return a.rotate ? launch_a<128, true>(a, num_sms, stream) : launch_a<128, false>(a, num_sms, stream);
    return a.rotate ? launch_a<64, true>(a, num_sms, stream) : launch_a<64, false>(a, num_sms, stream);
}

}  // namespace tq
