// tq_decode.cu -- split-K decode attention over the TQ4/4 cache and the
// log-sum-exp combine of the splits.
//
// Scores: H is symmetric and orthogonal, so <q, k_hat_t> = n_t <H q, C[idx_t]>.
// The query is rotated once (q~ = H q) and every score is formed in the
// rotated domain against the stored centroids; keys are never un-rotated.
// Values: v_hat = code * s + z per group of 32, so
//   o = sum_t p_t v_hat_t = sum_t (p_t s_t,g) code_t + sum_t p_t z_t,g.
//
// Work.  An item is (sequence, kv head, group of four query heads), or at d = 64
// with more than four query heads per kv head two such groups, whose records are
// then staged and unpacked once for both.  The virtual record space items x
// nmax (nmax = blocks of the longest sequence) is cut into ranges: evenly over
// every half of a full grid, or into ceil(nmax / S) records per range with S
// splits.  The grid is persistent: one CTA of 12 warps per SM, made of two
// independent halves of 6 warps, half h taking ranges h, h + H, ...  Within a
// range's part of an item (a segment) the 6 warps take its 16-token blocks
// round-robin.  Each warp streams its records through a private ring of
// shared-memory stages with bulk asynchronous copies (cp.async.bulk +
// mbarrier); the ring runs across segment boundaries, so the next segment's
// first records are in flight while a segment's partial results are merged.
//
// Per record every product runs on the tensor cores (mma.sync m16n8k16, fp32
// accumulate), with exact fp16 operands only:
//   q.K  A = centroids of the 16 tokens from a byte -> (C[lo], C[hi]) table
//        with one copy per lane (one prmt forms each table address), B = q~
//        with head h's high fp16 part in column 2h and its low part in 2h+1,
//        so the scores carry q~ to ~22 bits.  Four shuffles move each head's
//        weights into the layout p.V takes them in.
//   p.V  A = value codes as fp16 subnormals (the nibble masked in place is
//        n 2^-24, or n 2^-20 for a high nibble: exact, no bias to remove);
//        B = p_t s_t,g as an exact two-part fp16 product, the high part in
//        column 2h and the low part in column 2h+1 of head h.
//   p.z  A = fp16 zero points (rows 0-7) and ones (rows 8-15), B = p as fp16
//        parts: gives sum_t p_t z_t,g and the softmax denominator.
// Softmax runs online in base 2 (scale * log2 e is folded into q~) and the
// accumulators are rescaled only when a running maximum moves.  An item
// that lies wholly inside one range is written directly; the others leave an
// unnormalised partial (o, m, l) per range that the combine kernel merges.
#include <mutex>

#include "tq_kernels.cuh"

namespace tq {
namespace {

constexpr int kNW = 6;                   // warps per half (per range)
constexpr int kHalves = 2;               // independent halves per CTA
constexpr int kWarps = kNW * kHalves;    // 12 warps, 384 threads
constexpr int kStages = 4;               // records per warp ring: two pairs
constexpr int kPairs = kStages / 2;      // pair slots per ring (one mbarrier each)
constexpr int kMergeSlots = kNW / 2;     // partials a half's merge tree holds at once
constexpr int kHeads = 4;                // query heads per mma group (an item holds 1 or 2)
constexpr uint32_t kLutBytes = 1u << 16; // 256 byte values x (2 halves x 32 lanes x 4 B)
constexpr uint32_t kOnes = 0x3C003C00u;  // fp16 (1, 1)

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(v));
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(v));
}
// barrier among the threads of one half (ids 1, 2; 0 is __syncthreads)
__device__ __forceinline__ void half_sync(int half) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + half), "n"(kNW * 32) : "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
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
// The same for a whole warp, kept out of line: the common case (the phase has
// completed) is one try_wait and one vote at the call site.
__device__ __noinline__ bool mbar_wait_warp_slow(uint32_t bar, uint32_t phase) {
    return __all_sync(0xffffffffu, mbar_wait(bar, phase));
}
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t phase) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, phase))) return true;
    return mbar_wait_warp_slow(bar, phase);
}
// OR bits into the status word from lane 0 only, without a branch
__device__ __forceinline__ void flag_lane0(int32_t* status, int bits, int lane) {
    const uint32_t p = (uint32_t)(lane == 0 && status != nullptr);
    asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %0, 0;\n @p red.global.or.b32 [%1], %2;\n}\n"
                 ::"r"(p), "l"(status), "r"(bits) : "memory");
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

// the same with a zero accumulator in
__device__ __forceinline__ void mma16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
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

// The two fp16 operand parts of p for this lane's column: a high-part lane
// (sel = 0) gets u = 0, w = fp16(p); a low-part lane (sel = 1) gets
// u = fp16(p), w = fp16(p - u).  p0 goes to the low half of each pair.
__device__ __forceinline__ void split_uw(float p0, float p1, float sel, uint32_t mask, uint32_t& u,
                                         uint32_t& w) {
    const __half2 h = __floats2half2_rn(p0, p1);
    const float2 f = __half22float2(h);
    w = h2u(__floats2half2_rn(fmaf(-sel, f.x, p0), fmaf(-sel, f.y, p1)));
    u = h2u(h) & mask;
}

// This lane's part of p * s: fl(w s + (u s - fl(u s))).  With u = 0 it is
// fl(p_hi s); with (u, w) = (p_hi, p_lo) it is the remainder of p_hi s (exact
// by the fma two-product) plus p_lo s, so the two columns sum to p s within
// ~2^-21 relative.
__device__ __forceinline__ uint32_t ps_part(uint32_t u, uint32_t w, uint32_t s) {
    const __half2 x = __hmul2(u2h(u), u2h(s));
    const __half2 r = __hfma2(u2h(u), u2h(s), __hneg2(x));
    return h2u(__hfma2(u2h(w), u2h(s), r));
}

// ------------------------------------------------------------------ shared memory plan
// Floats of one warp's partial per lane, for one item: per group of four heads,
// 2 D/16 output values (two dims per m-tile) plus the head's sum l and maximum m,
// padded to whole 16-byte vectors.
template <int D, int QPI>
struct Part {
    static constexpr int kPerQ = 2 * (D / 16) + 2;
    static constexpr int kFloats = (QPI * kPerQ + 3) / 4 * 4;
    static constexpr uint32_t kSlotBytes = 32u * kFloats * 4u;  // [vector][lane][4 floats]
};

// Shared-window addresses for a dynamic region that starts at s0.  The table
// must sit on a 64 KB boundary so that one prmt can splice a code byte into
// the address.  The small buffers come first, whole warp rings fill the space
// below the table, and the remaining rings follow it.
template <int D, int QPI>
struct Plan {
    static constexpr int HPI = kHeads * QPI;
    static constexpr uint32_t kRec = Rec<D>::kBytes;
    static constexpr uint32_t kRing = kStages * kRec;  // one warp's stages, contiguous
    static constexpr uint32_t kMergeHalf = kMergeSlots * Part<D, QPI>::kSlotBytes;
    uint32_t merge, qh, ql, ids, bars, rings, lut, low, hi, end;
    __host__ __device__ explicit Plan(uint32_t s0) {
        merge = (s0 + 15) & ~15u;
        qh = merge + kHalves * kMergeHalf;
        ql = qh + kHalves * HPI * D * 2;
        ids = ql + kHalves * HPI * D * 2;
        bars = ids + kWarps * kStages * 4;
        rings = (bars + kWarps * kPairs * 8 + 127) & ~127u;
        lut = (rings + kLutBytes - 1) & ~(kLutBytes - 1);
        const uint32_t n = (lut - rings) / kRing;
        low = n < (uint32_t)kWarps ? n : (uint32_t)kWarps;
        hi = lut + kLutBytes;
        end = hi + (kWarps - low) * kRing;
    }
    // first stage of warp w's ring
    __host__ __device__ uint32_t ring(int w) const {
        return (uint32_t)w < low ? rings + w * kRing : hi + (w - low) * kRing;
    }
};

// Bytes to request so that the plan fits wherever the dynamic region starts
// (the start depends on the reserved shared memory of the device).
template <int D, int QPI>
uint32_t plan_bytes() {
    uint32_t worst = 0;
    for (uint32_t s0 = 0; s0 <= 8192; s0 += 16) {
        const Plan<D, QPI> p(s0);
        if (p.end - s0 > worst) worst = p.end - s0;
    }
    return worst;
}

// ------------------------------------------------------------------ segments
// The work is the virtual record space items x nmax (nmax = blocks of the
// longest sequence), cut into ranges of R consecutive records; half h takes
// ranges h, h + H, ...  A segment is the part of one item inside one range.
// An item that lies wholly inside a range is finished there ("direct"); the
// others leave one partial per range, in slot 0 if the item is the range's
// first, else slot 1 (only the range's last item can be split besides the first).
struct Seg {
    int r;                  // range (>= nranges: past the end)
    int i, i_first, i_last; // item, and the first and last items of the range
    int b, kv, quad;
    int L;                  // tokens of the sequence (clamped)
    int jb;                 // first block of the segment
    int nk;                 // records of this warp in the segment
    bool direct;
    const int32_t* bt;      // block-table entry of this warp's first record
    const unsigned char* src;  // record of block 0 for this kv head
};

template <int D>
__device__ __forceinline__ void seg_item(Seg& s, const DecodeArgs& a, int warp, bool report) {
    const int base = s.i * a.nmax;
    const int p0 = s.r * a.R;
    const int p1 = min(p0 + a.R, a.vrec);
    const int lo = max(p0, base) - base, hi = min(p1, base + a.nmax) - base;
    s.direct = lo == 0 && hi == a.nmax;
    const int bk = (int)fast_div((uint32_t)s.i, a.div_quads);
    s.quad = s.i - bk * a.quads;
    s.b = (int)fast_div((uint32_t)bk, a.div_hkv);
    s.kv = bk - s.b * a.Hkv;
    int L = a.seq_lens[s.b];
    const bool first = report && s.kv == 0 && s.quad == 0 && lo == 0;
    if (L < 0 || L > a.max_blocks * kBlock) {
        if (first) flag_status(a.status, TQ_STATUS_BAD_LEN);
        L = 0;
    }
    if (L > a.nmax * kBlock) {
        if (first) flag_status(a.status, TQ_STATUS_BAD_LEN);
        L = a.nmax * kBlock;
    }
    s.L = L;
    const int nblk = (L + kBlock - 1) / kBlock;
    s.jb = lo;
    const int left = min(hi, nblk) - lo - warp;
    s.nk = left > 0 ? (left + kNW - 1) / kNW : 0;
    s.bt = a.block_tables + (size_t)s.b * a.max_blocks + lo + warp;
    s.src = a.cache + (size_t)s.kv * Rec<D>::kBytes;
}

// first segment of range r (or past the end)
template <int D>
__device__ __forceinline__ void seg_range(Seg& s, int r, const DecodeArgs& a, int warp, bool report) {
    s.r = r;
    s.nk = 0;
    if (r >= a.nranges) return;
    const int p0 = r * a.R;
    const int p1 = min(p0 + a.R, a.vrec);
    s.i = s.i_first = (int)fast_div((uint32_t)p0, a.div_nmax);
    s.i_last = (int)fast_div((uint32_t)(p1 - 1), a.div_nmax);
    seg_item<D>(s, a, warp, report);
}

template <int D>
__device__ __forceinline__ void seg_next(Seg& s, int stride, const DecodeArgs& a, int warp,
                                         bool report) {
    if (s.i < s.i_last) {
        s.i++;
        seg_item<D>(s, a, warp, report);
    } else {
        seg_range<D>(s, s.r + stride, a, warp, report);
    }
}

// N consecutive 32-bit words (N = 2 or 4) of shared memory
template <int N>
__device__ __forceinline__ void ldw(uint32_t a, uint32_t (&w)[N]) {
    static_assert(N == 2 || N == 4, "8- or 16-byte loads");
    if constexpr (N == 4) {
        const uint4 v = lds128(a);
        w[0] = v.x;
        w[1] = v.y;
        w[2] = v.z;
        w[3] = v.w;
    } else {
        const uint2 v = lds64(a);
        w[0] = v.x;
        w[1] = v.y;
    }
}

// ------------------------------------------------------------------ merge tree
// The warps of a half merge their partials in rounds: in a round over `act`
// warps, warps [h, act) (h = ceil(act / 2)) hand their partials to warps
// [0, act - h) through the merge slots, and the next round is over h warps.  A
// writer uses the slot it read itself in an earlier round (else its own index
// minus h), so a slot is never overwritten while another warp may still be
// reading it, and one barrier per round suffices.
__host__ __device__ constexpr int tree_act(int k) {
    int act = kNW;
    for (int r = 0; r < k; r++) act = (act + 1) / 2;
    return act;
}
__host__ __device__ constexpr int tree_rounds() {
    int k = 0;
    while (tree_act(k) > 1) k++;
    return k;
}
// The slot each writer of round k uses, 4 bits per warp.
__host__ __device__ constexpr uint32_t tree_wslot(int k) {
    int rd[16] = {-1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1};
    for (int r = 0;; r++) {
        const int act = tree_act(r), h = (act + 1) / 2;
        uint32_t ws = 0;
        for (int w = h; w < act; w++) {
            const int sl = rd[w] >= 0 ? rd[w] : w - h;
            ws |= (uint32_t)sl << (4 * w);
            rd[w - h] = sl;
        }
        if (r == k) return ws;
    }
}
// Checks of the schedule: every slot index is below kMergeSlots, and no writer
// of round k uses a slot that a reader of round k - 1 other than itself read.
__host__ __device__ constexpr bool tree_ok() {
    for (int k = 0; k < tree_rounds(); k++) {
        const int act = tree_act(k), h = (act + 1) / 2;
        for (int w = h; w < act; w++) {
            const int sl = (int)((tree_wslot(k) >> (4 * w)) & 15u);
            if (sl >= kMergeSlots) return false;
            if (k > 0) {
                const int pa = tree_act(k - 1), ph = (pa + 1) / 2;
                for (int r = 0; r < pa - ph; r++)
                    if (r != w && (int)((tree_wslot(k - 1) >> (4 * (r + ph))) & 15u) == sl) return false;
            }
        }
    }
    return true;
}
static_assert(kNW <= 16 && tree_ok(), "merge tree schedule");

// ------------------------------------------------------------------ split kernel
// The scores of one record for QPI groups of four heads: s[q] rows g (token g)
// and g + 8 (token g + 8), columns 2c, 2c+1 (head 4q + c, high and low part of q~).
template <int D, int QPI>
__device__ __forceinline__ void record_scores(uint32_t rec, int g, int c, uint32_t lanebase,
                                              const uint32_t (&qb)[QPI][D / 16][2],
                                              float (&sc)[QPI][4]) {
    constexpr int KS = D / 16, KB = D / 8, KW = KB / 4;
    uint32_t kw0[KW], kw1[KW];
    ldw<KW>(rec + g * (D / 2) + c * KB, kw0);
    ldw<KW>(rec + (g + 8) * (D / 2) + c * KB, kw1);
#pragma unroll
    for (int ks = 0; ks < KS; ks++) {
        // table address: the code byte spliced into byte 1 of lanebase
        const uint32_t sa = (ks & 1) ? 0x7624u : 0x7604u;
        const uint32_t sb = (ks & 1) ? 0x7634u : 0x7614u;
        const uint32_t w0 = kw0[ks >> 1], w1 = kw1[ks >> 1];
        const uint32_t a0 = lds32(__byte_perm(w0, lanebase, sa));
        const uint32_t a2 = lds32(__byte_perm(w0, lanebase, sb));
        const uint32_t a1 = lds32(__byte_perm(w1, lanebase, sa));
        const uint32_t a3 = lds32(__byte_perm(w1, lanebase, sb));
#pragma unroll
        for (int q = 0; q < QPI; q++) {
            if (ks == 0)
                mma16816_z(sc[q], a0, a1, a2, a3, qb[q][ks][0], qb[q][ks][1]);
            else
                mma16816(sc[q], a0, a1, a2, a3, qb[q][ks][0], qb[q][ks][1]);
        }
    }
}

// p.z (and sum p) and p.V of one record for QPI groups of heads, given this
// lane's fp16 parts of the weights (u, w: tokens 2c, 2c+1 | 2c+8, 2c+9 of head
// g/2 of each group) and the valid-token masks of the fp16 lanes (mA: tokens
// 2c, 2c+1; mB: tokens 2c+8, 2c+9; all ones for a full record).
template <int D, int QPI, bool MASK>
__device__ __forceinline__ void record_values(uint32_t rec, int g, int c, uint32_t mA, uint32_t mB,
                                              const uint32_t (&u01)[QPI], const uint32_t (&w01)[QPI],
                                              const uint32_t (&u89)[QPI], const uint32_t (&w89)[QPI],
                                              float (&O)[QPI][D / 16][4], float (&Z)[QPI][4]) {
    constexpr int NG = D / 32, KB = D / 8, KW = KB / 4;
    using R = Rec<D>;
    uint2 zz = lds64(rec + R::kVZero + (c * NG + (g & (NG - 1))) * 8);
    uint32_t sw[2 * NG];
#pragma unroll
    for (int i = 0; i < 2 * NG; i += 4) {
        uint32_t t4[4];
        ldw<4>(rec + R::kVScale + c * NG * 8 + 4 * i, t4);
#pragma unroll
        for (int e = 0; e < 4; e++) sw[i + e] = t4[e];
    }
    if (MASK) {  // stale fields of unwritten tokens must not reach the products
        zz.x &= mA;
        zz.y &= mB;
#pragma unroll
        for (int G_ = 0; G_ < NG; G_++) {
            sw[2 * G_] &= mA;
            sw[2 * G_ + 1] &= mB;
        }
    }
#pragma unroll
    for (int q = 0; q < QPI; q++) mma16816(Z[q], zz.x, kOnes, zz.y, kOnes, w01[q], w89[q]);
    // word G of a chunk holds m-tiles 2G (bytes 0, 2) and 2G + 1 (bytes 1, 3) of
    // tokens 2c, 2c+1 (va) and 2c+8, 2c+9 (vb)
    uint32_t va[KW], vb[KW];
    // chunk r = g of token pairs c and c + 4, rotated by 2c (2 (c + 4) = 2c mod 8)
    const int rr = (g + 2 * c) & 7;
    ldw<KW>(rec + R::kVCodes + (c * 8 + rr) * KB, va);
    ldw<KW>(rec + R::kVCodes + ((c + 4) * 8 + rr) * KB, vb);
#pragma unroll
    for (int G_ = 0; G_ < NG; G_++) {
        const uint32_t A0 = va[G_], B0 = vb[G_], A1 = A0 >> 8, B1 = B0 >> 8;
#pragma unroll
        for (int q = 0; q < QPI; q++) {
            const uint32_t b0 = ps_part(u01[q], w01[q], sw[2 * G_]);
            const uint32_t b1 = ps_part(u89[q], w89[q], sw[2 * G_ + 1]);
            mma16816(O[q][2 * G_], A0 & 0x000F000Fu, A0 & 0x00F000F0u, B0 & 0x000F000Fu,
                     B0 & 0x00F000F0u, b0, b1);
            mma16816(O[q][2 * G_ + 1], A1 & 0x000F000Fu, A1 & 0x00F000F0u, B1 & 0x000F000Fu,
                     B1 & 0x00F000F0u, b0, b1);
        }
    }
}

// Token masks of a record with n valid tokens (n = 16: everything valid):
// tokens g, g + 8 of the score rows, and the fp16 lanes of tokens 2c, 2c+1 |
// 2c+8, 2c+9 of the value operands.
struct Mask {
    bool va, vb;
    uint32_t mA, mB;
};
__device__ __forceinline__ Mask token_mask(int n, int g, int c) {
    const int t = 2 * c;
    Mask m;
    m.va = g < n;
    m.vb = g + 8 < n;
    m.mA = (t < n ? 0xffffu : 0u) | (t + 1 < n ? 0xffff0000u : 0u);
    m.mB = (t + 8 < n ? 0xffffu : 0u) | (t + 9 < n ? 0xffff0000u : 0u);
    return m;
}

// Merge partial (pm, pl, po) into (m, l, o): both relative to their own maxima
// in base 2; an empty partial has maximum -inf and contributes nothing.
template <int N>
__device__ __forceinline__ void merge_into(float& m, float& l, float (&o)[N], float pm, float pl,
                                           const float* po) {
    const float M = fmaxf(m, pm);
    const float f0 = m == -INFINITY ? 0.f : ex2(m - M);
    const float f1 = pm == -INFINITY ? 0.f : ex2(pm - M);
#pragma unroll
    for (int j = 0; j < N; j++) o[j] = fmaf(f1, po[j], f0 * o[j]);
    l = fmaf(f1, pl, f0 * l);
    m = M;
}

template <int D, int QPI>
__global__ void __launch_bounds__(kWarps * 32, 1) decode_split_kernel(DecodeArgs a) {
    constexpr int HPI = kHeads * QPI;  // query heads per item
    constexpr int KS = D / 16;   // k-steps of q.K = m-tiles of p.V
    constexpr int KB = D / 8;    // key bytes of a lane per token = bytes of a value chunk
    constexpr int EPL = D / 32;  // query elements per lane in the rotation
    constexpr int PQ = 2 * KS;   // output values of a lane per group of heads
    constexpr uint32_t REC = Rec<D>::kBytes;
    using R = Rec<D>;
    using PT = Part<D, QPI>;
    extern __shared__ __align__(128) unsigned char dsm[];

    const int tid = threadIdx.x, lane = tid & 31, wa = tid >> 5;
    const int half = wa / kNW, warp = wa % kNW;
    const int g = lane >> 2, c = lane & 3;
    const uint32_t s0 = smem_u32(dsm);
    const Plan<D, QPI> P(s0);
    if (P.end - s0 > a.smem_bytes) {  // cannot happen with the launcher's size; never touch memory
        if (tid == 0 && blockIdx.x == 0) flag_status(a.status, TQ_STATUS_INTERNAL);
        return;
    }
    const int G = a.Hq / a.Hkv;
    const int stride = kHalves * gridDim.x;  // ranges per round over all halves
    const int v = kHalves * blockIdx.x + half;

    // ---- this warp's ring: kStages record stages, one mbarrier per pair of
    // stages, and the block ids of each stage
    const uint32_t bar0 = P.bars + wa * kPairs * 8;
    const uint32_t idw = P.ids + wa * kStages * 4;
    const uint32_t ringw = P.ring(wa);
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kPairs; s++) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();

    const long long rec_stride = (long long)a.Hkv * REC;  // bytes between blocks of one kv head
    // ---- issue cursor: the next pair of records of this warp's stream (all its
    // segments in order; a pair never spans two segments, so a segment with an
    // odd number of records ends with a single record)
    Seg is;
    seg_range<D>(is, v, a, warp, false);
    while (is.r < a.nranges && is.nk == 0) seg_next<D>(is, stride, a, warp, false);
    int irem = is.nk, ipair = 0, issued = 0;
    const int32_t* ibt = is.bt;
    int nid0 = -1, nid1 = -1;
    if (is.r < a.nranges) {
        nid0 = ibt[0];
        if (irem > 1) nid1 = ibt[kNW];
    }
    // Copy the next pair into pair slot ipair (one elected lane, no branch), note
    // the block ids for the consumer, and move the cursor on.
    auto issue = [&]() {
        if (is.r >= a.nranges) return;
        const int n = irem > 1 ? 2 : 1;
        const uint32_t bar = bar0 + 8 * ipair;
        const uint32_t v0 = (uint32_t)((uint32_t)nid0 < (uint32_t)a.num_blocks);
        const uint32_t v1 = (uint32_t)(n == 2 && (uint32_t)nid1 < (uint32_t)a.num_blocks);
        const uint32_t me = (uint32_t)(lane == 0);
        const uint32_t dst = ringw + (2 * ipair) * REC;
        const unsigned char* src0 = is.src + (long long)nid0 * rec_stride;  // used only if v0
        const unsigned char* src1 = is.src + (long long)nid1 * rec_stride;  // used only if v1
        asm volatile(
            "{\n .reg .pred pm, pa, pz, p0, p1;\n"
            " setp.ne.u32 pm, %0, 0;\n"
            " setp.ne.and.u32 pa, %9, 0, pm;\n"
            " setp.eq.and.u32 pz, %9, 0, pm;\n"
            " setp.ne.and.u32 p0, %1, 0, pm;\n"
            " setp.ne.and.u32 p1, %2, 0, pm;\n"
            " @pa fence.proxy.async.shared::cta;\n"
            " @pa mbarrier.arrive.expect_tx.shared::cta.b64 _, [%3], %9;\n"
            " @pz mbarrier.arrive.shared::cta.b64 _, [%3];\n"
            " @p0 cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%4], [%5], %10, [%3];\n"
            " @p1 cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%6], [%7], %10, [%3];\n"
            " @pm st.shared.v2.b32 [%8], {%11, %12};\n"
            "}\n" ::"r"(me), "r"(v0), "r"(v1), "r"(bar), "r"(dst), "l"(src0), "r"(dst + REC),
            "l"(src1), "r"(idw + 8 * ipair), "r"((v0 + v1) * REC), "r"(REC), "r"(nid0), "r"(nid1)
            : "memory");
        ipair ^= 1;
        issued++;
        irem -= n;
        if (irem == 0) {
            do seg_next<D>(is, stride, a, warp, false);
            while (is.r < a.nranges && is.nk == 0);
            irem = is.nk;
            ibt = is.bt;
        } else {
            ibt += 2 * kNW;
        }
        if (is.r < a.nranges) {
            nid0 = ibt[0];
            nid1 = irem > 1 ? ibt[kNW] : -1;
        }
    };
#pragma unroll 1
    for (int k = 0; k < kPairs; k++) issue();
    __syncwarp();

    // ---- per-lane constants of the consumer
    const uint32_t lanebase = P.lut | ((uint32_t)half << 7) | ((uint32_t)lane << 2);
    const float lo_sel = (float)(g & 1);  // this lane feeds the low part of its head
    const uint32_t lo_mask = (g & 1) ? 0xffffffffu : 0u;
    const uint32_t qsrc = ((g & 1) ? P.ql : P.qh) + (uint32_t)((half * HPI + (g >> 1)) * D * 2);
    const uint32_t mslots = P.merge + half * Plan<D, QPI>::kMergeHalf;
    int slot = 0, consumed = 0;
    uint32_t phase = 0;
    bool aborted = false;
    const uint16_t* lut_tab = nullptr;  // table held by this half's side of the LUT
    const int s_even = 8 * c + (g >> 1), s_odd = s_even + 4;  // weight sources of the p.V operand

    Seg cu;
    seg_range<D>(cu, v, a, warp, warp == 0 && lane == 0);
    bool first_seg = true;
#pragma unroll 1
    for (; cu.r < a.nranges; seg_next<D>(cu, stride, a, warp, warp == 0 && lane == 0)) {
        const int h0 = cu.kv * G + cu.quad * HPI;  // first query head of the item
        const int nh = min(HPI, G - cu.quad * HPI);

        // ---- the centroid-pair table of this kv head, on this half's side of
        // each 256-byte row: word (row, lane) = (C[row & 15], C[row >> 4])
        const uint16_t* tab = a.k_tables ? a.k_tables + cu.kv * 16 : nullptr;
        if (first_seg || tab != lut_tab) {
            first_seg = false;
            lut_tab = tab;
#pragma unroll 1
            for (int r4 = warp; r4 < 64; r4 += kNW) {  // 4 rows per warp and step
                const int row = 4 * r4 + (lane >> 3);
                const uint32_t lo = tab ? tab[row & 15] : a.default_table[row & 15];
                const uint32_t hi = tab ? tab[row >> 4] : a.default_table[row >> 4];
                sts128(P.lut + row * 256 + half * 128 + (lane & 7) * 16, lo | (hi << 16));
            }
        }
        // ---- rotate this item's queries: q~ = H q * scale log2(e) / sqrt(D), as
        // fp16 parts (the half's warps take the heads in turn)
#pragma unroll 1
        for (int hw = warp; hw < HPI; hw += kNW) {
            float x[EPL];
            if (hw < nh) {
                const uint16_t* src = a.q + ((size_t)cu.b * a.Hq + h0 + hw) * D + lane * EPL;
#pragma unroll
                for (int e = 0; e < EPL; e++) x[e] = __uint_as_float((uint32_t)src[e] << 16);
            } else {
#pragma unroll
                for (int e = 0; e < EPL; e++) x[e] = 0.f;
            }
            if (a.rotate) {
#pragma unroll
                for (int m = 1; m < EPL; m <<= 1)
#pragma unroll
                    for (int e = 0; e < EPL; e++)
                        if (!(e & m)) {
                            const float p = x[e], q = x[e | m];
                            x[e] = p + q;
                            x[e | m] = p - q;
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
            }
            // the +-1 butterfly leaves a factor sqrt(D) that the scale takes out
            const float sc = a.rotate ? a.scale_log2 * rsqrtf((float)D) : a.scale_log2;
            const uint32_t dh = P.qh + (uint32_t)(((half * HPI + hw) * D + lane * EPL) * 2);
            const uint32_t dl = P.ql + (uint32_t)(((half * HPI + hw) * D + lane * EPL) * 2);
#pragma unroll
            for (int e = 0; e < EPL; e += 2) {
                const float y0 = x[e] * sc, y1 = x[e + 1] * sc;
                const __half2 hp = __floats2half2_rn(y0, y1);
                const float2 hf = __half22float2(hp);
                sts32(dh + 2 * e, h2u(hp));
                sts32(dl + 2 * e, h2u(__floats2half2_rn(y0 - hf.x, y1 - hf.y)));
            }
        }
        half_sync(half);

        // ---- q.K B fragments of each group q of four heads: column g is head
        // 4q + g/2, its high fp16 part for even g and its low part for odd g;
        // k = 2c, 2c+1 | 2c+8, 2c+9 of step ks are the dims of key bytes
        // j = c*KB + 2ks and j + 1 (a fixed permutation)
        uint32_t qb[QPI][KS][2];
#pragma unroll
        for (int q = 0; q < QPI; q++)
#pragma unroll
            for (int ks = 0; ks < KS; ks++) {
                const uint2 v2 = lds64(qsrc + (uint32_t)(q * kHeads * D * 2) + 4 * (c * KB + 2 * ks));
                qb[q][ks][0] = v2.x;
                qb[q][ks][1] = v2.y;
            }

        // ---- this warp's records of the segment, two per iteration
        float O[QPI][KS][4];  // p.V: rows = dims (16m + 2g, 16m + 2g + 1), cols = head c (hi, lo)
        float Z[QPI][4];      // p.z: rows g = zero sums of group g, rows g + 8 = sum of p
        float mrun[QPI];      // running maximum of head 4q + c
#pragma unroll
        for (int q = 0; q < QPI; q++) {
            mrun[q] = -INFINITY;
#pragma unroll
            for (int i = 0; i < 4; i++) {
                Z[q][i] = 0.f;
#pragma unroll
                for (int m = 0; m < KS; m++) O[q][m][i] = 0.f;
            }
        }
        const int nk = aborted ? 0 : cu.nk;
        // tokens in this warp's last record of the segment (< 16 only at the end of the sequence)
        const int last_valid = cu.L - (cu.jb + warp + kNW * (nk - 1)) * kBlock;
#pragma unroll 1
        for (int k = 0; k < nk; k += 2) {
            if (!mbar_wait_warp(bar0 + 8 * slot, phase)) {
                flag_lane0(a.status, TQ_STATUS_TIMEOUT, lane);
                aborted = true;
                break;
            }
            const uint2 ids = lds64(idw + 8 * slot);
            const bool has1 = k + 1 < nk;
            const bool ok0 = (uint32_t)ids.x < (uint32_t)a.num_blocks;
            const bool ok1 = has1 && (uint32_t)ids.y < (uint32_t)a.num_blocks;
            if (!ok0 || (has1 && !ok1)) flag_lane0(a.status, TQ_STATUS_BAD_BLOCK, lane);
            // valid tokens of the two records (a bad or missing record has none)
            const int n0 = ok0 ? (k == nk - 1 ? last_valid : kBlock) : 0;
            const int n1 = ok1 ? (k + 1 == nk - 1 ? last_valid : kBlock) : 0;
            if (n0 + n1 > 0) {
                const uint32_t rec0 = ringw + (2 * slot) * REC, rec1 = rec0 + REC;
                // -------- q.K of both records
                float sc0[QPI][4], sc1[QPI][4];
                record_scores<D, QPI>(rec0, g, c, lanebase, qb, sc0);
                record_scores<D, QPI>(rec1, g, c, lanebase, qb, sc1);
                // scores of head 4q + c at tokens g and g + 8 (base 2): columns 2c,
                // 2c+1 hold the high and low parts of the query; the norm after the dot
                const uint32_t nw0 = lds32(rec0 + R::kKNorm + 4 * (g >> 1));
                const uint32_t nw0b = lds32(rec0 + R::kKNorm + 16 + 4 * (g >> 1));
                const uint32_t nw1 = lds32(rec1 + R::kKNorm + 4 * (g >> 1));
                const uint32_t nw1b = lds32(rec1 + R::kKNorm + 16 + 4 * (g >> 1));
                const int sh = (g & 1) * 16;
                const float na0 = __half2float(__ushort_as_half((uint16_t)(nw0 >> sh)));
                const float nb0 = __half2float(__ushort_as_half((uint16_t)(nw0b >> sh)));
                const float na1 = __half2float(__ushort_as_half((uint16_t)(nw1 >> sh)));
                const float nb1 = __half2float(__ushort_as_half((uint16_t)(nw1b >> sh)));
                Mask m0 = {true, true, 0xffffffffu, 0xffffffffu}, m1 = m0;
                const bool masked = n0 < kBlock || n1 < kBlock;  // a sequence's last block, or a bad one
                if (masked) {
                    m0 = token_mask(n0, g, c);
                    m1 = token_mask(n1, g, c);
                }

                // -------- online softmax over the 32 tokens (head 4q + c: lanes with
                // the same c), and the weights moved to the p.V operand: head g/2 at
                // tokens 2c, 2c+1, 2c+8, 2c+9 lives in lanes (2c, g/2) and (2c+1, g/2)
                uint32_t u01[2][QPI], w01[2][QPI], u89[2][QPI], w89[2][QPI];
#pragma unroll
                for (int q = 0; q < QPI; q++) {
                    const float xa0 = m0.va ? (sc0[q][0] + sc0[q][1]) * na0 : -INFINITY;
                    const float xb0 = m0.vb ? (sc0[q][2] + sc0[q][3]) * nb0 : -INFINITY;
                    const float xa1 = m1.va ? (sc1[q][0] + sc1[q][1]) * na1 : -INFINITY;
                    const float xb1 = m1.vb ? (sc1[q][2] + sc1[q][3]) * nb1 : -INFINITY;
                    float mx = fmaxf(fmaxf(xa0, xb0), fmaxf(xa1, xb1));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
                    const float mn = fmaxf(mrun[q], mx);
                    if (__any_sync(kFull, mn > mrun[q])) {
                        const float corr = ex2(mrun[q] - mn);
#pragma unroll
                        for (int i = 0; i < 4; i++) {
                            Z[q][i] *= corr;
#pragma unroll
                            for (int m = 0; m < KS; m++) O[q][m][i] *= corr;
                        }
                    }
                    mrun[q] = mn;
                    const float pa0 = ex2(xa0 - mn), pb0 = ex2(xb0 - mn);
                    const float pa1 = ex2(xa1 - mn), pb1 = ex2(xb1 - mn);
                    split_uw(__shfl_sync(kFull, pa0, s_even), __shfl_sync(kFull, pa0, s_odd), lo_sel,
                             lo_mask, u01[0][q], w01[0][q]);
                    split_uw(__shfl_sync(kFull, pb0, s_even), __shfl_sync(kFull, pb0, s_odd), lo_sel,
                             lo_mask, u89[0][q], w89[0][q]);
                    split_uw(__shfl_sync(kFull, pa1, s_even), __shfl_sync(kFull, pa1, s_odd), lo_sel,
                             lo_mask, u01[1][q], w01[1][q]);
                    split_uw(__shfl_sync(kFull, pb1, s_even), __shfl_sync(kFull, pb1, s_odd), lo_sel,
                             lo_mask, u89[1][q], w89[1][q]);
                }

                // -------- p.z, sum p and p.V of both records
                if (masked) {
                    record_values<D, QPI, true>(rec0, g, c, m0.mA, m0.mB, u01[0], w01[0], u89[0], w89[0], O, Z);
                    record_values<D, QPI, true>(rec1, g, c, m1.mA, m1.mB, u01[1], w01[1], u89[1], w89[1], O, Z);
                } else {
                    record_values<D, QPI, false>(rec0, g, c, 0u, 0u, u01[0], w01[0], u89[0], w89[0], O, Z);
                    record_values<D, QPI, false>(rec1, g, c, 0u, 0u, u01[1], w01[1], u89[1], w89[1], O, Z);
                }
            }
            __syncwarp();
            consumed++;
            issue();  // the pair after the ring's last: into the slot just read
            slot ^= 1;
            if (slot == 0) phase ^= 1u;
        }

        // ---- this warp's partial, per group q of heads: the outputs of head
        // 4q + c at dims 16m + 2g, 16m + 2g + 1 (zero-point term added), its
        // sum of weights and its running maximum
        float po[QPI][PQ], pl[QPI];
#pragma unroll
        for (int q = 0; q < QPI; q++) {
            float zs[KS / 2];
#pragma unroll
            for (int G_ = 0; G_ < KS / 2; G_++) zs[G_] = __shfl_sync(kFull, Z[q][0] + Z[q][1], 4 * G_ + c);
#pragma unroll
            for (int m = 0; m < KS; m++) {
                po[q][2 * m] = fmaf(O[q][m][0] + O[q][m][1], 0x1p24f, zs[m >> 1]);
                po[q][2 * m + 1] = fmaf(O[q][m][2] + O[q][m][3], 0x1p20f, zs[m >> 1]);
            }
            pl[q] = Z[q][2] + Z[q][3];
        }

        // ---- merge the half's warps in a tree; warp 0 ends with the sum
#pragma unroll
        for (int k = 0; k < tree_rounds(); k++) {
            const int act = tree_act(k), h = (act + 1) / 2;
            const uint32_t ws = tree_wslot(k);
            if (warp >= h && warp < act) {
                const int sl = (int)((ws >> (4 * warp)) & 15u);
                const uint32_t base = mslots + sl * PT::kSlotBytes + lane * 16;
                float buf[PT::kFloats];
#pragma unroll
                for (int q = 0; q < QPI; q++) {
#pragma unroll
                    for (int j = 0; j < PQ; j++) buf[q * (PQ + 2) + j] = po[q][j];
                    buf[q * (PQ + 2) + PQ] = pl[q];
                    buf[q * (PQ + 2) + PQ + 1] = mrun[q];
                }
#pragma unroll
                for (int j = QPI * (PQ + 2); j < PT::kFloats; j++) buf[j] = 0.f;
#pragma unroll
                for (int j = 0; j < PT::kFloats; j += 4)
                    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(base + (j / 4) * 512),
                                 "f"(buf[j]), "f"(buf[j + 1]), "f"(buf[j + 2]), "f"(buf[j + 3])
                                 : "memory");
            }
            half_sync(half);
            if (warp < act - h) {
                const int sl = (int)((ws >> (4 * (warp + h))) & 15u);
                const uint32_t base = mslots + sl * PT::kSlotBytes + lane * 16;
                float buf[PT::kFloats];
#pragma unroll
                for (int j = 0; j < PT::kFloats; j += 4)
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(buf[j]), "=f"(buf[j + 1]), "=f"(buf[j + 2]), "=f"(buf[j + 3])
                                 : "r"(base + (j / 4) * 512)
                                 : "memory");
#pragma unroll
                for (int q = 0; q < QPI; q++)
                    merge_into<PQ>(mrun[q], pl[q], po[q], buf[q * (PQ + 2) + PQ + 1],
                                   buf[q * (PQ + 2) + PQ], &buf[q * (PQ + 2)]);
            }
        }

        // ---- warp 0 writes the segment's output (a whole item) or its partial
        if (warp == 0) {
#pragma unroll
            for (int q = 0; q < QPI; q++) {
                const int hq = q * kHeads + c;
                if (hq < nh) {
                    if (cu.direct) {
                        float* dst = a.out + ((size_t)cu.b * a.Hq + h0 + hq) * D + 2 * g;
#pragma unroll
                        for (int m = 0; m < KS; m++)
                            *reinterpret_cast<float2*>(dst + 16 * m) =
                                pl[q] > 0.f ? make_float2(po[q][2 * m] / pl[q], po[q][2 * m + 1] / pl[q])
                                            : make_float2(0.f, 0.f);
                    } else {
                        const size_t pr = ((size_t)cu.r * 2 + (cu.i == cu.i_first ? 0 : 1)) * HPI + hq;
                        float* dst = a.ws_o + pr * D + 2 * g;
#pragma unroll
                        for (int m = 0; m < KS; m++)
                            *reinterpret_cast<float2*>(dst + 16 * m) = make_float2(po[q][2 * m], po[q][2 * m + 1]);
                        if (g == 0) a.ws_ml[pr] = make_float2(mrun[q], pl[q]);
                    }
                }
            }
        }
    }

    if (aborted) {  // give the copies still in flight a bounded chance to land
#pragma unroll 1
        for (int j = consumed; j < issued; j++) mbar_wait(bar0 + 8 * (j & 1), (uint32_t)(j >> 1) & 1u);
    }
}

// Items cut by range boundaries: out[b][h] = sum_r 2^(m_r - M) o_r / sum_r 2^(m_r - M) l_r
// over the ranges r that hold part of the item, M = max_r m_r.  Whole items
// were written by the split kernel and are skipped.  One warp per (sequence,
// query head) pair, each lane D / 32 dims; two ranges' loads in flight at once.
template <int D, int QPI>
__global__ void __launch_bounds__(32) combine_kernel(DecodeArgs a) {
    constexpr int HPI = kHeads * QPI;
    constexpr int DPL = D / 32;
    const int lane = threadIdx.x;
    const int G = a.Hq / a.Hkv;
#pragma unroll 1
    for (int bh = blockIdx.x; bh < a.B * a.Hq; bh += gridDim.x) {
        const int b = bh / a.Hq, hh = bh % a.Hq;
        const int kv = hh / G, quad = (hh % G) / HPI, h = (hh % G) % HPI;
        const int item = (b * a.Hkv + kv) * a.quads + quad;
        const int base = item * a.nmax;
        const int rA = base / a.R, rB = (base + a.nmax - 1) / a.R;
        if (rA == rB) continue;  // whole inside one range: already written
        float M = -INFINITY, l = 0.f, o[DPL];
#pragma unroll
        for (int j = 0; j < DPL; j++) o[j] = 0.f;
#pragma unroll 1
        for (int r0 = rA; r0 <= rB; r0 += 2) {  // two ranges' loads in flight at a time
            float2 ml[2];
            float po[2][DPL];
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int r = r0 + u;
                ml[u] = make_float2(-INFINITY, 0.f);
#pragma unroll
                for (int j = 0; j < DPL; j++) po[u][j] = 0.f;
                if (r <= rB) {
                    const int slot = r * a.R / a.nmax == item ? 0 : 1;
                    const size_t pr = ((size_t)r * 2 + slot) * HPI + h;
                    ml[u] = a.ws_ml[pr];
#pragma unroll
                    for (int j = 0; j < DPL; j++) po[u][j] = a.ws_o[pr * D + j * 32 + lane];
                }
            }
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const float Mn = fmaxf(M, ml[u].x);
                const float f0 = M == -INFINITY ? 0.f : ex2(M - Mn);
                const float f1 = ml[u].x == -INFINITY ? 0.f : ex2(ml[u].x - Mn);
#pragma unroll
                for (int j = 0; j < DPL; j++) o[j] = fmaf(f1, po[u][j], f0 * o[j]);
                l = fmaf(f1, ml[u].y, f0 * l);
                M = Mn;
            }
        }
#pragma unroll
        for (int j = 0; j < DPL; j++) a.out[(size_t)bh * D + j * 32 + lane] = l > 0.f ? o[j] / l : 0.f;
    }
}

template <int D, int QPI>
cudaError_t launch_d(DecodeArgs a, int num_sms, cudaStream_t stream) {
    // the kernel's shared-memory size, set once per device (under a lock: the
    // library may be called from several host threads)
    static std::mutex mu;
    static bool configured[64] = {};
    static const uint32_t smem = plan_bytes<D, QPI>();
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (dev < 0 || dev >= 64 || !configured[dev]) {
            e = cudaFuncSetAttribute(decode_split_kernel<D, QPI>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) configured[dev] = true;
        }
    }
    a.smem_bytes = smem;
    const int halves = (a.nranges + kHalves - 1) / kHalves;
    const int grid = halves < num_sms ? halves : num_sms;
    decode_split_kernel<D, QPI><<<grid, kWarps * 32, smem, stream>>>(a);
    if (decode_needs_combine(a)) combine_kernel<D, QPI><<<a.B * a.Hq, 32, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

uint32_t decode_smem_bytes(int head_dim) {  // the largest plan of the head_dim's kernels
    return head_dim == 128 ? plan_bytes<128, 1>() : plan_bytes<64, 2>();
}

// Ranges: with num_splits = 0 the virtual records are cut evenly over every
// half of a full grid; with num_splits = S each range is ceil(nmax / S) records
// (S = 1: one range per item, nothing to combine).
bool decode_plan(DecodeArgs& a, int head_dim, int num_sms) {
    const int G = a.Hq / a.Hkv;
    // at d = 64 an item takes two groups of four query heads when there are more
    // than four per kv head: the record is staged and dequantised once for both
    a.qpi = head_dim == 64 && G > kHeads ? 2 : 1;
    a.quads = (G + kHeads * a.qpi - 1) / (kHeads * a.qpi);
    a.items = a.B * a.Hkv * a.quads;
    a.nmax = a.max_seq_len > 0 ? (a.max_seq_len + kBlock - 1) / kBlock : 1;
    const long long V = (long long)a.items * a.nmax;
    if (V >= (1LL << 30)) return false;
    long long R;
    if (a.num_splits > 0) {
        R = (a.nmax + a.num_splits - 1) / a.num_splits;
    } else {
        const long long H = (long long)kHalves * num_sms;
        R = (V + H - 1) / H;
    }
    if (R < 1) R = 1;
    a.vrec = (int)V;
    a.R = (int)R;
    a.nranges = (int)((V + R - 1) / R);
    a.div_nmax = div_magic((uint32_t)a.nmax);
    a.div_hkv = div_magic((uint32_t)a.Hkv);
    a.div_quads = div_magic((uint32_t)a.quads);
    return true;
}

bool decode_needs_combine(const DecodeArgs& a) { return a.nranges > 1 && a.R % a.nmax != 0; }

size_t decode_workspace_for(const DecodeArgs& a, int head_dim) {
    if (!decode_needs_combine(a)) return 0;
    return (size_t)a.nranges * 2 * kHeads * a.qpi * (head_dim * sizeof(float) + sizeof(float2));
}

cudaError_t launch_decode(const DecodeArgs& args, int head_dim, int num_sms, cudaStream_t stream) {
    DecodeArgs a = args;
    if (num_sms < 1) num_sms = 1;
    if (!decode_plan(a, head_dim, num_sms)) return cudaErrorInvalidValue;
    if (head_dim == 128) return launch_d<128, 1>(a, num_sms, stream);
    return a.qpi == 2 ? launch_d<64, 2>(a, num_sms, stream) : launch_d<64, 1>(a, num_sms, stream);
}

}  // namespace tq
