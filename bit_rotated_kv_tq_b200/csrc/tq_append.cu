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
// Work split: one vector (token, kv head) is spread over D/8 lanes holding 8
// elements each, so a warp handles 2 (D=128) or 4 (D=64) vectors per pass;
// loads are 16-byte per lane and fully coalesced.  The grid is persistent
// (one wave of resident CTAs) and every warp loads its next pass before it
// computes the current one, so the global-load latency overlaps the math.
// The rotation is an in-register butterfly over 3 index bits plus
// xor-shuffles over the lane bits (a sign-FMA per element and stage).
//
// Exactness: the fast path runs in fp32.  Every decision it takes (fp16
// rounding of the norm, the nearest centroid, the rounding of (v - z)/s and
// the fp16 rounding up of the scale) is re-taken in fp64 from the bf16
// inputs whenever the fp32 input lies inside the fp32 error bound of the
// decision threshold.  The fp64 recomputation forms the +-1 Hadamard sums
// exactly and divides once by n*sqrt(D), which is the definition evaluated
// with exact sums, so the stored codes are those of the exact-arithmetic
// definition except within ~1e-15 of a threshold.
#include "tq_kernels.cuh"

namespace tq {

// Relative margin on the norm before its fp16 rounding (fp32 sum of squares
// of at most 128 exact products: error <= 11 ulp relative, 6.6e-7).
constexpr float kNormMargin = 1.5e-6f;
// Margin, in value-code units, around the .5 rounding points of (v - z)/s
// (fp32 error <= 3 ulp of 15, i.e. 2.7e-6).
constexpr float kValueMargin = 1.0f / 4096.0f;

// Bin tables in shared memory (called by the whole CTA).  Without per-head
// tables every head uses the default table, whose bins the launcher computed
// once on the host: they are copied, and every head indexes them as head 0.
// Per-head tables are binned here, one thread per (head, bin).
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

// 1/x by the hardware approximation (relative error ~2^-22): (v - z) * (1/s)
// then errs by < 15 * 2^-21 code units, far inside kValueMargin
__device__ __forceinline__ float fast_rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// fp32 neighbours of 1/15: the value rounded up and rounded down.
__device__ __forceinline__ float inv15_up() { return __uint_as_float(0x3d888889u); }
__device__ __forceinline__ float inv15_dn() { return __uint_as_float(0x3d888888u); }

// One warp pass's inputs (prefetched one pass ahead).
struct Pass {
    uint4 k, v;  // this lane's 8 bf16 keys / values
    int slot;    // slot_mapping entry of the token (-1: skip)
    int pb;      // physical block read from the block table (when one is given)
    uint32_t vec;
    bool in;
};

template <int D>
__device__ __forceinline__ void load_pass(const AppendArgs& a, uint32_t p, uint32_t npass,
                                          uint32_t total, int grp, int sub, Pass& L) {
    constexpr int VPW = 32 / (D / 8);
    L.vec = p * VPW + grp;
    L.in = p < npass && L.vec < total;
    L.slot = -1;
    L.pb = -1;
    L.k = make_uint4(0, 0, 0, 0);
    L.v = make_uint4(0, 0, 0, 0);
    if (L.in) {
        const uint32_t t = fast_div(L.vec, a.div_hkv);
        L.slot = __ldg(a.slots + t);
        const size_t eoff = (size_t)L.vec * D + sub * 8;  // vec = t * Hkv + h
        L.k = ld_stream_u4(a.K + eoff);
        L.v = ld_stream_u4(a.V + eoff);
    }
}

// With a block table, fetch the physical block of the pass's slot (issued one
// pass before it is used).
__device__ __forceinline__ void fetch_block(const AppendArgs& a, Pass& L) {
    if (a.block_table && L.in && L.slot >= 0) {
        const uint32_t s = (uint32_t)L.slot;
        const uint32_t seq = fast_div(s, a.div_cap);
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
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// 1.5 * 2^23: x + kRound rounds x (0 <= x < 2^22) to the nearest integer,
// ties to even, and leaves that integer in the low mantissa bits.
constexpr float kRound = 12582912.0f;

template <int D>
__global__ void __launch_bounds__(256, 3) append_kernel(AppendArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    HeadBins* hb = reinterpret_cast<HeadBins*>(smem);
    BinEntry* bins = reinterpret_cast<BinEntry*>(hb + a.Hkv);

    constexpr int LPV = D / 8;     // lanes per vector
    constexpr int VPW = 32 / LPV;  // vectors per warp pass
    using R = Rec<D>;
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPV;
    const int grp = lane / LPV;
    const uint32_t total = (uint32_t)a.T * (uint32_t)a.Hkv;
    const uint32_t npass = (total + VPW - 1) / VPW;
    const uint32_t nwarps = gridDim.x * (blockDim.x / 32);
    const uint32_t cap = (uint32_t)(a.max_blocks * kBlock);

    // the first pass's loads go out before the bins are built, so the two overlap
    Pass cur, nxt;
    uint32_t pass = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    load_pass<D>(a, pass, npass, total, grp, sub, cur);
    build_bins(hb, bins, a);
    fetch_block(a, cur);

    for (; pass < npass; pass += nwarps) {
        load_pass<D>(a, pass + nwarps, npass, total, grp, sub, nxt);
        const uint32_t t = fast_div(cur.vec, a.div_hkv);
        const int h = cur.in ? (int)(cur.vec - t * (uint32_t)a.Hkv) : 0;

        // ---- key: norm (elements 2i, 2i+1 in P[i])
        float2 P[4];
        P[0] = make_float2(bf16_lo(cur.k.x), bf16_hi(cur.k.x));
        P[1] = make_float2(bf16_lo(cur.k.y), bf16_hi(cur.k.y));
        P[2] = make_float2(bf16_lo(cur.k.z), bf16_hi(cur.k.z));
        P[3] = make_float2(bf16_lo(cur.k.w), bf16_hi(cur.k.w));
        float2 q2 = mul2(P[0], P[0]);
        q2 = __ffma2_rn(P[1], P[1], q2);
        q2 = __ffma2_rn(P[2], P[2], q2);
        q2 = __ffma2_rn(P[3], P[3], q2);
        float ss = q2.x + q2.y;
#pragma unroll
        for (int m = 1; m < LPV; m <<= 1) ss += __shfl_xor_sync(kFull, ss, m);
        const float n = sqrtf(ss);
        uint16_t n16 = __half_as_ushort(__float2half_rn(n));
        bool near = __half_as_ushort(__float2half_rn(n * (1.0f - kNormMargin))) !=
                    __half_as_ushort(__float2half_rn(n * (1.0f + kNormMargin)));
        // squares that leave the normal fp32 range (or a non-finite key) lose the
        // fp32 error bound: take the fp64 path
        near |= !(ss >= 1e-30f && ss <= 1e30f) && ss != 0.f;

        // ---- key: unnormalised Hadamard butterfly.  Index bit 0 lies inside a
        // pair, bits 1-2 across pairs (packed adds), the rest across lanes.
        float2 Q[4];
#pragma unroll
        for (int i = 0; i < 4; i++) Q[i] = make_float2(P[i].x + P[i].y, P[i].x - P[i].y);
        {
            const float2 a0 = add2(Q[0], Q[1]), a1 = sub2(Q[0], Q[1]);
            const float2 a2 = add2(Q[2], Q[3]), a3 = sub2(Q[2], Q[3]);
            Q[0] = add2(a0, a2); Q[2] = sub2(a0, a2);
            Q[1] = add2(a1, a3); Q[3] = sub2(a1, a3);
        }
#pragma unroll
        for (int m = 1; m < LPV; m <<= 1) {
            const float sg = (sub & m) ? -1.f : 1.f;  // upper half: partner - own
            const float2 sg2 = make_float2(sg, sg);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float2 pr = make_float2(__shfl_xor_sync(kFull, Q[i].x, m),
                                              __shfl_xor_sync(kFull, Q[i].y, m));
                Q[i] = __ffma2_rn(sg2, Q[i], pr);
            }
        }
        const float inv = ss > 0.f ? rsqrtf(ss * (float)D) : 0.f;

        // ---- key: nearest centroid through the per-head bins
        const int hs = a.k_tables ? h : 0;  // whose bins (one shared set without per-head tables)
        const HeadBins& B = hb[hs];
        const BinEntry* hbins = bins + hs * kBins;
        uint32_t kw = 0;
        float y[8];
        {
            const float2 inv2 = make_float2(inv, inv);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float2 yy = mul2(Q[i], inv2);
                y[2 * i] = yy.x;
                y[2 * i + 1] = yy.y;
            }
        }
        if (!B.dense) {
            uint32_t nib[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float2 ps = __ffma2_rn(make_float2(y[2 * i], y[2 * i + 1]),
                                            make_float2(kBinScale, kBinScale),
                                            make_float2(kBinScale, kBinScale));
                const int b0 = max(min((int)ps.x, kBins - 1), 0);
                const int b1 = max(min((int)ps.y, kBins - 1), 0);
                const BinEntry e0 = hbins[b0], e1 = hbins[b1];
                const float d0 = y[2 * i] - e0.mid, d1 = y[2 * i + 1] - e1.mid;
                nib[2 * i] = (uint32_t)(e0.k_lo + (d0 > 0.f ? 1 : 0));
                nib[2 * i + 1] = (uint32_t)(e1.k_lo + (d1 > 0.f ? 1 : 0));
                near |= fmaxf(fabsf(d0), fabsf(d1)) < kKeyMargin;
            }
            // bytes (nib[2j] | nib[2j+1] << 4), j = 0..3, into one word
            const uint32_t b01 = __byte_perm(nib[0] | (nib[1] << 4), nib[2] | (nib[3] << 4), 0x0040);
            const uint32_t b23 = __byte_perm(nib[4] | (nib[5] << 4), nib[6] | (nib[7] << 4), 0x0040);
            kw = __byte_perm(b01, b23, 0x5410);
        } else {
#pragma unroll
            for (int e = 0; e < 8; e++) {
                int idx = 0;
                for (int j = 0; j < 15; j++) {
                    const float dm = y[e] - 0.5f * (B.c[j] + B.c[j + 1]);
                    idx += dm > 0.f ? 1 : 0;
                    near |= fabsf(dm) < kKeyMargin;
                }
                kw |= (uint32_t)idx << (4 * e);
            }
        }
        near = near && cur.in && cur.slot >= 0;

        // ---- key: fp64 recomputation when any decision of the warp is close
        if (__any_sync(kFull, near)) {
            double Sd[8];
            double ssd = 0.0;
#pragma unroll
            for (int i = 0; i < 4; i++) {
                Sd[2 * i] = (double)P[i].x;
                Sd[2 * i + 1] = (double)P[i].y;
            }
#pragma unroll
            for (int e = 0; e < 8; e++) ssd = fma(Sd[e], Sd[e], ssd);
#pragma unroll
            for (int m = 1; m < LPV; m <<= 1) ssd += __shfl_xor_sync(kFull, ssd, m);
            const double nd = sqrt(ssd);
#pragma unroll
            for (int b = 1; b < 8; b <<= 1) {
#pragma unroll
                for (int e = 0; e < 8; e++)
                    if (!(e & b)) {
                        const double x = Sd[e], yv = Sd[e | b];
                        Sd[e] = x + yv;
                        Sd[e | b] = x - yv;
                    }
            }
#pragma unroll
            for (int m = 1; m < LPV; m <<= 1) {
                const bool upper = sub & m;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    const double p = __shfl_xor_sync(kFull, Sd[e], m);
                    Sd[e] = upper ? p - Sd[e] : Sd[e] + p;
                }
            }
            if (cur.in) {
                n16 = __half_as_ushort(__double2half(nd));
                const double denom = nd * sqrt((double)D);
                kw = 0;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    const double yd = nd > 0.0 ? Sd[e] / denom : 0.0;
                    int idx = 0;
                    for (int j = 0; j < 15; j++)
                        idx += yd > 0.5 * ((double)B.c[j] + (double)B.c[j + 1]) ? 1 : 0;
                    kw |= (uint32_t)idx << (4 * e);
                }
            }
        }

        // the next pass's block-table entry: its slot has arrived by now, and the
        // lookup overlaps this pass's value work and stores
        fetch_block(a, nxt);

        // ---- values: group of 32 = 4 lanes
        float2 V2[4];
        V2[0] = make_float2(bf16_lo(cur.v.x), bf16_hi(cur.v.x));
        V2[1] = make_float2(bf16_lo(cur.v.y), bf16_hi(cur.v.y));
        V2[2] = make_float2(bf16_lo(cur.v.z), bf16_hi(cur.v.z));
        V2[3] = make_float2(bf16_lo(cur.v.w), bf16_hi(cur.v.w));
        float mn = fminf(fminf(fminf(V2[0].x, V2[0].y), fminf(V2[1].x, V2[1].y)),
                         fminf(fminf(V2[2].x, V2[2].y), fminf(V2[3].x, V2[3].y)));
        float mx = fmaxf(fmaxf(fmaxf(V2[0].x, V2[0].y), fmaxf(V2[1].x, V2[1].y)),
                         fmaxf(fmaxf(V2[2].x, V2[2].y), fmaxf(V2[3].x, V2[3].y)));
#pragma unroll
        for (int m = 1; m < 4; m <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(kFull, mn, m));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
        }
        const __half zh = __float2half_rd(mn);  // exact: mn is a bf16 value
        const float zf = __half2float(zh);
        // s = fp16 rounded up from (mx - z)/15: bracket the quotient in fp32 with
        // directed roundings; if both ends round up to the same fp16 value it is
        // the answer, otherwise (an fp16 value inside the bracket) use fp64.
        uint16_t s16;
        {
            const float hi = __fmul_ru(__fsub_ru(mx, zf), inv15_up());
            const float lo = __fmul_rd(__fsub_rd(mx, zf), inv15_dn());
            const uint16_t s_hi = __half_as_ushort(__float2half_ru(hi));
            const uint16_t s_lo = __half_as_ushort(__float2half_ru(lo));
            s16 = s_hi;
            if (s_hi != s_lo) s16 = double_to_half_up_nonneg(((double)mx - (double)zf) / 15.0);
        }
        const float sf = half_bits_to_float(s16);
        uint32_t vw = 0;
        if (sf > 0.f) {
            const float inv_s = fast_rcp(sf);  // its error is far inside kValueMargin
            const float2 z2 = make_float2(zf, zf), is2 = make_float2(inv_s, inv_s);
            const float2 rnd = make_float2(kRound, kRound);
            uint32_t qb[8];
            bool tie = false;
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float2 r = mul2(sub2(V2[i], z2), is2);  // (v - z) / s, in [0, 15]
                const float2 tr = add2(r, rnd);               // round half to even
                const float2 d = sub2(r, sub2(tr, rnd));      // r - round(r)
                tie |= fmaxf(fabsf(d.x), fabsf(d.y)) > 0.5f - kValueMargin;
                qb[2 * i] = __float_as_uint(tr.x);            // low byte = code
                qb[2 * i + 1] = __float_as_uint(tr.y);
            }
            if (tie) {  // a .5 point within the fp32 error: exact quotients in fp64
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    qb[2 * i] = (uint32_t)rint(((double)V2[i].x - (double)zf) / (double)sf);
                    qb[2 * i + 1] = (uint32_t)rint(((double)V2[i].y - (double)zf) / (double)sf);
                }
            }
            const uint32_t even = __byte_perm(__byte_perm(qb[0], qb[2], 0x0040),
                                              __byte_perm(qb[4], qb[6], 0x0040), 0x5410);
            const uint32_t odd = __byte_perm(__byte_perm(qb[1], qb[3], 0x0040),
                                             __byte_perm(qb[5], qb[7], 0x0040), 0x5410);
            vw = ((even & 0x0f0f0f0fu) | ((odd & 0x0f0f0f0fu) << 4));
        }

        // ---- where this vector goes (the block-table read was issued a pass ago)
        int blk = -1, off = 0;
        if (cur.in && cur.slot >= 0) {
            if (a.block_table) {
                if (cur.pb >= 0 && cur.pb < a.num_blocks) {
                    blk = cur.pb;
                    off = (int)(((uint32_t)cur.slot - fast_div((uint32_t)cur.slot, a.div_cap) * cap) %
                                kBlock);
                } else if (sub == 0) {
                    flag_status(a.status, cur.pb == -2 ? TQ_STATUS_BAD_SLOT : TQ_STATUS_BAD_BLOCK);
                }
            } else if (cur.slot / kBlock < a.num_blocks) {
                blk = cur.slot / kBlock;
                off = cur.slot % kBlock;
            } else if (sub == 0) {
                flag_status(a.status, TQ_STATUS_BAD_SLOT);
            }
        }
        if (blk >= 0) {
            unsigned char* rec = a.cache + ((size_t)blk * a.Hkv + h) * (size_t)R::kBytes;
            *reinterpret_cast<uint32_t*>(rec + R::kKCodes + off * R::kCodeRow + sub * 4) = kw;
            // bytes j = 4 sub + i share m = sub / 2 and spread over r = 4 (sub % 2) + i
            unsigned char* vdst = rec + R::kVCodes + R::vcode_pos(off, 4 * sub);
#pragma unroll
            for (int i = 0; i < 4; i++) vdst[i * R::kPairChunk] = (unsigned char)(vw >> (8 * i));
            if (sub == 0) *reinterpret_cast<uint16_t*>(rec + R::kKNorm + off * 2) = n16;
            if ((sub & 3) == 0) {
                const int gp = R::group_pos(off, sub / 4);
                *reinterpret_cast<uint16_t*>(rec + R::kVScale + gp) = s16;
                *reinterpret_cast<uint16_t*>(rec + R::kVZero + gp) = __half_as_ushort(zh);
                const bool bad = !isfinite(sf) || !isfinite(zf) ||
                                 (sub == 0 && !isfinite(half_bits_to_float(n16)));
                if (bad) flag_status(a.status, TQ_STATUS_RANGE);
            }
        }

        cur = nxt;
    }
}

size_t append_smem_bytes(int Hkv) {
    return (size_t)Hkv * sizeof(HeadBins) + (size_t)Hkv * kBins * sizeof(BinEntry);
}


template <int D>
static int resident_ctas(int num_sms, size_t smem) {
    static int per_sm[2] = {0, 0};  // by (smem size class); set once per process
    const int key = smem > 16384 ? 1 : 0;
    if (!per_sm[key]) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, append_kernel<D>, 256, smem) !=
                cudaSuccess || n <= 0)
            n = 1;
        per_sm[key] = n;
    }
    return per_sm[key] * num_sms;
}

// The bins of the default table of head_dim d, computed once per process.
static void default_bins(int d, const uint16_t* table16, HeadBins& hb, BinEntry* bins) {
    static HeadBins cached_hb[2];
    static BinEntry cached[2][kBins];
    static bool ready[2] = {false, false};
    const int key = d == 128 ? 1 : 0;
    if (!ready[key]) {
        HeadBins& h = cached_hb[key];
        for (int k = 0; k < 16; k++) h.c[k] = __half2float(__ushort_as_half(table16[k]));
        h.dense = 0;
        h.pad = 0;
        for (int b = 0; b < kBins; b++)
            if (bin_entry(h.c, b, cached[key][b])) h.dense = 1;
        ready[key] = true;
    }
    hb = cached_hb[key];
    memcpy(bins, cached[key], sizeof cached[key]);
}

cudaError_t launch_append(const AppendArgs& args, int head_dim, int num_sms, cudaStream_t stream) {
    AppendArgs a = args;
    if (!a.k_tables) default_bins(head_dim, a.default_table, a.default_hb, a.default_bins);
    a.div_hkv = div_magic((uint32_t)a.Hkv);
    a.div_cap = div_magic((uint32_t)(a.max_blocks > 0 ? a.max_blocks * kBlock : 1));
    const int threads = 256;
    const long long vectors = (long long)a.T * a.Hkv;
    const int vpw = 32 / (head_dim / 8);
    const long long warps_needed = (vectors + vpw - 1) / vpw;
    long long blocks = (warps_needed + threads / 32 - 1) / (threads / 32);
    const size_t smem = append_smem_bytes(a.Hkv);
    const long long cap = head_dim == 128 ? resident_ctas<128>(num_sms, smem)
                                          : resident_ctas<64>(num_sms, smem);
    if (blocks > cap) blocks = cap;  // one wave; warps loop over the passes
    if (blocks < 1) blocks = 1;
    if (head_dim == 128)
        append_kernel<128><<<(unsigned)blocks, threads, smem, stream>>>(a);
    else
        append_kernel<64><<<(unsigned)blocks, threads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace tq
