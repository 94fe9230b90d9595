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
// loads are 16-byte per lane and fully coalesced.  The rotation is an in-
// register butterfly over 3 index bits plus xor-shuffles over the rest.
//
// Exactness: the fast path runs in fp32.  Every decision it takes (fp16
// rounding of the norm, the nearest centroid, the rounding of (v - z)/s) is
// re-taken in fp64 from the bf16 inputs whenever the fp32 input lies inside
// the fp32 error bound of the decision threshold.  The fp64 recomputation
// forms the +-1 Hadamard sums exactly and divides once by n*sqrt(D), which is
// the definition evaluated with exact sums, so the stored codes are those of
// the exact-arithmetic definition except within ~1e-15 of a threshold.
#include "tq_kernels.cuh"

namespace tq {

// Absolute margin, in rotated unit-vector units, inside which an fp32
// centroid decision is re-taken in fp64.  The fp32 butterfly of a bf16 key
// followed by one scaling is accurate to ~1.3e-6 in the worst case
// (7 stages, rsqrt within 2 ulp); typical errors are ~1e-7.
constexpr float kKeyMargin = 3.0e-6f;
// Relative margin on the norm before its fp16 rounding (fp32 sum of squares
// of at most 128 exact products: error <= 11 ulp relative, 6.6e-7).
constexpr float kNormMargin = 1.5e-6f;
// Margin, in value-code units, around the .5 rounding points of (v - z)/s
// (fp32 error <= 3 ulp of 15, i.e. 2.7e-6).
constexpr float kValueMargin = 1.0f / 4096.0f;

constexpr int kBins = 128;  // uniform bins over the midpoint range, per head

struct HeadBins {
    float c[16];    // the head's table
    float mid[16];  // fp32 midpoints m_0..m_14; mid[15] = +inf
    float lo, inv_w, w;
    int dense;      // 1: some bin holds more than one midpoint -> exact count path
};
struct BinEntry {
    float mid;  // the one midpoint inside the bin (with margins), or +inf
    int k_lo;   // number of midpoints strictly below the bin
};

// Build the per-head bin tables in shared memory (called by the whole CTA).
__device__ void build_bins(HeadBins* hb, BinEntry* bins, int Hkv, const uint16_t* k_tables,
                           const uint16_t* default_table) {
    for (int h = threadIdx.x; h < Hkv; h += blockDim.x) {
        HeadBins& b = hb[h];
        const uint16_t* src = k_tables ? k_tables + 16 * h : default_table;
        for (int k = 0; k < 16; k++) b.c[k] = half_bits_to_float(src[k]);
        for (int k = 0; k < 15; k++) b.mid[k] = 0.5f * (b.c[k] + b.c[k + 1]);
        b.mid[15] = __int_as_float(0x7f800000);
        float range = b.mid[14] - b.mid[0];
        float w = (range > 0.f ? range : 1e-3f) / (kBins - 4);
        b.w = w;
        b.inv_w = 1.0f / w;
        b.lo = b.mid[0] - 2.0f * w;
        b.dense = 0;
    }
    __syncthreads();
    const float delta = 2.0f * kKeyMargin;
    for (int e = threadIdx.x; e < Hkv * kBins; e += blockDim.x) {
        int h = e / kBins, bin = e % kBins;
        const HeadBins& b = hb[h];
        float ext_lo = b.lo + bin * b.w - delta;
        float ext_hi = b.lo + (bin + 1) * b.w + delta;
        int below = 0, inside = 0;
        float m_in = __int_as_float(0x7f800000);
        for (int k = 0; k < 15; k++) {
            float m = b.mid[k];
            if (m < ext_lo) below++;
            else if (m <= ext_hi) { inside++; m_in = m; }
        }
        bins[e].mid = m_in;
        bins[e].k_lo = below;
        if (inside > 1) hb[h].dense = 1;  // benign race: every writer stores 1
    }
    __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    HeadBins* hb = reinterpret_cast<HeadBins*>(smem);
    BinEntry* bins = reinterpret_cast<BinEntry*>(hb + a.Hkv);
    build_bins(hb, bins, a.Hkv, a.k_tables, a.default_table);

    constexpr int LPV = D / 8;      // lanes per vector
    constexpr int VPW = 32 / LPV;   // vectors per warp pass
    using R = Rec<D>;
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPV;
    const int grp = lane / LPV;
    const long long total = (long long)a.T * a.Hkv;
    const long long warps = (long long)gridDim.x * (blockDim.x / 32);
    const long long warp_id = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;

    for (long long base = warp_id * VPW; base < total; base += warps * VPW) {
        const long long vec = base + grp;
        int t = 0, h = 0, blk = -1, off = 0;
        if (vec < total) {
            t = (int)(vec / a.Hkv);
            h = (int)(vec - (long long)t * a.Hkv);
            int s = a.slots[t];
            if (s >= 0) {
                if (a.block_table) {
                    long long cap = (long long)a.max_blocks * kBlock;
                    long long seq = s / cap, pos = s - seq * cap;
                    if (seq < a.num_seqs) {
                        int pb = a.block_table[seq * a.max_blocks + pos / kBlock];
                        if (pb >= 0 && pb < a.num_blocks) {
                            blk = pb;
                            off = (int)(pos % kBlock);
                        } else if (sub == 0) {
                            flag_status(a.status, TQ_STATUS_BAD_BLOCK);
                        }
                    } else if (sub == 0) {
                        flag_status(a.status, TQ_STATUS_BAD_SLOT);
                    }
                } else {
                    if (s / kBlock < a.num_blocks) {
                        blk = s / kBlock;
                        off = s % kBlock;
                    } else if (sub == 0) {
                        flag_status(a.status, TQ_STATUS_BAD_SLOT);
                    }
                }
            }
        }
        const bool work = blk >= 0;
        // every lane takes part in the shuffles; lanes without work carry zeros
        uint4 kraw = make_uint4(0, 0, 0, 0), vraw = make_uint4(0, 0, 0, 0);
        if (work) {
            const size_t eoff = ((size_t)t * a.Hkv + h) * D + sub * 8;
            kraw = ld_stream_u4(a.K + eoff);
            vraw = ld_stream_u4(a.V + eoff);
        }
        float k[8];
        k[0] = bf16_lo(kraw.x); k[1] = bf16_hi(kraw.x);
        k[2] = bf16_lo(kraw.y); k[3] = bf16_hi(kraw.y);
        k[4] = bf16_lo(kraw.z); k[5] = bf16_hi(kraw.z);
        k[6] = bf16_lo(kraw.w); k[7] = bf16_hi(kraw.w);

        // ---- key: norm
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; e++) ss = fmaf(k[e], k[e], ss);
#pragma unroll
        for (int m = 1; m < LPV; m <<= 1) ss += __shfl_xor_sync(kFull, ss, m);
        const float n = sqrtf(ss);
        uint16_t n16 = __half_as_ushort(__float2half_rn(n));
        bool near = __half_as_ushort(__float2half_rn(n * (1.0f - kNormMargin))) !=
                    __half_as_ushort(__float2half_rn(n * (1.0f + kNormMargin)));
        // squares that leave the normal fp32 range (or a non-finite key) lose the
        // fp32 error bound: take the fp64 path
        near |= !(ss >= 1e-30f && ss <= 1e30f) && ss != 0.f;

        // ---- key: unnormalised Hadamard butterfly (3 in-lane bits, log2(LPV) lane bits)
        float S[8];
#pragma unroll
        for (int e = 0; e < 8; e++) S[e] = k[e];
#pragma unroll
        for (int b = 1; b < 8; b <<= 1) {
#pragma unroll
            for (int e = 0; e < 8; e++)
                if (!(e & b)) {
                    float x = S[e], y = S[e | b];
                    S[e] = x + y;
                    S[e | b] = x - y;
                }
        }
#pragma unroll
        for (int m = 1; m < LPV; m <<= 1) {
            const bool upper = sub & m;
#pragma unroll
            for (int e = 0; e < 8; e++) {
                float p = __shfl_xor_sync(kFull, S[e], m);
                S[e] = upper ? p - S[e] : S[e] + p;
            }
        }
        const float inv = ss > 0.f ? rsqrtf(ss * (float)D) : 0.f;

        // ---- key: nearest centroid through the per-head bins
        const HeadBins& B = hb[h];
        const BinEntry* hbins = bins + h * kBins;
        uint32_t kw = 0;
        if (!B.dense) {
#pragma unroll
            for (int e = 0; e < 8; e++) {
                float y = S[e] * inv;
                float pos = fminf(fmaxf((y - B.lo) * B.inv_w, 0.f), (float)(kBins - 1));
                BinEntry be = hbins[(int)pos];
                int idx = be.k_lo + (y > be.mid ? 1 : 0);
                near |= fabsf(y - be.mid) < kKeyMargin;
                kw |= (uint32_t)idx << (4 * e);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; e++) {
                float y = S[e] * inv;
                int idx = 0;
                for (int j = 0; j < 15; j++) {
                    idx += y > B.mid[j] ? 1 : 0;
                    near |= fabsf(y - B.mid[j]) < kKeyMargin;
                }
                kw |= (uint32_t)idx << (4 * e);
            }
        }
        near = near && work;

        // ---- key: fp64 recomputation when any decision of the warp is close
        if (__any_sync(kFull, near)) {
            double kd[8], Sd[8];
            double ssd = 0.0;
#pragma unroll
            for (int e = 0; e < 8; e++) {
                kd[e] = (double)k[e];
                ssd = fma(kd[e], kd[e], ssd);
                Sd[e] = kd[e];
            }
#pragma unroll
            for (int m = 1; m < LPV; m <<= 1) ssd += __shfl_xor_sync(kFull, ssd, m);
            const double nd = sqrt(ssd);
#pragma unroll
            for (int b = 1; b < 8; b <<= 1) {
#pragma unroll
                for (int e = 0; e < 8; e++)
                    if (!(e & b)) {
                        double x = Sd[e], y = Sd[e | b];
                        Sd[e] = x + y;
                        Sd[e | b] = x - y;
                    }
            }
#pragma unroll
            for (int m = 1; m < LPV; m <<= 1) {
                const bool upper = sub & m;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    double p = __shfl_xor_sync(kFull, Sd[e], m);
                    Sd[e] = upper ? p - Sd[e] : Sd[e] + p;
                }
            }
            if (work) {
                n16 = __half_as_ushort(__double2half(nd));
                const double denom = nd * sqrt((double)D);
                kw = 0;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    double y = nd > 0.0 ? Sd[e] / denom : 0.0;
                    int idx = 0;
                    for (int j = 0; j < 15; j++)
                        idx += y > 0.5 * ((double)B.c[j] + (double)B.c[j + 1]) ? 1 : 0;
                    kw |= (uint32_t)idx << (4 * e);
                }
            }
        }

        // ---- values: group of 32 = 4 lanes
        float v[8];
        v[0] = bf16_lo(vraw.x); v[1] = bf16_hi(vraw.x);
        v[2] = bf16_lo(vraw.y); v[3] = bf16_hi(vraw.y);
        v[4] = bf16_lo(vraw.z); v[5] = bf16_hi(vraw.z);
        v[6] = bf16_lo(vraw.w); v[7] = bf16_hi(vraw.w);
        float mn = v[0], mx = v[0];
#pragma unroll
        for (int e = 1; e < 8; e++) {
            mn = fminf(mn, v[e]);
            mx = fmaxf(mx, v[e]);
        }
#pragma unroll
        for (int m = 1; m < 4; m <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(kFull, mn, m));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
        }
        const __half zh = __float2half_rd(mn);  // exact: mn is a bf16 value
        const float zf = __half2float(zh);
        const uint16_t s16 = double_to_half_up_nonneg(((double)mx - (double)zf) / 15.0);
        const float sf = half_bits_to_float(s16);
        uint32_t vw = 0;
        if (sf > 0.f) {
            const float inv_s = 1.0f / sf;
#pragma unroll
            for (int e = 0; e < 8; e++) {
                float r = (v[e] - zf) * inv_s;
                unsigned q;
                if (fabsf(r - floorf(r) - 0.5f) < kValueMargin) {
                    // near a .5 rounding point: exact quotient in fp64
                    double rd = ((double)v[e] - (double)zf) / (double)sf;
                    q = (unsigned)rint(rd);
                } else {
                    q = __float2uint_rn(r);
                }
                vw |= (q > 15u ? 15u : q) << (4 * e);
            }
        }

        if (work) {
            unsigned char* rec =
                a.cache + ((size_t)blk * a.Hkv + h) * (size_t)R::kBytes;
            *reinterpret_cast<uint32_t*>(rec + R::kKCodes + off * R::kCodeRow + sub * 4) = kw;
            unsigned char* vrow = rec + R::kVCodes + off * R::kCodeRow;
#pragma unroll
            for (int i = 0; i < 4; i++) vrow[R::vpos(sub * 4 + i)] = (unsigned char)(vw >> (8 * i));
            if (sub == 0) *reinterpret_cast<uint16_t*>(rec + R::kKNorm + off * 2) = n16;
            if ((sub & 3) == 0) {
                const uint16_t z16 = __half_as_ushort(zh);
                *reinterpret_cast<uint32_t*>(rec + R::kVGroups +
                                             (off * R::kGroups + sub / 4) * 4) =
                    (uint32_t)s16 | ((uint32_t)z16 << 16);
                bool bad = !isfinite(sf) || !isfinite(zf) ||
                           (sub == 0 && !isfinite(half_bits_to_float(n16)));
                if (bad) flag_status(a.status, TQ_STATUS_RANGE);
            }
        }
    }
}

size_t append_smem_bytes(int Hkv) {
    return (size_t)Hkv * sizeof(HeadBins) + (size_t)Hkv * kBins * sizeof(BinEntry);
}

cudaError_t launch_append(const AppendArgs& a, int head_dim, int num_sms, cudaStream_t stream) {
    const int threads = 256;
    const long long vectors = (long long)a.T * a.Hkv;
    const int vpw = 32 / (head_dim / 8);
    long long warps_needed = (vectors + vpw - 1) / vpw;
    long long blocks = (warps_needed + threads / 32 - 1) / (threads / 32);
    const long long cap = (long long)num_sms * 8;  // grid-stride beyond 8 CTAs per SM
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const size_t smem = append_smem_bytes(a.Hkv);
    if (head_dim == 128) {
        append_kernel<128><<<(unsigned)blocks, threads, smem, stream>>>(a);
    } else {
        append_kernel<64><<<(unsigned)blocks, threads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace tq
