// tq_prefill.cu -- chunked-prefill attention over the TQ4/4 cache on the
// fifth-generation tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// A prompt chunk of q_len tokens is appended to the cache first (the same
// order as the decode: tq_quantize_append, then attention); chunk token i of
// sequence b then attends to the cached positions 0 .. L_b - q_len + i.  Many
// queries share every cached block here, so the work is a dense contraction
// and runs on tcgen05: one CTA takes a tile of 128 query rows -- (chunk token,
// query head) pairs of one kv head -- and walks the sequence's blocks in steps
// of 64 tokens:
//   1. the step's four records arrive by bulk copy;
//   2. all threads dequantise them into shared memory: the keys as their fp16
//      centroids (in the rotated domain, C[idx], K-major), the values as v_hat
//      = code * s + z split into fp16 high and low parts (MN-major);
//   3. one thread issues S = q~ . C^T into tensor memory (M 128, N 64), with
//      the rotated query's fp16 high and low parts side by side along K;
//   4. each thread owns one query row: it loads the row of S, applies the key
//      norms and the causal limit, runs the online softmax in base 2 (the
//      accumulator is rescaled only when the row maximum grows by more than
//      2^8), and writes p as fp16 high and low parts;
//   5. one thread issues O += [p_hi | p_hi | p_lo] . [v_hi ; v_lo ; v_hi]
//      (M 128, N d, K 3 x 64) into tensor memory.
// Every operand the tensor cores see is exact fp16 except the value and weight
// splits (22 significant bits each), so the output carries ~2^-21 relative
// error against the fp64 attention over the same dequantised K/V.
//
// The value operand's N order follows the record's byte order: column
// n = (d/8) r + 2m + e holds dim 16m + 2r + e (r = 0..7, m = 0..d/16-1), so a
// thread dequantises one 16-byte record chunk into one contiguous run of n;
// the output is written back in dim order.
#include <mutex>

#include "tq_kernels.cuh"

namespace tq {
namespace {

constexpr int kRows = 128;      // query rows per tile (the M of every MMA)
constexpr int kStep = 64;       // cached tokens per step (four blocks; the N of S)
constexpr int kThreads = 128;   // one thread per query row
constexpr int kRecStages = 2;   // steps whose records are in flight

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint32_t ld_s32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 ld_s128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void st_s32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void st_s64(uint32_t a, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void st_s128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
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
// Wait for a phase of the barrier, giving up after ~2^31 clocks (about a second).
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t phase) {
    if (bar_try(bar, phase)) return true;
    const long long t0 = clock64();
    while (!bar_try(bar, phase))
        if (clock64() - t0 > (1LL << 31)) return false;
    return true;
}
__device__ __forceinline__ float exp2a(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}
// fp16 high and low parts of a pair of floats: hi = fp16(x), lo = fp16(x - hi)
__device__ __forceinline__ void split_h2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 f = __half22float2(h);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = pack_h2(a - f.x, b - f.y);
}

// Shared-memory matrix descriptor, no swizzle: start address, the byte offset
// between core matrices adjacent along the leading dimension (K for K-major
// operands, K for MN-major ones as well) and along the strided dimension, and
// the descriptor version of this architecture (bit 46).
__device__ __forceinline__ uint64_t mdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Instruction descriptor of kind::f16: fp32 accumulator (bit 4), fp16 A and B
// (format 0), A K-major, B K-major (0) or MN-major (1) at bit 16, N / 8 at
// bits 17-22, M / 16 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int b_mn_major) {
    return (1u << 4) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_f16(uint32_t tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void async_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// 16 consecutive fp32 columns of this thread's tensor-memory lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 16; j++) v[j] = __uint_as_float(r[j]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ shared memory plan
// All operand tiles use the no-swizzle core-matrix layout: a core matrix is 8
// rows of 16 bytes, stored as 128 contiguous bytes.
//   Q  [128 rows][2d] K-major: (r/8) 32d + (k/8) 128 + (r%8) 16 + (k%8) 2
//   K  [64 tokens][d] K-major: (t/8) 16d + (k/8) 128 + (t%8) 16 + (k%8) 2
//   V  hi, lo: [d cols][64 tokens] MN-major: (n/8) 1024 + (t/8) 128 + (t%8) 16 + (n%8) 2
//   P  hi, lo: [128 rows][64 tokens] K-major: (r/8) 1024 + (t/8) 128 + (r%8) 16 + (t%8) 2
template <int D>
struct PPlan {
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + 512u * D;
    static constexpr uint32_t kV = kK + 128u * D;          // hi, then lo at + 128 d
    static constexpr uint32_t kP = kV + 256u * D;          // hi, then lo at + 16 KB
    static constexpr uint32_t kRec = kP + 32768u;
    static constexpr uint32_t kRecStage = 4u * Rec<D>::kBytes;
    static constexpr uint32_t kLut = kRec + kRecStages * kRecStage;
    static constexpr uint32_t kNorm = kLut + 1024u;
    static constexpr uint32_t kIds = kNorm + kStep * 4u;
    static constexpr uint32_t kBars = kIds + kRecStages * 16u;  // record stages, S, O
    static constexpr uint32_t kMisc = kBars + (kRecStages + 2) * 8u;  // tensor-memory base, abort flag
    static constexpr uint32_t kEnd = kMisc + 16u;
    static constexpr uint32_t kCols = D == 128 ? 256u : 128u;  // S (64 columns) + O (d columns)
    static_assert(kRec % 16 == 0 && Rec<D>::kBytes % 16 == 0, "bulk copies need 16-byte alignment");
};

struct PrefillArgs {
    const uint16_t* q;            // bf16 [T][Hq][D]
    const unsigned char* cache;   // [num_blocks][Hkv][record]
    int num_blocks, Hkv, Hq, B;
    const uint16_t* k_tables;     // fp16 [Hkv][16] or null
    uint16_t default_table[16];
    const int32_t* block_tables;  // [B][max_blocks]
    int max_blocks;
    const int32_t* seq_lens;      // [B]
    const int32_t* q_start;       // [B + 1]
    int T;                        // rows of q and out
    int max_q_len;
    float scale_log2;             // scale * log2(e)
    float* out;                   // [T][Hq][D]
    int32_t* status;
    int rotate;                   // 0: TQ_CACHE_UNROTATED (the query is not rotated)
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(PrefillArgs a) {
    using R = Rec<D>;
    using PL = PPlan<D>;
    constexpr uint32_t REC = R::kBytes;
    constexpr int EPL = D / 32;  // query elements per lane in the rotation
    extern __shared__ __align__(1024) unsigned char psm[];
    const uint32_t base = saddr(psm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.z, kv = blockIdx.y, tile = blockIdx.x;
    const int G = a.Hq / a.Hkv;

    const int q0 = a.q_start[b];
    int qlen = a.q_start[b + 1] - q0;
    if (q0 < 0 || qlen < 0 || q0 + qlen > a.T) {  // rows outside q / out: nothing is touched
        if (tid == 0 && kv == 0 && tile == 0) flag_status(a.status, TQ_STATUS_BAD_LEN);
        return;
    }
    if (qlen > a.max_q_len) {  // beyond the grid: the chunk is cut (its last rows are not written)
        if (tid == 0 && kv == 0 && tile == 0) flag_status(a.status, TQ_STATUS_BAD_LEN);
        qlen = a.max_q_len;
    }
    const int rows_b = qlen * G;
    if (qlen <= 0 || tile * kRows >= rows_b) return;  // the whole CTA leaves together
    int L = a.seq_lens[b];
    if (L < a.q_start[b + 1] - q0 || L > a.max_blocks * kBlock) {  // no valid context: rows get 0
        if (tid == 0 && kv == 0 && tile == 0) flag_status(a.status, TQ_STATUS_BAD_LEN);
        L = -1;
    }
    const int qlen_full = a.q_start[b + 1] - q0;  // positions count from the chunk's full length
    // this thread's row: chunk token i, query head kv * G + hh; it sees positions < lim
    const int R_ = tile * kRows + tid;
    const bool row_ok = R_ < rows_b;  // a row of the chunk (its output is written)
    const int ri = R_ / G, rh = R_ % G;
    const int lim = row_ok && L >= 0 ? L - qlen_full + ri + 1 : 0;
    const int last_row = min(tile * kRows + kRows, rows_b) - 1;
    const int maxlim = L >= 0 ? L - qlen_full + last_row / G + 1 : 0;  // the tile's widest row
    const int nblk = (maxlim + kBlock - 1) / kBlock;
    const int nsteps = (maxlim + kStep - 1) / kStep;

    const uint32_t sQ = base + PL::kQ, sK = base + PL::kK, sV = base + PL::kV, sP = base + PL::kP;
    const uint32_t sRec = base + PL::kRec, sLut = base + PL::kLut, sNorm = base + PL::kNorm;
    const uint32_t sIds = base + PL::kIds, sBars = base + PL::kBars;
    const uint32_t barS = sBars + kRecStages * 8, barO = barS + 8;
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(psm + PL::kMisc);

    // ---- set-up: barriers, tensor memory, the centroid-pair table
    if (tid == 0) {
        for (int s = 0; s < kRecStages + 2; s++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sBars + 8 * s) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        misc[1] = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(base + PL::kMisc),
                     "r"(PL::kCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    {
        const uint16_t* tab = a.k_tables ? a.k_tables + kv * 16 : nullptr;
        for (int v = tid; v < 256; v += kThreads) {
            const uint32_t lo = tab ? tab[v & 15] : a.default_table[v & 15];
            const uint32_t hi = tab ? tab[v >> 4] : a.default_table[v >> 4];
            st_s32(sLut + 4 * v, lo | (hi << 16));
        }
    }
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = misc[0];
    const uint32_t tS = tmem, tO = tmem + kStep;  // column offsets of S and O
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;  // this warp's tensor-memory lanes

    const int32_t* bt = a.block_tables + (size_t)b * a.max_blocks;
    const long long rec_stride = (long long)a.Hkv * REC;
    // The records of step s into stage s % kRecStages (thread 0): blocks 4s .. 4s+3
    // that exist; the ids of the others are noted as -1.
    auto issue = [&](int s) {
        if (s >= nsteps || tid != 0) return;
        const uint32_t st = sRec + (uint32_t)(s % kRecStages) * PL::kRecStage;
        const uint32_t bar = sBars + 8 * (uint32_t)(s % kRecStages);
        int ids[4];
        uint32_t bytes = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int jb = 4 * s + j;
            int id = jb < nblk ? bt[jb] : -1;
            if (jb < nblk && (uint32_t)id >= (uint32_t)a.num_blocks) {
                flag_status(a.status, TQ_STATUS_BAD_BLOCK);
                id = -1;
            }
            ids[j] = id;
            if (id >= 0) bytes += REC;
        }
        st_s128(sIds + 16 * (uint32_t)(s % kRecStages),
                make_uint4((uint32_t)ids[0], (uint32_t)ids[1], (uint32_t)ids[2], (uint32_t)ids[3]));
        async_proxy_fence();
        if (bytes)
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
        else
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
#pragma unroll
        for (int j = 0; j < 4; j++)
            if (ids[j] >= 0) {
                const unsigned char* src = a.cache + (long long)ids[j] * rec_stride + (long long)kv * REC;
                asm volatile(
                    "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                        st + (uint32_t)j * REC),
                    "l"(src), "r"(REC), "r"(bar)
                    : "memory");
            }
    };
    issue(0);
    issue(1);

    // ---- the rotated queries: q~ = H q * scale log2(e) / sqrt(D) as fp16 high
    // (K 0 .. D-1) and low (K D .. 2D-1) parts; warp w rotates rows w, w + 4, ...
    for (int r = warp; r < kRows; r += 4) {
        const int Rr = tile * kRows + r;
        float x[EPL];
        if (Rr < rows_b && L >= 0) {
            const int i = Rr / G, h = kv * G + Rr % G;
            const uint16_t* src = a.q + ((size_t)(q0 + i) * a.Hq + h) * D + lane * EPL;
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
        uint32_t hi[EPL / 2], lo[EPL / 2];
#pragma unroll
        for (int e = 0; e < EPL; e += 2) split_h2(x[e] * sc, x[e + 1] * sc, hi[e / 2], lo[e / 2]);
        const int k = lane * EPL;  // EPL consecutive dims: inside one 8-dim chunk
        const uint32_t oh = sQ + (uint32_t)((r / 8) * (32 * D) + (k / 8) * 128 + (r % 8) * 16 + (k % 8) * 2);
        const uint32_t ol = oh + (uint32_t)((D / 8) * 128);  // K + D: D / 8 chunks further
        if constexpr (EPL == 4) {
            st_s64(oh, hi[0], hi[1]);
            st_s64(ol, lo[0], lo[1]);
        } else {
            st_s32(oh, hi[0]);
            st_s32(ol, lo[0]);
        }
    }
    async_proxy_fence();

    float m_run = -INFINITY, l_run = 0.f;
    bool o_started = false;
    int s = 0, o_issued = 0;
    bool aborted = false;
#pragma unroll 1
    for (; s < nsteps; s++) {
        const int stage = s % kRecStages;
        bool ok = bar_wait(sBars + 8 * (uint32_t)stage, (uint32_t)(s / kRecStages) & 1u);
        if (o_issued > 0) ok = ok && bar_wait(barO, (uint32_t)(o_issued - 1) & 1u);  // it read V, P
        if (__syncthreads_or(!ok)) {
            if (tid == 0) flag_status(a.status, TQ_STATUS_TIMEOUT);
            aborted = true;
            break;
        }
        tc_after_sync();
        const uint32_t st = sRec + (uint32_t)stage * PL::kRecStage;
        const uint4 idv = ld_s128(sIds + 16 * (uint32_t)stage);
        // block id of the step's record j (selects, not an indexed local array)
        auto id_of = [&](int j) {
            return (int)(j == 0 ? idv.x : j == 1 ? idv.y : j == 2 ? idv.z : idv.w);
        };
        // ---- keys: token tt, dims 8c .. 8c+7 -> one 16-byte row of a core matrix
        // (consecutive threads take consecutive tokens: eight of them fill one
        // 128-byte core matrix, so the stores do not collide on banks)
#pragma unroll 2
        for (int u = tid; u < kStep * (D / 8); u += kThreads) {
            const int tt = u % kStep, c = u / kStep;
            const int j = tt >> 4, o = tt & 15;
            uint4 w4 = make_uint4(0, 0, 0, 0);
            if (id_of(j) >= 0 && kStep * s + tt < maxlim) {
                const uint32_t w = ld_s32(st + (uint32_t)j * REC + (uint32_t)(o * (D / 2) + 4 * c));
                w4.x = ld_s32(sLut + 4 * (w & 0xFFu));
                w4.y = ld_s32(sLut + 4 * ((w >> 8) & 0xFFu));
                w4.z = ld_s32(sLut + 4 * ((w >> 16) & 0xFFu));
                w4.w = ld_s32(sLut + 4 * (w >> 24));
            }
            st_s128(sK + (uint32_t)((tt / 8) * (16 * D) + c * 128 + (tt % 8) * 16), w4);
        }
        // ---- values: token tt, byte row r of its pair chunk -> columns (D/8) r ..
        // (D/8) r + D/8 - 1 (dims 16m + 2r + e), high and low parts
#pragma unroll 1
        for (int u = tid; u < kStep * 8; u += kThreads) {
            const int tt = u % kStep, r = u / kStep;  // consecutive tokens: bank-free stores
            const int j = tt >> 4, o = tt & 15;
            const bool valid = id_of(j) >= 0 && kStep * s + tt < maxlim;
            float v[D / 8];
            if (valid) {
                const uint32_t rec = st + (uint32_t)j * REC;
                const uint32_t ch =
                    rec + R::kVCodes + (uint32_t)((8 * (o >> 1) + ((r + 2 * (o >> 1)) & 7)) * (D / 8));
                float sc[D / 32], zr[D / 32];
#pragma unroll
                for (int g = 0; g < D / 32; g++) {
                    const uint32_t gp = (uint32_t)R::group_pos(o, g);
                    const uint32_t sw = ld_s32(rec + R::kVScale + (gp & ~3u));
                    const uint32_t zw = ld_s32(rec + R::kVZero + (gp & ~3u));
                    sc[g] = half_bits_to_float((uint16_t)(sw >> (8 * (gp & 2))));
                    zr[g] = half_bits_to_float((uint16_t)(zw >> (8 * (gp & 2))));
                }
#pragma unroll
                for (int q = 0; q < D / 32; q++) {  // word q: bytes of m = 2q, 2q + 1 of both tokens
                    const uint32_t w = ld_s32(ch + 4 * q) >> (16 * (o & 1));
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const int m = 2 * q + e;
                        const uint32_t byte = (w >> (8 * e)) & 0xFFu;
                        const int g = m >> 1;
                        v[2 * m] = fmaf((float)(byte & 15u), sc[g], zr[g]);
                        v[2 * m + 1] = fmaf((float)(byte >> 4), sc[g], zr[g]);
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < D / 8; e++) v[e] = 0.f;
            }
#pragma unroll
            for (int n8 = 0; n8 < D / 64; n8++) {  // one 8-column group: 16 bytes of each part
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; e++) split_h2(v[8 * n8 + 2 * e], v[8 * n8 + 2 * e + 1], hi[e], lo[e]);
                const int n = (D / 8) * r + 8 * n8;
                const uint32_t off = (uint32_t)((n / 8) * 1024 + (tt / 8) * 128 + (tt % 8) * 16);
                st_s128(sV + off, make_uint4(hi[0], hi[1], hi[2], hi[3]));
                st_s128(sV + 128u * D + off, make_uint4(lo[0], lo[1], lo[2], lo[3]));
            }
        }
        if (tid < kStep) {  // the key norms of the step
            const int j = tid >> 4, o = tid & 15;
            float n = 0.f;
            if (id_of(j) >= 0 && kStep * s + tid < maxlim) {
                const uint32_t w = ld_s32(st + (uint32_t)j * REC + R::kKNorm + 4 * (o >> 1));
                n = half_bits_to_float((uint16_t)(w >> (16 * (o & 1))));
            }
            st_s32(sNorm + 4 * tid, __float_as_uint(n));
        }
        async_proxy_fence();
        tc_before_sync();
        __syncthreads();
        tc_after_sync();

        // ---- S = q~ C^T (thread 0), then the next records into the stage just read
        if (tid == 0) {
            constexpr uint32_t idS = idesc_f16(kRows, kStep, 0);
#pragma unroll 1
            for (int ks = 0; ks < 2 * D / 16; ks++) {
                const uint64_t ad = mdesc(sQ + 256u * ks, 128, 32 * D);
                const uint64_t bd = mdesc(sK + 256u * (ks % (D / 16)), 128, 16 * D);
                mma_f16(tS, ad, bd, idS, ks > 0);
            }
            mma_commit(barS);
        }
        issue(s + kRecStages);
        if (!__all_sync(kFull, bar_wait(barS, (uint32_t)s & 1u))) {
            if (lane == 0) misc[1] = 1;
        }
        tc_after_sync();

        // ---- online softmax of this thread's row over the step's 64 tokens
        float x[kStep];
#pragma unroll
        for (int c0 = 0; c0 < kStep; c0 += 16) {
            float t16[16];
            tmem_ld16(tS + lane_off + (uint32_t)c0, t16);
#pragma unroll
            for (int j = 0; j < 16; j++) x[c0 + j] = t16[j];
        }
        const bool whole = kStep * (s + 1) <= lim;  // the row sees every token of the step
        if (__all_sync(kFull, whole)) {  // no mask: the norms by packed multiplies
#pragma unroll
            for (int c0 = 0; c0 < kStep; c0 += 4) {
                const uint4 nw = ld_s128(sNorm + 4 * c0);
                const float2 a = __fmul2_rn(make_float2(x[c0], x[c0 + 1]),
                                            make_float2(__uint_as_float(nw.x), __uint_as_float(nw.y)));
                const float2 b = __fmul2_rn(make_float2(x[c0 + 2], x[c0 + 3]),
                                            make_float2(__uint_as_float(nw.z), __uint_as_float(nw.w)));
                x[c0] = a.x;
                x[c0 + 1] = a.y;
                x[c0 + 2] = b.x;
                x[c0 + 3] = b.y;
            }
        } else {
#pragma unroll
            for (int c0 = 0; c0 < kStep; c0 += 4) {
                const uint4 nw = ld_s128(sNorm + 4 * c0);
                const float nn[4] = {__uint_as_float(nw.x), __uint_as_float(nw.y), __uint_as_float(nw.z),
                                     __uint_as_float(nw.w)};
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const int t = kStep * s + c0 + j;
                    x[c0 + j] = whole || t < lim ? x[c0 + j] * nn[j] : -INFINITY;
                }
            }
        }
        // the row maximum: four independent chains
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < kStep; j++) m4[j & 3] = fmaxf(m4[j & 3], x[j]);
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        // the reference maximum moves only when the row maximum passes it by 2^8;
        // the accumulator row is rescaled then (tensor-memory loads and stores are
        // warp-wide: a lane whose row keeps its maximum scales by 1)
        const bool grow = mx > m_run + 8.0f;
        const float corr = grow && m_run != -INFINITY ? exp2a(m_run - mx) : 1.0f;
        if (grow) {
            l_run *= corr;
            m_run = mx;
        }
        if (o_started && __any_sync(kFull, corr != 1.0f)) {
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 16) {
                float t16[16];
                tmem_ld16(tO + lane_off + (uint32_t)c0, t16);
#pragma unroll
                for (int j = 0; j < 16; j++) t16[j] *= corr;
                tmem_st16(tO + lane_off + (uint32_t)c0, t16);
            }
        }
        // p = 2^(x - m) as fp16 high and low parts, 8 tokens per 16-byte row.  A row
        // that has seen no token yet has every x at -inf and takes 0 as its maximum
        // here: 2^-inf = 0 without a per-token test
        const uint32_t prow = sP + (uint32_t)((tid / 8) * 1024 + (tid % 8) * 16);
        const float m_eff = m_run == -INFINITY ? 0.f : m_run;
        const float2 nm2 = make_float2(-m_eff, -m_eff);
        float2 l2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int t8 = 0; t8 < kStep / 8; t8++) {
            float p[8];
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                const float2 d2 = __fadd2_rn(make_float2(x[8 * t8 + j], x[8 * t8 + j + 1]), nm2);
                p[j] = exp2a(d2.x);
                p[j + 1] = exp2a(d2.y);
                l2 = __fadd2_rn(l2, make_float2(p[j], p[j + 1]));
            }
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const __half2 h = __floats2half2_rn(p[2 * e], p[2 * e + 1]);
                const float2 f = __half22float2(h);
                const float2 r = __ffma2_rn(f, make_float2(-1.f, -1.f), make_float2(p[2 * e], p[2 * e + 1]));
                hi[e] = *reinterpret_cast<const uint32_t*>(&h);
                lo[e] = pack_h2(r.x, r.y);
            }
            st_s128(prow + 128u * t8, make_uint4(hi[0], hi[1], hi[2], hi[3]));
            st_s128(prow + 16384u + 128u * t8, make_uint4(lo[0], lo[1], lo[2], lo[3]));
        }
        l_run += l2.x + l2.y;
        async_proxy_fence();
        tc_before_sync();
        __syncthreads();
        tc_after_sync();
        if (misc[1]) {  // an S MMA that never completed: leave (its O is not issued)
            if (tid == 0) flag_status(a.status, TQ_STATUS_TIMEOUT);
            aborted = true;
            s++;  // this step's records were read
            break;
        }

        // ---- O += [p_hi | p_hi | p_lo] [v_hi ; v_lo ; v_hi] (thread 0)
        if (tid == 0) {
            constexpr uint32_t idO = idesc_f16(kRows, D, 1);
#pragma unroll 1
            for (int seg = 0; seg < 3; seg++) {
                const uint32_t pa = sP + (seg == 2 ? 16384u : 0u);
                const uint32_t vb = sV + (seg == 1 ? 128u * D : 0u);
#pragma unroll 1
                for (int ks = 0; ks < kStep / 16; ks++) {
                    const uint64_t ad = mdesc(pa + 256u * ks, 128, 1024);
                    const uint64_t bd = mdesc(vb + 256u * ks, 128, 1024);
                    mma_f16(tO, ad, bd, idO, (o_issued > 0 || seg > 0 || ks > 0) ? 1u : 0u);
                }
            }
            mma_commit(barO);
        }
        o_started = true;
        o_issued++;
    }

    // ---- the last O MMA, then this row's output in dim order (an aborted tile,
    // or one with nothing to attend to, leaves zeros; the status says why)
    bool done = o_issued > 0 && bar_wait(barO, (uint32_t)(o_issued - 1) & 1u);
    done = __syncthreads_and(done) && !aborted;
    if (o_issued > 0 && !done && tid == 0) flag_status(a.status, TQ_STATUS_TIMEOUT);
    tc_after_sync();
    {
        const int tok = q0 + ri, h = kv * G + rh;
        float* dst = a.out + ((size_t)tok * a.Hq + h) * D;
        const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
            float t16[16];
            if (done) {  // CTA-uniform: every lane of the warp loads
                tmem_ld16(tO + lane_off + (uint32_t)c0, t16);
            } else {
#pragma unroll
                for (int j = 0; j < 16; j++) t16[j] = 0.f;
            }
            if (row_ok) {
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    const int n = c0 + j;
                    const int rr = n / (D / 8), rem = n % (D / 8);
                    const int dim = 16 * (rem >> 1) + 2 * rr;  // e = 0; dim + 1 is e = 1
                    *reinterpret_cast<float2*>(dst + dim) = make_float2(t16[j] * inv, t16[j + 1] * inv);
                }
            }
        }
    }
    if (aborted) {  // copies still in flight get a bounded chance to land
        for (int j = s; j < min(s + kRecStages, nsteps); j++)
            bar_wait(sBars + 8 * (uint32_t)(j % kRecStages), (uint32_t)(j / kRecStages) & 1u);
    }
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(PL::kCols)
                     : "memory");
}

template <int D>
cudaError_t launch_p(const PrefillArgs& a, int max_q_len, cudaStream_t stream) {
    static std::mutex mu;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (dev < 0 || dev >= 64 || !configured[dev]) {
            e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)PPlan<D>::kEnd);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) configured[dev] = true;
        }
    }
    const int G = a.Hq / a.Hkv;
    const long long tiles = ((long long)max_q_len * G + kRows - 1) / kRows;
    const dim3 grid((unsigned)tiles, (unsigned)a.Hkv, (unsigned)a.B);
    prefill_kernel<D><<<grid, kThreads, PPlan<D>::kEnd, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const void* q, const unsigned char* cache, int num_blocks, int Hkv, int Hq, int B,
                           const uint16_t* k_tables, const uint16_t* default_table,
                           const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                           const int32_t* q_start, int T, int max_q_len, float scale, float* out,
                           int32_t* status, int head_dim, int rotate, cudaStream_t stream) {
    PrefillArgs a;
    a.q = static_cast<const uint16_t*>(q);
    a.cache = cache;
    a.num_blocks = num_blocks;
    a.Hkv = Hkv;
    a.Hq = Hq;
    a.B = B;
    a.k_tables = k_tables;
    for (int i = 0; i < 16; i++) a.default_table[i] = default_table[i];
    a.block_tables = block_tables;
    a.max_blocks = max_blocks;
    a.seq_lens = seq_lens;
    a.q_start = q_start;
    a.T = T;
    a.max_q_len = max_q_len;
    a.scale_log2 = scale * 1.44269504088896340736f;
    a.out = out;
    a.status = status;
    a.rotate = rotate;
    return head_dim == 128 ? launch_p<128>(a, max_q_len, stream) : launch_p<64>(a, max_q_len, stream);
}

size_t prefill_smem_bytes(int head_dim) {
    return head_dim == 128 ? PPlan<128>::kEnd : PPlan<64>::kEnd;
}

}  // namespace tq
