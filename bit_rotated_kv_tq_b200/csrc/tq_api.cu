// tq_api.cu -- the C ABI (include/tq.h): argument checks, default tables,
// split planning and kernel launches.  No call here allocates device memory
// or synchronises the stream.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "tq_kernels.cuh"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int ok() {
    g_err[0] = 0;
    return TQ_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool supported_d(int d) { return d == 64 || d == 128; }

int cuda_fail(cudaError_t e, const char* what) {
    return fail(TQ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

int device_sms() {
    static std::mutex mu;
    static std::vector<int> sms;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    std::lock_guard<std::mutex> lk(mu);
    if ((int)sms.size() <= dev) sms.resize(dev + 1, 0);
    if (!sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        sms[dev] = n;
    }
    return sms[dev];
}

// ---------------------------------------------------------------------------
// Lloyd-Max levels of N(0,1) with 16 cells, on the positive half-line.
// By symmetry the cells are [0,b1),[b1,b2),...,[b7,inf) mirrored, and each
// level is the mean of N(0,1) restricted to its cell:
//   c_j = (phi(b_{j-1}) - phi(b_j)) / (Q(b_{j-1}) - Q(b_j)),  Q the upper tail,
// with b_j = (c_j + c_{j+1})/2 and b_0 = 0.  Iterated until it stops moving.
void lloyd_max_half(double c[8]) {
    const double inv_sqrt_2pi = 0.39894228040143267794;
    auto phi = [&](double x) { return x == INFINITY ? 0.0 : inv_sqrt_2pi * exp(-0.5 * x * x); };
    auto Q = [](double x) { return x == INFINITY ? 0.0 : 0.5 * erfc(x * 0.70710678118654752440); };
    for (int j = 0; j < 8; j++) c[j] = 0.15 + 0.33 * j;
    int settle = -1;  // extra rounds once the step is below 1e-15, to reach the floor
    for (int it = 0; it < 200000; it++) {
        double b[9];
        b[0] = 0.0;
        for (int j = 1; j < 8; j++) b[j] = 0.5 * (c[j - 1] + c[j]);
        b[8] = INFINITY;
        double moved = 0.0;
        for (int j = 0; j < 8; j++) {
            double nc = (phi(b[j]) - phi(b[j + 1])) / (Q(b[j]) - Q(b[j + 1]));
            moved = std::max(moved, fabs(nc - c[j]));
            c[j] = nc;
        }
        if (moved == 0.0) break;
        if (settle < 0 && moved < 1e-15) settle = 2000;
        if (settle >= 0 && settle-- == 0) break;
    }
}

uint16_t to_half_bits(double x) { return __half_as_ushort(__double2half(x)); }

void scaled_table(int d, uint16_t out[16]) {
    double c[8];
    lloyd_max_half(c);
    const double s = 1.0 / sqrt((double)d);
    for (int j = 0; j < 8; j++) {
        out[8 + j] = to_half_bits(c[j] * s);
        out[7 - j] = to_half_bits(-c[j] * s);
    }
}

struct DefaultTables {
    std::once_flag once[2];
    uint16_t t[2][16];
};
DefaultTables g_tables;

const uint16_t* default_table(int d) {
    const int k = d == 128 ? 1 : 0;
    std::call_once(g_tables.once[k], [&] { scaled_table(d, g_tables.t[k]); });
    return g_tables.t[k];
}

bool check_cache(const tq_cache_t* c, int* err) {
    if (!c || !c->data || c->num_blocks <= 0 || c->num_kv_heads <= 0) {
        *err = fail(TQ_ERR_INVALID_ARG, "cache: null data or non-positive num_blocks/num_kv_heads");
        return false;
    }
    if ((c->flags & ~(TQ_CACHE_UNROTATED | TQ_CACHE_BF16)) ||
        c->flags == (TQ_CACHE_UNROTATED | TQ_CACHE_BF16)) {
        *err = fail(TQ_ERR_INVALID_ARG, "cache: unknown flags 0x%x", (unsigned)c->flags);
        return false;
    }
    if (!supported_d(c->head_dim)) {
        *err = fail(TQ_ERR_UNSUPPORTED, "cache: head_dim %d (supported: 64, 128)", c->head_dim);
        return false;
    }
    if (c->num_kv_heads > 32) {
        *err = fail(TQ_ERR_UNSUPPORTED, "cache: num_kv_heads %d > 32", c->num_kv_heads);
        return false;
    }
    if (!aligned(c->data, 16)) {
        *err = fail(TQ_ERR_ALIGNMENT, "cache: data must be 16-byte aligned");
        return false;
    }
    return true;
}

}  // namespace

namespace tq {
// Record a failure for tq_last_error() from another translation unit.
int set_last_error(int code, const char* msg) { return fail(code, "%s", msg); }

// Every host check of a decode call, then its split plan.  On TQ_OK with B > 0,
// `a` is ready for decode_launch and `need` holds the workspace bytes the plan
// uses (0 when nothing has to be combined); nothing has been enqueued.
int decode_prepare(const void* q, const tq_cache_t* cache, const uint16_t* k_tables,
                   const int32_t* block_tables, int max_blocks, const int32_t* seq_lens, int B,
                   int H_q, int max_seq_len, float scale, float* out, int num_splits,
                   int32_t* status, DecodeArgs& a, size_t& need) {
    int err;
    need = 0;
    if (!check_cache(cache, &err)) return err;
    if (B < 0 || H_q <= 0 || max_blocks <= 0 || max_seq_len < 0 ||
        (long long)max_seq_len > (long long)max_blocks * kBlock)
        return fail(TQ_ERR_INVALID_ARG,
                    "tq_decode_attention: need B >= 0, H_q > 0, 0 <= max_seq_len <= max_blocks*16");
    if (num_splits < 0 || num_splits > 1024)
        return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attention: num_splits %d (0..1024)", num_splits);
    if (B == 0) return ok();
    if (B > 65535) return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attention: B %d > 65535", B);
    if (!q || !block_tables || !seq_lens || !out)
        return fail(TQ_ERR_INVALID_ARG, "tq_decode_attention: q, block_tables, seq_lens, out required");
    const int Hkv = cache->num_kv_heads;
    if (H_q % Hkv)
        return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attention: H_q %d not a multiple of H_kv %d", H_q, Hkv);
    const int G = H_q / Hkv;
    if (G > 64)
        return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attention: GQA group %d (supported 1..64)", G);
    if (!isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "tq_decode_attention: scale not finite");
    // the split kernel stores its outputs as pairs of floats
    if (!aligned(out, 8)) return fail(TQ_ERR_ALIGNMENT, "tq_decode_attention: out must be 8-byte aligned");
    if (!aligned(q, 4) || !aligned(block_tables, 4) || !aligned(seq_lens, 4) ||
        (k_tables && !aligned(k_tables, 4)) || (status && !aligned(status, 4)))
        return fail(TQ_ERR_ALIGNMENT, "tq_decode_attention: q and the tables must be 4-byte aligned");
    const int d = cache->head_dim;
    const bool bf16 = (cache->flags & TQ_CACHE_BF16) != 0;
    if (bf16 && k_tables)
        return fail(TQ_ERR_INVALID_ARG, "tq_decode_attention: a bf16 cache takes no key tables");
    a = DecodeArgs{};
    a.q = static_cast<const uint16_t*>(q);
    a.cache = static_cast<const unsigned char*>(cache->data);
    a.num_blocks = cache->num_blocks;
    a.Hkv = Hkv;
    a.Hq = H_q;
    a.B = B;
    a.k_tables = k_tables;
    memcpy(a.default_table, default_table(d), sizeof a.default_table);
    a.block_tables = block_tables;
    a.max_blocks = max_blocks;
    a.seq_lens = seq_lens;
    a.scale_log2 = scale * 1.44269504088896340736f;
    a.rotate = (cache->flags & TQ_CACHE_UNROTATED) ? 0 : 1;
    a.out = out;
    a.num_splits = num_splits;
    a.max_seq_len = max_seq_len;
    a.status = status;
    if (bf16) {
        // items of up to 8 query heads; S ranges of blocks per item.  The kernel is
        // bound by HBM, not by how evenly the SMs are loaded (an SM whose neighbours
        // are done streams faster), so by default S is the fewest ranges that give
        // every SM a CTA (one CTA keeps 96 KB of copies in flight), at most 16, at
        // most the longest sequence's blocks, with partials inside the
        // num_splits = 0 workspace
        a.bf16 = 1;
        a.bf_hgroups = (G + 7) / 8;
        const long long items = (long long)B * Hkv * a.bf_hgroups;
        int S = num_splits;
        if (S == 0) {
            const long long per = (long long)B * H_q * (4LL * d + 8);
            long long cap = (long long)tq_decode_workspace_bytes(B, H_q, d, 0) / per;
            cap = std::min(cap, 16LL);
            cap = std::min(cap, (long long)std::max(1, (max_seq_len + kBlock - 1) / kBlock));
            cap = std::max(cap, 1LL);
            const long long sms = device_sms();
            S = (int)std::min(cap, std::max(1LL, (sms + items - 1) / items));
        }
        if (items * S > 0x7fffffffLL)
            return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attention: B * H_kv * num_splits too large");
        a.bf_splits = S;
        need = S > 1 ? (size_t)B * H_q * S * ((size_t)d * sizeof(float) + sizeof(float2)) : 0;
        return ok();
    }
    if (!decode_plan(a, d, device_sms()))
        return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attention: B * H_kv * num_splits too large");
    need = decode_workspace_for(a, d);
    return ok();
}

// Launch a prepared decode with its partials in `workspace` (the plan's
// decode_workspace_for bytes, 16-byte aligned; unused when that is 0).
int decode_launch(DecodeArgs& a, int head_dim, void* workspace, void* stream) {
    a.ws_o = static_cast<float*>(workspace);
    if (a.bf16) {  // [B][H_q][S][d] partial outputs, then [B][H_q][S] (m, l)
        a.ws_ml = workspace ? reinterpret_cast<float2*>(static_cast<float*>(workspace) +
                                                        (size_t)a.B * a.Hq * a.bf_splits * head_dim)
                            : nullptr;
        cudaError_t e = launch_bf16_decode(a, head_dim, (cudaStream_t)stream);
        if (e != cudaSuccess) return cuda_fail(e, "tq_decode_attention launch");
        return ok();
    }
    // [ranges][2][heads per item][d] partial outputs, then [ranges][2][heads per item] (m, l)
    a.ws_ml = workspace ? reinterpret_cast<float2*>(static_cast<float*>(workspace) +
                                                    (size_t)a.nranges * 2 * 4 * a.qpi * head_dim)
                        : nullptr;
    cudaError_t e = launch_decode(a, head_dim, device_sms(), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tq_decode_attention launch");
    return ok();
}
}  // namespace tq

extern "C" {

TQ_API size_t tq_record_bytes(int head_dim) {
    if (!supported_d(head_dim)) return 0;
    return head_dim == 128 ? (size_t)tq::Rec<128>::kBytes : (size_t)tq::Rec<64>::kBytes;
}

TQ_API size_t tq_cache_record_bytes(int head_dim, int flags) {
    if (!supported_d(head_dim)) return 0;
    if ((flags & ~(TQ_CACHE_UNROTATED | TQ_CACHE_BF16)) || flags == (TQ_CACHE_UNROTATED | TQ_CACHE_BF16))
        return 0;
    return (flags & TQ_CACHE_BF16) ? (size_t)64 * head_dim : tq_record_bytes(head_dim);
}

TQ_API size_t tq_cache_bytes(int num_blocks, int num_kv_heads, int head_dim) {
    if (num_blocks <= 0 || num_kv_heads <= 0) return 0;
    return (size_t)num_blocks * (size_t)num_kv_heads * tq_record_bytes(head_dim);
}

TQ_API int tq_lloyd_max_table(int head_dim, uint16_t out16[16]) {
    if (!out16) return fail(TQ_ERR_INVALID_ARG, "tq_lloyd_max_table: out16 is NULL");
    if (head_dim <= 0 || (head_dim & (head_dim - 1)))
        return fail(TQ_ERR_UNSUPPORTED, "tq_lloyd_max_table: head_dim %d", head_dim);
    if (supported_d(head_dim))
        memcpy(out16, default_table(head_dim), 16 * sizeof(uint16_t));
    else
        scaled_table(head_dim, out16);
    return ok();
}

TQ_API int tq_fit_k_table(const uint16_t* keys_bf16, int n, int head_dim,
                          const uint16_t init16[16], int max_iter, uint16_t out16[16]) {
    if (!keys_bf16 || !init16 || !out16 || n < 0 || max_iter < 0)
        return -fail(TQ_ERR_INVALID_ARG, "tq_fit_k_table: bad argument");
    if (head_dim <= 0 || (head_dim & (head_dim - 1)) || head_dim > 4096)
        return -fail(TQ_ERR_UNSUPPORTED, "tq_fit_k_table: head_dim %d", head_dim);
    const int d = head_dim;
    // rotated unit coordinates: (S k)/(||k|| sqrt(d)) with the exact +-1 butterfly
    std::vector<double> ys((size_t)n * d);
    std::vector<double> buf(d);
    for (int v = 0; v < n; v++) {
        double ss = 0.0;
        for (int i = 0; i < d; i++) {
            uint32_t w = (uint32_t)keys_bf16[(size_t)v * d + i] << 16;
            float f;
            memcpy(&f, &w, 4);
            buf[i] = f;
            ss += buf[i] * buf[i];
        }
        for (int len = 1; len < d; len <<= 1)
            for (int i = 0; i < d; i += 2 * len)
                for (int j = i; j < i + len; j++) {
                    double x = buf[j], y = buf[j + len];
                    buf[j] = x + y;
                    buf[j + len] = x - y;
                }
        const double nrm = sqrt(ss);
        const double den = nrm * sqrt((double)d);
        for (int i = 0; i < d; i++) ys[(size_t)v * d + i] = nrm > 0.0 ? buf[i] / den : 0.0;
    }
    double c[16];
    for (int j = 0; j < 16; j++) c[j] = (double)__half2float(__ushort_as_half(init16[j]));
    const size_t N = ys.size();
    std::vector<int> cell(N, -1);
    int it = 0;
    for (; it < max_iter; it++) {
        bool moved = false;
        for (size_t i = 0; i < N; i++) {
            int best = 0;
            double bd = fabs(ys[i] - c[0]);
            for (int j = 1; j < 16; j++) {
                double dj = fabs(ys[i] - c[j]);
                if (dj < bd) {
                    bd = dj;
                    best = j;
                }
            }
            if (best != cell[i]) {
                cell[i] = best;
                moved = true;
            }
        }
        if (!moved) break;
        double sum[16] = {0};
        int cnt[16] = {0};
        for (size_t i = 0; i < N; i++) {
            sum[cell[i]] += ys[i];
            cnt[cell[i]]++;
        }
        for (int j = 0; j < 16; j++)
            if (cnt[j]) c[j] = sum[j] / cnt[j];
    }
    std::sort(c, c + 16);
    for (int j = 0; j < 16; j++) out16[j] = to_half_bits(c[j]);
    ok();
    return it;
}

TQ_API int tq_quantize_append(const void* K, const void* V, const int32_t* block_table, int num_seqs,
                       int max_blocks, const int32_t* slot_mapping, int T,
                       const tq_cache_t* cache, const uint16_t* k_tables, int32_t* status,
                       void* stream) {
    int err;
    if (!check_cache(cache, &err)) return err;
    if (T < 0) return fail(TQ_ERR_INVALID_ARG, "tq_quantize_append: T < 0");
    if (T == 0) return ok();
    if ((long long)T * cache->num_kv_heads >= 0x7fffffffLL)
        return fail(TQ_ERR_UNSUPPORTED, "tq_quantize_append: T * H_kv must stay below 2^31");
    if (!K || !V || !slot_mapping)
        return fail(TQ_ERR_INVALID_ARG, "tq_quantize_append: K, V and slot_mapping are required");
    if (block_table && (num_seqs <= 0 || max_blocks <= 0))
        return fail(TQ_ERR_INVALID_ARG, "tq_quantize_append: block_table needs num_seqs, max_blocks > 0");
    if ((long long)num_seqs * max_blocks * tq::kBlock > 0x7fffffffLL)
        return fail(TQ_ERR_UNSUPPORTED, "tq_quantize_append: logical slots exceed int32");
    if (!aligned(K, 16) || !aligned(V, 16))
        return fail(TQ_ERR_ALIGNMENT, "tq_quantize_append: K and V must be 16-byte aligned");
    if (!aligned(slot_mapping, 4) || (block_table && !aligned(block_table, 4)) ||
        (k_tables && !aligned(k_tables, 4)) || (status && !aligned(status, 4)))
        return fail(TQ_ERR_ALIGNMENT, "tq_quantize_append: int32 arrays and tables must be 4-byte aligned");
    tq::AppendArgs a;
    a.K = static_cast<const uint16_t*>(K);
    a.V = static_cast<const uint16_t*>(V);
    a.block_table = block_table;
    a.num_seqs = num_seqs;
    a.max_blocks = max_blocks;
    a.slots = slot_mapping;
    a.T = T;
    a.cache = static_cast<unsigned char*>(cache->data);
    a.num_blocks = cache->num_blocks;
    a.Hkv = cache->num_kv_heads;
    a.k_tables = k_tables;
    memcpy(a.default_table, default_table(cache->head_dim), sizeof a.default_table);
    a.status = status;
    a.rotate = (cache->flags & TQ_CACHE_UNROTATED) ? 0 : 1;
    cudaError_t e;
    if (cache->flags & TQ_CACHE_BF16) {
        if (k_tables) return fail(TQ_ERR_INVALID_ARG, "tq_quantize_append: a bf16 cache takes no key tables");
        e = tq::launch_bf16_append(a, cache->head_dim, device_sms(), (cudaStream_t)stream);
    } else {
        e = tq::launch_append(a, cache->head_dim, device_sms(), (cudaStream_t)stream);
    }
    if (e != cudaSuccess) return cuda_fail(e, "tq_quantize_append launch");
    return ok();
}

TQ_API int tq_decode_default_splits(int B, int H_kv, int max_seq_len) {
    (void)B;
    (void)H_kv;
    (void)max_seq_len;
    return 0;  // the library cuts the work evenly over the whole GPU
}

TQ_API size_t tq_decode_workspace_bytes(int B, int H_q, int head_dim, int num_splits) {
    if (B <= 0 || H_q <= 0 || !supported_d(head_dim) || num_splits == 1 || num_splits < 0) return 0;
    // Even cut: at most two ranges per SM (one per half), each with partials of
    // up to 8 heads per item at d = 64 (two groups of four) and 4 at d = 128.
    // S splits: at most items * S + 1 ranges, and items * (heads per item) is at
    // most B * H_kv * (G + 3) with 4 heads per item, B * H_kv * (G + 7) with 8
    // (only when G > 4); both leave items * S * heads + heads within
    // 4 (B * H_q * S + 1) head partials
    const long long ranges =
        num_splits == 0 ? 2LL * device_sms() : (long long)B * H_q * num_splits + 1;
    const long long heads = num_splits == 0 && head_dim == 64 ? 8 : 4;
    const size_t per_head = (size_t)head_dim * sizeof(float) + sizeof(float2);
    size_t n = (size_t)ranges * 2 * heads * per_head;
    // the default plan of a bf16 cache: up to 8 ranges per query head, within the
    // static entry's 8 MiB
    if (num_splits == 0) n = std::max(n, std::min((size_t)8 * B * H_q * per_head, (size_t)8 << 20));
    return n;
}

TQ_API int tq_decode_attention(const void* q, const tq_cache_t* cache, const uint16_t* k_tables,
                        const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                        int B, int H_q, int max_seq_len, float scale, float* out,
                        void* workspace, size_t ws_bytes, int num_splits, int32_t* status,
                        void* stream) {
    tq::DecodeArgs a;
    size_t need = 0;
    const int err = tq::decode_prepare(q, cache, k_tables, block_tables, max_blocks, seq_lens, B, H_q,
                                       max_seq_len, scale, out, num_splits, status, a, need);
    if (err != TQ_OK || B == 0) return err;
    if (need) {
        if (!workspace || ws_bytes < need)
            return fail(TQ_ERR_WORKSPACE, "tq_decode_attention: workspace %zu bytes < %zu needed",
                        workspace ? ws_bytes : (size_t)0, need);
        if (!aligned(workspace, 16))
            return fail(TQ_ERR_ALIGNMENT, "tq_decode_attention: workspace must be 16-byte aligned");
    }
    return tq::decode_launch(a, cache->head_dim, need ? workspace : nullptr, stream);
}

TQ_API int tq_prefill_attention(const void* q, const tq_cache_t* cache, const uint16_t* k_tables,
                                const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                                const int32_t* q_start, int B, int H_q, int T, int max_q_len, float scale,
                                float* out, int32_t* status, void* stream) {
    int err;
    if (!check_cache(cache, &err)) return err;
    if (cache->flags & TQ_CACHE_BF16)
        return fail(TQ_ERR_UNSUPPORTED, "tq_prefill_attention: not available for a bf16 cache");
    if (B < 0 || H_q <= 0 || T < 0 || max_q_len < 0 || max_blocks <= 0)
        return fail(TQ_ERR_INVALID_ARG,
                    "tq_prefill_attention: need B, T, max_q_len >= 0, H_q > 0, max_blocks > 0");
    if (B == 0 || T == 0 || max_q_len == 0) return ok();
    if (B > 65535) return fail(TQ_ERR_UNSUPPORTED, "tq_prefill_attention: B %d > 65535", B);
    if (!q || !block_tables || !seq_lens || !q_start || !out)
        return fail(TQ_ERR_INVALID_ARG,
                    "tq_prefill_attention: q, block_tables, seq_lens, q_start and out are required");
    const int Hkv = cache->num_kv_heads;
    if (H_q % Hkv)
        return fail(TQ_ERR_UNSUPPORTED, "tq_prefill_attention: H_q %d not a multiple of H_kv %d", H_q, Hkv);
    if ((long long)max_q_len * (H_q / Hkv) > (1LL << 30))
        return fail(TQ_ERR_UNSUPPORTED, "tq_prefill_attention: max_q_len * GQA group too large");
    if (!isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "tq_prefill_attention: scale not finite");
    if (!aligned(q, 16) || !aligned(out, 16))
        return fail(TQ_ERR_ALIGNMENT, "tq_prefill_attention: q and out must be 16-byte aligned");
    if (!aligned(block_tables, 4) || !aligned(seq_lens, 4) || !aligned(q_start, 4) ||
        (k_tables && !aligned(k_tables, 4)) || (status && !aligned(status, 4)))
        return fail(TQ_ERR_ALIGNMENT, "tq_prefill_attention: int32 arrays and tables must be 4-byte aligned");
    cudaError_t e = tq::launch_prefill(q, static_cast<const unsigned char*>(cache->data), cache->num_blocks, Hkv,
                                       H_q, B, k_tables, default_table(cache->head_dim), block_tables, max_blocks,
                                       seq_lens, q_start, T, max_q_len, scale, out, status, cache->head_dim,
                                       (cache->flags & TQ_CACHE_UNROTATED) ? 0 : 1, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tq_prefill_attention launch");
    return ok();
}

TQ_API int tq_dequantize(const tq_cache_t* cache, const uint16_t* k_tables, const int32_t* block_tables,
                  int max_blocks, const int32_t* seq_lens, int B, int max_len, float* K_hat,
                  float* V_hat, int32_t* status, void* stream) {
    int err;
    if (!check_cache(cache, &err)) return err;
    if (B < 0 || max_len < 0 || max_blocks <= 0)
        return fail(TQ_ERR_INVALID_ARG, "tq_dequantize: need B >= 0, max_len >= 0, max_blocks > 0");
    if (B == 0 || max_len == 0) return ok();
    if (!block_tables || !seq_lens || !K_hat || !V_hat)
        return fail(TQ_ERR_INVALID_ARG, "tq_dequantize: block_tables, seq_lens, K_hat, V_hat required");
    if (!aligned(K_hat, 16) || !aligned(V_hat, 16))
        return fail(TQ_ERR_ALIGNMENT, "tq_dequantize: K_hat and V_hat must be 16-byte aligned");
    if (!aligned(block_tables, 4) || !aligned(seq_lens, 4) || (k_tables && !aligned(k_tables, 4)) ||
        (status && !aligned(status, 4)))
        return fail(TQ_ERR_ALIGNMENT, "tq_dequantize: int32 arrays and tables must be 4-byte aligned");
    tq::DequantArgs a;
    a.cache = static_cast<const unsigned char*>(cache->data);
    a.num_blocks = cache->num_blocks;
    a.Hkv = cache->num_kv_heads;
    a.k_tables = k_tables;
    memcpy(a.default_table, default_table(cache->head_dim), sizeof a.default_table);
    a.block_tables = block_tables;
    a.max_blocks = max_blocks;
    a.seq_lens = seq_lens;
    a.B = B;
    a.max_len = max_len;
    a.K_hat = K_hat;
    a.V_hat = V_hat;
    a.status = status;
    a.rotate = (cache->flags & TQ_CACHE_UNROTATED) ? 0 : 1;
    cudaError_t e;
    if (cache->flags & TQ_CACHE_BF16) {
        if (k_tables) return fail(TQ_ERR_INVALID_ARG, "tq_dequantize: a bf16 cache takes no key tables");
        e = tq::launch_bf16_dequant(a, cache->head_dim, device_sms(), (cudaStream_t)stream);
    } else {
        e = tq::launch_dequant(a, cache->head_dim, device_sms(), (cudaStream_t)stream);
    }
    if (e != cudaSuccess) return cuda_fail(e, "tq_dequantize launch");
    return ok();
}

TQ_API const char* tq_last_error(void) { return g_err; }

}  // extern "C"
