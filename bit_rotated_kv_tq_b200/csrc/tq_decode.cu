// tq_decode.cu -- split-K decode attention over the TQ4/4 cache and the
// log-sum-exp combine of the splits.
//
// For one sequence b and kv head kv, the G = Hq/Hkv query heads that read kv
// are handled together.  Because the Hadamard matrix H is symmetric and
// orthogonal, <q, k_hat_t> = <H q, H k_hat_t> = n_t <q~, C[idx_t]> with
// q~ = H q: the query is rotated once and the scores are formed against the
// stored centroids in the rotated domain (the key is never un-rotated).
// Values are dequantised as code * s + z per group of 32.  Softmax runs
// online in base 2 (scale * log2(e) is folded into q~), one block of 16
// tokens at a time, and each split of the context leaves an unnormalised
// partial (o, m, l) that the combine kernel merges.
#include "tq_kernels.cuh"

namespace tq {

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(kFull, x, m);
    return x;
}

// Rotate q for the G heads of this kv head into shared memory, scaled by
// scale*log2(e)/sqrt(D).  Warp w handles heads w, w+nwarps, ...
template <int D, int G>
__device__ void rotate_queries(const DecodeArgs& a, int b, int kv, float* qs) {
    constexpr int EPL = D / 32;  // elements per lane
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const float sc = a.scale_log2 * rsqrtf((float)D);
    for (int g = warp; g < G; g += nw) {
        const uint16_t* src = a.q + ((size_t)b * a.Hq + kv * G + g) * D + lane * EPL;
        float x[EPL];
#pragma unroll
        for (int e = 0; e < EPL; e++) x[e] = __uint_as_float((uint32_t)src[e] << 16);
#pragma unroll
        for (int m = 1; m < EPL; m <<= 1) {
#pragma unroll
            for (int e = 0; e < EPL; e++)
                if (!(e & m)) {
                    float u = x[e], w = x[e | m];
                    x[e] = u + w;
                    x[e | m] = u - w;
                }
        }
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const bool upper = lane & m;
#pragma unroll
            for (int e = 0; e < EPL; e++) {
                float p = __shfl_xor_sync(kFull, x[e], m);
                x[e] = upper ? p - x[e] : x[e] + p;
            }
        }
#pragma unroll
        for (int e = 0; e < EPL; e++) qs[g * D + lane * EPL + e] = x[e] * sc;
    }
}

// One CTA per (split, kv head, sequence); 4 warps take the split's blocks
// round-robin, each with its own online-softmax state, merged at the end.
template <int D, int G>
__global__ void __launch_bounds__(128) decode_split_kernel(DecodeArgs a) {
    constexpr int EPL = D / 32;
    constexpr int NW = 4;
    using R = Rec<D>;
    __shared__ float qs[G * D];
    __shared__ float ctab[16];
    __shared__ float sc_s[NW][kBlock][G];
    __shared__ float red_m[NW][G], red_l[NW][G];
    __shared__ float red_o[NW][G][D];

    const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    int L = a.seq_lens[b];
    if (L < 0 || L > a.max_blocks * kBlock) {
        if (threadIdx.x == 0 && split == 0 && kv == 0) flag_status(a.status, TQ_STATUS_BAD_LEN);
        L = 0;
    }
    if (L > a.num_splits * a.blocks_per_split * kBlock) {  // longer than max_seq_len promised
        if (threadIdx.x == 0 && split == 0 && kv == 0) flag_status(a.status, TQ_STATUS_BAD_LEN);
        L = a.num_splits * a.blocks_per_split * kBlock;
    }
    const int nblk = (L + kBlock - 1) / kBlock;
    const int jb = split * a.blocks_per_split;
    const int je = min(jb + a.blocks_per_split, nblk);

    if (threadIdx.x < 16)
        ctab[threadIdx.x] = half_bits_to_float(a.k_tables ? a.k_tables[kv * 16 + threadIdx.x]
                                                          : a.default_table[threadIdx.x]);
    rotate_queries<D, G>(a, b, kv, qs);
    __syncthreads();

    float qr[G][EPL];
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int e = 0; e < EPL; e++) qr[g][e] = qs[g * D + lane * EPL + e];

    float m_run[G], l_run[G], acc[G][EPL];
#pragma unroll
    for (int g = 0; g < G; g++) {
        m_run[g] = -INFINITY;
        l_run[g] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; e++) acc[g][e] = 0.f;
    }

    const int grp = (lane * EPL) / kGroup;  // value group of this lane's elements
    for (int j = jb + warp; j < je; j += NW) {
        const int pb = a.block_tables[(size_t)b * a.max_blocks + j];
        if (pb < 0 || pb >= a.num_blocks) {
            if (lane == 0) flag_status(a.status, TQ_STATUS_BAD_BLOCK);
            continue;
        }
        const unsigned char* rec = a.cache + ((size_t)pb * a.Hkv + kv) * (size_t)R::kBytes;
        const int valid = min(kBlock, L - j * kBlock);
        // scores of the block's tokens
        for (int t = 0; t < valid; t++) {
            uint32_t codes;
            if (EPL == 4)
                codes = *reinterpret_cast<const uint16_t*>(rec + R::kKCodes + t * R::kCodeRow + lane * 2);
            else
                codes = rec[R::kKCodes + t * R::kCodeRow + lane];
            float kval[EPL];
#pragma unroll
            for (int e = 0; e < EPL; e++) kval[e] = ctab[(codes >> (4 * e)) & 15];
            const float nrm = half_bits_to_float(
                *reinterpret_cast<const uint16_t*>(rec + R::kKNorm + t * 2));
#pragma unroll
            for (int g = 0; g < G; g++) {
                float p = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; e++) p = fmaf(qr[g][e], kval[e], p);
                p = warp_sum(p);
                if (lane == 0) sc_s[warp][t][g] = p * nrm;
            }
        }
        __syncwarp();
        // online softmax update with this block, then the weighted values
#pragma unroll
        for (int g = 0; g < G; g++) {
            float bm = -INFINITY;
            for (int t = 0; t < valid; t++) bm = fmaxf(bm, sc_s[warp][t][g]);
            const float mn = fmaxf(m_run[g], bm);
            const float corr = exp2f(m_run[g] - mn);
            l_run[g] *= corr;
#pragma unroll
            for (int e = 0; e < EPL; e++) acc[g][e] *= corr;
            m_run[g] = mn;
        }
        for (int t = 0; t < valid; t++) {
            uint32_t codes;
            if (EPL == 4)
                codes = *reinterpret_cast<const uint16_t*>(rec + R::kVCodes + t * R::kCodeRow + lane * 2);
            else
                codes = rec[R::kVCodes + t * R::kCodeRow + lane];
            const uint32_t sz =
                *reinterpret_cast<const uint32_t*>(rec + R::kVGroups + (t * R::kGroups + grp) * 4);
            const float s = half_bits_to_float((uint16_t)(sz & 0xffff));
            const float z = half_bits_to_float((uint16_t)(sz >> 16));
            float vval[EPL];
#pragma unroll
            for (int e = 0; e < EPL; e++) vval[e] = fmaf((float)((codes >> (4 * e)) & 15), s, z);
#pragma unroll
            for (int g = 0; g < G; g++) {
                const float p = exp2f(sc_s[warp][t][g] - m_run[g]);
                l_run[g] += p;
#pragma unroll
                for (int e = 0; e < EPL; e++) acc[g][e] = fmaf(p, vval[e], acc[g][e]);
            }
        }
        __syncwarp();
    }

    // merge the warps
#pragma unroll
    for (int g = 0; g < G; g++) {
        if (lane == 0) {
            red_m[warp][g] = m_run[g];
            red_l[warp][g] = l_run[g];
        }
#pragma unroll
        for (int e = 0; e < EPL; e++) red_o[warp][g][lane * EPL + e] = acc[g][e];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int g = idx / D, i = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; w++) M = fmaxf(M, red_m[w][g]);
        float o = 0.f, l = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; w++) {
                const float f = exp2f(red_m[w][g] - M);
                o = fmaf(f, red_o[w][g][i], o);
                l = fmaf(f, red_l[w][g], l);
            }
        }
        const int h = kv * G + g;
        if (a.num_splits == 1) {
            a.out[((size_t)b * a.Hq + h) * D + i] = l > 0.f ? o / l : 0.f;
        } else {
            const size_t row = ((size_t)b * a.Hq + h) * a.num_splits + split;
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
            const float f = exp2f(ml.x - M);
            o = fmaf(f, a.ws_o[(row0 + s) * D + i], o);
            l = fmaf(f, ml.y, l);
        }
    }
    a.out[(size_t)bh * D + i] = l > 0.f ? o / l : 0.f;
}

template <int D, int G>
static cudaError_t launch_dg(const DecodeArgs& a, cudaStream_t stream) {
    dim3 grid(a.num_splits, a.Hkv, a.B);
    decode_split_kernel<D, G><<<grid, 128, 0, stream>>>(a);
    if (a.num_splits > 1) combine_kernel<D><<<a.B * a.Hq, D, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_d(const DecodeArgs& a, cudaStream_t stream) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_dg<D, 1>(a, stream);
        case 2: return launch_dg<D, 2>(a, stream);
        case 4: return launch_dg<D, 4>(a, stream);
        case 8: return launch_dg<D, 8>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const DecodeArgs& a, int head_dim, cudaStream_t stream) {
    return head_dim == 128 ? launch_d<128>(a, stream) : launch_d<64>(a, stream);
}

}  // namespace tq
