// tq_dequant.cu -- gather and dequantise the cache back to fp32 (checks only).
//   k_hat = fp16 norm * H_d * C[idx]   (H_d symmetric and involutive, so the
//                                      same butterfly undoes the rotation;
//                                      fp16 norm * C[idx] for an unrotated cache)
//   v_hat = code * scale + zero
// One vector (sequence, position, kv head) per D/8 lanes, 8 elements per lane.
#include "tq_kernels.cuh"

namespace tq {

template <int D>
__global__ void __launch_bounds__(256) dequant_kernel(DequantArgs a) {
    constexpr int LPV = D / 8;
    constexpr int VPW = 32 / LPV;
    using R = Rec<D>;
    __shared__ float ctab[64][16];
    for (int i = threadIdx.x; i < a.Hkv * 16 && i < 64 * 16; i += blockDim.x)
        ctab[i / 16][i % 16] = half_bits_to_float(a.k_tables ? a.k_tables[i] : a.default_table[i % 16]);
    __syncthreads();

    const int lane = threadIdx.x & 31, sub = lane % LPV, grp = lane / LPV;
    const long long total = (long long)a.B * a.max_len * a.Hkv;
    const long long warps = (long long)gridDim.x * (blockDim.x / 32);
    const long long warp_id = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const float inv_sqrt_d = rsqrtf((float)D);

    for (long long base = warp_id * VPW; base < total; base += warps * VPW) {
        const long long vec = base + grp;
        const bool in = vec < total;
        int h = 0, t = 0, b = 0;
        if (in) {
            h = (int)(vec % a.Hkv);
            long long bt = vec / a.Hkv;
            t = (int)(bt % a.max_len);
            b = (int)(bt / a.max_len);
        }
        int L = in ? a.seq_lens[b] : 0;
        if (L < 0 || L > a.max_blocks * kBlock) {
            if (sub == 0 && t == 0 && h == 0) flag_status(a.status, TQ_STATUS_BAD_LEN);
            L = 0;
        }
        const unsigned char* rec = nullptr;
        if (in && t < L) {
            const int pb = a.block_tables[(size_t)b * a.max_blocks + t / kBlock];
            if (pb >= 0 && pb < a.num_blocks)
                rec = a.cache + ((size_t)pb * a.Hkv + h) * (size_t)R::kBytes;
            else if (sub == 0)
                flag_status(a.status, TQ_STATUS_BAD_BLOCK);
        }
        const int off = t % kBlock;
        float kx[8], vx[8];
        float nrm = 0.f, s = 0.f, z = 0.f;
        uint32_t kw = 0, vw = 0;
        if (rec) {
            kw = *reinterpret_cast<const uint32_t*>(rec + R::kKCodes + off * R::kCodeRow + sub * 4);
#pragma unroll
            for (int i = 0; i < 4; i++)
                vw |= (uint32_t)rec[R::kVCodes + R::vcode_pos(off, 4 * sub + i)] << (8 * i);
            nrm = half_bits_to_float(*reinterpret_cast<const uint16_t*>(rec + R::kKNorm + off * 2));
            const int gp = R::group_pos(off, sub / 4);
            s = half_bits_to_float(*reinterpret_cast<const uint16_t*>(rec + R::kVScale + gp));
            z = half_bits_to_float(*reinterpret_cast<const uint16_t*>(rec + R::kVZero + gp));
        }
        const float* C = ctab[h < 64 ? h : 0];
#pragma unroll
        for (int e = 0; e < 8; e++) {
            kx[e] = C[(kw >> (4 * e)) & 15];
            vx[e] = fmaf((float)((vw >> (4 * e)) & 15), s, z);
        }
        // inverse rotation: the same +-1 butterfly, then 1/sqrt(D) (none for an
        // unrotated cache; the branch is uniform over the grid)
        if (a.rotate) {
#pragma unroll
            for (int m = 1; m < 8; m <<= 1) {
#pragma unroll
                for (int e = 0; e < 8; e++)
                    if (!(e & m)) {
                        float x = kx[e], y = kx[e | m];
                        kx[e] = x + y;
                        kx[e | m] = x - y;
                    }
            }
#pragma unroll
            for (int m = 1; m < LPV; m <<= 1) {
                const bool upper = sub & m;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    float p = __shfl_xor_sync(kFull, kx[e], m);
                    kx[e] = upper ? p - kx[e] : kx[e] + p;
                }
            }
        }
        if (in) {
            const float f = rec ? (a.rotate ? nrm * inv_sqrt_d : nrm) : 0.f;
            const size_t o = (size_t)vec * D + sub * 8;
            float4* kd = reinterpret_cast<float4*>(a.K_hat + o);
            float4* vd = reinterpret_cast<float4*>(a.V_hat + o);
            kd[0] = make_float4(kx[0] * f, kx[1] * f, kx[2] * f, kx[3] * f);
            kd[1] = make_float4(kx[4] * f, kx[5] * f, kx[6] * f, kx[7] * f);
            if (rec) {
                vd[0] = make_float4(vx[0], vx[1], vx[2], vx[3]);
                vd[1] = make_float4(vx[4], vx[5], vx[6], vx[7]);
            } else {
                vd[0] = make_float4(0.f, 0.f, 0.f, 0.f);
                vd[1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
}

cudaError_t launch_dequant(const DequantArgs& a, int head_dim, int num_sms, cudaStream_t stream) {
    const int threads = 256;
    const long long vectors = (long long)a.B * a.max_len * a.Hkv;
    const int vpw = 32 / (head_dim / 8);
    long long blocks = ((vectors + vpw - 1) / vpw + threads / 32 - 1) / (threads / 32);
    const long long cap = (long long)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (head_dim == 128)
        dequant_kernel<128><<<(unsigned)blocks, threads, 0, stream>>>(a);
    else
        dequant_kernel<64><<<(unsigned)blocks, threads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace tq
