// tq_append.cu -- the TQ4/4 write path as its own kernel: one wave of
// resident CTAs whose warps loop over the passes (tq_append_impl.cuh).
#include "tq_append_impl.cuh"

namespace tq {

template <int D>
__global__ void __launch_bounds__(256, 3) append_kernel(AppendArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    HeadBins* hb = reinterpret_cast<HeadBins*>(smem);
    BinEntry* bins = reinterpret_cast<BinEntry*>(hb + a.Hkv);
    app::append_warps<D>(a, hb, bins, blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32,
                         gridDim.x * (blockDim.x / 32));
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

void prepare_append(AppendArgs& a, int head_dim) {
    if (!a.k_tables) default_bins(head_dim, a.default_table, a.default_hb, a.default_bins);
    a.div_hkv = div_magic((uint32_t)a.Hkv);
    a.div_cap = div_magic((uint32_t)(a.max_blocks > 0 ? a.max_blocks * kBlock : 1));
}

cudaError_t launch_append(const AppendArgs& args, int head_dim, int num_sms, cudaStream_t stream) {
    AppendArgs a = args;
    prepare_append(a, head_dim);
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
