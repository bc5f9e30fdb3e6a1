// ss2d_launch.cu -- the table of kernel variants and their launchers.
#include "ss2d_launch.h"

#include <cuda_bf16.h>

#include "ss2d_kernels.cuh"

namespace ss2d {

namespace {

template <typename Tin, int G, int JW, int J, int WC, int I, int MINB>
cudaError_t launch_scan(const ScanParams &p, cudaStream_t st)
{
    using Sh = ScanShape<G, JW, J, WC, I>;
    auto kern = scan_fwd_kernel<Tin, G, JW, J, WC, I, MINB>;
    const size_t smem = Sh::SMEM_BYTES;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(
            kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    dim3 grid((unsigned)((p.D + Sh::DC - 1) / Sh::DC), (unsigned)p.K, (unsigned)p.B);
    kern<<<grid, Sh::NT, smem, st>>>(p);
    return cudaGetLastError();
}

template <int G, int JW, int J, int WC, int I, int MINB>
VariantInfo make_variant(const char *name)
{
    using Sh = ScanShape<G, JW, J, WC, I>;
    VariantInfo v;
    v.name = name;
    v.G = G;
    v.JW = JW;
    v.J = J;
    v.WC = WC;
    v.I = I;
    v.channels_per_cta = Sh::DC;
    v.threads = Sh::NT;
    v.chunk = Sh::LC;
    v.smem_bytes = Sh::SMEM_BYTES;
    v.launch_f32 = &launch_scan<float, G, JW, J, WC, I, MINB>;
    v.launch_bf16 = &launch_scan<__nv_bfloat16, G, JW, J, WC, I, MINB>;
    return v;
}

// name: <path>_g<G>_jw<JW>_j<J>_wc<WC>_i<I>
const VariantInfo kVariants[] = {
    // direct: one lane per channel (G = 1) or per quarter channel (G = 4)
    make_variant<1, 1, 1, 2, 16, 8>("direct_g1_jw1_j1_wc2_i16"),
    make_variant<1, 1, 1, 4, 16, 4>("direct_g1_jw1_j1_wc4_i16"),
    make_variant<4, 1, 1, 4, 32, 4>("direct_g4_jw1_j1_wc4_i32"),
    make_variant<4, 1, 1, 2, 64, 6>("direct_g4_jw1_j1_wc2_i64"),
    // split in time: NS = J * JW segments per chunk
    make_variant<4, 1, 4, 1, 16, 4>("split_g4_jw1_j4_wc1_i16"),
    make_variant<4, 2, 2, 1, 16, 8>("split_g4_jw2_j2_wc1_i16"),
    make_variant<4, 2, 1, 1, 16, 12>("split_g4_jw2_j1_wc1_i16"),
    make_variant<4, 4, 2, 1, 16, 8>("split_g4_jw4_j2_wc1_i16"),
    make_variant<4, 8, 1, 1, 16, 12>("split_g4_jw8_j1_wc1_i16"),
    make_variant<4, 8, 2, 1, 16, 8>("split_g4_jw8_j2_wc1_i16"),
    make_variant<4, 8, 4, 1, 16, 4>("split_g4_jw8_j4_wc1_i16"),
    make_variant<4, 4, 1, 1, 8, 16>("split_g4_jw4_j1_wc1_i8"),
};
constexpr int kNumVariants = sizeof(kVariants) / sizeof(kVariants[0]);

template <int K>
cudaError_t launch_merge_k(const float *part, float *y, long long DL, long long total,
                           cudaStream_t st)
{
    const int threads = 256;
    long long work = (DL % 4 == 0) ? total / 4 : total;
    long long blocks = (work + threads - 1) / threads;
    const long long cap = 148LL * 16;
    if (blocks > cap)
        blocks = cap;
    if (blocks < 1)
        blocks = 1;
    merge_kernel<K><<<(unsigned)blocks, threads, 0, st>>>(part, y, DL, total);
    return cudaGetLastError();
}

}  // namespace

int num_variants() { return kNumVariants; }

const VariantInfo *variant(int i)
{
    if (i < 0 || i >= kNumVariants)
        return nullptr;
    return &kVariants[i];
}

int pick_variant(int two_d, int B, int D, int H, int W, int N, int K)
{
    (void)two_d;
    (void)N;
    const long long L = (long long)H * W;
    const long long seqs = (long long)B * K * D;
    // Lanes wanted on the GPU at once: ~4 warps per SM sub-partition on
    // 148 SMs.  A G = 1 lane carries one channel; a G = 4 lane a quarter.
    const long long want = 148LL * 4 * 4 * 32;
    if (seqs >= want)
        return 1;                        // direct_g1_wc4
    if (seqs * 4 >= want || L <= 256)
        return 2;                        // direct_g4_wc4
    // split in time: pick the segment count that reaches the target
    const long long per_seg = seqs * 4;
    if (per_seg * 4 >= want)
        return 5;                        // split_g4_jw2_j2 (NS = 4)
    if (per_seg * 8 >= want)
        return 7;                        // split_g4_jw4_j2 (NS = 8)
    if (per_seg * 16 >= want)
        return 9;                        // split_g4_jw8_j2 (NS = 16)
    return 10;                           // split_g4_jw8_j4 (NS = 32)
}

cudaError_t launch_scan_variant(int v, bool bf16, const ScanParams &p, cudaStream_t st)
{
    const VariantInfo *vi = variant(v);
    if (!vi)
        return cudaErrorInvalidValue;
    return bf16 ? vi->launch_bf16(p, st) : vi->launch_f32(p, st);
}

cudaError_t launch_merge(int K, const float *part, float *y, long long DL, long long total,
                         cudaStream_t st)
{
    switch (K) {
    case 2:
        return launch_merge_k<2>(part, y, DL, total, st);
    case 4:
        return launch_merge_k<4>(part, y, DL, total, st);
    default:
        return cudaErrorInvalidValue;
    }
}

}  // namespace ss2d
