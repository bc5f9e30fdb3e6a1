// ss2d_launch.cu -- the table of kernel variants and their launchers.
#include "ss2d_launch.h"

#include <cuda_bf16.h>

#include "ss2d_kernels.cuh"

namespace ss2d {

namespace {

template <typename Tin, int WC, int LC, int MINB>
cudaError_t launch_direct(const ScanParams &p, cudaStream_t st)
{
    using Sh = DirectShape<WC, LC>;
    dim3 grid((unsigned)p.K, (unsigned)((p.D + Sh::NT - 1) / Sh::NT), (unsigned)p.B);
    scan_direct_kernel<Tin, WC, LC, MINB><<<grid, Sh::NT, 0, st>>>(p);
    return cudaGetLastError();
}

template <typename Tin, int JW, int J, int I, int MINB>
cudaError_t launch_split(const ScanParams &p, cudaStream_t st)
{
    using Sh = SplitShape<Tin, JW, J, I>;
    auto kern = scan_split_kernel<Tin, JW, J, I, MINB>;
    const size_t smem = Sh::SMEM_BYTES;
    if (smem > 48 * 1024) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    dim3 grid((unsigned)p.K, (unsigned)((p.D + Sh::DC - 1) / Sh::DC), (unsigned)p.B);
    kern<<<grid, Sh::NT, smem, st>>>(p);
    return cudaGetLastError();
}

template <int WC, int LC, int MINB>
VariantInfo direct_variant(const char *name)
{
    using Sh = DirectShape<WC, LC>;
    VariantInfo v{};
    v.name = name;
    v.split = 0;
    v.channels_per_cta = Sh::NT;
    v.threads = Sh::NT;
    v.chunk = LC;
    v.segments = 1;
    v.smem_bytes = sizeof(float4) * 2 * LC * 8;
    v.launch_f32 = &launch_direct<float, WC, LC, MINB>;
    v.launch_bf16 = &launch_direct<__nv_bfloat16, WC, LC, MINB>;
    return v;
}

template <int JW, int J, int I, int MINB>
VariantInfo split_variant(const char *name)
{
    using Sh = SplitShape<__nv_bfloat16, JW, J, I>;
    VariantInfo v{};
    v.name = name;
    v.split = 1;
    v.channels_per_cta = Sh::DC;
    v.threads = Sh::NT;
    v.chunk = Sh::LC;
    v.segments = Sh::NS;
    v.smem_bytes = Sh::SMEM_BYTES;
    v.launch_f32 = &launch_split<float, JW, J, I, MINB>;
    v.launch_bf16 = &launch_split<__nv_bfloat16, JW, J, I, MINB>;
    return v;
}

// direct_wc<W>_lc<LC>: 32*W threads, one channel per thread, chunks of LC steps.
// split_jw<JW>_j<J>_i<I>: 4 lanes per channel, JW segments per warp, J warps,
// I steps per segment.
const VariantInfo kVariants[] = {
    direct_variant<4, 64, 4>("direct_wc4_lc64"),
    direct_variant<2, 64, 6>("direct_wc2_lc64"),
    direct_variant<4, 32, 4>("direct_wc4_lc32"),
    split_variant<2, 4, 16, 4>("split_jw2_j4_i16"),
    split_variant<2, 2, 16, 8>("split_jw2_j2_i16"),
    split_variant<1, 4, 16, 4>("split_jw1_j4_i16"),
    split_variant<4, 2, 16, 8>("split_jw4_j2_i16"),
    split_variant<4, 4, 16, 4>("split_jw4_j4_i16"),
    split_variant<8, 2, 16, 8>("split_jw8_j2_i16"),
    split_variant<8, 4, 16, 4>("split_jw8_j4_i16"),
    split_variant<8, 1, 16, 8>("split_jw8_j1_i16"),
    split_variant<1, 8, 16, 2>("split_jw1_j8_i16"),
    split_variant<2, 1, 16, 8>("split_jw2_j1_i16"),
};
constexpr int kNumVariants = sizeof(kVariants) / sizeof(kVariants[0]);

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
    // Lanes wanted resident at once: about four warps per SM sub-partition.
    const long long want = 148LL * 4 * 4 * 32;
    if (seqs * 2 >= want || L <= 256)
        return 0;                                 // direct_wc4_lc64
    const long long lanes4 = seqs * 4;            // split: 4 lanes per channel
    if (lanes4 * 4 >= want)
        return 4;                                 // split_jw2_j2 (4 segments)
    if (lanes4 * 8 >= want)
        return 6;                                 // split_jw4_j2 (8 segments)
    if (lanes4 * 16 >= want)
        return 8;                                 // split_jw8_j2 (16 segments)
    return 9;                                     // split_jw8_j4 (32 segments)
}

cudaError_t launch_scan_variant(int v, bool bf16, const ScanParams &p, cudaStream_t st)
{
    const VariantInfo *vi = variant(v);
    if (!vi)
        return cudaErrorInvalidValue;
    return bf16 ? vi->launch_bf16(p, st) : vi->launch_f32(p, st);
}

}  // namespace ss2d
