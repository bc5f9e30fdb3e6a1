// ss2d_launch.cu -- kernel variants, the execution plan of a call, launchers.
#include "ss2d_launch.h"

#include <cuda_bf16.h>

#include "ss2d_kernels.cuh"

namespace ss2d {

namespace {

// name: wc<W>_<chunking>; wc = 32-channel warps per CTA.
const VariantInfo kVariants[] = {
    {"wc2_auto", 2, 0},    {"wc4_auto", 4, 0},    {"wc1_auto", 1, 0},
    {"wc2_lc16", 2, 16},   {"wc4_lc64", 4, 64},   {"wc2_nochunk", 2, -1},
    {"wc2_lc256", 2, 256}, {"wc4_lc512", 4, 512}, {"wc1_lc128", 1, 128},
};
constexpr int kNumVariants = sizeof(kVariants) / sizeof(kVariants[0]);

// Minimum resident CTAs per SM the kernels are compiled for: 20 warps per
// SM, a register cap of 65536 / 640 = 102 per thread.
template <int WC>
struct MinBlocks {
    static constexpr int value = 20 / WC;
};

template <typename Tin, int WC, int MODE>
cudaError_t launch_chunk(const ScanParams &p, int ncg, cudaStream_t st)
{
    using Sh = ChunkShape<WC>;
    auto kern = chunk_scan_kernel<Tin, WC, MODE, MinBlocks<WC>::value>;
    const size_t smem = Sh::SMEM_BYTES;
    if (smem > 48 * 1024) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    dim3 grid((unsigned)p.K, (unsigned)((p.D + Sh::NT - 1) / Sh::NT), (unsigned)(p.B * ncg));
    kern<<<grid, Sh::NT, smem, st>>>(p);
    return cudaGetLastError();
}

template <typename Tin, int WC>
cudaError_t launch_passes(const Plan &plan, ScanParams &p, cudaStream_t st, cudaEvent_t *ev)
{
    cudaError_t e;
    if (plan.NC > 1) {
        if (ev)
            cudaEventRecord(ev[0], st);
        e = launch_chunk<Tin, WC, kModeState>(p, plan.NC - 1, st);
        if (e != cudaSuccess)
            return e;
        if (ev)
            cudaEventRecord(ev[1], st);
        const long long total = (long long)p.B * p.K * p.D * kNP;
        const int threads = 256;
        carry_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, st>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    if (ev)
        cudaEventRecord(ev[2], st);
    e = launch_chunk<Tin, WC, kModeOutput>(p, plan.NC, st);
    if (ev)
        cudaEventRecord(ev[3], st);
    return e;
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
    (void)B;
    (void)H;
    (void)W;
    (void)N;
    (void)K;
    if (D <= 32)
        return 2;   // wc1_auto
    return 0;       // wc2_auto
}

Plan make_plan(int v, int B, int D, int L, int K)
{
    const VariantInfo *vi = variant(v);
    Plan pl;
    pl.variant = v;
    pl.wc = vi->wc;
    int lc;
    if (vi->chunk > 0) {
        lc = vi->chunk;
    } else if (vi->chunk < 0) {
        lc = L;
    } else {
        // enough lanes for about four resident warps per SM sub-partition on
        // 148 SMs; short sequences are never split
        const long long want = 148LL * 16 * 32;
        const long long seqs = (long long)B * K * D;
        long long nc = (seqs >= want / 2 || L <= 512) ? 1 : (want + seqs - 1) / seqs;
        if (nc < 1)
            nc = 1;
        lc = (int)((L + nc - 1) / nc);
    }
    lc = ((lc + kT - 1) / kT) * kT;
    if (lc < kT)
        lc = kT;
    pl.LC = lc;
    pl.NC = (L + lc - 1) / lc;
    pl.launches = (pl.NC > 1 ? 3 : 1) + (K > 1 ? 1 : 0);
    return pl;
}

cudaError_t launch_scan(const Plan &plan, bool bf16, ScanParams &p, cudaStream_t st,
                        cudaEvent_t *ev)
{
    p.LC = plan.LC;
    p.NC = plan.NC;
    switch (plan.wc) {
    case 1:
        return bf16 ? launch_passes<__nv_bfloat16, 1>(plan, p, st, ev)
                    : launch_passes<float, 1>(plan, p, st, ev);
    case 2:
        return bf16 ? launch_passes<__nv_bfloat16, 2>(plan, p, st, ev)
                    : launch_passes<float, 2>(plan, p, st, ev);
    case 4:
        return bf16 ? launch_passes<__nv_bfloat16, 4>(plan, p, st, ev)
                    : launch_passes<float, 4>(plan, p, st, ev);
    default:
        return cudaErrorInvalidValue;
    }
}

namespace {
// merge work unit: cpb channels x R image rows, about 2048 pixels
void merge_shape(int H, int W, int K, int two_d, int *R, int *cpb)
{
    const bool cols = two_d && K == 4;
    int r = cols ? 2048 / (W > 0 ? W : 1) : H;
    if (r < 8)
        r = 8;
    if (r > H)
        r = H;
    *R = r;
    const long long px = (long long)r * W;
    long long c = px >= 2048 ? 1 : 2048 / (px > 0 ? px : 1);
    if (c < 1)
        c = 1;
    *cpb = (int)c;
}
}  // namespace

size_t merge_smem_bytes(int H, int W, int K, int two_d)
{
    if (!(two_d && K == 4))
        return 0;
    int R, cpb;
    merge_shape(H, W, K, two_d, &R, &cpb);
    return sizeof(float) * (size_t)cpb * 2 * W * (R + 1);
}

cudaError_t launch_merge(const float *part, float *y, int B, int D, int H, int W, int K,
                         int two_d, int sum, cudaStream_t st)
{
    int R, cpb;
    merge_shape(H, W, K, two_d, &R, &cpb);
    const size_t smem = merge_smem_bytes(H, W, K, two_d);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(merge_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    const int nblk = (H + R - 1) / R;
    const long long groups = ((long long)B * D + cpb - 1) / cpb;
    merge_kernel<<<(unsigned)(groups * nblk), 256, smem, st>>>(part, y, B, D, H, W, K, two_d,
                                                               sum, R, cpb);
    return cudaGetLastError();
}

}  // namespace ss2d
