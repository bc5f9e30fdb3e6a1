// ss2d_launch.cu -- kernel variants, the execution plan of a call, launchers.
#include "ss2d_launch.h"

#include <cuda_bf16.h>

#include "ss2d_kernels.cuh"
#include "ss2d_scan.cuh"

namespace ss2d {

namespace {

// name: wc<W>_<chunking>: one lane per channel, wc = 32-channel warps per CTA;
// chunking: auto (from the shape), lc<N> (N steps), nochunk, lcfit (the
// multiple of 16 in 96..160 that pads the sequence least, ties toward 128);
// lane<W>_<chunking>: the cp.async lane kernel (wave: chunks for about one wave).
const VariantInfo kVariants[] = {
    {"wc2_auto", 2, 0, 128},       {"wc4_auto", 4, 0, 128},       {"wc1_auto", 1, 0, 128},
    {"wc2_lc16", 2, 16, 128},      {"wc4_lc64", 4, 64, 128},      {"wc2_nochunk", 2, -1, 128},
    {"wc2_lc256", 2, 256, 128},    {"wc4_lc512", 4, 512, 128},    {"wc1_lc128", 1, 128, 128},
    {"wc2_auto_r168", 2, 0, 168},  {"wc4_auto_r168", 4, 0, 168},  {"wc4_lc64_r168", 4, 64, 168},
    {"wc2_lc128_r168", 2, 128, 168},
    {"wc2_lc256_r168", 2, 256, 168}, {"wc2_lc512_r168", 2, 512, 168},
    {"wc2_lcfit_r168", 2, -2, 168},
    {"lane2_wave", 2, -3, 128, 2},   {"lane2_nochunk", 2, -1, 128, 2},
    {"lane2_lc128", 2, 128, 128, 2}, {"lane2_lc16", 2, 16, 128, 2},
};
constexpr int kNumVariants = sizeof(kVariants) / sizeof(kVariants[0]);

}  // namespace

int num_variants() { return kNumVariants; }

int variant_index(const char *name)
{
    for (int i = 0; i < kNumVariants; ++i) {
        const char *a = kVariants[i].name, *b = name;
        while (*a && *a == *b) {
            ++a;
            ++b;
        }
        if (*a == 0 && *b == 0)
            return i;
    }
    return -1;
}

const VariantInfo *variant(int i)
{
    if (i < 0 || i >= kNumVariants)
        return nullptr;
    return &kVariants[i];
}

namespace {
// CTAs of lane_scan_kernel (two warps, 2-byte inputs, aligned rows, 128
// registers per thread) resident on one SM: limited by registers and by the
// 228 KB of shared memory per SM (1 KB of it reserved per CTA)
int lane_ctas_per_sm(bool cols)
{
    const size_t smem = cols ? LaneShape<__nv_bfloat16, 2, true, true>::SMEM_BYTES
                             : LaneShape<__nv_bfloat16, 2, false, true>::SMEM_BYTES;
    const int by_regs = 65536 / (32 * 2 * 128);
    const int by_smem = (int)((228u * 1024u) / (smem + 1024u));
    int n = by_regs < by_smem ? by_regs : by_smem;
    return n < 1 ? 1 : (n > 32 ? 32 : n);
}

// Sequences of a call are split into chunks when there are too few of them
// to give every SM sub-partition about four resident warps.
constexpr long long kWantLanes = 148LL * 16 * 32;

bool wants_chunks(long long seqs, long long L)
{
    return seqs < kWantLanes / 2 && L > 512;
}
}  // namespace

int pick_variant(int two_d, int B, int D, int H, int W, int N, int K)
{
    (void)N;
    const long long L = two_d ? (long long)H * W : (long long)W;
    // chunked shapes: 128-step chunks with the 168-register kernels (fewer,
    // fuller warps hide the longer per-chunk dependency chains better)
    if (wants_chunks((long long)B * K * D, L))
        return variant_index("wc2_lcfit_r168");
    // a handful of sequences of 64..512 steps (at most 1024 channels in all:
    // a few warps on the whole GPU): 16-step chunks, so that the scan's
    // latency is a chunk's and not a sequence's (B = 1, D = 8, 8 x 8, K = 4:
    // 28.9 -> 23.2 us per call with the extra carry launch)
    if ((long long)B * K * D <= 1024 && L >= 64 && L <= 512)
        return variant_index("wc2_lc16");
    // SS2D (four directions, two column-major) unchunked: 64-channel CTAs at
    // 168 registers
    if (two_d && K == 4 && D % 64 == 0)
        return variant_index("wc2_auto_r168");
    // otherwise the widest CTA that leaves no channel tile mostly empty
    if (D % 128 == 0)
        return variant_index("wc4_auto");
    if (D % 64 == 0 || D > 64)
        return variant_index("wc2_auto");
    return variant_index("wc1_auto");
}

Plan make_plan(int v, int B, int D, int L, int K)
{
    const VariantInfo *vi = variant(v);
    Plan pl;
    pl.variant = v;
    pl.wc = vi->wc;
    pl.regs = vi->regs;
    pl.layout = vi->layout;
    int lc;
    if (vi->chunk > 0) {
        lc = vi->chunk;
    } else if (vi->chunk == -2) {
        // chunks of about 128 steps that leave the last one as full as possible
        lc = 128;
        long long best = -1;
        for (int c = 96; c <= 160; c += kT) {
            const long long pad = ((L + c - 1) / c) * (long long)c - L;
            const long long key = pad * 1024 + (c > 128 ? c - 128 : 128 - c);
            if (best < 0 || key < best) {
                best = key;
                lc = c;
            }
        }
        if (lc > L)
            lc = L;
    } else if (vi->chunk == -3) {
        // about one wave of CTAs: the chunks that fill the CTAs resident on
        // 148 SMs (2-byte inputs, 128 registers per thread), at least 64 steps each
        const long long seqs = (long long)B * K * D;
        long long nc = 1;
        if (wants_chunks(seqs, L)) {
            const int ch = 32 * vi->wc;   // channels per CTA
            const long long ctas_per_chunk = (long long)((D + ch - 1) / ch) * K * B;
            nc = (148LL * lane_ctas_per_sm(K == 4)) / (ctas_per_chunk > 0 ? ctas_per_chunk : 1);
            if (nc < 2)
                nc = 2;
        }
        lc = (int)((L + nc - 1) / nc);
        if (lc < 64)
            lc = L < 64 ? L : 64;
    } else if (vi->chunk < 0) {
        lc = L;
    } else {
        // enough lanes for about four resident warps per SM sub-partition on
        // 148 SMs; short sequences are never split
        const long long seqs = (long long)B * K * D;
        long long nc = wants_chunks(seqs, L) ? (kWantLanes + seqs - 1) / seqs : 1;
        if (nc < 1)
            nc = 1;
        lc = (int)((L + nc - 1) / nc);
    }
    lc = ((lc + kT - 1) / kT) * kT;
    if (lc < kT)
        lc = kT;
    pl.LC = lc;
    pl.NC = (L + lc - 1) / lc;
    // chunked: state pass, carry (none with two chunks), output pass
    pl.launches = (pl.NC > 2 ? 3 : pl.NC > 1 ? 2 : 1) + (K > 1 ? 1 : 0);
    return pl;
}

cudaError_t launch_scan(const Plan &plan, int dtype, ScanParams &p, cudaStream_t st,
                        cudaEvent_t *ev)
{
    if (p.front && plan.layout != 2)
        return cudaErrorInvalidValue;   // only the lane kernel reads the front's rows
    if (p.ymerge && (p.K != 2 || p.N > kNP))
        return cudaErrorInvalidValue;   // the merge by adds: two directions, one state group
    p.LC = plan.LC;
    p.NC = plan.NC;
    // more than 16 states: the passes once per group of at most 16 states, in
    // order on the stream, the later groups adding to the first group's rows
    const int ns = p.N;
    cudaError_t e = cudaSuccess;
    for (int n0 = 0; n0 < ns && e == cudaSuccess; n0 += kNP) {
        ScanParams q = p;
        q.n0 = n0;
        q.NS = ns;
        q.N = ns - n0 < kNP ? ns - n0 : kNP;
        q.accum = n0 > 0 ? 1 : 0;
        cudaEvent_t *qev = n0 == 0 ? ev : nullptr;
        switch (dtype) {
        case 1:
            e = launch_scan_bf16(plan, q, st, qev);
            break;
        case 2:
            e = launch_scan_f16(plan, q, st, qev);
            break;
        default:
            e = launch_scan_f32(plan, q, st, qev);
            break;
        }
    }
    return e;
}

namespace {
// merge work unit (see merge2_kernel): bands of R full image rows holding
// about kMergeTarget pixels, and CG channels per CTA so that a CTA moves
// about kMergeTarget pixels of every direction; the column-major tiles of a
// CTA stay within 48 KB of shared memory.  Maps 128 pixels wide or more
// with column-major directions take half the pixels per CTA: their tiles
// then use half the shared memory and twice as many CTAs fit on an SM
// (256x256: 67.6 -> 55.3 us; narrower maps measured the same or slower).
constexpr int kMergeTarget = 4096;
constexpr size_t kMergeSmemMax = 48 * 1024;

struct MergeShape {
    int cols, vec, R, CG, nbands, whole, flat;
    size_t smem;
};

MergeShape merge_shape(int D, int H, int W, int K, int two_d)
{
    MergeShape m{};
    m.cols = (two_d && K == 4) ? 1 : 0;
    m.vec = (W % 4 == 0 && (!m.cols || H % 4 == 0)) ? 4 : 1;
    const int target = (m.cols && W >= 128) ? kMergeTarget / 2 : kMergeTarget;
    int R = W >= target ? 1 : target / W;
    if (R > H)
        R = H;
    if (m.vec == 4 && m.cols)
        R = R < 4 ? 4 : (R & ~3);   // H % 4 == 0, so R <= H stays true
    m.R = R;
    m.nbands = (H + R - 1) / R;
    const long long band = (long long)R * W;
    int cg = (int)(target / band);
    if (cg < 1)
        cg = 1;
    // a band that is the whole image whose column-major rows cannot use the
    // float4 transpose: copy those rows as they are
    const long long L = (long long)H * W;
    m.whole = (m.cols && m.vec == 1 && R == H && L % 4 == 0 &&
               sizeof(float) * 2 * L <= kMergeSmemMax) ? 1 : 0;
    const size_t per_ch = !m.cols ? 0
                          : m.whole ? sizeof(float) * 2 * (size_t)L
                                    : sizeof(float) * 2 * (size_t)R * (W + 1);
    while (cg > 1 && per_ch * cg > kMergeSmemMax)
        --cg;
    int cgp = 1;   // compiled channel-group sizes: 1, 2, 4, 8, 16
    while (cgp * 2 <= cg && cgp < 16)
        cgp *= 2;
    m.CG = cgp;
    m.smem = per_ch * cgp;
    m.flat = (!m.cols && m.nbands == 1 && D % cgp == 0 && cgp % 4 == 0) ? 1 : 0;
    return m;
}

template <int VEC, int CG>
cudaError_t launch_merge2(const MergeShape &m, const float *part, float *y, int B, int D,
                          int H, int W, int K, int sum, cudaStream_t st, const void *z,
                          int zt)
{
    const long long groups = ((long long)B * D + CG - 1) / CG;
    dim3 grid((unsigned)groups, (unsigned)m.nbands);
    // the gate is compiled in only for gated calls
    auto kern = z ? merge2_kernel<VEC, CG, true> : merge2_kernel<VEC, CG, false>;
    return launch_kernel(kern, grid, dim3(kMerge2Threads), m.smem, st, true, part, y, B, D, H,
                         W, K, m.cols, sum, m.R, m.whole, m.flat, z, zt);
}
}  // namespace


cudaError_t launch_merge(const float *part, float *y, int B, int D, int H, int W, int K,
                         int two_d, int sum, cudaStream_t st, const void *z, int zt)
{
    const MergeShape m = merge_shape(D, H, W, K, two_d);
    if (m.smem > kMergeSmemMax || m.nbands > 65535 || (long long)B * D > 0x7fffffffLL) {
        // too wide (or too many bands) for the band form: one pixel per thread
        const long long total = (long long)B * D * H * W;
        long long blocks = (total + 255) / 256;
        if (blocks > 148LL * 64)
            blocks = 148LL * 64;
        return launch_kernel(merge1_kernel, dim3((unsigned)blocks), dim3(256), 0, st, true, part,
                             y, B, D, H, W, K, m.cols, sum, z, zt);
    }
#define SS2D_MERGE(V, C)                                                             \
    if (m.vec == V && m.CG == C)                                                     \
        return launch_merge2<V, C>(m, part, y, B, D, H, W, K, sum, st, z, zt);
    SS2D_MERGE(4, 1) SS2D_MERGE(4, 2) SS2D_MERGE(4, 4) SS2D_MERGE(4, 8) SS2D_MERGE(4, 16)
    SS2D_MERGE(1, 1) SS2D_MERGE(1, 2) SS2D_MERGE(1, 4) SS2D_MERGE(1, 8) SS2D_MERGE(1, 16)
#undef SS2D_MERGE
    return cudaErrorInvalidValue;
}

}  // namespace ss2d
