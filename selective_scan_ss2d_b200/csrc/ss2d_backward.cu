// ss2d_backward.cu -- plan and launch sequence of the backward pass (kernels
// in ss2d_backward.cuh), for the three input dtypes.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ss2d_backward.cuh"
#include "ss2d_scan.cuh"
#include "ss2d_launch.h"

namespace ss2d {

namespace {
// CTAs (one per channel group and chunk range) wanted per launch: 2960 = 148
// SMs x 20, about 6.7 waves of the final pass (3 four-warp CTAs per SM);
// fewer ranges would leave SMs idle on the small-batch shapes, more would
// add carry work
constexpr long long kBwdWantCtas = 148LL * 5 * 4;

template <typename Tin>
cudaError_t launch_bwd_t(const BwdParams &p, cudaStream_t st)
{
    const dim3 grid((unsigned)((long long)p.G * p.B * p.K), (unsigned)p.CGN);
    if (p.NC > 1) {
        bwd_local4_kernel<Tin><<<grid, kBwd4Threads, 0, st>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
        // the forward's carry scan over the chunk end states, then over the
        // reversed local adjoints
        ScanParams c{};
        c.A_log = p.A_log;
        c.B = p.B;
        c.D = p.D;
        c.K = p.K;
        c.N = p.N;      // this state group's states, rows n0.. of A_log
        c.n0 = p.n0;
        c.NS = p.NS;
        c.L = p.L;
        c.NC = p.NC;
        c.hstate = p.hfwd;
        c.dtsum = p.dtf;
        e = launch_carry_scan(c, st, false);
        if (e == cudaSuccess && p.adj_chunks) {
            c.hstate = p.hadj;
            c.dtsum = p.dta;
            e = launch_carry_scan(c, st, false);
        }
        if (e != cudaSuccess)
            return e;
    }
    // the final pass: 4 warps per channel group, 4 states each
    auto kern = bwd_final4_kernel<Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kBwd4Smem);
    if (e != cudaSuccess)
        return e;
    kern<<<grid, kBwd4Threads, kBwd4Smem, st>>>(p);
    return cudaGetLastError();
}
}  // namespace

BwdShape backward_shape(int B, int D, int L, int K)
{
    BwdShape s;
    s.NC = (L + kT - 1) / kT;
    s.G = (D + kBwdLanes - 1) / kBwdLanes;
    const long long ctas = (long long)s.G * B * K;
    long long cgn = ctas > 0 ? (kBwdWantCtas + ctas - 1) / ctas : 1;
    if (cgn > s.NC)
        cgn = s.NC;
    if (cgn < 1)
        cgn = 1;
    long long cpb = (s.NC + cgn - 1) / cgn;
    const long long min_cpb = (s.NC + 65534) / 65535;   // gridDim.y <= 65535
    if (cpb < min_cpb)
        cpb = min_cpb;
    if (cpb < 1)
        cpb = 1;
    s.CPB = (int)cpb;
    s.CGN = (int)((s.NC + cpb - 1) / cpb);
    return s;
}

cudaError_t launch_backward(const BwdParams &p, int dtype, cudaStream_t st)
{
    // more than 16 states: the passes once per group of at most 16, in order
    // on the stream, later groups adding to the first group's rows
    const int ns = p.NS;
    if (p.dxmerge && (p.K != 2 || ns > kNP))
        return cudaErrorInvalidValue;   // the dx merge by adds: two directions, one group
    cudaError_t e = cudaSuccess;
    for (int n0 = 0; n0 < ns && e == cudaSuccess; n0 += kNP) {
        BwdParams q = p;
        q.n0 = n0;
        q.N = ns - n0 < kNP ? ns - n0 : kNP;
        q.accum = n0 > 0 ? 1 : 0;
        switch (dtype) {
        case 1:
            e = launch_bwd_t<__nv_bfloat16>(q, st);
            break;
        case 2:
            e = launch_bwd_t<__half>(q, st);
            break;
        default:
            e = launch_bwd_t<float>(q, st);
            break;
        }
    }
    return e;
}

cudaError_t launch_backward_reduce(const BwdParams &p, float *dBs, float *dCs, float *dA_log,
                                   float *dDskip, float *ddelta_bias, cudaStream_t st)
{
    const long long rows = (long long)p.B * p.K * 2 * p.NS;   // one CTA per dBs | dCs row
    if (rows > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    const int vec = ((p.L & 3) == 0 && ((reinterpret_cast<uintptr_t>(dBs) |
                                         reinterpret_cast<uintptr_t>(dCs) |
                                         reinterpret_cast<uintptr_t>(p.bc_part)) & 15) == 0)
                        ? 1
                        : 0;
    bwd_reduce_bc_kernel<<<(unsigned)rows, kReduceBcThreads, 0, st>>>(p.bc_part, dBs, dCs, p.G,
                                                                     p.NS, p.L, vec);
    const long long npr = (long long)p.K * p.D * (p.NS + 2);   // one warp each
    long long blocks = (npr + kReduceParamThreads / 32 - 1) / (kReduceParamThreads / 32);
    if (blocks > 148LL * 64)
        blocks = 148LL * 64;
    bwd_reduce_param_kernel<<<(unsigned)blocks, kReduceParamThreads, 0, st>>>(
        p.prm_part, p.A_log, dA_log, dDskip, ddelta_bias, p.B, p.K, p.D, p.NS, p.CGN);
    return cudaGetLastError();
}

}  // namespace ss2d
