// ss2d_scan_launch.cuh -- launchers of the scan passes (state pass, carry,
// output pass) for one input dtype; included by ss2d_scan_bf16.cu and
// ss2d_scan_f32.cu so that the two dtypes compile as separate units.
#pragma once

#include <cuda_bf16.h>

#include "ss2d_kernels.cuh"
#include "ss2d_launch.h"
#include "ss2d_scan.cuh"

namespace ss2d {
namespace {

// Minimum resident CTAs per SM the kernels are compiled for, from a register
// cap R per thread: R = 128 gives 16 warps per SM, R = 168 gives 12 (more room
// for the compiler to keep loads in flight and interleave steps).
template <int WC, int R>
struct MinBlocks {
    static constexpr int value = 65536 / (32 * WC * R);
};

template <typename Tin, int WC, int MODE, int R>
cudaError_t launch_chunk(const ScanParams &p, int ncg, cudaStream_t st, bool dependent)
{
    using Sh = ChunkShape<WC>;
    constexpr int MB = MinBlocks<WC, R>::value;
    // the column-major path only where a direction is column-major; half the
    // state work when this call (or state group) has at most 8 states
    const bool cols = p.two_d && p.K == 4, eight = p.N <= 8;
    auto kern = cols ? (eight ? chunk_scan_kernel<Tin, WC, MODE, MB, true, 2>
                              : chunk_scan_kernel<Tin, WC, MODE, MB, true, 4>)
                     : (eight ? chunk_scan_kernel<Tin, WC, MODE, MB, false, 2>
                              : chunk_scan_kernel<Tin, WC, MODE, MB, false, 4>);
    const size_t smem = Sh::SMEM_BYTES;
    if (smem > 48 * 1024) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    const long long nz = (long long)p.B * ncg;   // (b, chunk) pairs, looped past 65535
    dim3 grid((unsigned)p.K, (unsigned)((p.D + Sh::NT - 1) / Sh::NT),
              (unsigned)(nz < 65535 ? nz : 65535));
    return launch_kernel(kern, grid, dim3(Sh::NT), smem, st, dependent, p);
}

// lane_scan_kernel with a cap of R registers per thread (128: 16 warps per SM)
template <typename Tin, int WC, int R, int MODE, int CPL, bool C, int Q, bool A, bool F = false>
cudaError_t launch_lane_k(const ScanParams &p, int ncg, cudaStream_t st, bool dependent)
{
    using Sh = LaneShape<Tin, WC, C, A, F, CPL>;
    constexpr int MB = 65536 / (32 * WC * R);
    auto kern = lane_scan_kernel<Tin, WC, MODE, MB, C, Q, A, F, CPL>;
    const size_t smem = Sh::SMEM_BYTES;
    // the largest shared-memory carveout, so that 16 warps per SM fit
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    const long long blocks = (long long)((p.D + Sh::CH - 1) / Sh::CH) * p.K * p.B * ncg;
    if (blocks > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    return launch_kernel(kern, dim3((unsigned)blocks), dim3(Sh::NT), smem, st, dependent, p);
}

template <typename Tin, int WC, int R, int MODE, int CPL>
cudaError_t launch_lane(const ScanParams &p, int ncg, cudaStream_t st, bool dependent)
{
    // the column-major path only where a direction is column-major; half the
    // state work when this call (or state group) has at most 8 states; packed
    // row copies when every row starts on an 8-byte boundary
    const bool cols = p.two_d && p.K == 4, eight = p.N <= 8, aligned = p.vec >= 8;
    if (p.front)   // the fused front's scratch rows: 1D, aligned
        return eight ? launch_lane_k<Tin, WC, R, MODE, CPL, false, 2, true, true>(p, ncg, st, dependent)
                     : launch_lane_k<Tin, WC, R, MODE, CPL, false, 4, true, true>(p, ncg, st, dependent);
    if (cols) {
        if (eight)
            return aligned ? launch_lane_k<Tin, WC, R, MODE, CPL, true, 2, true>(p, ncg, st, dependent)
                           : launch_lane_k<Tin, WC, R, MODE, CPL, true, 2, false>(p, ncg, st, dependent);
        return aligned ? launch_lane_k<Tin, WC, R, MODE, CPL, true, 4, true>(p, ncg, st, dependent)
                       : launch_lane_k<Tin, WC, R, MODE, CPL, true, 4, false>(p, ncg, st, dependent);
    }
    if (eight)
        return aligned ? launch_lane_k<Tin, WC, R, MODE, CPL, false, 2, true>(p, ncg, st, dependent)
                       : launch_lane_k<Tin, WC, R, MODE, CPL, false, 2, false>(p, ncg, st, dependent);
    return aligned ? launch_lane_k<Tin, WC, R, MODE, CPL, false, 4, true>(p, ncg, st, dependent)
                   : launch_lane_k<Tin, WC, R, MODE, CPL, false, 4, false>(p, ncg, st, dependent);
}

template <typename Tin, int LAYOUT, int WC, int R, int MODE>
cudaError_t launch_pass(const ScanParams &p, int ncg, cudaStream_t st, bool dependent)
{
    if constexpr (LAYOUT == 0)
        return launch_chunk<Tin, WC, MODE, R>(p, ncg, st, dependent);
    else
        return launch_lane<Tin, WC, R, MODE, 1>(p, ncg, st, dependent);
}

template <typename Tin, int LAYOUT, int WC, int R>
cudaError_t launch_passes(const Plan &plan, ScanParams &p, cudaStream_t st, cudaEvent_t *ev)
{
    cudaError_t e;
    if (plan.NC > 1) {
        if (ev)
            cudaEventRecord(ev[0], st);
        e = launch_pass<Tin, LAYOUT, WC, R, kModeState>(p, plan.NC - 1, st, false);
        if (e != cudaSuccess)
            return e;
        if (ev)
            cudaEventRecord(ev[1], st);
        // with two chunks the end state of the first is already the entry
        // state of the second: no carry to combine
        if (plan.NC > 2)
            e = launch_carry_scan(p, st, ev == nullptr);
        if (e != cudaSuccess)
            return e;
    }
    if (ev)
        cudaEventRecord(ev[2], st);
    e = launch_pass<Tin, LAYOUT, WC, R, kModeOutput>(p, plan.NC, st, plan.NC > 1 && ev == nullptr);
    if (ev)
        cudaEventRecord(ev[3], st);
    return e;
}

}  // namespace

// The scan passes of a plan for input dtype Tin (see launch_scan).
template <typename Tin>
cudaError_t launch_scan_t(const Plan &plan, ScanParams &p, cudaStream_t st, cudaEvent_t *ev)
{
#define SS2D_DISPATCH(LY, WCV, RV)                                       \
    if (plan.layout == LY && plan.wc == WCV && plan.regs == RV)          \
        return launch_passes<Tin, LY, WCV, RV>(plan, p, st, ev);
    SS2D_DISPATCH(0, 1, 128)
    SS2D_DISPATCH(0, 2, 128)
    SS2D_DISPATCH(0, 4, 128)
    SS2D_DISPATCH(0, 2, 168)
    SS2D_DISPATCH(0, 4, 168)
    SS2D_DISPATCH(2, 2, 128)
#undef SS2D_DISPATCH
    return cudaErrorInvalidValue;
}

}  // namespace ss2d
