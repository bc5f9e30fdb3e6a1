// ss2d_kernels.cuh -- sm_100a kernels of the SS2D forward path.
//
// Recurrence ("Vision Mamba" tutorial, section "Background: State Space
// Models and Mamba", SelectiveSSM; "Vision Mamba ..." summary, section 4.1),
// per direction k, channel d and state n:
//     dt_l = softplus(delta_l + bias)
//     h_l  = exp(dt_l * A_n) * h_{l-1} + dt_l * B_{n,l} * u_l        (h_{-1} = 0)
//     y_l  = sum_n C_{n,l} h_l + Dskip * u_l
// with u_l = x[pixel(k, l)]: the cross_scan is folded into the address
// generation; no unfolded copy of x exists.
//
// Work decomposition.  One lane owns one (b, k, d) channel with all 16
// states in registers; a CTA holds 32*WC channels of one (b, k).  Long
// sequences with few channels are cut into NC chunks of LC steps so that
// enough lanes exist; the chunks are independent given their entry state:
//   1. chunk_scan_kernel<..., kModeState>: every chunk but the last runs
//      from a zero state and stores its end state and its sum of dt;
//   2. carry_kernel: per (b,k,d,n), sequentially over the chunks,
//      h_in[c+1] = exp(A_n * sum_c(dt)) * h_in[c] + h_end[c];
//   3. chunk_scan_kernel<..., kModeOutput>: every chunk from its true entry
//      state, writing y_k in scan order (per-direction scratch, or y when
//      K = 1);
//   4. merge_kernel (K > 1): y[p] = ((Y_0[s_0(p)] + Y_1[s_1(p)]) +
//      Y_2[s_2(p)]) + Y_3[s_3(p)], s_k the pixel -> scan-step map of
//      direction k (cross_merge), always in that order.
// Chunking costs one extra exp per update on the chunked workloads only,
// and keeps every pass a uniform mix of MUFU and FMA work.
//
// Memory traffic is coalesced: per 32-step sub-chunk, each warp loads delta
// and x for its 32 channels two channels per instruction (lanes = 16 steps x
// 2 channels), applies softplus to delta as it stores them transposed into a
// warp-private shared-memory tile, and the outputs go back the same way.  B and C of a sub-chunk (shared by every channel of the CTA)
// are staged once per CTA as a float32 [step][32] tile, read with broadcast
// float4 loads.  The next sub-chunk's loads are spread over the current
// sub-chunk's compute (software pipelining; nothing waits on a flag).
//
// exp(dt*A) runs on the MUFU unit as 2^(dt * A*log2(e)).  The float32 pair
// arithmetic uses the sm_100 packed f32x2 instructions (__ffma2_rn,
// __fmul2_rn), which round each lane exactly as fmaf / a float multiply do.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ss2d_params.h"

namespace ss2d {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// 2^x on the multi-function unit (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float mufu_ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(z) = log(1 + e^z) = max(z, 0) + log1p(e), e = exp(-|z|) in (0, 1].
// log1p(e) = e * q(e) with q a degree-7 polynomial fitted (Chebyshev nodes,
// least squares) to log1p(e)/e on [0, 1]; evaluated in float32 its relative
// error stays below 4e-7 over the whole interval.  Never overflows: for large
// |z| the correction e underflows to 0.
__device__ __forceinline__ float softplus_f(float z)
{
    const float e = mufu_ex2(-fabsf(z) * kLog2e);
    float q = -8.574676205e-03f;
    q = fmaf(q, e, 4.421419234e-02f);
    q = fmaf(q, e, -1.078536792e-01f);
    q = fmaf(q, e, 1.775702399e-01f);
    q = fmaf(q, e, -2.449961172e-01f);
    q = fmaf(q, e, 3.327617657e-01f);
    q = fmaf(q, e, -4.999744938e-01f);
    q = fmaf(q, e, 9.999998102e-01f);
    return fmaf(e, q, fmaxf(z, 0.f));
}

// Walks direction k's scan -> pixel map (see include/ss2d.h) a fixed stride
// of steps at a time, without divisions.
struct PixWalk {
    int p;      // pixel of the current step (meaningful while the step is < L)
    int h, w;   // row and column, for the column-major directions
    int mode;   // 0: p = l; 1: p = L-1-l; 2: column-major; 3: reversed column-major

    __device__ __forceinline__ void init(int two_d, int k, int l, int H, int W, int L)
    {
        if (!two_d || k < 2) {
            mode = k & 1;
            p = (k & 1) ? L - 1 - l : l;
            h = w = 0;
        } else {
            mode = k;
            const int m = (k == 3) ? L - 1 - l : l;
            h = m % H;
            w = m / H;
            p = h * W + w;
        }
    }
    // advance by n = nq*H + nr steps (nq = n / H, nr = n % H precomputed)
    __device__ __forceinline__ void advance(int n, int nq, int nr, int H, int W)
    {
        if (mode == 0) {
            p += n;
        } else if (mode == 1) {
            p -= n;
        } else if (mode == 2) {
            h += nr;
            w += nq;
            if (h >= H) {
                h -= H;
                ++w;
            }
            p = h * W + w;
        } else {
            h -= nr;
            w -= nq;
            if (h < 0) {
                h += H;
                --w;
            }
            p = h * W + w;
        }
    }
};

enum ScanMode { kModeState = 0, kModeOutput = 1 };

template <int WC>
struct ChunkShape {
    static constexpr int NT = 32 * WC;                     // threads = channels per CTA
    static constexpr int TROW = 34;                        // padded row of a warp tile
    static constexpr int WTILE = kT * TROW;                // floats per warp tile
    static constexpr int BC_ENTRIES = kT * 8;              // float4 per B|C sub-chunk tile
    static constexpr int BC_PER_THREAD = (BC_ENTRIES + NT - 1) / NT;
    static_assert(kT == 16, "a warp stages two channels x 16 steps per load");
    static_assert(BC_PER_THREAD <= 4, "B|C staging spread over the 4 batches");
    // shared memory: B|C double buffer, then per warp the delta and x double
    // buffers (the delta tile is reused for the outputs)
    static constexpr size_t SMEM_BYTES =
        sizeof(float4) * 2 * BC_ENTRIES + sizeof(float) * WC * 4 * WTILE;
};

// One chunk of LC steps of 32*WC channels of one (b, k); see the header.
// grid: x = k, y = channel tile, z = b * NCg + chunk, NCg = chunks launched
// (NC - 1 in kModeState, NC in kModeOutput).
template <typename Tin, int WC, int MODE, int MINB, bool PACK>
__global__ void __launch_bounds__(32 * WC, MINB) chunk_scan_kernel(const ScanParams p)
{
    using Sh = ChunkShape<WC>;
    constexpr int NT = Sh::NT, TROW = Sh::TROW, WTILE = Sh::WTILE;
    constexpr int BCPT = Sh::BC_PER_THREAD;

    extern __shared__ float4 smem_f4[];
    float4 *sBC = smem_f4;   // [2][kT][8], slot q of step t stored at t*8 + (q ^ (t & 7))
    float *wtiles = reinterpret_cast<float *>(sBC + 2 * Sh::BC_ENTRIES);

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    float *sD = wtiles + warp * 4 * WTILE;   // [2][kT][TROW] raw delta, then outputs
    float *sX = sD + 2 * WTILE;              // [2][kT][TROW] u

    const int D = p.D, L = p.L, N = p.N, H = p.H, W = p.W, K = p.K;
    const int k = blockIdx.x, tile = blockIdx.y;
    const int ncg = (MODE == kModeState) ? p.NC - 1 : p.NC;
    const int b = blockIdx.z / ncg, chunk = blockIdx.z % ncg;
    const int d0 = tile * NT;
    const int wd0 = d0 + warp * 32;          // first channel of this warp
    const int d = d0 + tid;
    const bool cvalid = d < D;
    const int dc = cvalid ? d : D - 1;       // clamped channel for parameter reads
    const int kd = k * D + dc;
    const int l_begin = chunk * p.LC;
    const int l_end = min(l_begin + p.LC, L);

    float2 A2[8];   // A[n] * log2(e) for states (2j, 2j+1)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int n0 = 2 * j, n1 = 2 * j + 1;
        A2[j].x = (n0 < N) ? -expf(__ldg(p.A_log + (size_t)kd * N + n0)) * kLog2e : 0.f;
        A2[j].y = (n1 < N) ? -expf(__ldg(p.A_log + (size_t)kd * N + n1)) * kLog2e : 0.f;
    }
    const float dsk = __ldg(p.Dskip + kd);

    const size_t row_bk = ((size_t)b * K + k) * D;   // row index of (b, k, d = 0)
    const Tin *xg = static_cast<const Tin *>(p.x) + (size_t)b * D * L;
    const Tin *dg = static_cast<const Tin *>(p.delta) + row_bk * L;
    const Tin *Bg = static_cast<const Tin *>(p.Bs) + ((size_t)b * K + k) * N * L;
    const Tin *Cg = static_cast<const Tin *>(p.Cs) + ((size_t)b * K + k) * N * L;

    // entry state
    float2 h2[8];
    if (MODE == kModeOutput && chunk > 0) {
        const float4 *hs = reinterpret_cast<const float4 *>(
            p.hstate + ((row_bk + dc) * (p.NC - 1) + (chunk - 1)) * kNP);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = hs[q];
            h2[2 * q] = make_float2(v.x, v.y);
            h2[2 * q + 1] = make_float2(v.z, v.w);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            h2[j] = make_float2(0.f, 0.f);
    }
    float dtsum = 0.f;

    // ---- staging of the sub-chunk that starts at ld_l0 ------------------
    // delta / x: lane = (step t = lane & 15, channel parity lane >> 4); batch j
    // (0..3) loads channels 8j .. 8j+7 of this warp into registers, the next
    // batch stores them transposed into the warp tile [step][channel].
    const int st = lane & 15, sh = lane >> 4;
    PixWalk xw;   // pixel of step ld_l0 + st
    xw.init(p.two_d, k, l_begin + st, H, W, L);
    const int sq = kT / H, sr = kT % H;
    float rd[4], rx[4];
    int ld_l0 = l_begin;
    auto load_dx = [&](int j) {
        const int l = ld_l0 + st;
        const bool lok = l < l_end;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int cc = wd0 + 8 * j + 2 * i + sh;
            const bool ok = lok && cc < D;
            rd[i] = ok ? to_f32(dg[(size_t)cc * L + l]) : 0.f;
            rx[i] = ok ? to_f32(xg[(size_t)cc * L + xw.p]) : 0.f;
        }
    };
    // the staging lanes apply softplus once per (channel, step) and store dt
    // (and u), so each step of the scan loop starts from shared memory
    const float *bias_w = p.delta_bias + (size_t)k * D;
    auto store_dx = [&](int buf, int j) {
        float *td = sD + buf * WTILE + st * TROW + 8 * j + sh;
        float *tx = sX + buf * WTILE + st * TROW + 8 * j + sh;
        const bool lok = ld_l0 + st < l_end;   // the step these registers were loaded for
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int cc = wd0 + 8 * j + 2 * i + sh;
            td[2 * i] = (lok && cc < D) ? softplus_f(rd[i] + __ldg(bias_w + cc)) : 0.f;
            tx[2 * i] = rx[i];
        }
    };
    // B|C: float4 entry e = (slot q = e / kT, step t = e % kT) holds rows
    // 4q..4q+3 of B (q < 4) or C (q >= 4) at step t
    float4 rbc[BCPT];
    auto load_bc_one = [&](int r) {
        const int e = tid + r * NT;
        const int q = e / kT, t = e % kT;
        const int l = ld_l0 + t;
        const Tin *src = (q < 4) ? Bg : Cg;
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int n = (q & 3) * 4 + i;
            v[i] = (e < Sh::BC_ENTRIES && l < l_end && n < N) ? to_f32(src[(size_t)n * L + l])
                                                              : 0.f;
        }
        rbc[r] = make_float4(v[0], v[1], v[2], v[3]);
    };
    auto store_bc = [&](int buf) {
#pragma unroll
        for (int r = 0; r < BCPT; ++r) {
            const int e = tid + r * NT;
            if (e < Sh::BC_ENTRIES) {
                const int q = e / kT, t = e % kT;
                sBC[buf * Sh::BC_ENTRIES + t * 8 + (q ^ (t & 7))] = rbc[r];
            }
        }
    };

    // prologue: stage the first sub-chunk
#pragma unroll
    for (int r = 0; r < BCPT; ++r)
        load_bc_one(r);
    store_bc(0);
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
        load_dx(j);
        store_dx(0, j);
    }
    __syncthreads();

    int buf = 0;
    for (int l0 = l_begin; l0 < l_end; l0 += kT, buf ^= 1) {
        const bool more = l0 + kT < l_end;
        ld_l0 = l0 + kT;
        xw.advance(kT, sq, sr, H, W);
        const float4 *sb = sBC + buf * Sh::BC_ENTRIES;
        float *td = sD + buf * WTILE;
        const float *tx = sX + buf * WTILE;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // software-pipelined staging of the next sub-chunk
            if (more) {
                if (j > 0)
                    store_dx(buf ^ 1, j - 1);
                load_dx(j);
                if (j < BCPT)
                    load_bc_one(j);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = j * 4 + i;
                const float dt = td[t * TROW + lane];
                const float u = tx[t * TROW + lane];
                dtsum += dt;
                const float du = dt * u;
                const float2 dt2 = make_float2(dt, dt);
                const float2 du2 = make_float2(du, du);
                const float4 *row = sb + t * 8;
                const int sw = t & 7;
                float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 bv = row[q ^ sw];
                    if constexpr (PACK) {
                        const float2 arg0 = __fmul2_rn(dt2, A2[2 * q]);
                        const float2 arg1 = __fmul2_rn(dt2, A2[2 * q + 1]);
                        const float2 a0 = make_float2(mufu_ex2(arg0.x), mufu_ex2(arg0.y));
                        const float2 a1 = make_float2(mufu_ex2(arg1.x), mufu_ex2(arg1.y));
                        h2[2 * q] =
                            __ffma2_rn(a0, h2[2 * q], __fmul2_rn(du2, make_float2(bv.x, bv.y)));
                        h2[2 * q + 1] =
                            __ffma2_rn(a1, h2[2 * q + 1], __fmul2_rn(du2, make_float2(bv.z, bv.w)));
                        if (MODE == kModeOutput) {
                            const float4 cv = row[(4 + q) ^ sw];
                            acc0 = __ffma2_rn(make_float2(cv.x, cv.y), h2[2 * q], acc0);
                            acc1 = __ffma2_rn(make_float2(cv.z, cv.w), h2[2 * q + 1], acc1);
                        }
                    } else {
                        const float a0 = mufu_ex2(dt * A2[2 * q].x);
                        const float a1 = mufu_ex2(dt * A2[2 * q].y);
                        const float a2 = mufu_ex2(dt * A2[2 * q + 1].x);
                        const float a3 = mufu_ex2(dt * A2[2 * q + 1].y);
                        h2[2 * q].x = fmaf(a0, h2[2 * q].x, du * bv.x);
                        h2[2 * q].y = fmaf(a1, h2[2 * q].y, du * bv.y);
                        h2[2 * q + 1].x = fmaf(a2, h2[2 * q + 1].x, du * bv.z);
                        h2[2 * q + 1].y = fmaf(a3, h2[2 * q + 1].y, du * bv.w);
                        if (MODE == kModeOutput) {
                            const float4 cv = row[(4 + q) ^ sw];
                            acc0.x = fmaf(cv.x, h2[2 * q].x, acc0.x);
                            acc0.y = fmaf(cv.y, h2[2 * q].y, acc0.y);
                            acc1.x = fmaf(cv.z, h2[2 * q + 1].x, acc1.x);
                            acc1.y = fmaf(cv.w, h2[2 * q + 1].y, acc1.y);
                        }
                    }
                }
                if (MODE == kModeOutput)   // the output takes the consumed delta slot
                    td[t * TROW + lane] = fmaf(dsk, u, (acc0.x + acc0.y) + (acc1.x + acc1.y));
            }
        }
        if (MODE == kModeOutput) {
            // the sub-chunk's outputs: two channels x 16 consecutive steps per store
            __syncwarp();
            const int l = l0 + st;
            if (l < l_end) {
                float *orow = p.out + (row_bk + wd0 + sh) * L + l;
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    if (wd0 + 2 * i + sh < D)
                        orow[(size_t)(2 * i) * L] = td[st * TROW + 2 * i + sh];
                }
            }
        }
        if (more) {
            store_dx(buf ^ 1, 3);
            store_bc(buf ^ 1);
        }
        __syncthreads();
    }

    if (MODE == kModeState && cvalid) {
        float4 *hs = reinterpret_cast<float4 *>(
            p.hstate + ((row_bk + d) * (p.NC - 1) + chunk) * kNP);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            hs[q] = make_float4(h2[2 * q].x, h2[2 * q].y, h2[2 * q + 1].x, h2[2 * q + 1].y);
        p.dtsum[(row_bk + d) * (p.NC - 1) + chunk] = dtsum;
    }
}

// Entry states of every chunk after the first, in place over the chunk end
// states: slot c of (b,k,d) holds h_end of chunk c on entry and h_in of chunk
// c+1 on exit.  One thread per (b, k, d, n).
__global__ void carry_kernel(const ScanParams p)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = (long long)p.B * p.K * p.D * kNP;
    if (idx >= total)
        return;
    const int n = (int)(idx % kNP);
    const long long bkd = idx / kNP;
    const int d = (int)(bkd % p.D);
    const int k = (int)((bkd / p.D) % p.K);
    const float a2 =
        n < p.N ? -expf(__ldg(p.A_log + ((size_t)k * p.D + d) * p.N + n)) * kLog2e : 0.f;
    float *hs = p.hstate + (size_t)bkd * (p.NC - 1) * kNP + n;
    const float *ds = p.dtsum + (size_t)bkd * (p.NC - 1);
    const int nc1 = p.NC - 1;
    float h = 0.f;
    for (int c0 = 0; c0 < nc1; c0 += 8) {
        float he[8], dc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {   // the loads do not depend on h: issue them first
            const bool ok = c0 + i < nc1;
            he[i] = ok ? hs[(size_t)(c0 + i) * kNP] : 0.f;
            dc[i] = ok ? ds[c0 + i] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (c0 + i < nc1) {
                h = fmaf(mufu_ex2(a2 * dc[i]), h, he[i]);
                hs[(size_t)(c0 + i) * kNP] = h;
            }
        }
    }
}

// cross_merge: scan-order rows part[(b,k,d)][l] -> pixel order.  A CTA of
// kMergeThreads threads covers kMergePix "slots": 2^cpb_log2 consecutive
// (b,d) channels, each with one band of its pixels.  Two band shapes:
//  * cols = 1 (SS2D, K = 4): R image rows padded to 2^rp_log2 x 2^wp_log2
//    slots; the column-major directions are gathered through a shared-memory
//    tile, so global reads stay coalesced (the band of each image column is a
//    run of consecutive scan steps);
//  * cols = 0 (K <= 2, SS2D or 1D): 2^wp_log2 consecutive pixels.
// Slots map to (row, column) with shifts and masks, and every thread issues
// all of its loads before it uses any (memory-level parallelism).
//   sum = 1: y[b,d,p] = ((Y_0 + Y_1) + Y_2) + Y_3       (first K terms)
//   sum = 0: y[b,k,d,p] = Y_k                          (per-direction copy)
constexpr int kMergeThreads = 128;
constexpr int kMergePix = 512;
constexpr int kMergeIt = 4;   // kMergePix / kMergeThreads

__global__ void __launch_bounds__(kMergeThreads)
    merge_kernel(const float *__restrict__ part, float *__restrict__ y, int B, int D, int H,
                 int W, int K, int cols, int sum, int R, int rp_log2, int wp_log2,
                 int cpb_log2, int nblk)
{
    extern __shared__ float smem_m[];   // [cpb][2][W][R + 1] when cols
    const long long L = (long long)H * W;
    const size_t kstride = (size_t)D * L;
    const int RP = 1 << rp_log2, WP = 1 << wp_log2;
    const int S_log2 = rp_log2 + wp_log2;          // slots per channel band
    const long long ch_total = (long long)B * D;
    const int blk = blockIdx.x % nblk;
    const long long bd0 = (long long)(blockIdx.x / nblk) << cpb_log2;
    const int h0 = blk * R;
    const int hr = cols ? min(R, H - h0) : 0;
    const long long p0 = cols ? (long long)h0 * W : (long long)blk * WP;
    const size_t tile = 2 * (size_t)W * (R + 1);
    if (cols) {
        float g2[kMergeIt], g3[kMergeIt];
        int gi[kMergeIt];
#pragma unroll
        for (int i = 0; i < kMergeIt; ++i) {   // slot -> (channel, column, band row)
            const int e = threadIdx.x + i * kMergeThreads;
            const int c = e >> S_log2, sl = e & ((1 << S_log2) - 1);
            const int w = sl >> rp_log2, hh = sl & (RP - 1);
            const long long bd = bd0 + c;
            const bool ok = bd < ch_total && w < W && hh < hr;
            gi[i] = ok ? (int)(c * tile) + w * (R + 1) + hh : -1;
            g2[i] = g3[i] = 0.f;
            if (ok) {
                const float *rows = part + ((size_t)(bd / D) * K * D + (size_t)(bd % D)) * L;
                const long long s2 = (long long)w * H + h0 + hh;
                g2[i] = __ldg(rows + 2 * kstride + s2);
                g3[i] = __ldg(rows + 3 * kstride + (L - 1 - s2));
            }
        }
#pragma unroll
        for (int i = 0; i < kMergeIt; ++i) {
            if (gi[i] >= 0) {
                smem_m[gi[i]] = g2[i];
                smem_m[gi[i] + W * (R + 1)] = g3[i];
            }
        }
        __syncthreads();
    }
    float v0[kMergeIt], v1[kMergeIt];
    long long pixv[kMergeIt];   // pixel, -1 if the slot is empty
    size_t rowk[kMergeIt], rowy[kMergeIt];
    int si[kMergeIt];
#pragma unroll
    for (int i = 0; i < kMergeIt; ++i) {
        const int e = threadIdx.x + i * kMergeThreads;
        const int c = e >> S_log2, sl = e & ((1 << S_log2) - 1);
        const long long bd = bd0 + c;
        long long pix;
        bool ok;
        if (cols) {   // slot -> (channel, band row, column)
            const int hh = sl >> wp_log2, w = sl & (WP - 1);
            ok = bd < ch_total && hh < hr && w < W;
            pix = p0 + (long long)hh * W + w;
            si[i] = (int)(c * tile) + w * (R + 1) + hh;
        } else {      // slot -> (channel, pixel of the band)
            pix = p0 + sl;
            ok = bd < ch_total && pix < L;
            si[i] = 0;
        }
        const size_t b = ok ? (size_t)(bd / D) : 0, d = ok ? (size_t)(bd % D) : 0;
        rowk[i] = (b * K * D + d) * (size_t)L;
        rowy[i] = (b * D + d) * (size_t)L;
        pixv[i] = ok ? pix : -1;
        const float *rows = part + rowk[i];
        v0[i] = ok ? __ldg(rows + pix) : 0.f;
        v1[i] = (ok && K >= 2) ? __ldg(rows + kstride + (L - 1 - pix)) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kMergeIt; ++i) {
        const long long pix = pixv[i];
        if (pix < 0)
            continue;
        const float v2 = cols ? smem_m[si[i]] : 0.f;
        const float v3 = cols ? smem_m[si[i] + W * (R + 1)] : 0.f;
        if (sum) {
            float acc = v0[i];
            if (K >= 2)
                acc += v1[i];
            if (K == 4) {
                acc += v2;
                acc += v3;
            }
            y[rowy[i] + pix] = acc;
        } else {
            // per-direction layout (B, K, D, L): row (b, k, d) = rowk + k*D*L
            y[rowk[i] + pix] = v0[i];
            if (K >= 2)
                y[rowk[i] + kstride + pix] = v1[i];
            if (K == 4) {
                y[rowk[i] + 2 * kstride + pix] = v2;
                y[rowk[i] + 3 * kstride + pix] = v3;
            }
        }
    }
}

}  // namespace ss2d
