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
//   2. carry_scan_kernel (ss2d_scan.cuh): the entry state of every chunk,
//      an associative scan over the chunks of (exp(A_n * sum_c(dt)), h_end[c]);
//   3. chunk_scan_kernel<..., kModeOutput>: every chunk from its true entry
//      state, writing y_k in scan order (per-direction scratch, or y when
//      K = 1; with K = 2 and one state group both directions add into a
//      zeroed y with float atomic adds, and no merge runs: two terms give
//      the same bits in either order);
//   4. merge2_kernel (K > 1 otherwise): y[p] = ((Y_0[s_0(p)] + Y_1[s_1(p)]) +
//      Y_2[s_2(p)]) + Y_3[s_3(p)], s_k the pixel -> scan-step map of
//      direction k (cross_merge), always in that order.
// Chunking costs one extra exp per update on the chunked workloads only,
// and keeps every pass a uniform mix of MUFU and FMA work.
//
// Staging: each lane loads 16 steps of its own channel's delta and x with
// 16-byte vector loads (x of the column-major directions through the pixel
// walker), one 16-step sub-chunk ahead; it applies softplus once per
// (channel, step) and parks (dt, u) in a warp-private shared-memory tile, and
// its outputs go back as 16-byte vectors of its scan-order row.  B and C of a
// sub-chunk (shared by every channel of the CTA) are staged once per CTA as a
// float32 [slot][step] tile read with broadcast float4 loads, also one
// sub-chunk ahead.  Nothing waits on a flag.
//
// exp(dt*A) runs on the MUFU unit as 2^(dt * A*log2(e)).  The float32 pair
// arithmetic uses the sm_100 packed f32x2 instructions (__ffma2_rn,
// __fmul2_rn), which round each lane exactly as fmaf / a float multiply do.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <type_traits>
#include <stdint.h>

#include "ss2d_params.h"

namespace ss2d {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }

// float value of the 16 stored bits of a 2-byte input type
template <typename Tin>
__device__ __forceinline__ float half_bits_to_f32(uint32_t bits16)
{
    if constexpr (std::is_same_v<Tin, __half>)
        return __half2float(__ushort_as_half((unsigned short)bits16));
    else
        return __uint_as_float(bits16 << 16);
}

// Programmatic dependent launch (sm_90+): a kernel launched as a dependent
// of the previous one on the stream may start before that one has finished;
// grid_dependency_wait() blocks until it has completed and its writes are
// visible (a no-op for a kernel launched without the dependency), and
// allow_dependents() lets the next kernel start launching early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// 2^x on the multi-function unit (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float mufu_ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(z) = log(1 + e^z) = max(z, 0) + log1p(e), e = exp(-|z|) in (0, 1].
// log1p(e) = e * q(e) with q the degree-7 least-squares fit of log1p(e)/e on
// the 256 Chebyshev nodes of [0, 1] (fit_softplus.py in this directory prints
// these coefficients); evaluated in float32 its relative error stays below
// 4e-7 over the whole interval.  Never overflows: for large |z| the
// correction e underflows to 0.
__device__ __forceinline__ float softplus_f(float z)
{
    const float e = mufu_ex2(-fabsf(z) * kLog2e);
    float q = -8.574676204e-03f;
    q = fmaf(q, e, 4.421419234e-02f);
    q = fmaf(q, e, -1.078536792e-01f);
    q = fmaf(q, e, 1.775702399e-01f);
    q = fmaf(q, e, -2.449961172e-01f);
    q = fmaf(q, e, 3.327617657e-01f);
    q = fmaf(q, e, -4.999744938e-01f);
    q = fmaf(q, e, 9.999998102e-01f);
    return fmaf(e, q, fmaxf(z, 0.f));
}
// softplus_f of two values on the packed f32x2 instructions (each lane
// rounds as fmaf / a float multiply: the results equal softplus_f's)
__device__ __forceinline__ float2 softplus2_f(float2 z)
{
    const float2 a = __fmul2_rn(make_float2(fabsf(z.x), fabsf(z.y)), make_float2(-kLog2e, -kLog2e));
    const float2 e = make_float2(mufu_ex2(a.x), mufu_ex2(a.y));
    auto c2 = [](float v) { return make_float2(v, v); };
    float2 q = c2(-8.574676204e-03f);
    q = __ffma2_rn(q, e, c2(4.421419234e-02f));
    q = __ffma2_rn(q, e, c2(-1.078536792e-01f));
    q = __ffma2_rn(q, e, c2(1.775702399e-01f));
    q = __ffma2_rn(q, e, c2(-2.449961172e-01f));
    q = __ffma2_rn(q, e, c2(3.327617657e-01f));
    q = __ffma2_rn(q, e, c2(-4.999744938e-01f));
    q = __ffma2_rn(q, e, c2(9.999998102e-01f));
    return __ffma2_rn(e, q, make_float2(fmaxf(z.x, 0.f), fmaxf(z.y, 0.f)));
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
    // one step forward
    __device__ __forceinline__ void next(int H, int W)
    {
        if (mode == 0) {
            ++p;
        } else if (mode == 1) {
            --p;
        } else if (mode == 2) {
            if (++h == H) {
                h = 0;
                ++w;
                p = w;
            } else {
                p += W;
            }
        } else {
            if (--h < 0) {
                h = H - 1;
                --w;
                p = h * W + w;
            } else {
                p -= W;
            }
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
    static constexpr int BC_ENTRIES = kT * 8;              // float4 per B|C sub-chunk tile
    static constexpr int BC_PER_THREAD = (BC_ENTRIES + NT - 1) / NT;
    static constexpr int DU_WARP = 2 * kT * 32;            // float2 per warp: [2][kT][32] (dt, u)
    static constexpr int Y_WARP = kT * 33;                 // floats per warp: [kT][33] outputs
    static_assert(kT == 16, "sub-chunks of 16 steps: two 16-byte bf16 vectors per lane");
    static constexpr size_t SMEM_BYTES =
        sizeof(float4) * 2 * BC_ENTRIES +
        (size_t)WC * (sizeof(float2) * DU_WARP + sizeof(float) * Y_WARP);
};

// 16 consecutive values of one row, held as raw 32-bit words (bf16: 8 words,
// two values each; float: 16 words)
template <typename Tin>
struct Row16 {
    static constexpr int RW = kT * (int)sizeof(Tin) / 4;
    uint32_t w[RW];
    __device__ __forceinline__ float get(int i) const
    {
        if constexpr (std::is_same_v<Tin, __nv_bfloat16>) {
            const uint32_t v = w[i >> 1];
            return __uint_as_float((i & 1) ? (v & 0xffff0000u) : (v << 16));
        } else if constexpr (std::is_same_v<Tin, __half>) {
            return half_bits_to_f32<Tin>((i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xffffu));
        } else {
            return __uint_as_float(w[i]);
        }
    }
    // 16-byte vector loads; src 16-byte aligned
    __device__ __forceinline__ void load_vec(const Tin *src)
    {
        const uint4 *v = reinterpret_cast<const uint4 *>(src);
#pragma unroll
        for (int q = 0; q < RW / 4; ++q) {
            const uint4 x = __ldg(v + q);
            w[4 * q] = x.x;
            w[4 * q + 1] = x.y;
            w[4 * q + 2] = x.z;
            w[4 * q + 3] = x.w;
        }
    }
    // 8-byte vector loads; src 8-byte aligned
    __device__ __forceinline__ void load_vec8(const Tin *src)
    {
        const uint2 *v = reinterpret_cast<const uint2 *>(src);
#pragma unroll
        for (int q = 0; q < RW / 2; ++q) {
            const uint2 x = __ldg(v + q);
            w[2 * q] = x.x;
            w[2 * q + 1] = x.y;
        }
    }
    // 2-byte rows whose start is only 2-byte aligned: nine 4-byte word loads
    // from the aligned word at or before src, realigned with funnel shifts.
    // Reads up to two values past the sixteen; the caller guarantees they
    // exist.
    __device__ __forceinline__ void load_words(const Tin *src)
    {
        static_assert(sizeof(Tin) == 2, "4-byte words hold two 2-byte values");
        const uintptr_t a = reinterpret_cast<uintptr_t>(src);
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(a & ~(uintptr_t)3);
        const unsigned sh = (unsigned)(a & 2) * 8;   // 0 or 16
        uint32_t v[RW + 1];
#pragma unroll
        for (int j = 0; j <= RW; ++j)
            v[j] = __ldg(wp + j);
#pragma unroll
        for (int j = 0; j < RW; ++j)
            w[j] = __funnelshift_r(v[j], v[j + 1], sh);
    }
    // sixteen values loaded one by one (each in the low bits of e[i])
    __device__ __forceinline__ void pack(const uint32_t (&e)[kT])
    {
        if constexpr (sizeof(Tin) == 2) {
#pragma unroll
            for (int j = 0; j < RW; ++j)
                w[j] = __byte_perm(e[2 * j], e[2 * j + 1], 0x5410);
        } else {
#pragma unroll
            for (int i = 0; i < kT; ++i)
                w[i] = e[i];
        }
    }
    __device__ __forceinline__ void set_raw(int i, uint32_t bits)   // bits of one value
    {
        if constexpr (sizeof(Tin) == 2) {
            if (i & 1)
                w[i >> 1] = (w[i >> 1] & 0xffffu) | (bits << 16);
            else
                w[i >> 1] = (w[i >> 1] & 0xffff0000u) | (bits & 0xffffu);
        } else {
            w[i] = bits;
        }
    }
};

__device__ __forceinline__ uint32_t raw_bits(const float *p) { return __float_as_uint(__ldg(p)); }
__device__ __forceinline__ uint32_t raw_bits(const __nv_bfloat16 *p)
{
    return (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p));
}
__device__ __forceinline__ uint32_t raw_bits(const __half *p)
{
    return (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p));
}

// One chunk of LC steps of 32*WC channels of one (b, k); see the header.
// grid: x = k, y = channel tile, z = b * NCg + chunk (looped past 65535),
// NCg = chunks launched (NC - 1 in kModeState, NC in kModeOutput).
// COLS: the column-major directions (SS2D with K = 4) are compiled in.
// QN: groups of 4 states the lane runs (4: up to 16 states; 2: up to 8, half
// the exp2 and FMA work of a step).
template <typename Tin, int WC, int MODE, bool COLS, int QN>
__device__ __forceinline__ void chunk_scan_body(const ScanParams &p, int zz)
{
    static_assert(QN == 2 || QN == 4, "8 or 16 states per lane");
    using Sh = ChunkShape<WC>;
    constexpr int NT = Sh::NT, BCPT = Sh::BC_PER_THREAD;

    extern __shared__ float4 smem_f4[];
    float4 *sBC = smem_f4;   // [2][8][kT]: slot q of step t at q*kT + t
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    float2 *sDU = reinterpret_cast<float2 *>(sBC + 2 * Sh::BC_ENTRIES) + warp * Sh::DU_WARP;
    float *sY = reinterpret_cast<float *>(reinterpret_cast<float2 *>(sBC + 2 * Sh::BC_ENTRIES) +
                                          WC * Sh::DU_WARP) + warp * Sh::Y_WARP;

    const int D = p.D, L = p.L, N = p.N, H = p.H, W = p.W, K = p.K;
    const int k = blockIdx.x, tile = blockIdx.y;
    const int ncg = (MODE == kModeState) ? p.NC - 1 : p.NC;
    const int b = zz / ncg, chunk = zz % ncg;
    const int d0 = tile * NT;
    const int d = d0 + tid;
    const bool cvalid = d < D;
    const int dc = cvalid ? d : D - 1;       // clamped channel for addressing
    const int kd = k * D + dc;
    const int l_begin = chunk * p.LC;
    const int l_end = min(l_begin + p.LC, L);

    float2 A2[8];   // A[n] * log2(e) for states (2j, 2j+1)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int n0 = 2 * j, n1 = 2 * j + 1;
        const float *al = p.A_log + (size_t)kd * p.NS + p.n0;
        A2[j].x = (n0 < N) ? -expf(__ldg(al + n0)) * kLog2e : 0.f;
        A2[j].y = (n1 < N) ? -expf(__ldg(al + n1)) * kLog2e : 0.f;
    }
    const bool accum = p.accum != 0;   // a later state group: add to out, no skip term
    const bool ymode = MODE == kModeOutput && p.ymerge != nullptr;   // both directions add into y
    const float dsk = accum ? 0.f : __ldg(p.Dskip + kd);
    const float bias = __ldg(p.delta_bias + kd);

    const size_t row_bk = ((size_t)b * K + k) * D;   // row index of (b, k, d = 0)
    const Tin *drow = static_cast<const Tin *>(p.delta) + (row_bk + dc) * L;   // my delta row
    const Tin *xrow = static_cast<const Tin *>(p.x) + ((size_t)b * D + dc) * L;  // my x map
    const Tin *Bg = static_cast<const Tin *>(p.Bs) + (((size_t)b * K + k) * p.NS + p.n0) * L;
    const Tin *Cg = static_cast<const Tin *>(p.Cs) + (((size_t)b * K + k) * p.NS + p.n0) * L;
    // x order of this direction: 0 forward, 1 reversed (both contiguous),
    // 2 through the pixel walker (column-major directions)
    const int xmode = (COLS && k >= 2) ? 2 : (k & 1);
    const int vbytes = p.vec;   // 16 or 8: vector width of delta/x row loads; 0: scalar
    const bool ovec = p.ovec != 0;

    // entry state (chunks after the first of the output pass: loaded once the
    // carry kernel has finished, after the staging prologue below)
    float2 h2[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        h2[j] = make_float2(0.f, 0.f);
    float dtsum = 0.f;

    // ---- per-lane prefetch of 16 steps of this lane's delta and x ------
    PixWalk xw;   // column-major directions: pixel of the next step to prefetch
    xw.init(p.two_d, k, l_begin, H, W, L);
    Row16<Tin> pd, px;
    const int adv_q = kT / H, adv_r = kT % H;   // the walker's 16-step advance
    auto prefetch = [&](int ls) {   // steps ls .. ls + 15
        const bool whole = ls + kT <= L;
        // a row segment of 16 values starting at src (ascending), or the
        // values of steps ls.. one by one where it is cut by the row end
        auto load_row = [&](Row16<Tin> &r, const Tin *src, bool words_ok) {
            if (vbytes == 16)
                r.load_vec(src);
            else if (vbytes == 8)
                r.load_vec8(src);
            else if constexpr (sizeof(Tin) == 2) {
                if (words_ok) {
                    r.load_words(src);
                } else {
                    uint32_t e[kT];
#pragma unroll
                    for (int i = 0; i < kT; ++i)
                        e[i] = raw_bits(src + i);
                    r.pack(e);
                }
            } else {
                uint32_t e[kT];
#pragma unroll
                for (int i = 0; i < kT; ++i)
                    e[i] = raw_bits(src + i);
                r.pack(e);
            }
        };
        if (whole) {
            load_row(pd, drow + ls, ls + kT + 2 <= L);
        } else {
#pragma unroll
            for (int i = 0; i < kT; ++i)
                pd.set_raw(i, ls + i < L ? raw_bits(drow + ls + i) : 0u);
        }
        if (xmode == 0) {
            if (whole) {
                load_row(px, xrow + ls, ls + kT + 2 <= L);
            } else {
#pragma unroll
                for (int i = 0; i < kT; ++i)
                    px.set_raw(i, ls + i < L ? raw_bits(xrow + ls + i) : 0u);
            }
        } else if (xmode == 1) {   // pixels L-1-ls-i: load ascending, read reversed
            if (whole) {
                load_row(px, xrow + (L - kT - ls), ls > 0);
            } else {
#pragma unroll
                for (int i = 0; i < kT; ++i) {   // value of step ls + 15 - i
                    const int l = ls + kT - 1 - i;
                    px.set_raw(i, l < L ? raw_bits(xrow + (L - 1 - l)) : 0u);
                }
            }
        } else if constexpr (!COLS) {
            // no column-major direction in this instantiation
        } else if (whole && H >= 8) {
            // column-major directions: pixel of step ls + i without walking.
            // Each column wrap moves the pixel by L - 1 against the row
            // stride; with H >= 8 there are at most two wraps in 16 steps
            // (one when H >= 16).
            uint32_t e[kT];
            const int p0 = xw.p, h0 = xw.h, Lm1 = L - 1;
            if (k == 2) {
#pragma unroll
                for (int i = 0; i < kT; ++i) {
                    const int hh = h0 + i;
                    const int c = (hh >= H) + (H < kT && hh >= 2 * H);
                    e[i] = raw_bits(xrow + (p0 + i * W - c * Lm1));
                }
            } else {
#pragma unroll
                for (int i = 0; i < kT; ++i) {
                    const int hh = h0 - i;
                    const int c = (hh < 0) + (H < kT && hh < -H);
                    e[i] = raw_bits(xrow + (p0 - i * W + c * Lm1));
                }
            }
            px.pack(e);
            xw.advance(kT, adv_q, adv_r, H, W);
        } else {
#pragma unroll
            for (int i = 0; i < kT; ++i) {
                px.set_raw(i, ls + i < L ? raw_bits(xrow + xw.p) : 0u);
                xw.next(H, W);
            }
        }
    };
    // softplus once per (channel, step); dt and u to the warp tile [t][lane]
    auto unpack_store = [&](int buf, int ls) {
        float2 *du = sDU + buf * (kT * 32) + lane;
        if (ls + kT <= l_end) {   // whole sub-chunk inside the chunk
            // softplus of two steps at a time on the packed pair instructions
            if (xmode == 1) {
#pragma unroll
                for (int i = 0; i < kT; i += 2) {
                    const float2 sp = softplus2_f(make_float2(pd.get(i) + bias, pd.get(i + 1) + bias));
                    du[i * 32] = make_float2(sp.x, px.get(kT - 1 - i));
                    du[(i + 1) * 32] = make_float2(sp.y, px.get(kT - 2 - i));
                }
            } else {
#pragma unroll
                for (int i = 0; i < kT; i += 2) {
                    const float2 sp = softplus2_f(make_float2(pd.get(i) + bias, pd.get(i + 1) + bias));
                    du[i * 32] = make_float2(sp.x, px.get(i));
                    du[(i + 1) * 32] = make_float2(sp.y, px.get(i + 1));
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < kT; ++i) {
                const bool ok = ls + i < l_end;
                const float dt = ok ? softplus_f(pd.get(i) + bias) : 0.f;
                const float u = (xmode == 1) ? px.get(kT - 1 - i) : px.get(i);
                du[i * 32] = make_float2(dt, u);
            }
        }
    };
    // B|C: float4 entry e = (slot q = e / kT, step t = e % kT) holds rows
    // 4q..4q+3 of B (q < 4) or C (q >= 4) at step t
    float4 rbc[BCPT];
    auto load_bc = [&](int ls) {
        const bool whole = N == kNP && ls + kT <= l_end;
#pragma unroll
        for (int r = 0; r < BCPT; ++r) {
            const int e = tid + r * NT;
            const int q = e / kT, t = e % kT;
            const int l = ls + t;
            const Tin *src = (q < 4) ? Bg : Cg;
            const bool ok = (Sh::BC_ENTRIES % NT == 0 || e < Sh::BC_ENTRIES) &&
                            (whole || l < l_end);
            float v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int n = (q & 3) * 4 + i;
                v[i] = (ok && (whole || n < N)) ? to_f32(src[(size_t)n * L + l]) : 0.f;
            }
            rbc[r] = make_float4(v[0], v[1], v[2], v[3]);
        }
    };
    auto store_bc = [&](int buf) {
#pragma unroll
        for (int r = 0; r < BCPT; ++r) {
            const int e = tid + r * NT;
            if (Sh::BC_ENTRIES % NT == 0 || e < Sh::BC_ENTRIES)
                sBC[buf * Sh::BC_ENTRIES + e] = rbc[r];
        }
    };

    // prologue: sub-chunk 0 staged, sub-chunk 1 in flight (inputs only)
    prefetch(l_begin);
    load_bc(l_begin);
    unpack_store(0, l_begin);
    store_bc(0);
    if (l_begin + kT < l_end) {
        prefetch(l_begin + kT);
        load_bc(l_begin + kT);
    }
    // everything below may read or overwrite what the previous kernel on the
    // stream wrote (entry states, the output rows)
    grid_dependency_wait();
    if (MODE == kModeOutput && chunk > 0) {
        const float4 *hs = reinterpret_cast<const float4 *>(
            p.hstate + ((row_bk + dc) * (p.NC - 1) + (chunk - 1)) * kNP);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = hs[q];
            h2[2 * q] = make_float2(v.x, v.y);
            h2[2 * q + 1] = make_float2(v.z, v.w);
        }
    }
    __syncthreads();

    int buf = 0;
    for (int l0 = l_begin; l0 < l_end; l0 += kT, buf ^= 1) {
        const bool more = l0 + kT < l_end;
        const float4 *sb = sBC + buf * Sh::BC_ENTRIES;
        const float2 *du_t = sDU + buf * (kT * 32) + lane;
#pragma unroll 4
        for (int t = 0; t < kT; ++t) {
            const float2 dtu = du_t[t * 32];
            const float dt = dtu.x, u = dtu.y;
            dtsum += dt;
            const float du = dt * u;
            const float2 dt2 = make_float2(dt, dt);
            const float2 du2 = make_float2(du, du);
            const float4 *col = sb + t;   // slot q at col[q * kT]
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < QN; ++q) {
                const float4 bv = col[q * kT];
                const float2 arg0 = __fmul2_rn(dt2, A2[2 * q]);
                const float2 arg1 = __fmul2_rn(dt2, A2[2 * q + 1]);
                const float2 a0 = make_float2(mufu_ex2(arg0.x), mufu_ex2(arg0.y));
                const float2 a1 = make_float2(mufu_ex2(arg1.x), mufu_ex2(arg1.y));
                h2[2 * q] = __ffma2_rn(a0, h2[2 * q], __fmul2_rn(du2, make_float2(bv.x, bv.y)));
                h2[2 * q + 1] =
                    __ffma2_rn(a1, h2[2 * q + 1], __fmul2_rn(du2, make_float2(bv.z, bv.w)));
                if (MODE == kModeOutput) {
                    const float4 cv = col[(4 + q) * kT];
                    acc0 = __ffma2_rn(make_float2(cv.x, cv.y), h2[2 * q], acc0);
                    acc1 = __ffma2_rn(make_float2(cv.z, cv.w), h2[2 * q + 1], acc1);
                }
            }
            if (MODE == kModeOutput)
                sY[t * 33 + lane] = fmaf(dsk, u, (acc0.x + acc0.y) + (acc1.x + acc1.y));
        }
        if (MODE == kModeOutput && cvalid) {
            // this lane's 16 outputs, one segment of its output row: in scan
            // order, except direction 1 of a multi-direction call (the reversed
            // row-major order), which is stored flipped, in pixel order
            const bool flip = k == 1 && K > 1;
            float *rowp = ymode ? p.ymerge + ((size_t)b * D + d) * L : p.out + (row_bk + d) * L;
            if (ovec && l0 + kT <= l_end) {
                float4 *orow = reinterpret_cast<float4 *>(rowp + (flip ? L - kT - l0 : l0));
#pragma unroll
                for (int q = 0; q < kT / 4; ++q) {
                    float4 v = flip ? make_float4(sY[(15 - 4 * q) * 33 + lane],
                                                  sY[(14 - 4 * q) * 33 + lane],
                                                  sY[(13 - 4 * q) * 33 + lane],
                                                  sY[(12 - 4 * q) * 33 + lane])
                                    : make_float4(sY[(4 * q) * 33 + lane],
                                                  sY[(4 * q + 1) * 33 + lane],
                                                  sY[(4 * q + 2) * 33 + lane],
                                                  sY[(4 * q + 3) * 33 + lane]);
                    if (ymode) {
                        atomicAdd(orow + q, v);
                        continue;
                    }
                    if (accum) {
                        const float4 o = orow[q];
                        v = make_float4(o.x + v.x, o.y + v.y, o.z + v.z, o.w + v.w);
                    }
                    orow[q] = v;
                }
            } else {
#pragma unroll
                for (int t = 0; t < kT; ++t)
                    if (l0 + t < l_end) {
                        float *o = rowp + (flip ? L - 1 - l0 - t : l0 + t);
                        if (ymode)
                            atomicAdd(o, sY[t * 33 + lane]);
                        else
                            *o = accum ? *o + sY[t * 33 + lane] : sY[t * 33 + lane];
                    }
            }
        }
        if (more) {
            // stage the next sub-chunk (its loads were issued one sub-chunk
            // ago) and issue the loads of the one after it
            unpack_store(buf ^ 1, l0 + kT);
            store_bc(buf ^ 1);
            if (l0 + 2 * kT < l_end) {
                prefetch(l0 + 2 * kT);
                load_bc(l0 + 2 * kT);
            }
        }
        __syncthreads();
    }
    allow_dependents();

    if (MODE == kModeState && cvalid) {
        float4 *hs = reinterpret_cast<float4 *>(
            p.hstate + ((row_bk + d) * (p.NC - 1) + chunk) * kNP);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            hs[q] = make_float4(h2[2 * q].x, h2[2 * q].y, h2[2 * q + 1].x, h2[2 * q + 1].y);
        p.dtsum[(row_bk + d) * (p.NC - 1) + chunk] = dtsum;
    }
    // the state after the last step (steps past L stage dt = 0: identity)
    if (MODE == kModeOutput && p.hlast && cvalid && chunk == p.NC - 1) {
        float *hl = p.hlast + (row_bk + d) * p.NS + p.n0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (2 * j < N)
                hl[2 * j] = h2[j].x;
            if (2 * j + 1 < N)
                hl[2 * j + 1] = h2[j].y;
        }
    }
}

// The kernel: grid z runs over (b, chunk) pairs, more than 65535 of them by
// looping (z, z + gridDim.z, ...); every iteration ends on a CTA barrier.
template <typename Tin, int WC, int MODE, int MINB, bool COLS, int QN>
__global__ void __launch_bounds__(32 * WC, MINB) chunk_scan_kernel(const ScanParams p)
{
    const int ncg = (MODE == kModeState) ? p.NC - 1 : p.NC;
    const int nz = p.B * ncg;
    for (int zz = blockIdx.z; zz < nz; zz += gridDim.z)
        chunk_scan_body<Tin, WC, MODE, COLS, QN>(p, zz);
}

// cross_merge, band form: a CTA covers `rows` full image rows (the band
// starting at row h0 = blockIdx.y * R) of CG consecutive (b, d) channels.
//  * cols (SS2D, K = 4): the column-major directions' values of the band are
//    staged in shared memory first:
//      - whole (the band is the whole image, L % 4 == 0): their rows are
//        copied as they are (float4, scan order) and read at the scan index
//        of each pixel;
//      - otherwise column w of the band is the run of scan steps
//        w*H + h0 .. w*H + h0 + rows - 1 of direction 2 (the mirror run of
//        direction 3), read as runs and transposed to [rows][W + 1];
//  * the row-major directions (and every direction of K <= 2 or 1D) are
//    read at p: direction 0's row is in scan order = pixel order, and the
//    output pass stores direction 1's row flipped, in pixel order.
// Work units (float4 groups of pixels when VEC = 4 or whole, pixels when
// VEC = 1) of all CG channels are spread over the whole CTA.  flat (no
// column-major direction, one band per image, CG | D, 4 | CG): the CTA's
// channels form one contiguous block of each row set, streamed as float4.  VEC = 4 needs
// W % 4 == 0, and H % 4 == 0 and R % 4 == 0 when cols.
//   sum = 1: y[b,d,p] = ((Y_0 + Y_1) + Y_2) + Y_3       (first K terms)
//   sum = 0: y[b,k,d,p] = Y_k                          (per-direction copy)
constexpr int kMerge2Threads = 256;

// SiLU(z) = z / (1 + e^-z), the optional output gate of cross_merge (fast
// exp and division intrinsics; for z below about -88 the denominator is
// infinite and the result is -0)
__device__ __forceinline__ float silu_f(float z) { return __fdividef(z, 1.f + __expf(-z)); }
// gate factors of four consecutive y elements starting at index i of z
// (zt: 0 float32, 1 bfloat16, 2 float16 storage of z)
__device__ __forceinline__ float4 gate4(const void *z, int zt, size_t i)
{
    float4 g;
    if (zt == 0) {
        g = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(z) + i));
    } else {
        const uint2 r =
            __ldg(reinterpret_cast<const uint2 *>(static_cast<const unsigned short *>(z) + i));
        if (zt == 1)
            g = make_float4(half_bits_to_f32<__nv_bfloat16>(r.x & 0xffffu),
                            half_bits_to_f32<__nv_bfloat16>(r.x >> 16),
                            half_bits_to_f32<__nv_bfloat16>(r.y & 0xffffu),
                            half_bits_to_f32<__nv_bfloat16>(r.y >> 16));
        else
            g = make_float4(half_bits_to_f32<__half>(r.x & 0xffffu),
                            half_bits_to_f32<__half>(r.x >> 16),
                            half_bits_to_f32<__half>(r.y & 0xffffu),
                            half_bits_to_f32<__half>(r.y >> 16));
    }
    return make_float4(silu_f(g.x), silu_f(g.y), silu_f(g.z), silu_f(g.w));
}
__device__ __forceinline__ float gate1(const void *z, int zt, size_t i)
{
    float v;
    if (zt == 0) {
        v = __ldg(static_cast<const float *>(z) + i);
    } else {
        const uint32_t b = __ldg(static_cast<const unsigned short *>(z) + i);
        v = zt == 1 ? half_bits_to_f32<__nv_bfloat16>(b) : half_bits_to_f32<__half>(b);
    }
    return silu_f(v);
}
__device__ __forceinline__ float4 mul4(float4 a, float4 b)
{
    return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}

template <int VEC, int CG, bool GATE>
__global__ void __launch_bounds__(kMerge2Threads)
    merge2_kernel(const float *__restrict__ part, float *__restrict__ y, int B, int D, int H,
                  int W, int K, int cols, int sum, int R, int whole, int flat,
                  const void *__restrict__ z, int zt)
{
    extern __shared__ float smem_m2[];   // cols: [CG][2][R][W + 1], whole: [CG][2][L]
    grid_dependency_wait();   // the output pass's rows
    const int L = H * W;
    const size_t kstride = (size_t)D * L;
    const long long nch = (long long)B * D;
    const long long bd0 = (long long)blockIdx.x * CG;
    const int h0 = blockIdx.y * R;
    const int rows = min(R, H - h0);
    const int p0 = h0 * W, n = rows * W;
    const int WS = W + 1;
    const long long b0 = bd0 / D;
    const int d0 = (int)(bd0 - b0 * D);
    const int nc = (int)min((long long)CG, nch - bd0);   // channels of this CTA
    const size_t tile = whole ? 2 * (size_t)L : 2 * (size_t)R * WS;   // smem floats per channel
    // row (b, 0, d) of part for the c-th channel of the CTA
    auto part_row = [&](int c) {
        long long bb = b0;
        int dd = d0 + c;
        while (dd >= D) {
            dd -= D;
            ++bb;
        }
        return ((size_t)bb * K * D + dd) * (size_t)L;
    };
    auto y_row = [&](int c) {
        long long bb = b0;
        int dd = d0 + c;
        while (dd >= D) {
            dd -= D;
            ++bb;
        }
        return ((size_t)bb * D + dd) * (size_t)L;
    };

    if (flat) {
        // no column-major direction, whole rows, CG | D and 4 | CG: the CTA's
        // channels are one contiguous, 16-byte aligned block of every row set
        const size_t nb = (size_t)CG * L / 4;
        const size_t rk0 = part_row(0);
        const float4 *a = reinterpret_cast<const float4 *>(part + rk0);
        const float4 *m = reinterpret_cast<const float4 *>(part + rk0 + kstride);
        const size_t yr0 = y_row(0);
        float4 *yo = reinterpret_cast<float4 *>(sum ? y + yr0 : y + rk0);
        float4 *yo1 = reinterpret_cast<float4 *>(y + rk0 + kstride);
#pragma unroll 4
        for (size_t f = threadIdx.x; f < nb; f += kMerge2Threads) {
            const float4 v0 = __ldg(a + f);
            const float4 v1 = K >= 2 ? __ldg(m + f) : make_float4(0.f, 0.f, 0.f, 0.f);
            if (sum) {
                float4 v = make_float4(v0.x + v1.x, v0.y + v1.y, v0.z + v1.z, v0.w + v1.w);
                if constexpr (GATE)
                    v = mul4(v, gate4(z, zt, yr0 + 4 * f));
                yo[f] = v;
            } else {
                yo[f] = v0;
                if (K >= 2)
                    yo1[f] = v1;
            }
        }
        return;
    }

    // thread slice of each channel: TPC consecutive threads per channel
    constexpr int TPC = kMerge2Threads / CG;
    const int c = threadIdx.x / TPC, t0 = threadIdx.x % TPC;
    const bool active = c < nc;
    const size_t rk = active ? part_row(c) : 0;   // row (b, 0, d) of part

    if (cols) {
        if (active) {
            const float *r2 = part + rk + 2 * kstride;
            const float *r3 = r2 + kstride;
            float *s2 = smem_m2 + c * tile;
            if (whole) {
                const int q4 = L / 4;   // float4 per row
                float4 *t2 = reinterpret_cast<float4 *>(s2), *t3 = t2 + q4;
#pragma unroll 4
                for (int j = t0; j < q4; j += TPC) {
                    t2[j] = __ldg(reinterpret_cast<const float4 *>(r2) + j);
                    t3[j] = __ldg(reinterpret_cast<const float4 *>(r3) + j);
                }
            } else if (VEC == 4) {
                float *s3 = s2 + (size_t)R * WS;
                const int rq = rows / 4;   // float4 runs per column
                for (int e = t0; e < W * rq; e += TPC) {
                    const int w = e / rq, r = 4 * (e - w * rq);
                    const int sc = w * H + h0 + r;
                    const float4 a = __ldg(reinterpret_cast<const float4 *>(r2 + sc));
                    const float4 m = __ldg(reinterpret_cast<const float4 *>(r3 + (L - 4 - sc)));
                    s2[(r + 0) * WS + w] = a.x;
                    s2[(r + 1) * WS + w] = a.y;
                    s2[(r + 2) * WS + w] = a.z;
                    s2[(r + 3) * WS + w] = a.w;
                    s3[(r + 0) * WS + w] = m.w;
                    s3[(r + 1) * WS + w] = m.z;
                    s3[(r + 2) * WS + w] = m.y;
                    s3[(r + 3) * WS + w] = m.x;
                }
            } else {
                float *s3 = s2 + (size_t)R * WS;
                // element e of the band in column-major order: w = e / rows
                for (int e = t0; e < n; e += TPC) {
                    const int w = e / rows, r = e - w * rows;
                    const int sc = w * H + h0 + r;
                    s2[r * WS + w] = __ldg(r2 + sc);
                    s3[r * WS + w] = __ldg(r3 + (L - 1 - sc));
                }
            }
        }
        __syncthreads();
    }
    if (!active)
        return;

    const int vw = (whole || VEC == 4) ? 4 : 1;
    const int upc = n / vw;   // units per channel
    const float *r0 = part + rk, *r1 = r0 + kstride;
    const size_t yr = y_row(c);
    float *yo = sum ? y + yr : y + rk;
    for (int iu = t0; iu < upc; iu += TPC) {
        const int i = iu * vw;   // band pixel index
        const int p = p0 + i;
        if (vw == 4) {
            const float4 v0 = __ldg(reinterpret_cast<const float4 *>(r0 + p));
            float4 v1 = make_float4(0.f, 0.f, 0.f, 0.f), v2 = v1, v3 = v1;
            if (K >= 2)
                v1 = __ldg(reinterpret_cast<const float4 *>(r1 + p));
            if (cols) {
                float a2[4], a3[4];
                if (whole) {
                    const float *t2 = smem_m2 + c * tile, *t3 = t2 + L;
                    int h = p / W, w = p - h * W;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int sc = w * H + h;   // column-major scan index of pixel p + j
                        a2[j] = t2[sc];
                        a3[j] = t3[L - 1 - sc];
                        if (++w == W) {
                            w = 0;
                            ++h;
                        }
                    }
                } else {
                    const int r = i / W, w = i - r * W;
                    const float *s2 = smem_m2 + c * tile + r * WS + w;
                    const float *s3 = s2 + (size_t)R * WS;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        a2[j] = s2[j];
                        a3[j] = s3[j];
                    }
                }
                v2 = make_float4(a2[0], a2[1], a2[2], a2[3]);
                v3 = make_float4(a3[0], a3[1], a3[2], a3[3]);
            }
            if (sum) {
                float4 v = v0;
                if (K >= 2)
                    v = make_float4(v.x + v1.x, v.y + v1.y, v.z + v1.z, v.w + v1.w);
                if (cols)
                    v = make_float4((v.x + v2.x) + v3.x, (v.y + v2.y) + v3.y,
                                    (v.z + v2.z) + v3.z, (v.w + v2.w) + v3.w);
                if constexpr (GATE)
                    v = mul4(v, gate4(z, zt, yr + p));
                *reinterpret_cast<float4 *>(yo + p) = v;
            } else {
                *reinterpret_cast<float4 *>(yo + p) = v0;
                if (K >= 2)
                    *reinterpret_cast<float4 *>(yo + kstride + p) = v1;
                if (cols) {
                    *reinterpret_cast<float4 *>(yo + 2 * kstride + p) = v2;
                    *reinterpret_cast<float4 *>(yo + 3 * kstride + p) = v3;
                }
            }
        } else {
            float v = __ldg(r0 + p);
            const float v1 = K >= 2 ? __ldg(r1 + p) : 0.f;
            float v2 = 0.f, v3 = 0.f;
            if (cols) {
                const int r = i / W, w = i - r * W;
                const float *s2 = smem_m2 + c * tile;
                v2 = s2[r * WS + w];
                v3 = s2[(size_t)R * WS + r * WS + w];
            }
            if (sum) {
                if (K >= 2)
                    v += v1;
                if (cols)
                    v = (v + v2) + v3;
                if constexpr (GATE)
                    v *= gate1(z, zt, yr + p);
                yo[p] = v;
            } else {
                yo[p] = v;
                if (K >= 2)
                    yo[kstride + p] = v1;
                if (cols) {
                    yo[2 * kstride + p] = v2;
                    yo[3 * kstride + p] = v3;
                }
            }
        }
    }
}

// cross_merge, one pixel per thread: the plain form, for maps too wide for the
// band form's shared-memory tiles.  Pixel p = h*W + w of channel (b, d):
// direction 0's row is in pixel order, direction 1's too (the output pass
// stores it flipped), direction 2 visits p at scan step w*H + h, direction 3
// at L-1-(w*H + h).  sum = 1: y = ((Y_0 + Y_1) + Y_2) + Y_3 (first K terms),
// times SiLU(z) when z is given; sum = 0: y[b,k,d,p] = Y_k.
static __global__ void merge1_kernel(const float *__restrict__ part, float *__restrict__ y, int B,
                                     int D, int H, int W, int K, int cols, int sum,
                                     const void *__restrict__ z, int zt)
{
    grid_dependency_wait();   // the output pass's rows
    const long long L = (long long)H * W;
    const long long total = (long long)B * D * L;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long pix = i % L, bd = i / L;
        const long long b = bd / D, d = bd % D;
        const long long h = pix / W, w = pix % W;
        const long long s2 = w * H + h;
        float acc = 0.f;
        for (int k = 0; k < K; ++k) {
            const long long idx = (cols && k >= 2) ? (k == 2 ? s2 : L - 1 - s2) : pix;
            const float v = part[((b * K + k) * D + d) * L + idx];
            if (sum)
                acc = k == 0 ? v : acc + v;
            else
                y[((b * K + k) * D + d) * L + pix] = v;
        }
        if (sum)
            y[i] = z ? acc * gate1(z, zt, (size_t)i) : acc;
    }
}

}  // namespace ss2d

