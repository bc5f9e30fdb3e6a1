// ss2d_quad.cuh -- the scan kernel in the "quad" layout: four lanes per
// (b, k, d) channel, each holding four of its sixteen states.
//
// Same recurrence, chunking and passes as chunk_scan_kernel (ss2d_kernels.cuh);
// only the mapping of work to lanes differs.  With one lane per channel a
// sequence of L steps keeps one lane busy for L steps, so shapes with few
// channels and long sequences (B*K*D of a few thousand, L in the thousands)
// need many chunks, and every chunk but the last is scanned twice (state pass,
// then output pass).  Four lanes per channel give four times the lanes for the
// same channels, so such shapes need few chunks or none.
//
// Per warp: 8 channels x 4 state quarters, lane = 4*c + q holds states
// 4q..4q+3 of channel c.  Per step a lane reads (dt, dt, du, du) of its channel
// from a warp tile [step][channel] (8 distinct 16-byte words per warp load),
// and B[4q..4q+3], C[4q..4q+3] of the step from a CTA tile [step][B0..15 |
// C0..15] (4 distinct 16-byte words per warp load); both tiles are filled one
// 16-step sub-chunk ahead.  The C.h partial sums of a sub-chunk (16 per lane)
// are reduced over the 4 lanes of a channel with two rounds of shuffles
// (reduce-scatter), after which lane q holds the outputs of steps 4q..4q+3,
// the same steps whose delta and x it staged, and stores them as one 16-byte
// vector.
#pragma once

#include "ss2d_kernels.cuh"

namespace ss2d {

constexpr int kQLanes = 4;                 // lanes per channel
constexpr int kQStates = kNP / kQLanes;    // states per lane
constexpr int kQCh = 32 / kQLanes;         // channels per warp
static_assert(kQStates == 4 && kT == 16, "quad layout: 4 states per lane, 16-step sub-chunks");

// four consecutive values of one row as raw 32-bit words
template <typename Tin>
struct Quad4 {
    static constexpr int RW = (int)sizeof(Tin);   // words: 2-byte types 2, float 4
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
    // one vector load; src aligned to 4 * sizeof(Tin)
    __device__ __forceinline__ void load_vec(const Tin *src)
    {
        if constexpr (sizeof(Tin) == 2) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(src));
            w[0] = v.x;
            w[1] = v.y;
        } else {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src));
            w[0] = v.x;
            w[1] = v.y;
            w[2] = v.z;
            w[3] = v.w;
        }
    }
    __device__ __forceinline__ void set_raw(int i, uint32_t bits)
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

// One chunk of LC steps of 8*NW channels of one (b, k).
// grid: x = k, y = channel tile, z = b * NCg + chunk (NCg = NC - 1 in
// kModeState, NC in kModeOutput); block 32*NW.
template <typename Tin, int MODE, int NW, int MINB>
__global__ void __launch_bounds__(32 * NW, MINB) quad_scan_kernel(const ScanParams p)
{
    constexpr int NT = 32 * NW;
    constexpr int CH = kQCh * NW;
    __shared__ __align__(16) float sBC[2][kT][2 * kNP];          // [buf][t][B0..15 C0..15]
    __shared__ __align__(16) float4 sDU[NW][2][kT][kQCh];        // [warp][buf][t][c] (dt,dt,du,du)

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int c = lane >> 2, q = lane & 3;

    const int D = p.D, L = p.L, N = p.N, H = p.H, W = p.W, K = p.K;
    const int k = blockIdx.x, tile = blockIdx.y;
    const int ncg = (MODE == kModeState) ? p.NC - 1 : p.NC;
    const int b = blockIdx.z / ncg, chunk = blockIdx.z % ncg;
    const int d = tile * CH + warp * kQCh + c;
    const bool cvalid = d < D;
    const int dc = cvalid ? d : D - 1;
    const int kd = k * D + dc;
    const int l_begin = chunk * p.LC;
    const int l_end = min(l_begin + p.LC, L);
    const bool v4 = (L & 3) == 0;   // rows allow 4-element vector access

    float2 A2[2];   // A[n] * log2(e), n = 4q .. 4q+3
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int n0 = 4 * q + 2 * j, n1 = n0 + 1;
        const float *al = p.A_log + (size_t)kd * p.NS + p.n0;
        A2[j].x = (n0 < N) ? -expf(__ldg(al + n0)) * kLog2e : 0.f;
        A2[j].y = (n1 < N) ? -expf(__ldg(al + n1)) * kLog2e : 0.f;
    }
    const bool accum = p.accum != 0;   // a later state group: add to out, no skip term
    const float dsk = accum ? 0.f : __ldg(p.Dskip + kd);
    const float bias = __ldg(p.delta_bias + kd);

    const size_t row_bk = ((size_t)b * K + k) * D;
    const Tin *drow = static_cast<const Tin *>(p.delta) + (row_bk + dc) * L;
    const Tin *xrow = static_cast<const Tin *>(p.x) + ((size_t)b * D + dc) * L;
    // B|C staging: thread -> (row r of 32: B0..15 then C0..15, step group g of 4)
    const Tin *bcrow = nullptr;
    const int r = tid & 31;
    {
        const int n = r & 15;
        const Tin *base = static_cast<const Tin *>(r < 16 ? p.Bs : p.Cs);
        bcrow = n < N ? base + (((size_t)b * K + k) * p.NS + p.n0 + n) * L : nullptr;
    }
    constexpr int BC_ITEMS = 2 * kNP * (kT / 4);   // (row, group) items per sub-chunk: 128
    constexpr int BC_PER_THREAD = (BC_ITEMS + NT - 1) / NT;

    // x order of this direction: 0 forward, 1 reversed (both contiguous in
    // memory), 2 / 3 column-major through the pixel walker
    const int xmode = (p.two_d && k >= 2) ? 2 : (k & 1);
    PixWalk walk;
    walk.init(p.two_d, k, min(l_begin + 4 * q, L - 1), H, W, L);
    const int adv_q = kT / H, adv_r = kT % H;

    // entry state (written by the carry kernel, which may still be running
    // when this kernel starts as its dependent)
    grid_dependency_wait();
    float2 h2[2];
    if (MODE == kModeOutput && chunk > 0) {
        const float4 v = *reinterpret_cast<const float4 *>(
            p.hstate + ((row_bk + dc) * (p.NC - 1) + (chunk - 1)) * kNP + 4 * q);
        h2[0] = make_float2(v.x, v.y);
        h2[1] = make_float2(v.z, v.w);
    } else {
        h2[0] = make_float2(0.f, 0.f);
        h2[1] = make_float2(0.f, 0.f);
    }

    // prefetch registers: delta and x of steps l0+4q .. l0+4q+3, and this
    // thread's B|C items
    Quad4<Tin> rd, rx;
    Quad4<Tin> rbc[BC_PER_THREAD];
    float u_cur[4];
    float dts = 0.f;

    auto load = [&](int l0) {
        const int l = l0 + 4 * q;
        const bool full = l + 3 < l_end;
        if (v4 && full) {
            rd.load_vec(drow + l);
            if (xmode == 0)
                rx.load_vec(xrow + l);
            else if (xmode == 1)
                rx.load_vec(xrow + (L - 4 - l));   // pixels L-4-l .. L-1-l, reversed below
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                rd.set_raw(i, (l + i < l_end) ? raw_bits(drow + l + i) : 0u);
            if (xmode == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    rx.set_raw(i, (l + i < l_end) ? raw_bits(xrow + l + i) : 0u);
            } else if (xmode == 1) {
#pragma unroll
                for (int i = 0; i < 4; ++i)   // stored reversed, like the vector path
                    rx.set_raw(3 - i, (l + i < l_end) ? raw_bits(xrow + (L - 1 - l - i)) : 0u);
            }
        }
        if (xmode == 2) {
            PixWalk w2 = walk;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                rx.set_raw(i, (l + i < l_end) ? raw_bits(xrow + w2.p) : 0u);
                if (i < 3)
                    w2.next(H, W);
            }
            walk.advance(kT, adv_q, adv_r, H, W);
        }
#pragma unroll
        for (int j = 0; j < BC_PER_THREAD; ++j) {
            const int item = tid + j * NT;
            if (BC_ITEMS % NT == 0 || item < BC_ITEMS) {
                const int lg = l0 + 4 * (item >> 5);
                if (bcrow && v4 && lg + 3 < l_end) {
                    rbc[j].load_vec(bcrow + lg);
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        rbc[j].set_raw(i, (bcrow && lg + i < l_end) ? raw_bits(bcrow + lg + i) : 0u);
                }
            }
        }
    };

    auto store = [&](int buf, int l0) {
        const int l = l0 + 4 * q;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool ok = l + i < l_end;
            const float dt = ok ? softplus_f(rd.get(i) + bias) : 0.f;
            const float u = (xmode == 1) ? rx.get(3 - i) : rx.get(i);
            const float du = dt * u;
            sDU[warp][buf][4 * q + i][c] = make_float4(dt, dt, du, du);
            u_cur[i] = u;
            if (MODE == kModeState)
                dts += dt;
        }
#pragma unroll
        for (int j = 0; j < BC_PER_THREAD; ++j) {
            const int item = tid + j * NT;
            if (BC_ITEMS % NT == 0 || item < BC_ITEMS) {
                const int g = item >> 5;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    sBC[buf][4 * g + i][item & 31] = rbc[j].get(i);
            }
        }
    };

    float *orow = p.out + (row_bk + dc) * L;
    const int nsub = (l_end - l_begin + kT - 1) / kT;

    load(l_begin);
    store(0, l_begin);
    if (nsub > 1)
        load(l_begin + kT);
    __syncthreads();

    for (int s = 0; s < nsub; ++s) {
        const int buf = s & 1;
        const int l0 = l_begin + s * kT;
        const float4 *du_t = &sDU[warp][buf][0][c];
        const float *bc_t = &sBC[buf][0][4 * q];
        float yv[kT];
#pragma unroll
        for (int t = 0; t < kT; ++t) {
            const float4 e = du_t[t * kQCh];
            const float2 dt2 = make_float2(e.x, e.y), du2 = make_float2(e.z, e.w);
            const float2 g0 = __fmul2_rn(dt2, A2[0]), g1 = __fmul2_rn(dt2, A2[1]);
            const float2 a0 = make_float2(mufu_ex2(g0.x), mufu_ex2(g0.y));
            const float2 a1 = make_float2(mufu_ex2(g1.x), mufu_ex2(g1.y));
            const float4 bv = *reinterpret_cast<const float4 *>(bc_t + t * 2 * kNP);
            h2[0] = __ffma2_rn(a0, h2[0], __fmul2_rn(du2, make_float2(bv.x, bv.y)));
            h2[1] = __ffma2_rn(a1, h2[1], __fmul2_rn(du2, make_float2(bv.z, bv.w)));
            if (MODE == kModeOutput) {
                const float4 cv = *reinterpret_cast<const float4 *>(bc_t + t * 2 * kNP + kNP);
                float2 yp = __fmul2_rn(make_float2(cv.x, cv.y), h2[0]);
                yp = __ffma2_rn(make_float2(cv.z, cv.w), h2[1], yp);
                yv[t] = yp.x + yp.y;
            }
        }
        if (MODE == kModeOutput) {
            // reduce-scatter over the 4 lanes of the channel: lane q ends with
            // the sums of steps 4q .. 4q+3
            const bool hi = (q & 2) != 0, lo = (q & 1) != 0;
            float r8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float send = hi ? yv[i] : yv[i + 8];
                const float keep = hi ? yv[i + 8] : yv[i];
                r8[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
            }
            float r4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float send = lo ? r8[i] : r8[i + 4];
                const float keep = lo ? r8[i + 4] : r8[i];
                r4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
            }
            const int l = l0 + 4 * q;
            if (cvalid) {
                float o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    o[i] = fmaf(dsk, u_cur[i], r4[i]);
                auto put4 = [&](float *dst, float4 v) {
                    float4 *d4 = reinterpret_cast<float4 *>(dst);
                    if (accum) {
                        const float4 e = *d4;
                        v = make_float4(e.x + v.x, e.y + v.y, e.z + v.z, e.w + v.w);
                    }
                    *d4 = v;
                };
                auto put1 = [&](float *dst, float v) { *dst = accum ? *dst + v : v; };
                if (k == 1 && K > 1) {
                    // direction 1 of a multi-direction call: pixel order
                    if (v4 && l + 3 < l_end) {
                        put4(orow + (L - 4 - l), make_float4(o[3], o[2], o[1], o[0]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            if (l + i < l_end)
                                put1(orow + (L - 1 - l - i), o[i]);
                    }
                } else if (v4 && l + 3 < l_end) {
                    put4(orow + l, make_float4(o[0], o[1], o[2], o[3]));
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (l + i < l_end)
                            put1(orow + l + i, o[i]);
                }
            }
        }
        if (s + 1 < nsub)
            store(buf ^ 1, l0 + kT);
        if (s + 2 < nsub)
            load(l0 + 2 * kT);
        __syncthreads();
    }

    if (MODE == kModeState) {
        dts += __shfl_xor_sync(0xffffffffu, dts, 1);
        dts += __shfl_xor_sync(0xffffffffu, dts, 2);
        if (cvalid) {
            *reinterpret_cast<float4 *>(p.hstate + ((row_bk + d) * (p.NC - 1) + chunk) * kNP +
                                        4 * q) = make_float4(h2[0].x, h2[0].y, h2[1].x, h2[1].y);
            if (q == 0)
                p.dtsum[(row_bk + d) * (p.NC - 1) + chunk] = dts;
        }
    }
    // the state after the last step: states 4q .. 4q+3 of this lane
    if (MODE == kModeOutput && p.hlast && cvalid && chunk == p.NC - 1) {
        float *hl = p.hlast + (row_bk + d) * p.NS + p.n0 + 4 * q;
        const float hv[4] = {h2[0].x, h2[0].y, h2[1].x, h2[1].y};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (4 * q + i < p.N)
                hl[i] = hv[i];
    }
}

}  // namespace ss2d
