// ss2d_backward.cuh -- sm_100a kernels of the SS2D backward pass (gradients
// of sum(dy * y) with respect to every input of the forward).
//
// The pages ask for a backward that recomputes the scan instead of keeping
// the states in HBM ("Vision Mamba ..." summary, section 4.4).  With
// a_t = exp(dt_t A) and the adjoint g_t = dLoss/dh_t,
//     g_t   = dy_t C_t + a_{t+1} g_{t+1}
//     dC_t  = sum_d dy_t h_t            dB_t = sum_d g_t dt_t u_t
//     du_t  = Dskip dy_t + dt_t sum_n g_n B_t,n
//     ddt_t = sum_n g_n (A_n a_t h_{t-1} + B_t,n u_t),  a_t h_{t-1} = h_t - dt_t u_t B_t
//     dA_n  = sum_t g_n dt_t a_t h_{t-1},n
// then ddelta = ddt * sigmoid(delta + bias), dA_log = dA * A, dbias and
// dDskip the sums over (b, t), and dx gathers du of every direction back to
// its pixel (the adjoint of cross_scan is cross_merge).
//
// Work decomposition: chunks of kT = 16 steps; a CTA is one warp holding 32
// channels of one (b, k) and walks a range of chunks.
//   1. bwd_local_kernel: per chunk, from zero, the forward end state h_end[c]
//      and the local adjoint Q[c] = a_s g_s (g from zero at the chunk end),
//      each with the chunk's sum of dt.  Q is stored in reversed chunk
//      order, so that
//   2. carry_kernel (the forward's) run twice gives the entry state of every
//      chunk and, over the reversed order, the adjoint G[c] = a_{e+1} g_{e+1}
//      entering every chunk from its end: G[c-1] = exp(A sum_c dt) G[c] + Q[c].
//      The final pass needs G only at the top of each CTA's range of chunks;
//      when one range covers a whole sequence, Q and its carry are skipped.
//   3. bwd_final_kernel: per chunk, in descending order, h recomputed from
//      its entry state (the
//      16 states of 8 steps of every lane parked in shared memory at a time:
//      the chunk is walked back in two halves), then the reverse walk from
//      G[c] writes ddelta and du, reduces dB and dC over
//      the warp's channels (one reduce-scatter of 32 values per step) into a
//      per-channel-group partial, and accumulates the parameter gradients.
//   4. merge2_kernel (K > 1) sums du of the directions into dx; two fixed-order
//      reductions finish dBs, dCs and dA_log, dDskip, ddelta_bias.
// Every reduction runs in a fixed order: the result is reproducible.
#pragma once

#include "ss2d_bwd_params.h"
#include "ss2d_kernels.cuh"

namespace ss2d {

constexpr float kLn2 = 0.6931471805599453f;

// shared memory of both kernels (floats): B and C of the chunk [t][n], and the
// lanes' staged (dt, u, dy, sigmoid(delta + bias)) as float4 [t][lane]
constexpr int kBwdStage = 2 * kT * kNP + 4 * kT * kBwdLanes;
// the final kernel adds the recomputed states of half a chunk, float4
// [t][lane][4] with the float4 index XOR-swizzled by (lane >> 1) & 3 (no bank
// conflicts for the lanes' 16-byte accesses)
constexpr int kHalf = kT / 2;
constexpr int kBwdStates = kHalf * kNP * kBwdLanes;
constexpr size_t kBwdFinalSmem = sizeof(float) * (kBwdStage + kBwdStates);

struct BwdLane {
    int b, k, gi, d, bk;
    bool active;
    size_t bkd;   // row (b, k, d) (d clamped for idle lanes)
};

__device__ __forceinline__ BwdLane bwd_lane(const BwdParams &p)
{
    BwdLane r;
    const int lane = threadIdx.x;
    r.gi = (int)(blockIdx.x % (unsigned)p.G);
    r.bk = (int)(blockIdx.x / (unsigned)p.G);
    r.b = r.bk / p.K;
    r.k = r.bk - r.b * p.K;
    r.d = r.gi * kBwdLanes + lane;
    r.active = r.d < p.D;
    if (!r.active)
        r.d = p.D - 1;
    r.bkd = ((size_t)r.b * p.K + r.k) * p.D + r.d;
    return r;
}

// The raw inputs of one chunk (steps s .. s+nt-1) that a lane stages: its
// channel's delta, x and dy, and its share of the chunk's B and C (state
// n = lane >> 1, 8 steps), loaded one chunk ahead into registers and turned
// into the shared-memory tiles after the current chunk's work.
template <typename Tin>
struct BwdRaw {
    using RawT = std::conditional_t<sizeof(Tin) == 2, unsigned short, float>;
    RawT dl[kT], x[kT], b[kT / 2], c[kT / 2];
    float gy[kT];
    int nt;

    __device__ __forceinline__ static float f32(RawT v)
    {
        if constexpr (sizeof(Tin) == 2)
            return half_bits_to_f32<Tin>(v);
        else
            return v;
    }

    __device__ __forceinline__ void fetch(const BwdParams &p, const BwdLane &q, int s)
    {
        nt = min(kT, p.L - s);
        const int lane = threadIdx.x;
        const int n = lane >> 1, t0 = (lane & 1) * (kT / 2);
        const bool nok = n < p.N;
        const size_t row =
            (((size_t)q.b * p.K + q.k) * p.NS + p.n0 + (nok ? n : 0)) * p.L + s + t0;
        const RawT *Bp = static_cast<const RawT *>(p.Bs) + row;
        const RawT *Cp = static_cast<const RawT *>(p.Cs) + row;
#pragma unroll
        for (int i = 0; i < kT / 2; ++i) {
            const bool ok = nok && t0 + i < nt;
            b[i] = ok ? __ldg(Bp + i) : RawT(0);
            c[i] = ok ? __ldg(Cp + i) : RawT(0);
        }
        const RawT *dp = static_cast<const RawT *>(p.delta) + q.bkd * p.L + s;
        const size_t xrow = ((size_t)q.b * p.D + q.d) * p.L;
        const RawT *xp = static_cast<const RawT *>(p.x) + xrow;
        const float *gp = p.dy + xrow;
        PixWalk w;
        w.init(p.two_d, q.k, s, p.H, p.W, p.L);
#pragma unroll
        for (int t = 0; t < kT; ++t) {
            const bool ok = t < nt && q.active;   // idle lanes add nothing to dB, dC
            dl[t] = ok ? __ldg(dp + t) : RawT(0);
            x[t] = ok ? __ldg(xp + w.p) : RawT(0);
            gy[t] = ok ? __ldg(gp + w.p) : 0.f;
            if (t + 1 < nt)
                w.next(p.H, p.W);
        }
    }

    // sB, sC [t][n] and st4 [t][lane] = (dt, u, dy, sigmoid(z)), z = delta + bias;
    // steps past nt (and idle lanes) stage zeros: dt = 0 makes a step the identity
    __device__ __forceinline__ void commit(float *sB, float *sC, float4 *st4, float bias,
                                           bool active) const
    {
        const int lane = threadIdx.x;
        const int n = lane >> 1, t0 = (lane & 1) * (kT / 2);
#pragma unroll
        for (int i = 0; i < kT / 2; ++i) {
            sB[(t0 + i) * kNP + n] = f32(b[i]);
            sC[(t0 + i) * kNP + n] = f32(c[i]);
        }
#pragma unroll
        for (int t = 0; t < kT; ++t) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < nt && active) {
                const float z = f32(dl[t]) + bias;
                v.x = softplus_f(z);
                v.y = f32(x[t]);
                v.z = gy[t];
                // sigmoid(z) = 1 / (1 + e^-z); e^-z = inf gives 0
                v.w = __fdividef(1.f, 1.f + mufu_ex2(-z * kLog2e));
            }
            st4[t * kBwdLanes + lane] = v;
        }
    }
};

__device__ __forceinline__ void load16(float *v, const float *src)
{
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
    for (int i = 0; i < kNP / 4; ++i) {
        const float4 a = s4[i];
        v[4 * i] = a.x;
        v[4 * i + 1] = a.y;
        v[4 * i + 2] = a.z;
        v[4 * i + 3] = a.w;
    }
}

__device__ __forceinline__ void store16(float *dst, const float *v)
{
    float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
    for (int i = 0; i < kNP / 4; ++i)
        d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

// States in pairs (2j, 2j+1) for the sm_100 packed f32x2 instructions
// (__ffma2_rn, __fmul2_rn: each lane rounds as fmaf / a float multiply).
__device__ __forceinline__ float2 ex2_pair(float2 a)
{
    return make_float2(mufu_ex2(a.x), mufu_ex2(a.y));
}
__device__ __forceinline__ float2 dup2(float v) { return make_float2(v, v); }
// pair j of a 16-float shared-memory row (16-byte aligned)
__device__ __forceinline__ float2 row_pair(const float *row, int j)
{
    return reinterpret_cast<const float2 *>(row)[j];
}
__device__ __forceinline__ void load_a2(float2 *A2, const BwdParams &p, size_t kd)
{
#pragma unroll
    for (int j = 0; j < kNP / 2; ++j) {
        const int n0 = 2 * j, n1 = 2 * j + 1;
        const float *al = p.A_log + kd * p.NS + p.n0;
        A2[j].x = n0 < p.N ? -expf(__ldg(al + n0)) * kLog2e : 0.f;
        A2[j].y = n1 < p.N ? -expf(__ldg(al + n1)) * kLog2e : 0.f;
    }
}
// one step of the state recurrence, h = exp(dt A) h + dt u B, for all pairs
__device__ __forceinline__ void state_step(float2 *h, const float2 *A2, float dt, float dtu,
                                           const float *brow)
{
    const float2 dt2 = dup2(dt), dtu2 = dup2(dtu);
#pragma unroll
    for (int j = 0; j < kNP / 2; ++j)
        h[j] = __ffma2_rn(ex2_pair(__fmul2_rn(dt2, A2[j])), h[j],
                          __fmul2_rn(dtu2, row_pair(brow, j)));
}

template <typename Tin>
__global__ void __launch_bounds__(kBwdLanes) bwd_local_kernel(const BwdParams p)
{
    __shared__ float4 sm4[kBwdStage / 4];
    float *sB = reinterpret_cast<float *>(sm4), *sC = sB + kT * kNP;
    float4 *st4 = sm4 + 2 * kT * kNP / 4;
    const int lane = threadIdx.x;
    const BwdLane q = bwd_lane(p);
    const size_t kd = (size_t)q.k * p.D + q.d;
    float2 A2[kNP / 2];
    load_a2(A2, p, kd);
    const float bias = __ldg(p.delta_bias + kd);
    const int nc1 = p.NC - 1;
    const int c0 = blockIdx.y * p.CPB, c1 = min(p.NC, c0 + p.CPB);
    BwdRaw<Tin> raw;
    raw.fetch(p, q, c0 * kT);
    for (int c = c0; c < c1; ++c) {
        __syncwarp();
        raw.commit(sB, sC, st4, bias, q.active);
        __syncwarp();
        if (c + 1 < c1)
            raw.fetch(p, q, (c + 1) * kT);   // in flight during this chunk's work
        float dts = 0.f;
#pragma unroll
        for (int t = 0; t < kT; ++t)
            dts += st4[t * kBwdLanes + lane].x;
        if (c < nc1) {
            float2 h[kNP / 2];
#pragma unroll
            for (int j = 0; j < kNP / 2; ++j)
                h[j] = make_float2(0.f, 0.f);
#pragma unroll
            for (int t = 0; t < kT; ++t) {
                const float4 v = st4[t * kBwdLanes + lane];
                state_step(h, A2, v.x, v.x * v.y, sB + t * kNP);
            }
            if (q.active) {
                store16(p.hfwd + (q.bkd * nc1 + c) * kNP, reinterpret_cast<const float *>(h));
                p.dtf[q.bkd * nc1 + c] = dts;
            }
        }
        if (c > 0 && p.adj_chunks) {
            float2 g[kNP / 2];
#pragma unroll
            for (int j = 0; j < kNP / 2; ++j)
                g[j] = make_float2(0.f, 0.f);
#pragma unroll
            for (int t = kT - 1; t >= 0; --t) {
                const float4 v = st4[t * kBwdLanes + lane];
                const float2 dt2 = dup2(v.x), gy2 = dup2(v.z);
#pragma unroll
                for (int j = 0; j < kNP / 2; ++j)
                    g[j] = __fmul2_rn(ex2_pair(__fmul2_rn(dt2, A2[j])),
                                      __ffma2_rn(gy2, row_pair(sC + t * kNP, j), g[j]));
            }
            if (q.active) {
                const int r = nc1 - c;   // reversed chunk order
                store16(p.hadj + (q.bkd * nc1 + r) * kNP, reinterpret_cast<const float *>(g));
                p.dta[q.bkd * nc1 + r] = dts;
            }
        }
    }
}

// One halving exchange: lanes with bit M set keep v[M..2M) (moved to v[0..M)),
// the others v[0..M); each adds the half its partner sends.
template <int M>
__device__ __forceinline__ void halve(float *v)
{
    const bool hi = (threadIdx.x & M) != 0;
#pragma unroll
    for (int i = 0; i < M; ++i) {
        const float lo = v[i], up = v[i + M];
        const float send = hi ? lo : up;
        const float keep = hi ? up : lo;
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
    }
}

// Sum over the 32 lanes of v[j] for j = lane (v[0..15]: dB of the 16 states,
// v[16..31]: dC): five halving exchanges, 31 shuffles.
__device__ __forceinline__ float reduce_scatter32(float *v)
{
    halve<16>(v);
    halve<8>(v);
    halve<4>(v);
    halve<2>(v);
    halve<1>(v);
    return v[0];
}

template <typename Tin>
__global__ void __launch_bounds__(kBwdLanes) bwd_final_kernel(const BwdParams p)
{
    extern __shared__ float4 smem_bwd4[];
    float *sB = reinterpret_cast<float *>(smem_bwd4), *sC = sB + kT * kNP;
    float4 *st4 = smem_bwd4 + 2 * kT * kNP / 4;
    float4 *hs4 = st4 + kT * kBwdLanes;   // [t][lane][4 float4], half a chunk
    const int lane = threadIdx.x;
    const int swz = (lane >> 1) & 3;
    const BwdLane q = bwd_lane(p);
    const size_t kd = (size_t)q.k * p.D + q.d;
    float2 A2[kNP / 2];
    load_a2(A2, p, kd);
    const float bias = __ldg(p.delta_bias + kd);
    const bool accum = p.accum != 0;   // a later state group: add to the rows
    const float Dk = accum ? 0.f : __ldg(p.Dskip + kd);
    const int L = p.L, nc1 = p.NC - 1;
    const bool flip = p.flip1 && q.k == 1;
    float *durow = p.du + q.bkd * L;
    float *ddrow = p.ddelta + q.bkd * L;
    float *bcrow = p.bc_part + ((((size_t)q.bk * p.G + q.gi) * 2 + (lane >> 4)) * p.NS + p.n0 +
                                (lane & 15)) * L;
    const bool bc_ok = (lane & 15) < p.N;
    // rows of L floats: 16-byte segments at 16-step chunk starts when L % 4 == 0
    // (the scratch and gradient buffers are 16-byte aligned)
    const bool vec_rows = (L & 3) == 0;
    float2 dA[kNP / 2];
#pragma unroll
    for (int j = 0; j < kNP / 2; ++j)
        dA[j] = make_float2(0.f, 0.f);
    float dD = 0.f, db = 0.f;
    const int c0 = blockIdx.y * p.CPB, c1 = min(p.NC, c0 + p.CPB);
    // The chunks of the range in descending order: the walk back over chunk c
    // ends with g = a_s g_s, the adjoint entering chunk c - 1 at its end, so
    // only the range's top chunk takes its adjoint from the carry.
    float2 g[kNP / 2];
    BwdRaw<Tin> raw;
    raw.fetch(p, q, (c1 - 1) * kT);
    for (int c = c1 - 1; c >= c0; --c) {
        const int s = c * kT, nt = min(kT, L - s);
        __syncwarp();
        raw.commit(sB, sC, st4, bias, q.active);
        __syncwarp();
        if (c - 1 >= c0)
            raw.fetch(p, q, (c - 1) * kT);   // in flight during this chunk's work
        // The chunk in two halves of 8 steps, so that only half of its states
        // are parked at a time: the first recompute runs the whole chunk from
        // the entry state and parks steps 8..15 for the walk back over them;
        // the second recomputes steps 0..7 from the entry state again.
        auto entry = [&](float2 *h) {
            if (c > 0)
                load16(reinterpret_cast<float *>(h), p.hfwd + (q.bkd * nc1 + (c - 1)) * kNP);
            else
#pragma unroll
                for (int j = 0; j < kNP / 2; ++j)
                    h[j] = make_float2(0.f, 0.f);
        };
        auto recompute = [&](float2 *h, int t1, int park0) {
#pragma unroll 1
            for (int t = 0; t < t1; ++t) {
                const float4 v = st4[t * kBwdLanes + lane];
                state_step(h, A2, v.x, v.x * v.y, sB + t * kNP);
                if (t >= park0) {
                    float4 *row = hs4 + ((t - park0) * kBwdLanes + lane) * 4;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        row[j ^ swz] = make_float4(h[2 * j].x, h[2 * j].y, h[2 * j + 1].x,
                                                   h[2 * j + 1].y);
                }
            }
        };
        auto walk_back = [&](int t_hi, int base) {
#pragma unroll 2
            for (int t = t_hi; t >= base; --t) {
                const float4 v4 = st4[t * kBwdLanes + lane];
                const float dt = v4.x, u = v4.y, gy = v4.z;
                const float dtu = dt * u;
                const float2 dt2 = dup2(dt), dtu2 = dup2(dtu), ndtu2 = dup2(-dtu), gy2 = dup2(gy);
                const float4 *row = hs4 + ((t - base) * kBwdLanes + lane) * 4;
                float v[2 * kNP];
                // sum g A2 (a h_prev), sum g B: two-wide partial sums
                float2 s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const float4 h4 = row[qd ^ swz];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int j = 2 * qd + i;
                        const float2 B2 = row_pair(sB + t * kNP, j);
                        const float2 hv = i ? make_float2(h4.z, h4.w) : make_float2(h4.x, h4.y);
                        g[j] = __ffma2_rn(gy2, row_pair(sC + t * kNP, j), g[j]);
                        const float2 hp = __ffma2_rn(ndtu2, B2, hv);   // a_t h_{t-1}
                        const float2 vb = __fmul2_rn(g[j], dtu2);
                        const float2 vc = __fmul2_rn(gy2, hv);
                        v[2 * j] = vb.x;
                        v[2 * j + 1] = vb.y;
                        v[kNP + 2 * j] = vc.x;
                        v[kNP + 2 * j + 1] = vc.y;
                        s2 = __ffma2_rn(g[j], B2, s2);
                        s1 = __ffma2_rn(__fmul2_rn(g[j], A2[j]), hp, s1);
                        dA[j] = __ffma2_rn(__fmul2_rn(g[j], dt2), hp, dA[j]);
                        g[j] = __fmul2_rn(g[j], ex2_pair(__fmul2_rn(dt2, A2[j])));
                    }
                }
                const float red = reduce_scatter32(v);
                // this step's results replace its staged inputs in the lane's own
                // slot (consumed by now); the rows are written once per chunk
                const float S1 = s1.x + s1.y, S2 = s2.x + s2.y;
                const float ddl = fmaf(kLn2, S1, u * S2) * v4.w;
                st4[t * kBwdLanes + lane] = make_float4(ddl, fmaf(Dk, gy, dt * S2), red, 0.f);
                if (q.active && t < nt) {
                    dD = fmaf(gy, u, dD);
                    db += ddl;
                }
            }
        };
        // the adjoint entering the range's top chunk at its end (zero for the
        // sequence's last chunk)
        if (c == c1 - 1) {
            if (c < nc1)
                load16(reinterpret_cast<float *>(g),
                       p.hadj + (q.bkd * nc1 + (nc1 - 1 - c)) * kNP);
            else
#pragma unroll
                for (int j = 0; j < kNP / 2; ++j)
                    g[j] = make_float2(0.f, 0.f);
        }
        {
            float2 h[kNP / 2];
            entry(h);
            recompute(h, kT, kHalf);
        }
        walk_back(kT - 1, kHalf);
        {
            float2 h[kNP / 2];
            entry(h);
            recompute(h, kHalf, 0);
        }
        walk_back(kHalf - 1, 0);
        // the chunk's rows: ddelta and du of this lane's channel, and the
        // reduced dB | dC row this lane holds (16-byte segments when whole)
        const bool whole = nt == kT && vec_rows;
        if (q.active) {
            auto put4 = [&](float4 *dst, float4 v) {
                if (accum) {
                    const float4 e = *dst;
                    v = make_float4(e.x + v.x, e.y + v.y, e.z + v.z, e.w + v.w);
                }
                *dst = v;
            };
            if (whole) {
                float4 *dd4 = reinterpret_cast<float4 *>(ddrow + s);
                float4 *du4 = reinterpret_cast<float4 *>(durow + (flip ? L - kT - s : s));
#pragma unroll
                for (int i = 0; i < kT / 4; ++i) {
                    const float4 a = st4[(4 * i) * kBwdLanes + lane];
                    const float4 b = st4[(4 * i + 1) * kBwdLanes + lane];
                    const float4 c4 = st4[(4 * i + 2) * kBwdLanes + lane];
                    const float4 d4 = st4[(4 * i + 3) * kBwdLanes + lane];
                    put4(dd4 + i, make_float4(a.x, b.x, c4.x, d4.x));
                    if (flip)
                        put4(du4 + (kT / 4 - 1 - i), make_float4(d4.y, c4.y, b.y, a.y));
                    else
                        put4(du4 + i, make_float4(a.y, b.y, c4.y, d4.y));
                }
            } else {
                for (int t = 0; t < nt; ++t) {
                    const float4 r = st4[t * kBwdLanes + lane];
                    const int l = s + t;
                    float *o = durow + (flip ? L - 1 - l : l);
                    ddrow[l] = accum ? ddrow[l] + r.x : r.x;
                    *o = accum ? *o + r.y : r.y;
                }
            }
        }
        if (bc_ok) {
            if (whole) {
                float4 *bc4 = reinterpret_cast<float4 *>(bcrow + s);
#pragma unroll
                for (int i = 0; i < kT / 4; ++i)
                    bc4[i] = make_float4(st4[(4 * i) * kBwdLanes + lane].z,
                                         st4[(4 * i + 1) * kBwdLanes + lane].z,
                                         st4[(4 * i + 2) * kBwdLanes + lane].z,
                                         st4[(4 * i + 3) * kBwdLanes + lane].z);
            } else {
                for (int t = 0; t < nt; ++t)
                    bcrow[s + t] = st4[t * kBwdLanes + lane].z;
            }
        }
    }
    if (q.active) {
        // slots: dA of the call's NS states, dDskip, dbias; a later state group
        // writes its own dA and adds its share of dbias (same thread, later launch)
        float *pr = p.prm_part + (q.bkd * p.CGN + blockIdx.y) * (p.NS + 2);
#pragma unroll
        for (int j = 0; j < kNP / 2; ++j) {
            if (2 * j < p.N)
                pr[p.n0 + 2 * j] = dA[j].x;
            if (2 * j + 1 < p.N)
                pr[p.n0 + 2 * j + 1] = dA[j].y;
        }
        if (!accum) {
            pr[p.NS] = dD;
            pr[p.NS + 1] = db;
        } else {
            pr[p.NS + 1] += db;
        }
    }
}

// dBs, dCs (B,K,N,L) = the sum over the channel groups, in group order (the
// partial holds N rows per (b, k, group, B|C))
__global__ void bwd_reduce_bc_kernel(const float *__restrict__ part, float *__restrict__ dBs,
                                     float *__restrict__ dCs, int BK, int G, int N, int L)
{
    const long long total = (long long)BK * 2 * N * L;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int l = (int)(i % L);
        long long r = i / L;
        const int n = (int)(r % N);
        r /= N;
        const int which = (int)(r & 1);
        const long long bk = r >> 1;
        const float *src = part + (((size_t)bk * G * 2 + which) * N + n) * L + l;
        const size_t gstride = (size_t)2 * N * L;
        float s = 0.f;
        for (int g = 0; g < G; ++g)
            s += __ldg(src + g * gstride);
        (which ? dCs : dBs)[((size_t)bk * N + n) * L + l] = s;
    }
}

// dA_log = A * sum dA, dDskip, ddelta_bias: per (k, d), the sum over b and
// the chunk groups, in that order
__global__ void bwd_reduce_param_kernel(const float *__restrict__ prm,
                                        const float *__restrict__ A_log, float *__restrict__ dA_log,
                                        float *__restrict__ dDskip, float *__restrict__ dbias,
                                        int B, int K, int D, int N, int CGN)
{
    const long long total = (long long)K * D * (N + 2);
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int j = (int)(i % (N + 2));
        const long long kd = i / (N + 2);
        const int k = (int)(kd / D), d = (int)(kd % D);
        float s = 0.f;
        for (int b = 0; b < B; ++b) {
            const float *src = prm + ((((size_t)b * K + k) * D + d) * CGN) * (N + 2) + j;
            for (int cg = 0; cg < CGN; ++cg)
                s += __ldg(src + (size_t)cg * (N + 2));
        }
        if (j < N)
            dA_log[kd * N + j] = s * -expf(__ldg(A_log + kd * N + j));
        else if (j == N)
            dDskip[kd] = s;
        else
            dbias[kd] = s;
    }
}

}  // namespace ss2d
