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
// Work decomposition: chunks of kT = 16 steps; a CTA holds 32 channels of one
// (b, k) in four warps (warp w: states 4w .. 4w+3) and walks a range of
// chunks.
//   1. bwd_local4_kernel: per chunk, from zero, the forward end state h_end[c]
//      and the local adjoint Q[c] = a_s g_s (g from zero at the chunk end),
//      each with the chunk's sum of dt, in one forward walk with one exp2 per
//      state and step (Q as the sum of dy_t C_t weighted by the running
//      product of the a's).  Q is stored in reversed chunk order, so that
//   2. the forward's carry scan (launch_carry_scan) run twice gives the entry
//      state of every chunk and, over the reversed order, the adjoint G[c] = a_{e+1} g_{e+1}
//      entering every chunk from its end: G[c-1] = exp(A sum_c dt) G[c] + Q[c].
//      The final pass needs G only at the top of each CTA's range of chunks;
//      when one range covers a whole sequence, Q and its carry are skipped.
//   3. bwd_final4_kernel (4 warps per CTA, warp w holding states 4w..4w+3 of
//      the same 32 channels): per chunk of its range, in descending order
//      (the walk back over a chunk ends with the adjoint entering the chunk
//      below), each warp recomputes its states from the entry state and
//      parks them in shared memory, sums dC = dy h of its states over the
//      channels from there, then walks back from G[c] accumulating dA and
//      parking g dt u in the place of h, whose channel sums are dB; the
//      per-step sums over all 16 states that du and ddelta need are
//      combined through shared memory once per chunk.
//   4. merge2_kernel (K = 4, or K = 2 with N > 16) sums du of the
//      directions into dx (K = 2 otherwise: the final pass adds both into
//      dx); two fixed-order
//      reductions finish dBs, dCs and dA_log, dDskip, ddelta_bias.
// Every reduction runs in a fixed order: the result is reproducible.
#pragma once

#include "ss2d_bwd_params.h"
#include "ss2d_kernels.cuh"

namespace ss2d {

constexpr float kLn2 = 0.6931471805599453f;

// shared memory of the local pass (floats): B and C of the chunk [t][n], and
// the lanes' staged (dt, u, dy, sigmoid(delta + bias)) as float4 [t][lane]
// B and C tiles [t][kBCS]: rows of 16 states padded to 20 floats, so that
// the staging stores (16 consecutive steps of a state per half warp) fall
// into 16 different banks pairwise instead of two, and rows stay 16-byte
// aligned for the walks' float4 reads
constexpr int kBCS = 20;
constexpr int kBwdStage = 2 * kT * kBCS + 4 * kT * kBwdLanes;

struct BwdLane {
    int b, k, gi, d, bk;
    bool active;
    size_t bkd;   // row (b, k, d) (d clamped for idle lanes)
};

__device__ __forceinline__ BwdLane bwd_lane(const BwdParams &p)
{
    BwdLane r;
    const int lane = threadIdx.x & 31;
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

// States in pairs (2j, 2j+1) for the sm_100 packed f32x2 instructions
// (__ffma2_rn, __fmul2_rn: each lane rounds as fmaf / a float multiply).
__device__ __forceinline__ float2 ex2_pair(float2 a)
{
    return make_float2(mufu_ex2(a.x), mufu_ex2(a.y));
}
__device__ __forceinline__ float2 dup2(float v) { return make_float2(v, v); }
// pair j of a shared-memory row of states (16-byte aligned)
__device__ __forceinline__ float2 row_pair(const float *row, int j)
{
    return reinterpret_cast<const float2 *>(row)[j];
}

// ---------------------------------------------------------------------------
// The final pass with the 16 states of a channel group split over 4 warps
// (warp w: states 4w .. 4w+3 of the same 32 channels).  A warp parks the
// states of a whole chunk (8 KB), so a chunk is recomputed once; dC and dB
// of its 4 states are summed over the channels from that tile (lane_sums,
// before and after the walk back); the sums
// over all 16 states that du and ddelta need are combined through shared
// memory once per chunk, each warp finishing 4 of the 16 steps.
constexpr int kQuadWarps = 4;
constexpr int kBwd4Threads = kQuadWarps * kBwdLanes;
constexpr int kBwd4Stage = 2 * kT * kBCS + 4 * kT * kBwdLanes;   // B|C tiles, st4
constexpr int kBwd4Hs = kQuadWarps * kT * kBwdLanes * 4;         // per warp [t][lane] float4
constexpr int kBwd4Sums = kQuadWarps * kT * kBwdLanes * 2;       // per warp [t][lane] (s1, s2)
constexpr int kBwd4Red = kQuadWarps * kT * 8;                    // per warp [t][8] reduced dB|dC
constexpr int kBwd4Dy = kT * kBwdLanes;                          // [t][lane] dy, 4-byte stride
constexpr size_t kBwd4Smem =
    sizeof(float) * (kBwd4Stage + kBwd4Hs + kBwd4Sums + kBwd4Red + kBwd4Dy);

// Sums over the warp's 32 channels of a [t][lane] float4 tile of its 4
// states (hs), times dy of the channel (sdy[t][lane]) when weighted: lane
// 16 h + t sums channels 16 h .. 16 h + 15 of step t (16-byte loads, the
// channel order rotated by t so that each quarter-warp reads 8 different
// bank groups), then the two halves meet in one exchange: half h keeps
// states 2h, 2h + 1 and writes them to red[t * 8 + base + 2h + {0, 1}].
// The order is fixed, so every call gives the same sums.
__device__ __forceinline__ void lane_sums(const float4 *hs, const float *sdy, float *red,
                                          int lane, int base, bool weighted)
{
    const int t = lane & 15, hf = lane >> 4;
    const float4 *row = hs + t * kBwdLanes + 16 * hf;
    const float *dyrow = sdy + t * kBwdLanes + 16 * hf;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
        const int l = (i + t) & 15;
        const float4 v = row[l];
        if (weighted) {
            const float gy = dyrow[l];
            acc.x = fmaf(gy, v.x, acc.x);
            acc.y = fmaf(gy, v.y, acc.y);
            acc.z = fmaf(gy, v.z, acc.z);
            acc.w = fmaf(gy, v.w, acc.w);
        } else {
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
    }
    const float s0 = hf ? acc.x : acc.z, s1 = hf ? acc.y : acc.w;   // the other half's states
    const float k0 = hf ? acc.z : acc.x, k1 = hf ? acc.w : acc.y;   // this half's states
    const float r0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 16);
    const float r1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 16);
    *reinterpret_cast<float2 *>(red + t * 8 + base + 2 * hf) = make_float2(r0, r1);
}

// The raw inputs of one chunk, the staging split over the CTA's 128 threads:
// 4 of the 512 B|C values, and 4 steps (4w .. 4w+3) of the lane's channel.
template <typename Tin>
struct BwdRaw4 {
    using RawT = std::conditional_t<sizeof(Tin) == 2, unsigned short, float>;
    RawT bc[4], dl[4], x[4];
    float gy[4];
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
        const int tid = threadIdx.x, w = tid >> 5;
        const size_t bkrow = ((size_t)q.b * p.K + q.k) * p.NS + p.n0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int item = tid + i * kBwd4Threads;   // 0..511: (B|C, n, t)
            const int which = item >> 8, n = (item >> 4) & 15, t = item & 15;
            const bool ok = n < p.N && t < nt;
            const RawT *src = static_cast<const RawT *>(which ? p.Cs : p.Bs);
            bc[i] = ok ? __ldg(src + (bkrow + n) * p.L + s + t) : RawT(0);
        }
        const RawT *dp = static_cast<const RawT *>(p.delta) + q.bkd * p.L + s;
        const size_t xrow = ((size_t)q.b * p.D + q.d) * p.L;
        const RawT *xp = static_cast<const RawT *>(p.x) + xrow;
        const float *gp = p.dy + xrow;
        const int t0 = 4 * w;
        // the 4 steps whole and L % 4 == 0: the delta row segment is one
        // 8-byte (2-byte types) or 16-byte load, and so are x and dy of the
        // row-major directions (pixels s+t0.. ascending, or descending from
        // L-1-s-t0: loaded ascending from L-4-s-t0 and reversed); every such
        // segment starts on a multiple of 4 elements
        const bool vec = (p.L & 3) == 0 && t0 + 4 <= nt && q.active;
        const int xmode = (!p.two_d || q.k < 2) ? (q.k & 1) : 2;
        if (vec) {
            load4(dp + t0, dl);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const bool ok = t0 + i < nt && q.active;   // idle lanes add nothing to dB, dC
                dl[i] = ok ? __ldg(dp + t0 + i) : RawT(0);
            }
        }
        if (vec && xmode != 2) {
            const int base = xmode == 0 ? s + t0 : p.L - 4 - s - t0;
            RawT xv[4];
            load4(xp + base, xv);
            const float4 g4 = __ldg(reinterpret_cast<const float4 *>(gp + base));
            const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                x[i] = xmode == 0 ? xv[i] : xv[3 - i];
                gy[i] = xmode == 0 ? gv[i] : gv[3 - i];
            }
        } else {
            PixWalk pw;
            pw.init(p.two_d, q.k, min(s + t0, p.L - 1), p.H, p.W, p.L);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = t0 + i;
                const bool ok = t < nt && q.active;
                x[i] = ok ? __ldg(xp + pw.p) : RawT(0);
                gy[i] = ok ? __ldg(gp + pw.p) : 0.f;
                if (t + 1 < nt)
                    pw.next(p.H, p.W);
            }
        }
    }
    // 4 consecutive values from a 4-element-aligned address: one 8-byte
    // (2-byte types) or 16-byte load
    __device__ __forceinline__ static void load4(const RawT *src, RawT (&v)[4])
    {
        if constexpr (sizeof(RawT) == 2) {
            const uint2 r = __ldg(reinterpret_cast<const uint2 *>(src));
            v[0] = (RawT)(r.x & 0xffffu);
            v[1] = (RawT)(r.x >> 16);
            v[2] = (RawT)(r.y & 0xffffu);
            v[3] = (RawT)(r.y >> 16);
        } else {
            const float4 r = __ldg(reinterpret_cast<const float4 *>(src));
            v[0] = r.x;
            v[1] = r.y;
            v[2] = r.z;
            v[3] = r.w;
        }
    }

    // sdy (optional): dy again as a [t][lane] row of floats
    __device__ __forceinline__ void commit(float *sB, float *sC, float4 *st4, float bias,
                                           bool active, float *sdy = nullptr) const
    {
        const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int item = tid + i * kBwd4Threads;
            const int which = item >> 8, n = (item >> 4) & 15, t = item & 15;
            (which ? sC : sB)[t * kBCS + n] = f32(bc[i]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * w + i;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < nt && active) {
                const float z = f32(dl[i]) + bias;
                v.x = softplus_f(z);
                v.y = f32(x[i]);
                v.z = gy[i];
                v.w = __fdividef(1.f, 1.f + mufu_ex2(-z * kLog2e));   // sigmoid(z)
            }
            st4[t * kBwdLanes + lane] = v;
            if (sdy)
                sdy[t * kBwdLanes + lane] = v.z;
        }
    }
};

// One forward walk over a staged chunk from zero for the warp's 4 states
// (4w .. 4w+3: pairs A2[0], A2[1]), one exp2 per state and step serving both
// results:
//   HS: the end state h (h = a_t h + dt_t u_t B_t);
//   QS: the local adjoint Q = a_0 g_0 with g from zero at the chunk end,
//       g_t = a_t (dy_t C_t + g_{t+1}); unrolled, Q = sum_t P_t dy_t C_t with
//       P_t = a_0 a_1 ... a_t, which the walk accumulates forwards.
// Also returns the chunk's sum of dt in dts (the walk reads every step's dt).
template <bool HS, bool QS>
__device__ __forceinline__ void local_walk4(const float4 *st4, const float *sB, const float *sC,
                                            const float2 (&A2)[2], int nw, float2 (&h)[2],
                                            float2 (&Q)[2], float &dts)
{
    const int lane = threadIdx.x & 31;
    dts = 0.f;
    float2 P[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        h[j] = make_float2(0.f, 0.f);
        Q[j] = make_float2(0.f, 0.f);
        P[j] = make_float2(1.f, 1.f);
    }
#pragma unroll 4
    for (int t = 0; t < kT; ++t) {
        const float4 v = st4[t * kBwdLanes + lane];
        dts += v.x;
        const float2 dt2 = dup2(v.x), dtu2 = dup2(v.x * v.y), gy2 = dup2(v.z);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const float2 a = ex2_pair(__fmul2_rn(dt2, A2[j]));
            if constexpr (HS)
                h[j] = __ffma2_rn(a, h[j], __fmul2_rn(dtu2, row_pair(sB + t * kBCS + nw, j)));
            if constexpr (QS) {
                P[j] = __fmul2_rn(P[j], a);
                Q[j] = __ffma2_rn(P[j], __fmul2_rn(gy2, row_pair(sC + t * kBCS + nw, j)), Q[j]);
            }
        }
    }
}

// The local pass with the 16 states of a channel group split over 4 warps
// (warp w: states 4w .. 4w+3 of the same 32 channels), the chunk's inputs
// staged once for the CTA (BwdRaw4): per chunk of its range, from zero, the
// forward end state h_end[c] and the local adjoint Q[c], each with the
// chunk's sum of dt, in one forward walk.
template <typename Tin>
__global__ void __launch_bounds__(kBwd4Threads, 4) bwd_local4_kernel(const BwdParams p)
{
    __shared__ float4 sm4[kBwdStage / 4];
    float *sB = reinterpret_cast<float *>(sm4), *sC = sB + kT * kBCS;
    float4 *st4 = sm4 + 2 * kT * kBCS / 4;   // [t][lane]
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const BwdLane q = bwd_lane(p);
    const size_t kd = (size_t)q.k * p.D + q.d;
    const int nw = 4 * w;   // this warp's first state within the group
    float2 A2[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float *al = p.A_log + kd * p.NS + p.n0 + nw;
        A2[j].x = nw + 2 * j < p.N ? -expf(__ldg(al + 2 * j)) * kLog2e : 0.f;
        A2[j].y = nw + 2 * j + 1 < p.N ? -expf(__ldg(al + 2 * j + 1)) * kLog2e : 0.f;
    }
    const float bias = __ldg(p.delta_bias + kd);
    const int nc1 = p.NC - 1;
    const int c0 = blockIdx.y * p.CPB, c1 = min(p.NC, c0 + p.CPB);
    BwdRaw4<Tin> raw;
    raw.fetch(p, q, c0 * kT);
    for (int c = c0; c < c1; ++c) {
        __syncthreads();   // the previous chunk's tiles are read
        raw.commit(sB, sC, st4, bias, q.active);
        __syncthreads();
        if (c + 1 < c1)
            raw.fetch(p, q, (c + 1) * kT);   // in flight during this chunk's work
        const bool hs = c < nc1, qs = c > 0 && p.adj_chunks;
        float2 h[2], g[2];
        float dts = 0.f;   // the chunk's sum of dt (summed in step order by the walk)
        if (hs && qs)
            local_walk4<true, true>(st4, sB, sC, A2, nw, h, g, dts);
        else if (hs)
            local_walk4<true, false>(st4, sB, sC, A2, nw, h, g, dts);
        else if (qs)
            local_walk4<false, true>(st4, sB, sC, A2, nw, h, g, dts);
        if (hs && q.active) {
            *reinterpret_cast<float4 *>(p.hfwd + (q.bkd * nc1 + c) * kNP + nw) =
                make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
            if (w == 0)
                p.dtf[q.bkd * nc1 + c] = dts;
        }
        if (qs && q.active) {
            const int r = nc1 - c;   // reversed chunk order
            *reinterpret_cast<float4 *>(p.hadj + (q.bkd * nc1 + r) * kNP + nw) =
                make_float4(g[0].x, g[0].y, g[1].x, g[1].y);
            if (w == 0)
                p.dta[q.bkd * nc1 + r] = dts;
        }
    }
}

template <typename Tin>
__global__ void __launch_bounds__(kBwd4Threads) bwd_final4_kernel(const BwdParams p)
{
    extern __shared__ float4 smem_b4[];
    float *sB = reinterpret_cast<float *>(smem_b4), *sC = sB + kT * kBCS;
    float4 *st4 = smem_b4 + 2 * kT * kBCS / 4;                      // [t][lane]
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    float4 *hs = st4 + kT * kBwdLanes + w * kT * kBwdLanes;           // this warp's [t][lane]
    float2 *sums = reinterpret_cast<float2 *>(st4 + kT * kBwdLanes + kQuadWarps * kT * kBwdLanes);
    float *red = reinterpret_cast<float *>(sums + kQuadWarps * kT * kBwdLanes) + w * kT * 8;
    float *sdy = reinterpret_cast<float *>(sums + kQuadWarps * kT * kBwdLanes) + kBwd4Red;
    const BwdLane q = bwd_lane(p);
    const size_t kd = (size_t)q.k * p.D + q.d;
    const int nw = 4 * w;   // this warp's first state within the group
    float2 A2[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float *al = p.A_log + kd * p.NS + p.n0 + nw;
        A2[j].x = nw + 2 * j < p.N ? -expf(__ldg(al + 2 * j)) * kLog2e : 0.f;
        A2[j].y = nw + 2 * j + 1 < p.N ? -expf(__ldg(al + 2 * j + 1)) * kLog2e : 0.f;
    }
    const float bias = __ldg(p.delta_bias + kd);
    const bool accum = p.accum != 0;
    const float Dk = accum ? 0.f : __ldg(p.Dskip + kd);
    const int L = p.L, nc1 = p.NC - 1;
    const bool flip = p.flip1 && q.k == 1;
    const bool xmerge = p.dxmerge != nullptr;   // both directions add into dx
    float *durow = xmerge ? p.dxmerge + ((size_t)q.b * p.D + q.d) * L : p.du + q.bkd * L;
    float *ddrow = p.ddelta + q.bkd * L;
    const bool vec_rows = (L & 3) == 0;
    // the reduced row this lane writes (lanes 0..7 of each warp: j = lane)
    const int rj = lane & 7;
    const bool bc_ok = lane < 8 && nw + (rj & 3) < p.N;
    float *bcrow = p.bc_part + ((((size_t)q.bk * p.G + q.gi) * 2 + (rj >> 2)) * p.NS + p.n0 +
                                nw + (rj & 3)) * L;
    float2 dA[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float dD = 0.f, db = 0.f;
    const int c0 = blockIdx.y * p.CPB, c1 = min(p.NC, c0 + p.CPB);
    // chunks in descending order: the adjoint flows from chunk to chunk
    float2 g[2];
    BwdRaw4<Tin> raw;
    raw.fetch(p, q, (c1 - 1) * kT);
    for (int c = c1 - 1; c >= c0; --c) {
        const int s = c * kT, nt = min(kT, L - s);
        __syncthreads();   // every warp is done with the previous chunk's tiles
        raw.commit(sB, sC, st4, bias, q.active, sdy);
        __syncthreads();
        if (c - 1 >= c0)
            raw.fetch(p, q, (c - 1) * kT);   // in flight during this chunk's work
        // this warp's 4 states over the chunk, from the entry state
        {
            float2 h[2];
            if (c > 0) {
                const float4 e = *reinterpret_cast<const float4 *>(
                    p.hfwd + (q.bkd * nc1 + (c - 1)) * kNP + nw);
                h[0] = make_float2(e.x, e.y);
                h[1] = make_float2(e.z, e.w);
            } else {
                h[0] = h[1] = make_float2(0.f, 0.f);
            }
#pragma unroll 4
            for (int t = 0; t < kT; ++t) {
                const float4 v = st4[t * kBwdLanes + lane];
                const float4 b4 = *reinterpret_cast<const float4 *>(sB + t * kBCS + nw);
                const float2 dt2 = dup2(v.x), dtu2 = dup2(v.x * v.y);
                h[0] = __ffma2_rn(ex2_pair(__fmul2_rn(dt2, A2[0])), h[0],
                                  __fmul2_rn(dtu2, make_float2(b4.x, b4.y)));
                h[1] = __ffma2_rn(ex2_pair(__fmul2_rn(dt2, A2[1])), h[1],
                                  __fmul2_rn(dtu2, make_float2(b4.z, b4.w)));
                hs[t * kBwdLanes + lane] = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
            }
        }
        // dC of the warp's 4 states at every step of the chunk: lane (t, pair)
        // sums dy * h over the 32 channels
        __syncwarp();
        lane_sums(hs, sdy, red, lane, 4, true);
        __syncwarp();   // every lane is done with h before the walk back overwrites it
        if (c == c1 - 1) {   // the adjoint entering the range's top chunk at its end
            if (c < nc1) {
                const float4 e = *reinterpret_cast<const float4 *>(
                    p.hadj + (q.bkd * nc1 + (nc1 - 1 - c)) * kNP + nw);
                g[0] = make_float2(e.x, e.y);
                g[1] = make_float2(e.z, e.w);
            } else {
                g[0] = g[1] = make_float2(0.f, 0.f);
            }
        }
#pragma unroll 2
        for (int t = kT - 1; t >= 0; --t) {
            const float4 v4 = st4[t * kBwdLanes + lane];
            const float dt = v4.x, u = v4.y, gy = v4.z;
            const float2 dt2 = dup2(dt), dtu2 = dup2(dt * u), ndtu2 = dup2(-dt * u);
            const float2 gy2 = dup2(gy);
            const float4 b4 = *reinterpret_cast<const float4 *>(sB + t * kBCS + nw);
            const float4 c4 = *reinterpret_cast<const float4 *>(sC + t * kBCS + nw);
            const float4 h4 = hs[t * kBwdLanes + lane];
            const float2 B2[2] = {make_float2(b4.x, b4.y), make_float2(b4.z, b4.w)};
            const float2 C2[2] = {make_float2(c4.x, c4.y), make_float2(c4.z, c4.w)};
            const float2 H2[2] = {make_float2(h4.x, h4.y), make_float2(h4.z, h4.w)};
            float2 vb[2];
            float2 s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                g[j] = __ffma2_rn(gy2, C2[j], g[j]);
                const float2 hp = __ffma2_rn(ndtu2, B2[j], H2[j]);   // a_t h_{t-1}
                vb[j] = __fmul2_rn(g[j], dtu2);
                s2 = __ffma2_rn(g[j], B2[j], s2);
                s1 = __ffma2_rn(__fmul2_rn(g[j], A2[j]), hp, s1);
                dA[j] = __ffma2_rn(__fmul2_rn(g[j], dt2), hp, dA[j]);
                g[j] = __fmul2_rn(g[j], ex2_pair(__fmul2_rn(dt2, A2[j])));
            }
            // g dt u of the 4 states, in the place of h_t (read above)
            hs[t * kBwdLanes + lane] = make_float4(vb[0].x, vb[0].y, vb[1].x, vb[1].y);
            sums[(w * kT + t) * kBwdLanes + lane] = make_float2(s1.x + s1.y, s2.x + s2.y);
        }
        // dB of the warp's 4 states at every step: lane (t, pair) sums g dt u
        // over the 32 channels
        __syncwarp();
        lane_sums(hs, sdy, red, lane, 0, false);
        __syncthreads();   // every warp's (s1, s2) of the chunk
        // warp w finishes steps 4w .. 4w+3 of its lanes' channels
        float ddv[4], duv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * w + i;
            float S1 = 0.f, S2 = 0.f;
#pragma unroll
            for (int ww = 0; ww < kQuadWarps; ++ww) {
                const float2 e = sums[(ww * kT + t) * kBwdLanes + lane];
                S1 += e.x;
                S2 += e.y;
            }
            const float4 v4 = st4[t * kBwdLanes + lane];
            ddv[i] = fmaf(kLn2, S1, v4.y * S2) * v4.w;
            duv[i] = fmaf(Dk, v4.z, v4.x * S2);
            if (q.active && t < nt) {
                dD = fmaf(v4.z, v4.y, dD);
                db += ddv[i];
            }
        }
        if (q.active) {
            const int l0 = s + 4 * w;
            if (vec_rows && 4 * w + 4 <= nt) {
                float4 *dd4 = reinterpret_cast<float4 *>(ddrow + l0);
                float4 *du4 = reinterpret_cast<float4 *>(durow + (flip ? L - 4 - l0 : l0));
                float4 a = make_float4(ddv[0], ddv[1], ddv[2], ddv[3]);
                float4 b = flip ? make_float4(duv[3], duv[2], duv[1], duv[0])
                                : make_float4(duv[0], duv[1], duv[2], duv[3]);
                if (accum) {
                    const float4 ea = *dd4;
                    a = make_float4(ea.x + a.x, ea.y + a.y, ea.z + a.z, ea.w + a.w);
                }
                *dd4 = a;
                if (xmerge) {
                    atomicAdd(du4, b);
                } else {
                    if (accum) {
                        const float4 eb = *du4;
                        b = make_float4(eb.x + b.x, eb.y + b.y, eb.z + b.z, eb.w + b.w);
                    }
                    *du4 = b;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = 4 * w + i;
                    if (t < nt) {
                        const int l = s + t;
                        float *o = durow + (flip ? L - 1 - l : l);
                        ddrow[l] = accum ? ddrow[l] + ddv[i] : ddv[i];
                        if (xmerge)
                            atomicAdd(o, duv[i]);
                        else
                            *o = accum ? *o + duv[i] : duv[i];
                    }
                }
            }
        }
        // the warp's reduced dB | dC rows of the chunk (lanes 0..7: one row each)
        __syncwarp();
        if (bc_ok) {
            if (vec_rows && nt == kT) {
                float4 *r4 = reinterpret_cast<float4 *>(bcrow + s);
#pragma unroll
                for (int i = 0; i < kT / 4; ++i)
                    r4[i] = make_float4(red[(4 * i) * 8 + rj], red[(4 * i + 1) * 8 + rj],
                                        red[(4 * i + 2) * 8 + rj], red[(4 * i + 3) * 8 + rj]);
            } else {
                for (int t = 0; t < nt; ++t)
                    bcrow[s + t] = red[t * 8 + rj];
            }
        }
    }
    // parameter partials: this warp's dA; dDskip and dbias summed over the warps
    __syncthreads();
    float2 *acc = sums;   // reused: [warp][lane]
    acc[w * kBwdLanes + lane] = make_float2(dD, db);
    __syncthreads();
    if (q.active) {
        float *pr = p.prm_part + (q.bkd * p.CGN + blockIdx.y) * (p.NS + 2);
        const float dav[4] = {dA[0].x, dA[0].y, dA[1].x, dA[1].y};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (nw + i < p.N)
                pr[p.n0 + nw + i] = dav[i];
        if (w == 0) {
            float sD = 0.f, sb = 0.f;
#pragma unroll
            for (int ww = 0; ww < kQuadWarps; ++ww) {
                const float2 e = acc[ww * kBwdLanes + lane];
                sD += e.x;
                sb += e.y;
            }
            if (!accum) {
                pr[p.NS] = sD;
                pr[p.NS + 1] = sb;
            } else {
                pr[p.NS + 1] += sb;
            }
        }
    }
}

// dBs, dCs (B,K,N,L) = the sum over the channel groups, in group order (the
// partial holds N rows per (b, k, group, B|C)).  One CTA per output row
// r = (b * K + k) * 2N + which * N + n; vec: 16-byte pieces (L % 4 = 0).
constexpr int kReduceBcThreads = 256;
__global__ void __launch_bounds__(kReduceBcThreads)
    bwd_reduce_bc_kernel(const float *__restrict__ part, float *__restrict__ dBs,
                         float *__restrict__ dCs, int G, int N, int L, int vec)
{
    const unsigned r = blockIdx.x;
    const int n = (int)(r % (unsigned)N);
    const unsigned q = r / (unsigned)N;
    const int which = (int)(q & 1u);
    const size_t bk = q >> 1;
    const float *src = part + ((bk * G * 2 + which) * N + n) * (size_t)L;
    const size_t gstride = (size_t)2 * N * L;
    float *dst = (which ? dCs : dBs) + (bk * N + n) * (size_t)L;
    if (vec) {
        const int n4 = L / 4;
        for (int i = threadIdx.x; i < n4; i += kReduceBcThreads) {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int g = 0; g < G; ++g) {
                const float4 v = __ldg(reinterpret_cast<const float4 *>(src + g * gstride) + i);
                a = make_float4(a.x + v.x, a.y + v.y, a.z + v.z, a.w + v.w);
            }
            reinterpret_cast<float4 *>(dst)[i] = a;
        }
    } else {
        for (int l = threadIdx.x; l < L; l += kReduceBcThreads) {
            float a = 0.f;
            for (int g = 0; g < G; ++g)
                a += __ldg(src + g * gstride + l);
            dst[l] = a;
        }
    }
}

// dA_log = A * sum dA, dDskip, ddelta_bias: per (k, d, j) one warp; lane t
// sums b = t, t + 32, ... (each over the chunk groups in order), then the
// lanes' sums meet in a fixed butterfly, so every call adds in the same order
constexpr int kReduceParamThreads = 128;
__global__ void __launch_bounds__(kReduceParamThreads)
    bwd_reduce_param_kernel(const float *__restrict__ prm, const float *__restrict__ A_log,
                            float *__restrict__ dA_log, float *__restrict__ dDskip,
                            float *__restrict__ dbias, int B, int K, int D, int N, int CGN)
{
    const long long total = (long long)K * D * (N + 2);
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (kReduceParamThreads / 32);
    for (long long i = (long long)blockIdx.x * (kReduceParamThreads / 32) + (threadIdx.x >> 5);
         i < total; i += warps) {
        const int j = (int)(i % (N + 2));
        const long long kd = i / (N + 2);
        const int k = (int)(kd / D), d = (int)(kd % D);
        float s = 0.f;
        for (int b = lane; b < B; b += 32) {
            const float *src = prm + ((((size_t)b * K + k) * D + d) * CGN) * (N + 2) + j;
            float t = 0.f;
            for (int cg = 0; cg < CGN; ++cg)
                t += __ldg(src + (size_t)cg * (N + 2));
            s += t;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) {
            if (j < N)
                dA_log[kd * N + j] = s * -expf(__ldg(A_log + kd * N + j));
            else if (j == N)
                dDskip[kd] = s;
            else
                dbias[kd] = s;
        }
    }
}

}  // namespace ss2d
