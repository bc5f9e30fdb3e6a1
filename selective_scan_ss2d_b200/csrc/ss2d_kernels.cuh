// ss2d_kernels.cuh -- sm_100a kernels of the SS2D forward path.
//
// One launch of scan_fwd_kernel runs the selective scan of a tile of DC
// channels of one (batch b, direction k) over the whole sequence, with the
// cross_scan folded into its address generation and its output written in
// pixel order.  merge_kernel then adds the K per-direction outputs in the
// fixed order k = 0, 1, 2, 3 (cross_merge).
//
// Recurrence ("Vision Mamba" tutorial, SelectiveSSM; "Vision Mamba ..."
// summary, section 4.1), per channel and state n:
//     dt_l  = softplus(delta_l + bias)
//     h_l   = exp(dt_l * A_n) * h_{l-1} + dt_l * B_{n,l} * u_l
//     y_l   = sum_n C_{n,l} h_l + Dskip * u_l
// exp(dt*A) is evaluated as 2^(dt * A*log2(e)) on the MUFU unit.
//
// Work layout.  A CTA owns DC channels of one (b, k) and walks the sequence
// in chunks of LC = NS * I steps.  Per chunk it stages in shared memory:
//   * the B and C columns of the chunk, shared by all DC channels, as float32
//     rows of 16 states (zero padded past N);
//   * per channel: dt (softplus applied once per (channel, step)), dt*u and
//     u, gathered through the direction's scan->pixel map.
// Inside a warp, lanes are (channel cw, time segment jw, state group g):
// each lane owns S = 16/G states of one channel.  The C.h reduction over the
// G lanes of a channel is done for four steps at a time with a transposing
// butterfly (G-1 shuffles per four steps).
//
// Long sequences with few channels are split in time: a chunk is cut into
// NS = J*JW segments of I steps (JW inside a warp, J across warps).  Each
// lane first runs its segment from a zero state, keeping every exp(dt*A) in
// registers and accumulating the segment's transfer pair (P, Q) with
// h_out = P*h_in + Q.  The pairs are combined with the associative operator
// (P1,Q1) then (P2,Q2) = (P2*P1, P2*Q1 + Q2) -- shuffles inside a warp,
// shared memory across warps, plus the carry from the previous chunk -- and
// each lane replays its segment from its true entry state using the kept
// exponentials, so no exponential is evaluated twice.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ss2d {

constexpr int kNP = 16;  // states per channel held by the kernels (N <= 16)
constexpr float kLog2e = 1.4426950408889634f;

struct ScanParams {
    const void *x;           // (B,D,H,W) / (B,D,L)
    const void *delta;       // (B,K,D,L) scan order
    const float *A_log;      // (K*D,N)
    const void *Bs;          // (B,K,N,L) scan order
    const void *Cs;          // (B,K,N,L) scan order
    const float *Dskip;      // (K*D)
    const float *delta_bias; // (K*D)
    float *out;              // partials (B,K,D,L) or y (B,D,L), pixel order
    int B, D, H, W, L, N, K;
    int two_d;               // 1: SS2D scan orders; 0: 1D (k=1 reversed)
    long long out_b_stride;  // elements between batches in `out`
    long long out_k_stride;  // elements between directions in `out`
};

__device__ __forceinline__ float load_in(const float *p) { return __ldg(p); }
__device__ __forceinline__ float load_in(const __nv_bfloat16 *p)
{
    return __bfloat162float(__ldg(p));
}

// Pixel visited at scan step l of direction k (see include/ss2d.h).
__device__ __forceinline__ int scan_pixel(int two_d, int k, int l, int H, int W,
                                          int L)
{
    if (k & 1)
        l = L - 1 - l;
    if (two_d && k >= 2) {
        const int h = l % H;
        const int w = l / H;
        return h * W + w;
    }
    return l;
}

// 2^x on the multi-function unit (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float mufu_ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(z) = log(1 + e^z); above 20 the correction e^-z is below float32
// resolution of z and z itself is returned.
__device__ __forceinline__ float softplus_f(float z)
{
    return z > 20.f ? z : log1pf(__expf(z));
}

__device__ __forceinline__ float f4(const float4 &v, int i)
{
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// Reduce yp[0..3] (partial sums of four consecutive steps) over the G lanes
// of a channel and write y = sum + Dskip*u for those steps.  After the
// butterfly, lane g of the group holds whole sums for 4/G of the steps.
template <int G>
__device__ __forceinline__ void reduce_store(float (&yp)[4], float *ydst,
                                             const float *usrc, float dsk,
                                             int g)
{
    if constexpr (G == 1) {
        const float4 u4 = *reinterpret_cast<const float4 *>(usrc);
        float4 o;
        o.x = fmaf(dsk, u4.x, yp[0]);
        o.y = fmaf(dsk, u4.y, yp[1]);
        o.z = fmaf(dsk, u4.z, yp[2]);
        o.w = fmaf(dsk, u4.w, yp[3]);
        *reinterpret_cast<float4 *>(ydst) = o;
    } else if constexpr (G == 2) {
        const bool hi = g & 1;
        const float s0 = hi ? yp[0] : yp[2];
        const float s1 = hi ? yp[1] : yp[3];
        float k0 = hi ? yp[2] : yp[0];
        float k1 = hi ? yp[3] : yp[1];
        k0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        k1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        const int t = 2 * (g & 1);
        ydst[t] = fmaf(dsk, usrc[t], k0);
        ydst[t + 1] = fmaf(dsk, usrc[t + 1], k1);
    } else {
        static_assert(G == 4, "state groups of 1, 2 or 4 lanes");
        const bool b1 = (g >> 1) & 1;
        const float s0 = b1 ? yp[0] : yp[2];
        const float s1 = b1 ? yp[1] : yp[3];
        float k0 = b1 ? yp[2] : yp[0];
        float k1 = b1 ? yp[3] : yp[1];
        k0 += __shfl_xor_sync(0xffffffffu, s0, 2);
        k1 += __shfl_xor_sync(0xffffffffu, s1, 2);
        const bool b0 = g & 1;
        const float s = b0 ? k0 : k1;
        float v = b0 ? k1 : k0;
        v += __shfl_xor_sync(0xffffffffu, s, 1);
        ydst[g] = fmaf(dsk, usrc[g], v);
    }
}

template <int G, int JW, int J, int WC, int I>
struct ScanShape {
    static constexpr int S = kNP / G;          // states per lane
    static constexpr int CW = 32 / (G * JW);   // channels per warp
    static constexpr int DC = WC * CW;         // channels per CTA
    static constexpr int NT = 32 * WC * J;     // threads per CTA
    static constexpr int NS = J * JW;          // time segments per chunk
    static constexpr int LC = NS * I;          // steps per chunk
    static constexpr int SEG = I + 4;          // padded segment, channel rows
    static constexpr int RS0 = NS * SEG;
    // channel row stride: an odd number of 16-byte units, so float4 reads of
    // consecutive channels fall in distinct bank groups
    static constexpr int RS = RS0 + (((RS0 / 4) % 2 == 0) ? 4 : 8);
    static constexpr int BSEG = I * kNP + 4;   // padded segment, B/C tiles
    static constexpr bool SPLIT = NS > 1;
    static constexpr int TILE_FLOATS = NS * BSEG;       // one of sB, sC
    static constexpr int ROW_FLOATS = DC * RS;          // one of sDt..sY
    static constexpr int TOT_FLOATS = (SPLIT && J > 1) ? J * DC * kNP * 2 : 0;
    static constexpr int CAR_FLOATS = (SPLIT && J > 1) ? 2 * DC * kNP : 0;
    static constexpr int SMEM_FLOATS =
        2 * TILE_FLOATS + 4 * ROW_FLOATS + TOT_FLOATS + CAR_FLOATS;
    static constexpr size_t SMEM_BYTES = sizeof(float) * SMEM_FLOATS;
    static_assert(I % 4 == 0, "segments hold whole groups of four steps");
    static_assert(G == 1 || G == 2 || G == 4, "state groups of 1, 2 or 4 lanes");
    static_assert(32 % (G * JW) == 0 && CW >= 1, "lanes split evenly");
};

template <typename Tin, int G, int JW, int J, int WC, int I, int MINB>
__global__ void __launch_bounds__(32 * WC * J, MINB)
    scan_fwd_kernel(const ScanParams p)
{
    using Sh = ScanShape<G, JW, J, WC, I>;
    constexpr int S = Sh::S, CW = Sh::CW, DC = Sh::DC, NT = Sh::NT;
    constexpr int LC = Sh::LC, SEG = Sh::SEG, RS = Sh::RS, BSEG = Sh::BSEG;
    constexpr bool SPLIT = Sh::SPLIT;

    extern __shared__ float4 smem_f4[];
    float *sB = reinterpret_cast<float *>(smem_f4);
    float *sC = sB + Sh::TILE_FLOATS;
    float *sDt = sC + Sh::TILE_FLOATS;
    float *sDu = sDt + Sh::ROW_FLOATS;
    float *sU = sDu + Sh::ROW_FLOATS;
    float *sY = sU + Sh::ROW_FLOATS;
    float *sTot = sY + Sh::ROW_FLOATS;   // [J][DC][kNP][2]
    float *sCar = sTot + Sh::TOT_FLOATS; // [2][DC][kNP]

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int wc = warp % WC, j = warp / WC;
    const int g = lane % G;
    const int jw = (lane / G) % JW;
    const int cw = lane / (G * JW);
    const int c = wc * CW + cw;
    const int js = j * JW + jw;

    const int D = p.D, L = p.L, N = p.N, H = p.H, W = p.W;
    const int d0 = blockIdx.x * DC;
    const int k = blockIdx.y, b = blockIdx.z;
    const int d = d0 + c;
    const bool cvalid = d < D;
    const int kd = k * D + (cvalid ? d : 0);

    float A2[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const int n = g * S + s;
        A2[s] = (cvalid && n < N) ? -expf(__ldg(p.A_log + (size_t)kd * N + n)) * kLog2e
                                  : 0.f;
    }
    const float dsk = cvalid ? __ldg(p.Dskip + kd) : 0.f;

    const Tin *xg = static_cast<const Tin *>(p.x) + (size_t)b * D * L;
    const Tin *dg = static_cast<const Tin *>(p.delta) + ((size_t)b * p.K + k) * D * L;
    const Tin *Bg = static_cast<const Tin *>(p.Bs) + ((size_t)b * p.K + k) * N * L;
    const Tin *Cg = static_cast<const Tin *>(p.Cs) + ((size_t)b * p.K + k) * N * L;
    const float *biasg = p.delta_bias + (size_t)k * D;
    float *og = p.out + (size_t)b * p.out_b_stride + (size_t)k * p.out_k_stride;

    float h[S];      // state entering the current step (direct path)
    float hcar[S];   // state entering the current chunk (split path, J == 1)
#pragma unroll
    for (int s = 0; s < S; ++s) {
        h[s] = 0.f;
        hcar[s] = 0.f;
    }
    if constexpr (SPLIT && J > 1) {
        for (int e = tid; e < Sh::CAR_FLOATS; e += NT)
            sCar[e] = 0.f;
    }

    int chunk = 0;
    for (int l0 = 0; l0 < L; l0 += LC, ++chunk) {
        // ---------------- stage the chunk ----------------
        for (int e = tid; e < LC * (kNP / 4); e += NT) {
            const int nb = e & 3;
            const int t = e >> 2;
            const int l = l0 + t;
            float vb[4], vc[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int n = nb * 4 + q;
                const bool ok = (l < L) && (n < N);
                vb[q] = ok ? load_in(Bg + (size_t)n * L + l) : 0.f;
                vc[q] = ok ? load_in(Cg + (size_t)n * L + l) : 0.f;
            }
            const int off = (t / I) * BSEG + (t % I) * kNP + nb * 4;
            *reinterpret_cast<float4 *>(sB + off) = make_float4(vb[0], vb[1], vb[2], vb[3]);
            *reinterpret_cast<float4 *>(sC + off) = make_float4(vc[0], vc[1], vc[2], vc[3]);
        }
        for (int e = tid; e < DC * LC; e += NT) {
            const int t = e % LC;
            const int cc = e / LC;
            const int l = l0 + t;
            const int dd = d0 + cc;
            float dt = 0.f, du = 0.f, u = 0.f;
            if (l < L && dd < D) {
                const int pix = scan_pixel(p.two_d, k, l, H, W, L);
                u = load_in(xg + (size_t)dd * L + pix);
                const float z = load_in(dg + (size_t)dd * L + l) + __ldg(biasg + dd);
                dt = softplus_f(z);
                du = dt * u;
            }
            const int si = cc * RS + (t / I) * SEG + (t % I);
            sDt[si] = dt;
            sDu[si] = du;
            sU[si] = u;
        }
        __syncthreads();

        // ---------------- scan the chunk ----------------
        const int rb0 = c * RS + js * SEG;   // this lane's segment, channel rows
        const int bb0 = js * BSEG + g * S;   // this lane's segment, B/C tiles
        if constexpr (!SPLIT) {
#pragma unroll 1
            for (int i0 = 0; i0 < I; i0 += 4) {
                const float4 dt4 = *reinterpret_cast<const float4 *>(sDt + rb0 + i0);
                const float4 du4 = *reinterpret_cast<const float4 *>(sDu + rb0 + i0);
                float yp[4];
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const float dt = f4(dt4, tt), du = f4(du4, tt);
                    const float *rowB = sB + bb0 + (i0 + tt) * kNP;
                    const float *rowC = sC + bb0 + (i0 + tt) * kNP;
                    float acc = 0.f;
#pragma unroll
                    for (int s4 = 0; s4 < S; s4 += 4) {
                        const float4 bv = *reinterpret_cast<const float4 *>(rowB + s4);
                        const float4 cv = *reinterpret_cast<const float4 *>(rowC + s4);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int s = s4 + q;
                            const float a = mufu_ex2(dt * A2[s]);
                            h[s] = fmaf(a, h[s], du * f4(bv, q));
                            acc = fmaf(f4(cv, q), h[s], acc);
                        }
                    }
                    yp[tt] = acc;
                }
                reduce_store<G>(yp, sY + rb0 + i0, sU + rb0 + i0, dsk, g);
            }
        } else {
            // pass 1: run the segment from a zero state, keep exp(dt*A)
            float av[I][S];
            float P[S], Q[S];
#pragma unroll
            for (int s = 0; s < S; ++s) {
                P[s] = 1.f;
                Q[s] = 0.f;
            }
#pragma unroll
            for (int i0 = 0; i0 < I; i0 += 4) {
                const float4 dt4 = *reinterpret_cast<const float4 *>(sDt + rb0 + i0);
                const float4 du4 = *reinterpret_cast<const float4 *>(sDu + rb0 + i0);
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const float dt = f4(dt4, tt), du = f4(du4, tt);
                    const float *rowB = sB + bb0 + (i0 + tt) * kNP;
#pragma unroll
                    for (int s4 = 0; s4 < S; s4 += 4) {
                        const float4 bv = *reinterpret_cast<const float4 *>(rowB + s4);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int s = s4 + q;
                            const float a = mufu_ex2(dt * A2[s]);
                            av[i0 + tt][s] = a;
                            Q[s] = fmaf(a, Q[s], du * f4(bv, q));
                            P[s] *= a;
                        }
                    }
                }
            }
            // combine the segments' transfer pairs inside the warp
#pragma unroll
            for (int r = 1; r < JW; r <<= 1) {
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const float Pp = __shfl_up_sync(0xffffffffu, P[s], r * G);
                    const float Qp = __shfl_up_sync(0xffffffffu, Q[s], r * G);
                    if (jw >= r) {
                        Q[s] = fmaf(P[s], Qp, Q[s]);
                        P[s] *= Pp;
                    }
                }
            }
            float Pex[S], Qex[S];   // segments before mine, inside the warp
#pragma unroll
            for (int s = 0; s < S; ++s) {
                const float Pp = __shfl_up_sync(0xffffffffu, P[s], G);
                const float Qp = __shfl_up_sync(0xffffffffu, Q[s], G);
                Pex[s] = (jw == 0) ? 1.f : Pp;
                Qex[s] = (jw == 0) ? 0.f : Qp;
            }
            float hw[S];   // state entering this warp's first segment
            if constexpr (J == 1) {
                const int last = (cw * JW + JW - 1) * G + g;
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    hw[s] = hcar[s];
                    const float Pt = __shfl_sync(0xffffffffu, P[s], last);
                    const float Qt = __shfl_sync(0xffffffffu, Q[s], last);
                    hcar[s] = fmaf(Pt, hcar[s], Qt);
                }
            } else {
                if (jw == JW - 1) {
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        float *dst = sTot + ((j * DC + c) * kNP + g * S + s) * 2;
                        dst[0] = P[s];
                        dst[1] = Q[s];
                    }
                }
                __syncthreads();
                const float *car = sCar + (chunk & 1) * DC * kNP + c * kNP + g * S;
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    float hc = car[s];
                    for (int jj = 0; jj < j; ++jj) {
                        const float *tot = sTot + ((jj * DC + c) * kNP + g * S + s) * 2;
                        hc = fmaf(tot[0], hc, tot[1]);
                    }
                    hw[s] = hc;
                }
                if (j == J - 1 && jw == JW - 1) {
                    float *ncar = sCar + ((chunk + 1) & 1) * DC * kNP + c * kNP + g * S;
#pragma unroll
                    for (int s = 0; s < S; ++s)
                        ncar[s] = fmaf(P[s], hw[s], Q[s]);
                }
            }
            // pass 2: replay the segment from its entry state
#pragma unroll
            for (int s = 0; s < S; ++s)
                h[s] = fmaf(Pex[s], hw[s], Qex[s]);
#pragma unroll
            for (int i0 = 0; i0 < I; i0 += 4) {
                const float4 du4 = *reinterpret_cast<const float4 *>(sDu + rb0 + i0);
                float yp[4];
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const float du = f4(du4, tt);
                    const float *rowB = sB + bb0 + (i0 + tt) * kNP;
                    const float *rowC = sC + bb0 + (i0 + tt) * kNP;
                    float acc = 0.f;
#pragma unroll
                    for (int s4 = 0; s4 < S; s4 += 4) {
                        const float4 bv = *reinterpret_cast<const float4 *>(rowB + s4);
                        const float4 cv = *reinterpret_cast<const float4 *>(rowC + s4);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int s = s4 + q;
                            h[s] = fmaf(av[i0 + tt][s], h[s], du * f4(bv, q));
                            acc = fmaf(f4(cv, q), h[s], acc);
                        }
                    }
                    yp[tt] = acc;
                }
                reduce_store<G>(yp, sY + rb0 + i0, sU + rb0 + i0, dsk, g);
            }
        }
        __syncthreads();

        // ---------------- write the chunk's outputs in pixel order -------
        for (int e = tid; e < DC * LC; e += NT) {
            const int t = e % LC;
            const int cc = e / LC;
            const int l = l0 + t;
            const int dd = d0 + cc;
            if (l < L && dd < D) {
                const int pix = scan_pixel(p.two_d, k, l, H, W, L);
                og[(size_t)dd * L + pix] = sY[cc * RS + (t / I) * SEG + (t % I)];
            }
        }
    }
}

// y[b, r] = ((part[b,0,r] + part[b,1,r]) + part[b,2,r]) + part[b,3,r]
// for r over the D*L outputs of batch b; K = 2 stops after the first add.
template <int K>
__global__ void merge_kernel(const float *__restrict__ part, float *__restrict__ y,
                             long long DL, long long total)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    if ((DL & 3) == 0) {
        const long long total4 = total >> 2;
        for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total4;
             i += stride) {
            const long long e = i << 2;
            const long long bb = e / DL, r = e - bb * DL;
            const float *src = part + bb * K * DL + r;
            float4 acc = __ldg(reinterpret_cast<const float4 *>(src));
#pragma unroll
            for (int kk = 1; kk < K; ++kk) {
                const float4 v = __ldg(reinterpret_cast<const float4 *>(src + kk * DL));
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            }
            *reinterpret_cast<float4 *>(y + e) = acc;
        }
    } else {
        for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
             e += stride) {
            const long long bb = e / DL, r = e - bb * DL;
            const float *src = part + bb * K * DL + r;
            float acc = __ldg(src);
#pragma unroll
            for (int kk = 1; kk < K; ++kk)
                acc += __ldg(src + kk * DL);
            y[e] = acc;
        }
    }
}

}  // namespace ss2d
