// ss2d_scan.cuh -- the lane scan kernel with asynchronous staging, and the
// associative scan of the chunk carries.
//
// Recurrence ("Vision Mamba" tutorial, section "Background: State Space
// Models and Mamba", SelectiveSSM; "Vision Mamba ..." summary, section 4.1),
// per direction k, channel d and state n:
//     dt_l = softplus(delta_l + bias)
//     h_l  = exp(dt_l * A_n) * h_{l-1} + dt_l * B_{n,l} * u_l        (h_{-1} = 0)
//     y_l  = sum_n C_{n,l} h_l + Dskip * u_l
// with u_l = x[pixel(k, l)] (cross_scan folded into the addressing).
//
// lane_scan_kernel: one lane owns one (b, k, d) channel with its (up to 16)
// states in registers; a CTA holds 32*WC channels of one (b, k) and one
// chunk of the sequence.  Its inputs reach shared memory through cp.async
// (global -> shared copies that bypass the registers), one 16-step sub-chunk
// ahead of the arithmetic, so that no instruction of the step loop waits on
// global memory:
//   * each lane copies its own delta row segment and its own x values: as
//     packed 16- or 8-byte pieces of the row (rows whose start is aligned),
//     or as one 4-byte word per step (the column-major directions, whose
//     pixels are W apart, and rows that are only 2-byte aligned); the fused
//     front's bf16 u comes as 16-byte rows of its x_proj operand blocks;
//   * B and C of the sub-chunk (shared by every channel of the CTA) are
//     copied by the whole CTA two sub-chunks ahead, converted once to a
//     float32 [slot][step] tile one sub-chunk ahead, and read with broadcast
//     float4 loads.
// One barrier per sub-chunk orders the shared tiles; nothing spins.  Steps
// past the end of the sequence get delta = -inf in shared memory, so that
// dt = softplus(-inf) = 0 exactly and the step leaves the state unchanged.
//
// carry_scan_kernel: the state entering every chunk from the chunks' local
// end states.  Chunk c maps the state before it to a_c * h + e_c, with
// a_c = exp(A * sum(dt over c)) and e_c its end state from zero; maps compose
// as (a1, e1) then (a2, e2) = (a1 a2, a2 e1 + e2), an associative operator,
// so the entry states are an exclusive scan over the chunks: a serial run
// over each lane's segment of chunks, a Kogge-Stone scan across the lanes of
// a warp (shuffles) and across the warps of the CTA (shared memory), then a
// second run over the segment that writes the results.
#pragma once

#include "ss2d_kernels.cuh"

namespace ss2d {

// ---- cp.async: asynchronous copies global -> shared (sm_80 and later) ----
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// 4-byte word copy of the element at src (2-byte types: the aligned word that
// holds it); returns the element's half (0 low, 1 high) shifted to bit `bit`.
template <typename Tin>
__device__ __forceinline__ uint32_t cp_async_word(uint32_t dst, const Tin *src, int bit)
{
    const uintptr_t a = reinterpret_cast<uintptr_t>(src);
    if constexpr (sizeof(Tin) == 2) {
        cp_async4(dst, reinterpret_cast<const void *>(a & ~(uintptr_t)3));
        return (uint32_t)((a >> 1) & 1) << bit;
    } else {
        cp_async4(dst, src);
        return 0u;
    }
}

// float value of a staged raw value: `w` holds it (4-byte types) or holds it
// in its low (hi = 0) or high (hi = 1) half
template <typename Tin>
__device__ __forceinline__ float raw_value(uint32_t w, uint32_t hi)
{
    if constexpr (sizeof(Tin) == 4) {
        return __uint_as_float(w);
    } else if constexpr (std::is_same_v<Tin, __nv_bfloat16>) {
        return __uint_as_float(hi ? (w & 0xffff0000u) : (w << 16));
    } else {
        return __half2float(__ushort_as_half((unsigned short)(hi ? (w >> 16) : (w & 0xffffu))));
    }
}

__device__ __forceinline__ uint32_t u4c(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// raw bits of -inf in a staged delta slot (a whole word: both halves of a
// 2-byte word, so that either half reads -inf)
template <typename Tin>
__device__ __forceinline__ uint32_t neg_inf_word()
{
    if constexpr (sizeof(Tin) == 4)
        return 0xff800000u;
    else if constexpr (std::is_same_v<Tin, __nv_bfloat16>)
        return 0xff80ff80u;
    else
        return 0xfc00fc00u;
}

// Shared-memory plan of lane_scan_kernel (bytes; every offset a multiple of 16).
// FRONT: the fused front's inputs -- no delta rows (a dt_raw row of the
// direction is staged with B and C instead), float32 B and C.
// CPL: channels per lane.
template <typename Tin, int WC, bool COLS, bool ALIGNED, bool FRONT = false, int CPL = 1>
struct LaneShape {
    static constexpr int NT = 32 * WC;                  // threads per CTA
    static constexpr int CH = CPL * NT;                 // channels per CTA
    static constexpr int ESZ = (int)sizeof(Tin);
    static constexpr int EBC = FRONT ? 4 : ESZ;         // bytes of a B|C value
    // delta of 2-byte types from aligned rows: 16 values packed in 2 units of
    // 16 bytes; otherwise one word per step (4 units)
    static constexpr bool DPACK2 = ALIGNED && ESZ == 2;
    static constexpr int UD = FRONT ? 0 : (DPACK2 ? 2 : 4);   // units per channel and stage
    static constexpr int UX = (DPACK2 && !COLS) ? 2 : 4;
    static constexpr int RW = ALIGNED ? 4 * EBC : 16;   // words of a raw B|C row segment
    static constexpr int RS = RW;                       // their row stride
    static constexpr int BCS = 3;                       // raw B|C stages
    static constexpr int BCR = FRONT ? 33 : 32;         // raw rows: B, C (and dt_raw)
    static constexpr size_t OFF_X = sizeof(uint4) * 2 * CPL * UD * NT;
    static constexpr size_t OFF_BC = OFF_X + sizeof(uint4) * 2 * CPL * UX * NT;
    static constexpr size_t OFF_BCF = OFF_BC + sizeof(uint32_t) * BCS * BCR * RS;
    static constexpr size_t OFF_DT = OFF_BCF + sizeof(float4) * 2 * 8 * kT;
    static constexpr size_t OFF_DU = OFF_DT + (FRONT ? sizeof(float) * 2 * kT : 0);
    // per warp [kT][CPL][32] (dt, u) of the sub-chunk being computed; dt is
    // overwritten by the step's output
    static constexpr size_t SMEM_BYTES = OFF_DU + sizeof(float2) * WC * kT * CPL * 32;
};

// One chunk of LC steps of CPL*32*WC channels of one (b, k); see the header.
// grid: x = ((b * NCg + chunk) * K + k) * tiles + tile, NCg = chunks
// launched (NC - 1 in kModeState, NC in kModeOutput).
// COLS: the column-major directions (SS2D with K = 4) are compiled in.
// QN: groups of 4 states per channel (4: up to 16 states; 2: up to 8).
// ALIGNED: delta, x and B|C rows start on 8-byte boundaries (p.vec = 8 or
// 16): packed row copies; otherwise one word per step.
// FRONT: the inputs of the fused front (p.front): u of every direction in
// its scan order (B,K,D,LP) rows, or (p.utile) the x_proj A blocks, delta =
// w_dt * dt_raw, float32 B|C.
// CPL: channels per lane (channel c of thread t: tile * CPL*NT + c*NT + t);
// the B|C values of a step, read from shared memory once, serve all of them.
template <typename Tin, int WC, int MODE, int MINB, bool COLS, int QN, bool ALIGNED,
          bool FRONT = false, int CPL = 1>
__global__ void __launch_bounds__(32 * WC, MINB) lane_scan_kernel(const ScanParams p)
{
    static_assert(QN == 2 || QN == 4, "8 or 16 states per channel");
    static_assert(kT == 16, "16-step sub-chunks");
    static_assert(CPL == 1 || CPL == 2, "one or two channels per lane");
    static_assert(!FRONT || (ALIGNED && !COLS), "front inputs: aligned 1D rows");
    using Sh = LaneShape<Tin, WC, COLS, ALIGNED, FRONT, CPL>;
    using Tbc = std::conditional_t<FRONT, float, Tin>;   // type of the B|C rows
    constexpr int NT = Sh::NT, CH = Sh::CH, UD = Sh::UD, UX = Sh::UX, ESZ = Sh::ESZ;
    constexpr int RS = Sh::RS, EBC = Sh::EBC, BCR = Sh::BCR;
    constexpr bool DPACK2 = Sh::DPACK2;

    extern __shared__ __align__(16) unsigned char lane_smem[];
    uint4 *rawD = reinterpret_cast<uint4 *>(lane_smem);                   // [2][CPL][UD][NT]
    uint4 *rawX = reinterpret_cast<uint4 *>(lane_smem + Sh::OFF_X);       // [2][CPL][UX][NT]
    uint32_t *rawBC = reinterpret_cast<uint32_t *>(lane_smem + Sh::OFF_BC);   // [3][BCR][RS]
    float4 *BCf = reinterpret_cast<float4 *>(lane_smem + Sh::OFF_BCF);    // [2][8][kT]
    float *sDT = reinterpret_cast<float *>(lane_smem + Sh::OFF_DT);       // FRONT: [2][kT] dt_raw
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    // this lane's (dt, u) of step t, channel c at sDU[(t * CPL + c) * 32]
    float2 *sDU = reinterpret_cast<float2 *>(lane_smem + Sh::OFF_DU) + warp * (kT * CPL * 32) + lane;

    const int D = p.D, L = p.L, N = p.N, H = p.H, W = p.W, K = p.K;
    const int ncg = (MODE == kModeState) ? p.NC - 1 : p.NC;
    const int ntiles = (D + CH - 1) / CH;
    int rest = blockIdx.x;
    const int tile = rest % ntiles;
    rest /= ntiles;
    const int k = rest % K;
    rest /= K;
    const int chunk = rest % ncg;
    const int b = rest / ncg;
    const int l_begin = chunk * p.LC;
    const int l_end = min(l_begin + p.LC, L);
    const int nsub = (l_end - l_begin + kT - 1) / kT;
    const bool accum = p.accum != 0;   // a later state group: add to out, no skip term
    const bool ymode = MODE == kModeOutput && p.ymerge != nullptr;   // both directions add into y
    const size_t row_bk = ((size_t)b * K + k) * D;   // row index of (b, k, d = 0)
    const size_t LP = (size_t)p.LP;                  // row pitch of the input rows

    // the lane's channels
    int dch[CPL];           // channel
    bool cvalid[CPL];
    float2 A2[CPL][8];      // A[n] * log2(e) for states (2j, 2j+1)
    float dsk[CPL], bias[CPL], wdt[CPL];
    const Tin *drow[CPL], *xrow[CPL];
    size_t utb[CPL];        // p.utile: byte offset of the channel's rows in the A blocks
    float2 h2[CPL][8];
    float dtsum[CPL];
    const int ublk = (D + 63) / 64, utiles = (L + 127) / 128;   // A blocks: channel blocks, tiles
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        dch[c] = tile * CH + c * NT + tid;
        cvalid[c] = dch[c] < D;
        const int dc = cvalid[c] ? dch[c] : D - 1;   // clamped channel for addressing
        const int kd = k * D + dc;
        const float *al = p.A_log + (size_t)kd * p.NS + p.n0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            A2[c][j].x = (2 * j < N) ? -expf(__ldg(al + 2 * j)) * kLog2e : 0.f;
            A2[c][j].y = (2 * j + 1 < N) ? -expf(__ldg(al + 2 * j + 1)) * kLog2e : 0.f;
            h2[c][j] = make_float2(0.f, 0.f);
        }
        dsk[c] = accum ? 0.f : __ldg(p.Dskip + kd);
        bias[c] = __ldg(p.delta_bias + kd);
        wdt[c] = FRONT ? __ldg(p.w_dt + kd) : 0.f;
        drow[c] = FRONT ? nullptr : static_cast<const Tin *>(p.delta) + (row_bk + dc) * LP;
        // x rows: the caller's (b, d) map, or the front's u row of (b, k, d)
        xrow[c] = static_cast<const Tin *>(p.x) + (FRONT ? (row_bk + dc) : ((size_t)b * D + dc)) * LP;
        // u as the x_proj A blocks: block (b * K + k, tile 0, dc / 64), row dc % 64
        utb[c] = (((size_t)b * K + k) * utiles * ublk + (dc >> 6)) * 16384u + (size_t)(dc & 63) * 16u;
        dtsum[c] = 0.f;
    }
    const size_t bc_row0 = ((size_t)b * K + k) * p.NS + p.n0;   // row of this group's state 0
    const Tbc *Bg = static_cast<const Tbc *>(p.Bs) + bc_row0 * LP;
    const Tbc *Cg = static_cast<const Tbc *>(p.Cs) + bc_row0 * LP;
    const float *dtg = FRONT ? p.dt_raw + ((size_t)b * K + k) * LP : nullptr;
    // x order of this direction: 0 forward, 1 reversed (both contiguous),
    // 2 column-major (one word per step); the front's u rows are in scan order
    const int xmode = FRONT ? 0 : ((COLS && k >= 2) ? 2 : (k & 1));
    const int vec = p.vec;

    // ---- staging ---------------------------------------------------------
    // unit u of channel c, stage s: + ((s*CPL + c)*U + u)*NT*16
    const uint32_t sD0 = smem_u32(rawD) + tid * 16;
    const uint32_t sX0 = smem_u32(rawX) + tid * 16;
    // word halves of the staged values (2-byte types, one word per step):
    // bit i = half of step i, per stage and channel
    uint32_t dpar[2][CPL], xpar[2][CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c)
        dpar[0][c] = dpar[1][c] = xpar[0][c] = xpar[1][c] = 0u;
    PixWalk xw;   // column-major directions: pixel of the next step to copy
    xw.init(p.two_d, k, l_begin, H, W, L);
    const int adv_q = kT / H, adv_r = kT % H;

    // 16 elements e0.. of a row of length L, packed (row start and L * ESZ
    // are multiples of vec): 16-byte units, or pairs of 8-byte pieces.  A
    // piece that would start outside 0..L-1 reads the nearest piece inside
    // (its values belong to steps past the sequence end and are never used).
    auto copy_packed = [&](uint32_t dst, const Tin *row, int e0) {
        constexpr int UE = 16 / ESZ;   // elements per unit
        constexpr int NU = 16 / UE;    // units per 16 elements
        if (vec == 16) {
            const int lastu = ((L - 1) / UE) * UE;
#pragma unroll
            for (int u = 0; u < NU; ++u)
                cp_async16(dst + u * NT * 16, row + max(min(e0 + u * UE, lastu), 0));
        } else {
            constexpr int PE = UE / 2;
            const int lastp = ((L - 1) / PE) * PE;
#pragma unroll
            for (int u = 0; u < 2 * NU; ++u)
                cp_async8(dst + (u >> 1) * NT * 16 + (u & 1) * 8,
                          row + max(min(e0 + u * PE, lastp), 0));
        }
    };
    // the same 16 elements from the A blocks (p.utile, 2-byte u): 8 steps of
    // a channel are one 16-byte row, steps 128 apart are ublk blocks apart;
    // a row past the sequence end reads the last one inside
    auto copy_tile = [&](uint32_t dst, int c, int e0) {
        const unsigned char *base = static_cast<const unsigned char *>(p.x) + utb[c];
        const int lastu = ((L - 1) >> 3) << 3;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = max(min(e0 + u * 8, lastu), 0);
            cp_async16(dst + u * NT * 16,
                       base + ((size_t)(e >> 7) * ublk * 16384u + ((e >> 3) & 15) * 1024u));
        }
    };
    auto set_par = [&](uint32_t (&par)[2][CPL], int s, int c, uint32_t m) {
        if (s)
            par[1][c] = m;
        else
            par[0][c] = m;
    };
    auto issue_dx = [&](int s, int ls) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const uint32_t dD = sD0 + (s * CPL + c) * UD * NT * 16;
            const uint32_t dX = sX0 + (s * CPL + c) * UX * NT * 16;
            (void)dD;
            // delta: steps ls.. of the channel's row
            if constexpr (FRONT) {
                // delta comes from the dt_raw row staged with B and C
            } else if constexpr (ALIGNED) {
                copy_packed(dD, drow[c], ls);   // 4-byte types: one word per step as well
            } else {
                uint32_t m = 0;
#pragma unroll
                for (int i = 0; i < kT; ++i)
                    m |= cp_async_word(dD + (i >> 2) * NT * 16 + (i & 3) * 4,
                                       drow[c] + min(ls + i, L - 1), i);
                set_par(dpar, s, c, m);
            }
            // x of the row-major directions
            if (xmode == 0) {
                if constexpr (FRONT && ESZ == 2) {
                    if (p.utile)
                        copy_tile(dX, c, ls);
                    else
                        copy_packed(dX, xrow[c], ls);
                } else if constexpr (ALIGNED) {
                    copy_packed(dX, xrow[c], ls);
                } else {
                    uint32_t m = 0;
#pragma unroll
                    for (int i = 0; i < kT; ++i)
                        m |= cp_async_word(dX + (i >> 2) * NT * 16 + (i & 3) * 4,
                                           xrow[c] + min(ls + i, L - 1), i);
                    set_par(xpar, s, c, m);
                }
            } else if (xmode == 1) {   // pixels L-1-ls-i
                if constexpr (ALIGNED) {
                    copy_packed(dX, xrow[c], L - kT - ls);   // ascending; step i reads index 15 - i
                } else {
                    uint32_t m = 0;
#pragma unroll
                    for (int i = 0; i < kT; ++i)
                        m |= cp_async_word(dX + (i >> 2) * NT * 16 + (i & 3) * 4,
                                           xrow[c] + max(L - 1 - ls - i, 0), i);
                    set_par(xpar, s, c, m);
                }
            }
        }
        // x of the column-major directions: one word per step and channel
        // (the same pixel for every channel of the lane)
        if constexpr (COLS) {
            if (xmode == 2) {
                uint32_t m[CPL];
#pragma unroll
                for (int c = 0; c < CPL; ++c)
                    m[c] = 0u;
                auto copy_step = [&](int i, int pix) {
#pragma unroll
                    for (int c = 0; c < CPL; ++c)
                        m[c] |= cp_async_word(sX0 + (s * CPL + c) * UX * NT * 16 + (i >> 2) * NT * 16 +
                                                  (i & 3) * 4,
                                              xrow[c] + pix, i);
                };
                if (ls + kT <= L && H >= 8) {
                    // pixel of step ls + i without walking: each column wrap moves
                    // the pixel by L - 1 against the row stride; with H >= 8 at most
                    // two wraps fall in 16 steps (one when H >= 16)
                    const int p0 = xw.p, h0 = xw.h, Lm1 = L - 1;
#pragma unroll
                    for (int i = 0; i < kT; ++i) {
                        int pix;
                        if (k == 2) {
                            const int hh = h0 + i;
                            const int cw = (hh >= H) + (H < kT && hh >= 2 * H);
                            pix = p0 + i * W - cw * Lm1;
                        } else {
                            const int hh = h0 - i;
                            const int cw = (hh < 0) + (H < kT && hh < -H);
                            pix = p0 - i * W + cw * Lm1;
                        }
                        copy_step(i, pix);
                    }
                    xw.advance(kT, adv_q, adv_r, H, W);
                } else {
#pragma unroll
                    for (int i = 0; i < kT; ++i) {
                        copy_step(i, (ls + i < L) ? xw.p : 0);
                        xw.next(H, W);
                    }
                }
#pragma unroll
                for (int c = 0; c < CPL; ++c)
                    set_par(xpar, s, c, m[c]);
            }
        }
    };
    // B|C rows of sub-chunk ls into raw stage s: row r < 16 is B of state r,
    // r >= 16 is C of state r - 16; rows of states >= N are not copied
    const int bc_rows = (MODE == kModeOutput) ? 32 : 16;
    auto issue_bc = [&](int s, int ls) {
        const uint32_t base = smem_u32(rawBC) + s * BCR * RS * 4;
        if constexpr (FRONT) {
            // the direction's dt_raw row: row 32, four 16-byte units
            if (tid < 4)
                cp_async16(base + (32 * RS) * 4 + tid * 16,
                           dtg + min(ls + tid * 4, ((L - 1) / 4) * 4));
        }
        if constexpr (ALIGNED) {
            constexpr int UE = 16 / EBC, NU = 16 / UE;
            if (vec == 16) {
                const int lastu = ((L - 1) / UE) * UE;
                for (int t = tid; t < bc_rows * NU; t += NT) {
                    const int r = t / NU, j = t % NU, n = r & 15;
                    if (n < N)
                        cp_async16(base + (r * RS) * 4 + j * 16,
                                   ((r < 16) ? Bg : Cg) + (size_t)n * LP + min(ls + j * UE, lastu));
                }
            } else {
                constexpr int PE = UE / 2;
                const int lastp = ((L - 1) / PE) * PE;
                for (int t = tid; t < bc_rows * 2 * NU; t += NT) {
                    const int r = t / (2 * NU), j = t % (2 * NU), n = r & 15;
                    if (n < N)
                        cp_async8(base + (r * RS) * 4 + j * 8,
                                  ((r < 16) ? Bg : Cg) + (size_t)n * LP + min(ls + j * PE, lastp));
                }
            }
        } else {
            for (int t = tid; t < bc_rows * kT; t += NT) {
                const int r = t >> 4, i = t & 15, n = r & 15;
                if (n < N)
                    cp_async_word(base + (r * RS + i) * 4,
                                  ((r < 16) ? Bg : Cg) + (size_t)n * LP + min(ls + i, L - 1), 0);
            }
        }
    };
    // raw B|C stage s (sub-chunk ls) -> float32 tile buf: entry q*kT + t holds
    // rows 4q..4q+3 of B (q < 4) or C (q >= 4) at step t
    auto convert_bc = [&](int s, int buf, int ls) {
        const uint32_t *raw = rawBC + s * BCR * RS;
        float4 *dst = BCf + buf * 8 * kT;
        if constexpr (FRONT) {
            if (tid < kT)
                sDT[buf * kT + tid] = __uint_as_float(raw[32 * RS + tid]);
        }
        const int tasks = (MODE == kModeOutput) ? 8 * kT : 4 * kT;
        for (int t = tid; t < tasks; t += NT) {
            const int q = t >> 4, st = t & 15;
            const int r0 = (q >> 2) * 16 + (q & 3) * 4;
            float v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = r0 + i, n = r & 15;
                float f = 0.f;
                if (n < N) {
                    if constexpr (EBC == 4) {
                        f = __uint_as_float(raw[r * RS + st]);
                    } else if constexpr (ALIGNED) {
                        f = raw_value<Tbc>(raw[r * RS + (st >> 1)], st & 1);
                    } else {
                        const Tbc *src = ((r < 16) ? Bg : Cg) + (size_t)n * LP + min(ls + st, L - 1);
                        f = raw_value<Tbc>(raw[r * RS + st],
                                           (uint32_t)(reinterpret_cast<uintptr_t>(src) >> 1) & 1u);
                    }
                }
                v[i] = f;
            }
            dst[t] = make_float4(v[0], v[1], v[2], v[3]);
        }
    };
    // steps valid.. of raw delta stage s read -inf (dt = 0: identity steps)
    auto mask_tail = [&](int s, int valid) {
        if constexpr (FRONT) {
            (void)s;   // no final states here: steps past L are computed and never stored
            (void)valid;
        } else {
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                uint32_t *dw = reinterpret_cast<uint32_t *>(rawD + ((s * CPL + c) * UD) * NT + tid);
                for (int i = valid; i < kT; ++i) {
                    if constexpr (DPACK2) {
                        // step i: unit i / 8, word (i % 8) / 2, half i % 2
                        uint32_t *w = dw + (i >> 3) * NT * 4 + ((i & 7) >> 1);
                        const uint32_t ninf = neg_inf_word<Tin>();
                        *w = (i & 1) ? ((*w & 0xffffu) | (ninf & 0xffff0000u))
                                     : ((*w & 0xffff0000u) | (ninf & 0xffffu));
                    } else {
                        dw[(i >> 2) * NT * 4 + (i & 3)] = neg_inf_word<Tin>();
                    }
                }
            }
        }
    };

    // ---- the 16 steps of one sub-chunk --------------------------------------
    // (dt, u) of every step and channel from the raw tiles of stage s into
    // this lane's column of the du tile: softplus of 16 independent steps
    auto stage_du = [&](auto xm_c, int s, int buf) {
        constexpr int XM = decltype(xm_c)::value;
        (void)buf;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const uint4 *dU = rawD + ((s * CPL + c) * UD) * NT + tid;
            const uint4 *xU = rawX + ((s * CPL + c) * UX) * NT + tid;
            const uint32_t dp = s ? dpar[1][c] : dpar[0][c];
            const uint32_t xp = s ? xpar[1][c] : xpar[0][c];
            (void)dp;
            (void)xp;
            (void)dU;
            uint4 dv = make_uint4(0, 0, 0, 0), xv = make_uint4(0, 0, 0, 0);
            // raw delta and x of step t (t ascending: the vector registers
            // dv, xv are refilled at their first step)
            auto fetch = [&](int t, float &draw, float &u) {
                if constexpr (FRONT) {
                    draw = wdt[c] * sDT[buf * kT + t];
                } else if constexpr (DPACK2) {
                    if ((t & 7) == 0)
                        dv = dU[(t >> 3) * NT];
                    draw = raw_value<Tin>(u4c(dv, (t >> 1) & 3), t & 1);
                } else {
                    if ((t & 3) == 0)
                        dv = dU[(t >> 2) * NT];
                    draw = raw_value<Tin>(u4c(dv, t & 3), ESZ == 2 ? (dp >> t) & 1u : 0u);
                }
                // x of step t
                if constexpr (XM == 2 || !DPACK2) {
                    // one word per step (column-major, unaligned rows, 4-byte
                    // types); reversed rows of 4-byte types are packed
                    // ascending: index 15 - t
                    if constexpr (XM == 1 && ESZ == 4 && ALIGNED) {
                        const int ti = kT - 1 - t;
                        if ((t & 3) == 0)
                            xv = xU[(ti >> 2) * NT];
                        u = raw_value<Tin>(u4c(xv, ti & 3), 0u);
                    } else {
                        if ((t & 3) == 0)
                            xv = xU[(t >> 2) * NT];
                        u = raw_value<Tin>(u4c(xv, t & 3), ESZ == 2 ? (xp >> t) & 1u : 0u);
                    }
                } else {
                    // packed 2-byte row: forward index t, reversed index 15 - t
                    const int ti = (XM == 1) ? kT - 1 - t : t;
                    if ((t & 7) == 0)
                        xv = xU[(ti >> 3) * NT];
                    u = raw_value<Tin>(u4c(xv, (ti >> 1) & 3), ti & 1);
                }
            };
            // softplus of two steps at a time on the packed pair instructions
#pragma unroll
            for (int t = 0; t < kT; t += 2) {
                float d0, u0, d1, u1;
                fetch(t, d0, u0);
                fetch(t + 1, d1, u1);
                const float2 dt = softplus2_f(make_float2(d0 + bias[c], d1 + bias[c]));
                if (MODE == kModeState) {
                    dtsum[c] += dt.x;
                    dtsum[c] += dt.y;
                }
                sDU[(t * CPL + c) * 32] = make_float2(dt.x, u0);
                sDU[((t + 1) * CPL + c) * 32] = make_float2(dt.y, u1);
            }
        }
    };
    // the recurrence over the staged steps, B|C from tile buf (each value
    // read once for all channels of the lane); the outputs replace dt in the
    // du tile
    auto steps = [&](int buf) {
        const float4 *sb = BCf + buf * 8 * kT;
#pragma unroll(CPL == 1 ? 4 : 1)
        for (int t = 0; t < kT; ++t) {
            float2 dt2[CPL], du2[CPL], acc0[CPL], acc1[CPL];
            float uu[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const float2 dtu = sDU[(t * CPL + c) * 32];
                uu[c] = dtu.y;
                const float du = dtu.x * dtu.y;
                dt2[c] = make_float2(dtu.x, dtu.x);
                du2[c] = make_float2(du, du);
                acc0[c] = make_float2(0.f, 0.f);
                acc1[c] = make_float2(0.f, 0.f);
            }
            const float4 *col = sb + t;   // slot q at col[q * kT]
#pragma unroll
            for (int q = 0; q < QN; ++q) {
                const float4 bv = col[q * kT];
                float4 cv = make_float4(0.f, 0.f, 0.f, 0.f);
                if (MODE == kModeOutput)
                    cv = col[(4 + q) * kT];
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    const float2 arg0 = __fmul2_rn(dt2[c], A2[c][2 * q]);
                    const float2 arg1 = __fmul2_rn(dt2[c], A2[c][2 * q + 1]);
                    const float2 a0 = make_float2(mufu_ex2(arg0.x), mufu_ex2(arg0.y));
                    const float2 a1 = make_float2(mufu_ex2(arg1.x), mufu_ex2(arg1.y));
                    h2[c][2 * q] =
                        __ffma2_rn(a0, h2[c][2 * q], __fmul2_rn(du2[c], make_float2(bv.x, bv.y)));
                    h2[c][2 * q + 1] = __ffma2_rn(a1, h2[c][2 * q + 1],
                                                  __fmul2_rn(du2[c], make_float2(bv.z, bv.w)));
                    if (MODE == kModeOutput) {
                        acc0[c] = __ffma2_rn(make_float2(cv.x, cv.y), h2[c][2 * q], acc0[c]);
                        acc1[c] = __ffma2_rn(make_float2(cv.z, cv.w), h2[c][2 * q + 1], acc1[c]);
                    }
                }
            }
            if (MODE == kModeOutput) {
#pragma unroll
                for (int c = 0; c < CPL; ++c)
                    sDU[(t * CPL + c) * 32].x =
                        fmaf(dsk[c], uu[c], (acc0[c].x + acc0[c].y) + (acc1[c].x + acc1[c].y));
            }
        }
    };

    // ---- prologue: sub-chunk 0 staged, B|C of sub-chunk 1 in flight -------
    issue_dx(0, l_begin);
    issue_bc(0, l_begin);
    if (nsub > 1)
        issue_bc(1, l_begin + kT);
    cp_async_commit();
    // everything below may read or overwrite what the previous kernel on the
    // stream wrote (entry states, the output rows)
    grid_dependency_wait();
    if (MODE == kModeOutput && chunk > 0) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int dc = cvalid[c] ? dch[c] : D - 1;
            const float4 *hs = reinterpret_cast<const float4 *>(
                p.hstate + ((row_bk + dc) * (p.NC - 1) + (chunk - 1)) * kNP);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v = hs[q];
                h2[c][2 * q] = make_float2(v.x, v.y);
                h2[c][2 * q + 1] = make_float2(v.z, v.w);
            }
        }
    }
    cp_async_wait_all();
    if (l_end - l_begin < kT)
        mask_tail(0, l_end - l_begin);
    __syncthreads();
    convert_bc(0, 0, l_begin);
    __syncthreads();

    int sbc_conv = 1 % Sh::BCS, sbc_issue = 2 % Sh::BCS;   // raw B|C stages
    for (int i = 0; i < nsub; ++i) {
        const int l0 = l_begin + i * kT;
        const int s = i & 1;
        if (i + 1 < nsub)
            issue_dx(s ^ 1, l0 + kT);
        if (i + 2 < nsub)
            issue_bc(sbc_issue, l0 + 2 * kT);
        cp_async_commit();
        if (i + 1 < nsub)
            convert_bc(sbc_conv, s ^ 1, l0 + kT);
        sbc_conv = sbc_conv == Sh::BCS - 1 ? 0 : sbc_conv + 1;
        sbc_issue = sbc_issue == Sh::BCS - 1 ? 0 : sbc_issue + 1;

        if (xmode == 0)
            stage_du(std::integral_constant<int, 0>{}, s, s);
        else if (xmode == 1)
            stage_du(std::integral_constant<int, 1>{}, s, s);
        else if constexpr (COLS)
            stage_du(std::integral_constant<int, 2>{}, s, s);
        steps(s);

        if (MODE == kModeOutput) {
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                if (!cvalid[c])
                    continue;
                // this channel's 16 outputs, one segment of its output row: in
                // scan order, except direction 1 of a multi-direction call (the
                // reversed row-major order), which is stored flipped, in pixel order
                const bool flip = k == 1 && K > 1;
                float *rowp = ymode ? p.ymerge + ((size_t)b * D + dch[c]) * (size_t)L
                                    : p.out + (row_bk + dch[c]) * (size_t)L;
                const float2 *yc = sDU + c * 32;   // step t at yc[t * CPL * 32]
                if (p.ovec && l0 + kT <= l_end) {
                    float4 *orow = reinterpret_cast<float4 *>(rowp + (flip ? L - kT - l0 : l0));
#pragma unroll
                    for (int q = 0; q < kT / 4; ++q) {
                        float4 v = flip ? make_float4(yc[(15 - 4 * q) * CPL * 32].x,
                                                      yc[(14 - 4 * q) * CPL * 32].x,
                                                      yc[(13 - 4 * q) * CPL * 32].x,
                                                      yc[(12 - 4 * q) * CPL * 32].x)
                                        : make_float4(yc[(4 * q) * CPL * 32].x,
                                                      yc[(4 * q + 1) * CPL * 32].x,
                                                      yc[(4 * q + 2) * CPL * 32].x,
                                                      yc[(4 * q + 3) * CPL * 32].x);
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
                            const float y = yc[t * CPL * 32].x;
                            if (ymode)
                                atomicAdd(o, y);
                            else
                                *o = accum ? *o + y : y;
                        }
                }
            }
        }
        cp_async_wait_all();
        if (i + 1 < nsub && l_end - (l0 + kT) < kT)
            mask_tail(s ^ 1, l_end - (l0 + kT));
        __syncthreads();
    }
    allow_dependents();

#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        if (!cvalid[c])
            continue;
        if (MODE == kModeState) {
            float4 *hs = reinterpret_cast<float4 *>(
                p.hstate + ((row_bk + dch[c]) * (p.NC - 1) + chunk) * kNP);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                hs[q] = make_float4(h2[c][2 * q].x, h2[c][2 * q].y, h2[c][2 * q + 1].x,
                                    h2[c][2 * q + 1].y);
            p.dtsum[(row_bk + dch[c]) * (p.NC - 1) + chunk] = dtsum[c];
        }
        // the state after the last step (steps past L have dt = 0: identity)
        if (MODE == kModeOutput && p.hlast && chunk == p.NC - 1) {
            float *hl = p.hlast + (row_bk + dch[c]) * p.NS + p.n0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (2 * j < N)
                    hl[2 * j] = h2[c][j].x;
                if (2 * j + 1 < N)
                    hl[2 * j + 1] = h2[c][j].y;
            }
        }
    }
}

// Entry states of every chunk after the first, in place over the chunk end
// states: slot c of a (b,k,d) row holds h_end of chunk c (from a zero entry
// state) on entry and the state entering chunk c + 1 on exit.
//
// With a_c = exp(A * sum of dt over chunk c), chunk c maps an entry state h
// to a_c h + h_end(c); maps compose associatively,
//     (a1, e1) then (a2, e2) = (a1 a2, a2 e1 + e2),
// and the entry state of chunk c is the composition of chunks 0 .. c-1
// applied to zero.  Thread (row, segment, state n) owns a segment of
// seg_len chunks of one row (16 neighbouring threads read one chunk's 16
// states, one 64-byte piece; chunks stream through two register groups of
// 16, the next group's loads in flight while the current one is applied):
//   1. it composes its segment's maps in order;
//   2. a Kogge-Stone scan over the G segments of each (row, n) -- G lanes of
//      one warp, shuffles of width G -- gives every segment its entry state;
//   3. it walks its segment again, writing the entry states.
// G (a power of two <= 16) is chosen for parallelism: with rows * 16 threads
// already filling the GPU, G = 1 and steps 1-2 vanish (one sequential walk
// per (row, n)); small batches and long rows (the 256x256 map: 768 rows of
// 511 chunks) get up to 16 segments.  A CTA of kCarryThreads threads holds
// 16 / G rows.
constexpr int kCarryThreads = 256;
constexpr int kCarryGroup = 16;   // chunks per register group

static __global__ void __launch_bounds__(kCarryThreads)
    carry_scan_kernel(const ScanParams p, int G, int seg_len)
{
    constexpr int GB = kCarryGroup;
    __shared__ float s_a[kCarryThreads / kNP][kNP], s_e[kCarryThreads / kNP][kNP];
    // the chunk end states of the state pass (the output pass is let in only
    // after the last store: triggered earlier, its waiting CTAs held the SMs
    // and the 256x256 step ran about 9 % longer)
    grid_dependency_wait();
    const int tid = threadIdx.x;
    const int nc1 = p.NC - 1;
    const long long rows = (long long)p.B * p.K * p.D;
    const int rpc = (kCarryThreads / kNP) / G;   // rows per CTA
    const int slot = tid / kNP, n = tid % kNP;   // slot = (row, segment)
    const int rl = slot / G, sg = slot % G;
    const long long row = (long long)blockIdx.x * rpc + rl;
    const bool live = row < rows && n < p.N;
    const long long rr = live ? row : 0;
    const unsigned ur = (unsigned)rr;   // rows < 2^31 (checked at launch)
    const int d = (int)(ur % (unsigned)p.D), k = (int)((ur / (unsigned)p.D) % (unsigned)p.K);
    const int c0 = min(sg * seg_len, nc1);
    const int cnt = live ? min(seg_len, nc1 - c0) : 0;
    float *hs = p.hstate + (rr * (long long)nc1 + c0) * kNP + n;   // chunk c0 + j at [j * kNP]
    const float *ds = p.dtsum + rr * (long long)nc1 + c0;
    const float A2 = live ? -expf(__ldg(p.A_log + ((size_t)k * p.D + d) * p.NS + p.n0 + n)) * kLog2e
                          : 0.f;

    float hA[GB], dA[GB], hB[GB], dB[GB];
    auto load = [&](float *hv, float *dv, int j0) {
#pragma unroll
        for (int i = 0; i < GB; ++i) {
            const bool ok = j0 + i < cnt;
            hv[i] = ok ? hs[(size_t)(j0 + i) * kNP] : 0.f;
            dv[i] = ok ? ds[j0 + i] : 0.f;
        }
    };
    // the segment's chunks in order, group by group, f applied to each
    auto stream = [&](auto &&f) {
        load(hA, dA, 0);
        for (int j0 = 0; j0 < cnt; j0 += 2 * GB) {
            if (j0 + GB < cnt)
                load(hB, dB, j0 + GB);
#pragma unroll
            for (int i = 0; i < GB; ++i)
                if (j0 + i < cnt)
                    f(j0 + i, hA[i], dA[i]);
            if (j0 + GB >= cnt)
                break;
            if (j0 + 2 * GB < cnt)
                load(hA, dA, j0 + 2 * GB);
#pragma unroll
            for (int i = 0; i < GB; ++i)
                if (j0 + GB + i < cnt)
                    f(j0 + GB + i, hB[i], dB[i]);
        }
    };

    float h = 0.f;   // the state entering the segment
    if (G > 1) {
        // ---- 1. compose the segment's maps
        float a = 1.f, e = 0.f;
        stream([&](int, float he, float dsum) {
            const float ai = mufu_ex2(A2 * dsum);
            e = fmaf(ai, e, he);
            a *= ai;
        });
        s_a[slot][n] = a;
        s_e[slot][n] = e;
        __syncthreads();
        // ---- 2. scan over the segments of each (row, n): lane group of G lanes
        {
            const int pair = tid / G, q = tid % G;   // pair = (row, n)
            const int cs = (pair / kNP) * G + q, cn = pair % kNP;
            float ca = s_a[cs][cn], ce = s_e[cs][cn];
            for (int off = 1; off < G; off <<= 1) {
                const float au = __shfl_up_sync(0xffffffffu, ca, off, G);
                const float eu = __shfl_up_sync(0xffffffffu, ce, off, G);
                if (q >= off) {
                    ce = fmaf(ca, eu, ce);
                    ca *= au;
                }
            }
            // entry state of segment q: the inclusive result of segment q - 1
            const float pe = __shfl_up_sync(0xffffffffu, ce, 1, G);
            __syncthreads();   // every slot read before any is overwritten
            s_e[cs][cn] = q == 0 ? 0.f : pe;
        }
        __syncthreads();
        h = s_e[slot][n];
    }
    // ---- 3. the entry state of each chunk after this one
    stream([&](int j, float he, float dsum) {
        h = fmaf(mufu_ex2(A2 * dsum), h, he);
        hs[(size_t)j * kNP] = h;
    });
    allow_dependents();
}

// The carry scan of a plan's chunk end states (p.hstate, p.dtsum, p.NC),
// launched on st (as a programmatic dependent of the previous kernel when
// dependent is true).
inline cudaError_t launch_carry_scan(const ScanParams &p, cudaStream_t st, bool dependent)
{
    const int nc1 = p.NC - 1;
    if (nc1 < 1)
        return cudaSuccess;
    const long long rows = (long long)p.B * p.K * p.D;
    if (rows > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    // segments: double them while the threads number under 64K (about 3
    // resident CTAs of 256 on each of 148 SMs, twice) and segments keep at
    // least 8 chunks
    constexpr long long kWantThreads = 65536;
    int G = 1;
    while (G < 16 && rows * kNP * G < kWantThreads && nc1 >= 16 * G)
        G <<= 1;
    const int seg_len = (nc1 + G - 1) / G;
    const long long rpc = (kCarryThreads / kNP) / G;
    const long long blocks = (rows + rpc - 1) / rpc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kCarryThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (dependent) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, carry_scan_kernel, p, G, seg_len);
}

}  // namespace ss2d
