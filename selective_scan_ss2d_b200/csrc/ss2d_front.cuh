// ss2d_front.cuh -- the front of the selective scan in the tutorial's
// SelectiveSSM and the Vim block, on the 5th-generation tensor cores.
//
// "Vision Mamba" tutorial, section "Background: State Space Models and
// Mamba", SelectiveSSM.forward; "Vision Mamba ..." summary, section 4.3 (the
// Vim block: every direction its own conv1d and projections).  For
// direction k (0: the sequence as it is; 1: reversed along L), per batch
// element b and step l of the direction's own order:
//     c[l, d]  = conv_b[k, d] + sum_j conv_w[k, d, j] * s[l - 3 + j, d]   (causal, zeros before l = 0)
//     u[l, d]  = SiLU(c[l, d])
//     x_dbl[l] = W_x[k] u[l]            (x_proj: D -> 1 + 2N, no bias)
//     dt_raw[l] = x_dbl[l, 0], B[n, l] = x_dbl[l, 1 + n], C[n, l] = x_dbl[l, 1 + N + n]
// dt_proj (a Linear from 1 to D) is applied by the scan itself: its delta is
// w_dt[k, d] * dt_raw[l], its bias the scan's delta bias, so no (D, L) delta
// array is ever written.
//
// Two kernels:
//   front_conv_kernel: one CTA of 256 threads per (128-step tile, 64-channel
//     block, b * K + k); the tile's input steps (3-step halo) are staged in
//     shared memory with cp.async, then a thread holds a channel pair over 16
//     steps, convolves, applies SiLU and writes u rounded to bf16 as the
//     tile's x_proj A operand block, already in the tensor-core operand
//     layout (one 16 KB block per tile and channel block).  For bf16 inputs
//     of the fused call those blocks are the only copy of u: the scan reads
//     its rows from them (p.utile).  Otherwise it also writes u for the scan,
//     in the input dtype, as (B, K, D, LP) rows.  The CTAs of the first tile
//     of batch element 0 also convert W_x to the bf16 B operand blocks.
//   front_proj_kernel: one CTA of 128 threads per (128-step tile, k, b).  One
//     thread streams the tile's A blocks and the matching bf16 blocks of W_x
//     into a ring of shared-memory stages with cp.async.bulk, each stage completing
//     an mbarrier (expected bytes), and issues the tcgen05.mma instructions
//     (M = 128 steps, N = 1 + 2N rounded up to 16, K = 16 per instruction)
//     that accumulate x_dbl in tensor memory; a tcgen05.commit frees each
//     stage for the next copy.  The epilogue reads the accumulator back with
//     tcgen05.ld (warp w: steps 32w..32w+31, one step per lane) and stores
//     dt_raw, B and C.
// Every mbarrier wait gives up after a time limit, records the fault in a
// device word that ss2d_check_waits() reports, and lets the kernel finish.
//
// Operand layouts, no swizzle, core matrices of 8 rows x 16 bytes:
// A, MN-major (steps contiguous): element (step r, channel c) of a block at
//     (r / 8) * 1024 + c * 16 + (r % 8) * 2,
// core matrices 1024 bytes apart along the steps (SBO) and 128 bytes apart
// along the channels (LBO): each 16-byte run of 8 steps of one channel is one
// core-matrix row, which the conv kernel stores whole and the scan can read
// as a piece of its row.  B, K-major: element (row r, channel c) at
//     (r / 8) * 1024 + (c / 8) * 128 + (r % 8) * 16 + (c % 8) * 2
// (LBO = 128 along the channels, SBO = 1024 along the rows).  Both blocks
// are contiguous in global memory, so a block is one bulk copy.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ss2d_kernels.cuh"

namespace ss2d {

struct FrontParams {
    const void *x;          // (B, L, D) input branch, dtype
    const float *conv_w;    // (K, D, 4)
    const float *conv_b;    // (K, D)
    const float *W_x;       // (K, 1 + 2N, D)
    const void *Wb;         // W_x in bf16, per direction and 64-channel block, in the B layout
    void *Ab;               // u in bf16, per (b, k, tile, 64-channel block), in the A layout
    int utile;              // 1: Ab is the only copy of u (bf16 inputs of the fused call)
    void *u;                // (B, K, D, LP) u of every direction in its scan order, dtype
    float *dt_raw;          // (B, K, LP)
    float *Bs, *Cs;         // (B, K, N, LP)
    int *fault;             // set when a bounded wait ran out
    int B, D, L, LP, N, K;
    int NM;                 // MMA N: 1 + 2N rounded up to a multiple of 16
    int tcols;              // tensor-memory columns held (power of 2, >= 32, >= NM)
};

constexpr int kFrontConvThreads = 256;
constexpr int kFrontProjThreads = 128;
constexpr int kFrontTile = 128;       // steps per tile (MMA M)
constexpr int kFrontCh = 64;          // channels per block (4 MMAs of K = 16)
constexpr int kFrontLBO = 128;                               // B: channel stride; A: channel stride
constexpr int kFrontSBO = 1024;                              // B: row stride; A: step stride
constexpr int kFrontABytes = (kFrontTile / 8) * kFrontSBO;   // one A block (16 KB)
constexpr int kFrontStages = 2;                              // shared-memory ring

__host__ __device__ constexpr int front_bbytes(int NM) { return (NM / 8) * kFrontSBO; }
// dynamic shared memory of front_proj_kernel: the ring of (A, B) stages,
// 2 * stages + 1 mbarriers, the tensor-memory address
__host__ __device__ constexpr int front_smem_bytes(int NM)
{
    return kFrontStages * (kFrontABytes + front_bbytes(NM)) + 8 * (2 * kFrontStages + 1) + 16;
}

// codes written to the fault word
constexpr int kFaultFrontMma = 1;
constexpr int kFaultSelftest = 2;

// ---- mbarrier and tcgen05 wrappers -----------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase of `bar` with parity `parity` to complete, at most
// limit_ns nanoseconds; on time-out record `code` in *fault and return false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                                  int *fault, int code)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > limit_ns) {
            atomicCAS(fault, 0, code);
            return false;
        }
    }
    return true;
}
__device__ __forceinline__ void fence_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// shared-memory matrix descriptor: K-major, no swizzle, version 1 (sm_100)
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
    d |= (uint64_t)1 << 46;
    return d;   // base offset 0, layout type 0 (no swizzle)
}
// instruction descriptor of kind::f16: bf16 A and B, f32 accumulator,
// M = 128, N = nm, both operands K-major (the caller sets bit 15 for an
// MN-major A)
__device__ __forceinline__ uint32_t umma_idesc_bf16(int nm)
{
    return (1u << 4)                     // accumulator f32
           | (1u << 7) | (1u << 10)      // A, B bf16
           | ((uint32_t)(nm >> 3) << 17) // N / 8
           | ((uint32_t)(kFrontTile >> 4) << 24);   // M / 16
}
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void cp_async_16b(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}

// W_x (K, R, D) float32 -> Wb, one block: for direction k and 64-channel
// block cb, the NM x 64 bf16 B operand (rows >= R and channels >= D zero) in
// the layout (r / 8) * 1024 + (c / 8) * 128 + (r % 8) * 16 + (c % 8) * 2, by
// the calling CTA's threads.
__device__ __forceinline__ void front_wprep_block(const float *W_x, __nv_bfloat16 *Wb, int D,
                                                  int R, int NM, int k, int cb, int nblk)
{
    __nv_bfloat16 *dst = Wb + ((size_t)k * nblk + cb) * NM * kFrontCh;
    for (int i = threadIdx.x; i < NM * kFrontCh; i += blockDim.x) {
        const int r = i / kFrontCh, cc = i % kFrontCh, dd = cb * kFrontCh + cc;
        const float v = (r < R && dd < D) ? W_x[((size_t)k * R + r) * D + dd] : 0.f;
        dst[((r >> 3) * kFrontSBO + (cc >> 3) * kFrontLBO + (r & 7) * 16 + (cc & 7) * 2) / 2] =
            __float2bfloat16_rn(v);
    }
}

template <typename Tin>
__device__ __forceinline__ float front_load(const Tin *p)
{
    return to_f32(*p);
}

// bits of the stored value of u
__device__ __forceinline__ uint32_t store_bits(float v, float *) { return __float_as_uint(v); }
__device__ __forceinline__ uint32_t store_bits(float v, __nv_bfloat16 *)
{
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}
__device__ __forceinline__ uint32_t store_bits(float v, __half *)
{
    return (uint32_t)__half_as_ushort(__float2half_rn(v));
}

// cp.async of 16 bytes that reads `bytes` (0 or 16) and zero-fills the rest
__device__ __forceinline__ void cp_async_16b_zfill(uint32_t dst, const void *src, uint32_t bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}

constexpr int kFrontRows = kFrontTile + 3;   // input steps of a tile with the 3-step halo

// conv + SiLU of one (128-step tile, 64-channel block, b * K + k): the bf16
// A operand block and, unless p.utile, u for the scan.  grid: tiles *
// channel blocks * B * K CTAs in one dimension, the tile fastest.
// The CTA first copies the tile's 131 input steps (3-step halo) of its 64
// channels into shared memory (cp.async, 16-byte pieces, zeros outside the
// sequence and past channel D - 1), so that all its loads are in flight at
// once.  Thread t then owns the channel pair 2 * (t % 32), + 1 over steps
// 16 * (t / 32) .. + 15 of the tile: it writes per channel its 16 steps as
// two 16-byte A rows (and as u row segments).  Warps whose steps all lie
// past the end of the sequence do nothing (the A rows of those steps only
// feed accumulator rows that are never stored, and the scan never reads
// them).
template <typename Tin>
__global__ void __launch_bounds__(kFrontConvThreads) front_conv_kernel(const FrontParams p)
{
    constexpr int CP = 2, SG = 16;   // channels and steps per thread
    static_assert(kFrontCh / CP * (kFrontTile / SG) == kFrontConvThreads, "thread layout");
    constexpr int ROWB = kFrontCh * (int)sizeof(Tin);   // bytes of a staged row
    __shared__ __align__(16) unsigned char sx[kFrontRows * ROWB];
    const int tid = threadIdx.x;
    const int ntiles = (p.L + kFrontTile - 1) / kFrontTile;
    const int nblk = (p.D + kFrontCh - 1) / kFrontCh;
    const int tile = (int)(blockIdx.x % (unsigned)ntiles);
    const unsigned rest = blockIdx.x / (unsigned)ntiles;
    const int cb = (int)(rest % (unsigned)nblk), bk = (int)(rest / (unsigned)nblk);
    const int b = bk / p.K, k = bk % p.K;
    const int D = p.D, L = p.L, LP = p.LP;
    // the CTAs of the first tile of b = 0 also convert W_x's block (k, cb)
    // for x_proj (which runs after this kernel on the stream)
    if (tile == 0 && bk < p.K)
        front_wprep_block(p.W_x, static_cast<__nv_bfloat16 *>(const_cast<void *>(p.Wb)), D,
                          1 + 2 * p.N, p.NM, k, cb, nblk);
    const int lt = tile * kFrontTile;            // first step of the tile
    const int dblk = cb * kFrontCh;              // first channel of the block
    const Tin *xb = static_cast<const Tin *>(p.x) + (size_t)b * L * D;

    // ---- stage: row r holds step lt - 3 + r, which reads input position
    // l (k = 0) or L-1-l (k = 1)
    constexpr int EPV = 16 / (int)sizeof(Tin);   // elements per 16-byte piece
    const bool vec = D % EPV == 0 && (reinterpret_cast<uintptr_t>(p.x) & 15) == 0;
    if (vec) {
        constexpr int PPR = kFrontCh / EPV;      // pieces per row
        const uint32_t s0 = static_cast<uint32_t>(__cvta_generic_to_shared(sx));
        for (int i = tid; i < kFrontRows * PPR; i += kFrontConvThreads) {
            const int r = i / PPR, pc = i % PPR;
            const int l = lt - 3 + r, d = dblk + pc * EPV;
            const bool in = l >= 0 && l < L && d < D;
            const int pos = in ? (k == 0 ? l : L - 1 - l) : 0;
            cp_async_16b_zfill(s0 + r * ROWB + pc * 16, xb + (size_t)pos * D + (in ? d : 0),
                               in ? 16u : 0u);
        }
        asm volatile("cp.async.wait_all;\n" ::: "memory");
    } else {
        Tin *st = reinterpret_cast<Tin *>(sx);
        for (int i = tid; i < kFrontRows * kFrontCh; i += kFrontConvThreads) {
            const int r = i / kFrontCh, c = i % kFrontCh;
            const int l = lt - 3 + r, d = dblk + c;
            const bool in = l >= 0 && l < L && d < D;
            st[i] = in ? xb[(size_t)(k == 0 ? l : L - 1 - l) * D + d] : Tin(0.f);
        }
    }
    __syncthreads();

    const int pr = tid % (kFrontCh / CP), sg = tid / (kFrontCh / CP);
    const int c0 = pr * CP;                      // first channel of the pair in the block
    const int m0 = sg * SG;                      // first step of the thread in the tile
    const int l0 = lt + m0;
    if (l0 >= L)
        return;                                  // the whole warp: no step of it is stored
    const int d0 = dblk + c0;
    float w[CP][4], bias[CP];
#pragma unroll
    for (int j = 0; j < CP; ++j) {
        const int d = d0 + j;
        if (d < D) {
            const float4 wv = *reinterpret_cast<const float4 *>(p.conv_w + ((size_t)k * D + d) * 4);
            w[j][0] = wv.x;
            w[j][1] = wv.y;
            w[j][2] = wv.z;
            w[j][3] = wv.w;
            bias[j] = p.conv_b[(size_t)k * D + d];
        } else {
            w[j][0] = w[j][1] = w[j][2] = w[j][3] = bias[j] = 0.f;
        }
    }
    // the pair's value at staged row r
    auto xrow = [&](int r, float (&v)[CP]) {
        if constexpr (sizeof(Tin) == 2) {
            const uint32_t wd = *reinterpret_cast<const uint32_t *>(sx + r * ROWB + c0 * 2);
            v[0] = half_bits_to_f32<Tin>(wd & 0xffffu);
            v[1] = half_bits_to_f32<Tin>(wd >> 16);
        } else {
            const float2 f = *reinterpret_cast<const float2 *>(sx + r * ROWB + c0 * 4);
            v[0] = f.x;
            v[1] = f.y;
        }
    };
    float win[4][CP];   // steps m - 3 .. m of the pair
    xrow(m0, win[0]);
    xrow(m0 + 1, win[1]);
    xrow(m0 + 2, win[2]);
    unsigned char *ab = static_cast<unsigned char *>(p.Ab) +
                        (((size_t)bk * ntiles + tile) * nblk + cb) * kFrontABytes +
                        (m0 >> 3) * kFrontSBO + c0 * 16;   // channel c0, steps m0..m0+7
    // per step: the A operand word (the pair in bf16, one packed conversion);
    // 2-byte inputs: the pair in the input dtype, whose halves are u's values
    // (for bf16 the A word itself); float inputs: the float values
    uint32_t aw[SG], hw[sizeof(Tin) == 2 ? SG : 1];
    float uu[sizeof(Tin) == 4 ? CP : 1][sizeof(Tin) == 4 ? SG : 1];
#pragma unroll
    for (int i = 0; i < SG; ++i) {
        xrow(m0 + i + 3, win[(i + 3) & 3]);
        float v[CP];
#pragma unroll
        for (int j = 0; j < CP; ++j) {
            const float cv = fmaf(w[j][3], win[(i + 3) & 3][j],
                                  fmaf(w[j][2], win[(i + 2) & 3][j],
                                       fmaf(w[j][1], win[(i + 1) & 3][j], fmaf(w[j][0], win[i & 3][j], bias[j]))));
            v[j] = silu_f(cv);   // channels past D: zero inputs and taps give SiLU(0) = 0
        }
        const __nv_bfloat162 a2 = __floats2bfloat162_rn(v[0], v[1]);
        aw[i] = *reinterpret_cast<const uint32_t *>(&a2);
        if constexpr (std::is_same_v<Tin, __half>) {
            const __half2 h2 = __floats2half2_rn(v[0], v[1]);
            hw[i] = *reinterpret_cast<const uint32_t *>(&h2);
        } else if constexpr (sizeof(Tin) == 2) {
            hw[i] = aw[i];
        } else {
            uu[0][i] = v[0];
            uu[1][i] = v[1];
        }
    }
    // the A rows: per channel j and 8-step group q, the 8 bf16 values, the
    // low (j = 0) or high (j = 1) halves of the pair words
#pragma unroll
    for (int j = 0; j < CP; ++j) {
        const uint32_t sel = j == 0 ? 0x5410u : 0x7632u;
#pragma unroll
        for (int q = 0; q < SG / 8; ++q) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                w4[e] = __byte_perm(aw[q * 8 + 2 * e], aw[q * 8 + 2 * e + 1], sel);
            *reinterpret_cast<uint4 *>(ab + q * kFrontSBO + j * 16) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
    if (p.utile)
        return;   // the A rows are u
    // u for the scan, in the input dtype: 16-byte stores of 8 (2-byte) or 4
    // (float) steps; every store starts before L (LP is a multiple of 8)
    Tin *ub = static_cast<Tin *>(p.u) + (size_t)bk * D * LP;
    constexpr int PER = sizeof(Tin) == 2 ? 8 : 4;
#pragma unroll
    for (int j = 0; j < CP; ++j) {
        const int d = d0 + j;
        if (d >= D)
            continue;
#pragma unroll
        for (int q = 0; q < SG / PER; ++q) {
            const int lv = l0 + q * PER;
            if (lv >= L)
                continue;
            uint4 v;
            if constexpr (sizeof(Tin) == 2) {
                // channel j's values of steps 2e, 2e + 1: the low (j = 0) or
                // high (j = 1) halves of two pair words
                const uint32_t sel = j == 0 ? 0x5410u : 0x7632u;
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w4[e] = __byte_perm(hw[q * PER + 2 * e], hw[q * PER + 2 * e + 1], sel);
                v = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            } else {
                v = make_uint4(__float_as_uint(uu[j][q * PER]), __float_as_uint(uu[j][q * PER + 1]),
                               __float_as_uint(uu[j][q * PER + 2]), __float_as_uint(uu[j][q * PER + 3]));
            }
            *reinterpret_cast<uint4 *>(ub + (size_t)d * LP + lv) = v;
        }
    }
}

// bulk copy global -> shared completing `bytes` on the mbarrier (TMA, no
// tensor map, no multicast); src, dst 16-byte aligned, bytes a multiple of 16
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// x_proj of one (128-step tile, k, b) on the tensor cores; see the header.
// grid (tiles, K, B).
__global__ void __launch_bounds__(kFrontProjThreads) front_proj_kernel(const FrontParams p)
{
    extern __shared__ __align__(1024) unsigned char fsm[];
    const int NM = p.NM;
    const uint32_t bbytes = (uint32_t)front_bbytes(NM);
    const uint32_t stage_bytes = kFrontABytes + bbytes;
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(fsm));
    // stage s: A at sbase + s * stage_bytes, B right after it
    const uint32_t bars = sbase + kFrontStages * stage_bytes;   // full[s], empty[s], done
    uint32_t *tslot = reinterpret_cast<uint32_t *>(fsm + kFrontStages * stage_bytes +
                                                   8 * (2 * kFrontStages + 1));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, k = blockIdx.y, b = blockIdx.z;
    const int N = p.N, K = p.K, L = p.L, LP = p.LP;
    const int R = 1 + 2 * N;
    const int l0 = tile * kFrontTile;
    const int nblk = (p.D + kFrontCh - 1) / kFrontCh, ntiles = gridDim.x;
    const size_t bk = (size_t)b * K + k;
    const unsigned char *ag = static_cast<const unsigned char *>(p.Ab) +
                              ((bk * ntiles + tile) * nblk) * kFrontABytes;
    const unsigned char *wg = static_cast<const unsigned char *>(p.Wb) + (size_t)k * nblk * bbytes;
    constexpr uint64_t kLimitNs = 2000000000ull;   // 2 s

    if (tid == 0) {
        for (int i = 0; i < 2 * kFrontStages + 1; ++i)
            mbar_init(bars + 8 * i, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(tslot))), "r"(p.tcols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    bool ok = true;
    if (tid == 0) {
        const uint32_t idesc = umma_idesc_bf16(NM) | (1u << 15);   // A MN-major
        // the 8-step groups of A that hold steps before L (the last tile's
        // later rows only feed accumulator rows that are never stored)
        const uint32_t a_bytes = (uint32_t)min(kFrontTile / 8, (L - l0 + 7) / 8) * kFrontSBO;
        auto load = [&](int cb) {   // block cb into stage cb % S
            const int st = cb % kFrontStages;
            const uint32_t full = bars + 8 * st, dA = sbase + st * stage_bytes;
            mbar_expect_tx(full, a_bytes + bbytes);
            bulk_copy(dA, ag + (size_t)cb * kFrontABytes, a_bytes, full);
            bulk_copy(dA + kFrontABytes, wg + (size_t)cb * bbytes, bbytes, full);
        };
        for (int cb = 0; cb < kFrontStages && cb < nblk; ++cb)
            load(cb);
        for (int cb = 0; cb < nblk; ++cb) {
            const int st = cb % kFrontStages, use = cb / kFrontStages;
            const uint32_t full = bars + 8 * st, empty = bars + 8 * (kFrontStages + st);
            ok = ok && mbar_wait_bounded(full, use & 1, kLimitNs, p.fault, kFaultFrontMma);
            tc_fence_after();
            if (ok) {
                const uint32_t aS = sbase + st * stage_bytes, bS = aS + kFrontABytes;
#pragma unroll
                for (int kk = 0; kk < kFrontCh / 16; ++kk)
                    umma_bf16(tmem, umma_desc(aS + kk * 16 * 16, kFrontLBO, kFrontSBO),
                              umma_desc(bS + kk * 2 * kFrontLBO, kFrontLBO, kFrontSBO), idesc,
                              (cb > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(empty);
            if (cb + kFrontStages < nblk) {
                // the stage is refilled once its MMAs have read it
                ok = ok && mbar_wait_bounded(empty, use & 1, kLimitNs, p.fault, kFaultFrontMma);
                if (ok)
                    load(cb + kFrontStages);
            }
        }
        umma_commit(bars + 8 * (2 * kFrontStages));   // every MMA of the tile done
    }
    ok = mbar_wait_bounded(bars + 8 * (2 * kFrontStages), 0, kLimitNs, p.fault, kFaultFrontMma) &&
         ok;
    tc_fence_after();

    // ---- epilogue: x_dbl rows from tensor memory (warp w: lanes 32w..) ----
    const int l = l0 + warp * 32 + lane;
    for (int c0 = 0; c0 < NM; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
        if (ok && l < L) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int col = c0 + i;
                if (col == 0)
                    p.dt_raw[bk * LP + l] = v[i];
                else if (col <= N)
                    p.Bs[(bk * N + (col - 1)) * LP + l] = v[i];
                else if (col < R)
                    p.Cs[(bk * N + (col - 1 - N)) * LP + l] = v[i];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tcols)
                     : "memory");
    }
}

// A wait on an mbarrier that nothing arrives on: it must give up after
// limit_ns and record kFaultSelftest in *fault (the check of the bounded
// wait's time-out path).
static __global__ void wait_selftest_kernel(int *fault, unsigned long long limit_ns)
{
    __shared__ __align__(8) unsigned long long bar;
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    if (threadIdx.x == 0) {
        mbar_init(a, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    mbar_wait_bounded(a, 0, limit_ns, fault, kFaultSelftest);
}

}  // namespace ss2d
