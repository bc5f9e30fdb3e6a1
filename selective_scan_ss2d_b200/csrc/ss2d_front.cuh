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
// front_kernel: one CTA of 128 threads per (128-step tile, k, b).  Channels
// are taken 64 at a time: the CTA convolves its tile (3-step halo, taps in
// registers), applies SiLU, stores u for the scan (in the input dtype) and
// writes u, rounded to bf16, as the A operand of x_proj into shared memory;
// the matching 64 columns of W_x go in as the B operand.  One thread issues
// the tcgen05.mma instructions (M = 128 steps, N = 1 + 2N rounded up to 16,
// K = 16 per instruction) that accumulate x_dbl in tensor memory, and a
// tcgen05.commit tells an mbarrier when the buffers may be refilled (two
// buffers: the conv of the next 64 channels overlaps the MMAs of these).
// Every mbarrier wait gives up after a time limit, records the fault in a
// device word that ss2d_check_waits() reports, and lets the kernel finish.
// The epilogue reads the accumulator back with tcgen05.ld (warp w: steps
// 32w..32w+31, one step per lane) and stores dt_raw, B and C.
//
// Operand layout (K-major, no swizzle): core matrices of 8 rows x 16 bytes;
// element (row r, channel c) of a 64-channel block at byte
//     (r / 8) * kSBO + (c / 8) * kLBO + (r % 8) * 16 + (c % 8) * 2,
// kLBO = 144 (the 8 core matrices of a row group 144 bytes apart, which
// spreads a warp's stores of one row over 16 banks) and kSBO = 8 * kLBO.
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
    void *u;                // (B, K, D, LP) u of every direction in its scan order, dtype
    float *dt_raw;          // (B, K, LP)
    float *Bs, *Cs;         // (B, K, N, LP)
    int *fault;             // set when a bounded wait ran out
    int B, D, L, LP, N, K;
    int NM;                 // MMA N: 1 + 2N rounded up to a multiple of 16
    int tcols;              // tensor-memory columns held (power of 2, >= 32, >= NM)
};

constexpr int kFrontThreads = 128;
constexpr int kFrontTile = 128;       // steps per CTA (MMA M)
constexpr int kFrontCh = 64;          // channels per block (4 MMAs of K = 16)
constexpr int kFrontLBO = 144;
constexpr int kFrontSBO = 8 * kFrontLBO;
constexpr int kFrontABytes = (kFrontTile / 8) * kFrontSBO;   // one A buffer

__host__ __device__ constexpr int front_bbytes(int NM) { return (NM / 8) * kFrontSBO; }
// dynamic shared memory: two A buffers, two B buffers, three mbarriers, the
// tensor-memory address
__host__ __device__ constexpr int front_smem_bytes(int NM)
{
    return 2 * kFrontABytes + 2 * front_bbytes(NM) + 64;
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
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)((kFrontLBO >> 4) & 0x3fffu) << 16;
    d |= (uint64_t)((kFrontSBO >> 4) & 0x3fffu) << 32;
    d |= (uint64_t)1 << 46;
    return d;   // base offset 0, layout type 0 (no swizzle)
}
// instruction descriptor of kind::f16: bf16 A and B, f32 accumulator,
// both K-major, M = 128, N = nm
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

template <typename Tin>
__global__ void __launch_bounds__(kFrontThreads) front_kernel(const FrontParams p)
{
    extern __shared__ __align__(1024) unsigned char fsm[];
    const int NM = p.NM;
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(fsm));
    const uint32_t sA = sbase, sB = sbase + 2 * kFrontABytes;
    const uint32_t bbytes = (uint32_t)front_bbytes(NM);
    unsigned char *bars_g = fsm + 2 * kFrontABytes + 2 * bbytes;
    const uint32_t bar0 = sB + 2 * bbytes;              // buffer 0 free, buffer 1 free, done
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars_g + 32);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int l0 = blockIdx.x * kFrontTile;
    const int k = blockIdx.y, b = blockIdx.z;
    const int D = p.D, L = p.L, LP = p.LP, N = p.N, K = p.K;
    const int R = 1 + 2 * N;

    if (tid == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8, 1);
        mbar_init(bar0 + 16, 1);
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

    const Tin *xb = static_cast<const Tin *>(p.x) + (size_t)b * L * D;
    Tin *ub = static_cast<Tin *>(p.u) + ((size_t)b * K + k) * (size_t)D * LP;
    const uint32_t idesc = umma_idesc_bf16(NM);
    const int c = tid & 63, half = tid >> 6;          // this thread's channel and 64-step half
    const int nblk = (D + kFrontCh - 1) / kFrontCh;
    constexpr uint64_t kLimitNs = 2000000000ull;       // 2 s
    bool ok = true;

    for (int cb = 0; cb < nblk; ++cb) {
        const int buf = cb & 1;
        // the MMAs of block cb - 2 read this buffer
        if (cb >= 2)
            ok = ok && mbar_wait_bounded(bar0 + 8 * buf, ((cb >> 1) - 1) & 1, kLimitNs, p.fault,
                                         kFaultFrontMma);
        const uint32_t aBuf = sA + buf * kFrontABytes, bBuf = sB + buf * bbytes;
        unsigned char *aPtr = fsm + buf * kFrontABytes;
        unsigned char *bPtr = fsm + 2 * kFrontABytes + buf * bbytes;

        // ---- conv + SiLU of channel d over steps half*64 .. half*64 + 63 ----
        const int d = cb * kFrontCh + c;
        const bool dv = d < D;
        float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, bias = 0.f;
        if (dv) {
            const float4 wv = *reinterpret_cast<const float4 *>(p.conv_w + ((size_t)k * D + d) * 4);
            w0 = wv.x;
            w1 = wv.y;
            w2 = wv.z;
            w3 = wv.w;
            bias = p.conv_b[(size_t)k * D + d];
        }
        // the direction's step l reads input position l (k = 0) or L-1-l (k = 1)
        auto xat = [&](int l) -> float {
            if (!dv || l < 0 || l >= L)
                return 0.f;
            const int pos = k == 0 ? l : L - 1 - l;
            return front_load(xb + (size_t)pos * D + d);
        };
        const int m0 = half * 64;
        float s0 = xat(l0 + m0 - 3), s1 = xat(l0 + m0 - 2), s2 = xat(l0 + m0 - 1);
        constexpr int PER = sizeof(Tin) == 2 ? 8 : 4;   // steps per 16-byte store of u
        for (int mb = 0; mb < 64; mb += PER) {
            float xs[PER];
#pragma unroll
            for (int j = 0; j < PER; ++j)   // the group's inputs, loads in flight together
                xs[j] = xat(l0 + m0 + mb + j);
            uint32_t pack[PER];
#pragma unroll
            for (int j = 0; j < PER; ++j) {
                const int mt = m0 + mb + j;
                const float s3 = xs[j];
                const float cv = fmaf(w3, s3, fmaf(w2, s2, fmaf(w1, s1, fmaf(w0, s0, bias))));
                const float uu = dv ? silu_f(cv) : 0.f;
                s0 = s1;
                s1 = s2;
                s2 = s3;
                // A operand (bf16, nearest even)
                *reinterpret_cast<__nv_bfloat16 *>(aPtr + (mt >> 3) * kFrontSBO +
                                                   (c >> 3) * kFrontLBO + (mt & 7) * 16 +
                                                   (c & 7) * 2) = __float2bfloat16_rn(uu);
                pack[j] = store_bits(uu, static_cast<Tin *>(nullptr));
            }
            // u for the scan, in the input dtype: one 16-byte store of PER steps
            const int lv = l0 + m0 + mb;
            if (dv && lv < L) {
                uint4 v;
                if constexpr (sizeof(Tin) == 2)
                    v = make_uint4(pack[0] | (pack[1] << 16), pack[2] | (pack[3] << 16),
                                   pack[4] | (pack[5] << 16), pack[6] | (pack[7] << 16));
                else
                    v = make_uint4(pack[0], pack[1], pack[2], pack[3]);
                *reinterpret_cast<uint4 *>(ub + (size_t)d * LP + lv) = v;
            }
        }
        // ---- B operand: rows 0..NM-1 of W_x (zero beyond 1 + 2N and D) ----
        for (int i = tid; i < NM * kFrontCh; i += kFrontThreads) {
            const int r = i / kFrontCh, cc = i % kFrontCh, dd = cb * kFrontCh + cc;
            const float wv = (r < R && dd < D) ? p.W_x[((size_t)k * R + r) * D + dd] : 0.f;
            *reinterpret_cast<__nv_bfloat16 *>(bPtr + (r >> 3) * kFrontSBO + (cc >> 3) * kFrontLBO +
                                               (r & 7) * 16 + (cc & 7) * 2) = __float2bfloat16_rn(wv);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            if (ok) {
#pragma unroll
                for (int kk = 0; kk < kFrontCh / 16; ++kk)
                    umma_bf16(tmem, umma_desc(aBuf + kk * 2 * kFrontLBO),
                              umma_desc(bBuf + kk * 2 * kFrontLBO), idesc,
                              (cb > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(bar0 + 8 * buf);
        }
    }
    // every MMA of the tile done
    if (tid == 0)
        umma_commit(bar0 + 16);
    ok = mbar_wait_bounded(bar0 + 16, 0, kLimitNs, p.fault, kFaultFrontMma) && ok;
    tc_fence_after();

    // ---- epilogue: x_dbl rows from tensor memory ----
    const int l = l0 + warp * 32 + lane;
    const size_t row_bk = (size_t)b * K + k;
    for (int c0 = 0; c0 < NM; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
        if (ok && l < L) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int col = c0 + i;
                if (col == 0)
                    p.dt_raw[row_bk * LP + l] = v[i];
                else if (col <= N)
                    p.Bs[(row_bk * N + (col - 1)) * LP + l] = v[i];
                else if (col < R)
                    p.Cs[(row_bk * N + (col - 1 - N)) * LP + l] = v[i];
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
