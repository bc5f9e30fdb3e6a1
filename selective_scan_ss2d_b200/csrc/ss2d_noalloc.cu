// ss2d_noalloc.cu -- ss2d_forward_noalloc: the SS2D forward call with its
// scratch in a fixed device buffer that is part of this library's device
// image, so that a call allocates no memory.
//
// Who cannot allocate, and why:
//   * programs whose own caching allocator reserves (nearly) all device memory
//     when they start: a second allocator in the same process then fails, or
//     makes the first one give back cached blocks it will have to take again;
//   * latency-bound loops (serving, real-time pipelines): the stream-ordered
//     pool behind ss2d_forward grows on its first calls for each new largest
//     shape, and growing it calls into the driver;
//   * processes held to a fixed, known device footprint once they run (several
//     models packed on one GPU, hard per-process memory quotas).
//
// The scratch of a call is what ss2d_forward takes from its pool: the
// per-direction scan-order output rows (K > 1) and, when the sequences are
// split into chunks, the chunk end states and the sums of dt per chunk.
//
// Every call asks cudaGetSymbolAddress, with the call's device current, for
// the buffer's address in that device's context (after the first call it is
// a table lookup in the runtime).  Nothing is cached across calls, so a
// context that was torn down and created again (cudaDeviceReset) gives the
// new context's address, never a stale one.  The first call on a device loads
// this file's module, which is when the buffer's memory is reserved, so the
// first call on a device belongs before any stream capture begins.  No word of the buffer has to start at zero: the
// chunk state pass writes every end state and dt sum that the carry kernel
// and the output pass read, and the output pass writes every row element the
// merge kernel reads.  There is one buffer per device, so calls on one device
// whose work can overlap in time race on it: they must be serialised (one
// stream, or streams ordered by events).
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "ss2d.h"
#include "ss2d_launch.h"
#include "ss2d_params.h"

static __device__ __align__(256) char g_noalloc_scratch[SS2D_NOALLOC_SCRATCH_BYTES];

namespace {

// Address of g_noalloc_scratch on the current device, looked up on every call.
cudaError_t scratch_address(char **out)
{
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess)
        return e;
    *out = static_cast<char *>(ptr);
    return cudaSuccess;
}

size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

bool on_device(const void *q, int dev)
{
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, q) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return (a.type == cudaMemoryTypeDevice && a.device == dev) ||
           a.type == cudaMemoryTypeManaged;
}

}  // namespace

extern "C" int ss2d_forward_noalloc(const void *x, const void *delta, const float *A_log,
                                    const void *Bs, const void *Cs, const float *Dskip,
                                    const float *delta_bias, float *y, int B, int D, int H,
                                    int W, int N, int K, int dtype, void *stream)
{
    // shape, K and N rules of ss2d_forward (ss2d_plan applies the same checks)
    int LC = 0, NC = 0, launches = 0;
    int rc = ss2d_plan(1, B, D, H, W, N, K, -1, &LC, &NC, &launches);
    if (rc != SS2D_OK)
        return rc;
    if (dtype != SS2D_F32 && dtype != SS2D_BF16 && dtype != SS2D_F16)
        return SS2D_ERR_DTYPE;
    if (B == 0 || D == 0 || H == 0 || W == 0)
        return SS2D_OK;
    const void *ptrs[] = {x, delta, Bs, Cs, A_log, Dskip, delta_bias, y};
    for (const void *q : ptrs)
        if (!q)
            return SS2D_ERR_NULL;
    for (const void *q : ptrs)
        if (((uintptr_t)q & 15u) != 0)
            return SS2D_ERR_ALIGN;

    const int variant = ss2d::pick_variant(1, B, D, H, W, N, K);
    const long long L = (long long)H * W;
    const ss2d::Plan pl = ss2d::make_plan(variant, B, D, (int)L, K);
    const size_t rows = (size_t)B * K * D;
    // K = 2, one state group: both directions add into y (zeroed first)
    const bool add_merge = K == 2 && N <= ss2d::kNP;
    const size_t part_bytes = K > 1 && !add_merge ? round256(sizeof(float) * rows * (size_t)L) : 0;
    const size_t hs_bytes =
        pl.NC > 1 ? round256(sizeof(float) * rows * (size_t)(pl.NC - 1) * ss2d::kNP) : 0;
    const size_t ds_bytes = pl.NC > 1 ? round256(sizeof(float) * rows * (size_t)(pl.NC - 1)) : 0;
    const size_t need = part_bytes + hs_bytes + ds_bytes;
    if (need > (size_t)SS2D_NOALLOC_SCRATCH_BYTES) {
        char msg[160];
        snprintf(msg, sizeof(msg), "scratch needed: %zu bytes; fixed buffer: %zu bytes", need,
                 (size_t)SS2D_NOALLOC_SCRATCH_BYTES);
        ss2d::record_message(msg);
        return SS2D_ERR_SCRATCH;
    }

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        ss2d::record_error("cudaGetDevice", e);
        return SS2D_ERR_CUDA;
    }
    for (const void *q : ptrs)
        if (!on_device(q, dev))
            return SS2D_ERR_PTR;
    char *base = nullptr;
    e = scratch_address(&base);
    if (e != cudaSuccess) {
        ss2d::record_error("cudaGetSymbolAddress", e);
        return SS2D_ERR_CUDA;
    }

    ss2d::ScanParams p{};
    p.x = x;
    p.delta = delta;
    p.A_log = A_log;
    p.Bs = Bs;
    p.Cs = Cs;
    p.Dskip = Dskip;
    p.delta_bias = delta_bias;
    p.B = B;
    p.D = D;
    p.H = H;
    p.W = W;
    p.L = (int)L;
    p.LP = (int)L;
    p.N = N;
    p.NS = N;
    p.K = K;
    p.two_d = 1;
    p.out = K > 1 && !add_merge ? reinterpret_cast<float *>(base) : y;
    p.ymerge = add_merge ? y : nullptr;
    p.hstate = pl.NC > 1 ? reinterpret_cast<float *>(base + part_bytes) : nullptr;
    p.dtsum = pl.NC > 1 ? reinterpret_cast<float *>(base + part_bytes + hs_bytes) : nullptr;
    {
        // row vector width of delta/x (dtype) and of out (float32), as ss2d_forward
        const size_t esz = dtype == SS2D_F32 ? 4 : 2;
        const bool ptr_ok = (((uintptr_t)x | (uintptr_t)delta | (uintptr_t)p.out) & 15) == 0;
        const size_t rb = (size_t)L * esz;
        p.vec = !ptr_ok ? 0 : (rb % 16 == 0 ? 16 : (rb % 8 == 0 ? 8 : 0));
        p.ovec = (ptr_ok && ((size_t)L * 4) % 16 == 0) ? 1 : 0;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (add_merge)
        e = cudaMemsetAsync(y, 0, sizeof(float) * (size_t)B * D * L, st);
    if (e == cudaSuccess)
        e = ss2d::launch_scan(pl, dtype, p, st, nullptr);
    if (e == cudaSuccess && K > 1 && !add_merge)
        e = ss2d::launch_merge(p.out, y, B, D, H, W, K, 1, 1, st);
    if (e != cudaSuccess) {
        ss2d::record_error("kernel launch", e);
        return SS2D_ERR_CUDA;
    }
    return SS2D_OK;
}
