// ss2d_capi.cu -- the C ABI declared in include/ss2d.h: argument checks,
// scratch memory, the host-buffer path, and the launch sequence of a call
// (chunk state pass, carry, output pass, cross_merge).
#include <cuda_runtime.h>
#include <limits.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "ss2d.h"
#include "ss2d_bwd_params.h"
#include "ss2d_params.h"
#include "ss2d_launch.h"

namespace {

thread_local char g_last_error[512] = "";

void set_error(const char *what, cudaError_t e)
{
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", what,
             cudaGetErrorString(e), cudaGetErrorName(e));
}

// One stream-ordered pool per device, created on first use, that keeps its
// memory between calls (release threshold = max) so repeated calls do not
// go back to the driver.
constexpr int kMaxDevices = 64;
std::mutex g_pool_mutex;
cudaMemPool_t g_pools[kMaxDevices] = {};

cudaError_t device_pool(int dev, cudaMemPool_t *out)
{
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_pool_mutex);
    if (!g_pools[dev]) {
        cudaMemPoolProps props;
        memset(&props, 0, sizeof(props));
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool;
        cudaError_t e = cudaMemPoolCreate(&pool, &props);
        if (e != cudaSuccess)
            return e;
        uint64_t thr = UINT64_MAX;
        e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr);
        if (e != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return e;
        }
        g_pools[dev] = pool;
    }
    *out = g_pools[dev];
    return cudaSuccess;
}

int pool_alloc(void **ptr, size_t bytes, cudaStream_t st)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_error("cudaGetDevice", e);
        return SS2D_ERR_CUDA;
    }
    cudaMemPool_t pool;
    e = device_pool(dev, &pool);
    if (e != cudaSuccess) {
        set_error("cudaMemPoolCreate", e);
        return SS2D_ERR_CUDA;
    }
    e = cudaMallocFromPoolAsync(ptr, bytes, pool, st);
    if (e != cudaSuccess) {
        cudaGetLastError();
        set_error("cudaMallocFromPoolAsync", e);
        return SS2D_ERR_ALLOC;
    }
    return SS2D_OK;
}

enum PtrKind { kDevicePtr = 0, kHostPtr = 1, kBadPtr = 2 };

PtrKind pointer_kind(const void *ptr, int cur_dev)
{
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, ptr);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return kBadPtr;
    }
    switch (a.type) {
    case cudaMemoryTypeDevice:
        return a.device == cur_dev ? kDevicePtr : kBadPtr;
    case cudaMemoryTypeManaged:
        return kDevicePtr;
    default:
        return kHostPtr;
    }
}

struct Problem {
    const void *x, *delta, *Bs, *Cs;
    const float *A_log, *Dskip, *delta_bias;
    float *y;
    int B, D, H, W, N, K, dtype, two_d;
    const void *z = nullptr;   // output gate (gated calls)
    float *hlast = nullptr;    // final states (final-state calls)
};

int validate(const Problem &pr)
{
    if (pr.B < 0 || pr.D < 0 || pr.H < 0 || pr.W < 0)
        return SS2D_ERR_SHAPE;
    if (pr.dtype != SS2D_F32 && pr.dtype != SS2D_BF16 && pr.dtype != SS2D_F16)
        return SS2D_ERR_DTYPE;
    if (pr.two_d ? !(pr.K == 1 || pr.K == 2 || pr.K == 4) : !(pr.K == 1 || pr.K == 2))
        return SS2D_ERR_K;
    if (pr.N < 1 || pr.N > ss2d::kMaxN)
        return SS2D_ERR_N;
    const long long L = (long long)pr.H * pr.W;
    if (L > INT_MAX || pr.B > 65535 || (long long)pr.K * pr.D > INT_MAX)
        return SS2D_ERR_SHAPE;
    return SS2D_OK;
}

bool is_empty(const Problem &pr)
{
    return pr.B == 0 || pr.D == 0 || pr.H == 0 || pr.W == 0;
}

int check_pointers(const Problem &pr)
{
    const void *ptrs[] = {pr.x, pr.delta, pr.Bs, pr.Cs, pr.A_log, pr.Dskip, pr.delta_bias, pr.y,
                          pr.z ? pr.z : pr.x};
    for (const void *q : ptrs)
        if (!q)
            return SS2D_ERR_NULL;
    for (const void *q : ptrs)
        if (((uintptr_t)q & 15u) != 0)
            return SS2D_ERR_ALIGN;
    return SS2D_OK;
}

ss2d::ScanParams make_params(const Problem &pr)
{
    ss2d::ScanParams p{};
    p.x = pr.x;
    p.delta = pr.delta;
    p.A_log = pr.A_log;
    p.Bs = pr.Bs;
    p.Cs = pr.Cs;
    p.Dskip = pr.Dskip;
    p.delta_bias = pr.delta_bias;
    p.B = pr.B;
    p.D = pr.D;
    p.H = pr.H;
    p.W = pr.W;
    p.L = pr.H * pr.W;
    p.N = pr.N;
    p.K = pr.K;
    p.two_d = pr.two_d;
    p.hlast = pr.hlast;
    p.NS = pr.N;
    p.LP = pr.H * pr.W;
    return p;
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Device path: every pointer is device memory of the current device.
//   chunked (plan.NC > 1): state pass, carry, output pass;
//   K = 1: the output pass writes y (scan order of direction 0 = pixel order);
//   K > 1: the output pass writes per-direction scan-order rows to scratch
//   and the merge kernel sums them into y in fixed order (directions = true:
//   copies them to y as per-direction pixel-order outputs instead);
//   K = 2 without a gate, at most 16 states: y is zeroed and both
//   directions add into it in the output pass (no rows, no merge kernel).
// Scratch comes from the pool on the stream and goes back to it on the stream.
// plan_B: the batch size the chunk plan is made for (0: pr.B); a slice of a
// larger call keeps the whole call's plan, so that it computes the same bits.
int run_device(const Problem &pr, cudaStream_t st, int variant, bool directions,
               cudaEvent_t *ev = nullptr, int plan_B = 0)
{
    if (ev && pr.N > ss2d::kNP)
        return SS2D_ERR_N;   // per-launch timing covers one state group
    ss2d::ScanParams p = make_params(pr);
    const size_t in_esz = pr.dtype == SS2D_F32 ? 4 : 2;   // bytes per stored input value
    const long long L = p.L;
    const ss2d::Plan pl = ss2d::make_plan(variant, plan_B > 0 ? plan_B : pr.B, pr.D, (int)L, pr.K);
    // two directions, one state group, no gate: the output pass adds both into y
    const bool add_merge = pr.K == 2 && !pr.z && !directions && pr.N <= ss2d::kNP;
    const bool need_part = (pr.K > 1 || pr.z) && !add_merge;   // gated calls merge (the gate runs there)
    const size_t rows = (size_t)pr.B * pr.K * pr.D;
    const size_t part_bytes = need_part ? align256(sizeof(float) * rows * L) : 0;
    const size_t hs_bytes = pl.NC > 1 ? align256(sizeof(float) * rows * (pl.NC - 1) * ss2d::kNP) : 0;
    const size_t ds_bytes = pl.NC > 1 ? align256(sizeof(float) * rows * (pl.NC - 1)) : 0;
    const size_t total = part_bytes + hs_bytes + ds_bytes;
    void *scratch = nullptr;
    if (total > 0) {
        int rc = pool_alloc(&scratch, total, st);
        if (rc != SS2D_OK)
            return rc;
    }
    char *base = static_cast<char *>(scratch);
    p.out = need_part ? reinterpret_cast<float *>(base) : pr.y;
    {
        // vector access to the rows of delta and x (dtype) and of out (float32)
        // needs every row start on a boundary of the vector width
        const size_t esz = in_esz;
        const bool ptr_ok = (((uintptr_t)pr.x | (uintptr_t)pr.delta | (uintptr_t)p.out) & 15) == 0;
        const size_t rb = (size_t)L * esz;
        p.vec = !ptr_ok ? 0 : (rb % 16 == 0 ? 16 : (rb % 8 == 0 ? 8 : 0));
        p.ovec = (ptr_ok && ((size_t)L * 4) % 16 == 0) ? 1 : 0;
    }
    p.hstate = pl.NC > 1 ? reinterpret_cast<float *>(base + part_bytes) : nullptr;
    p.dtsum = pl.NC > 1 ? reinterpret_cast<float *>(base + part_bytes + hs_bytes) : nullptr;
    p.ymerge = add_merge ? pr.y : nullptr;
    cudaError_t e = cudaSuccess;
    if (add_merge)
        e = cudaMemsetAsync(pr.y, 0, sizeof(float) * (size_t)pr.B * pr.D * L, st);
    if (e == cudaSuccess)
        e = ss2d::launch_scan(pl, pr.dtype, p, st, ev);
    if (e == cudaSuccess && add_merge && ev)
        cudaEventRecord(ev[4], st);   // no merge launch
    if (e == cudaSuccess && need_part) {
        e = ss2d::launch_merge(p.out, pr.y, pr.B, pr.D, pr.H, pr.W, pr.K, pr.two_d,
                               directions ? 0 : 1, st, pr.z, pr.dtype);
        if (ev)
            cudaEventRecord(ev[4], st);
    }
    cudaError_t ef = cudaSuccess;
    if (scratch)
        ef = cudaFreeAsync(scratch, st);
    if (e != cudaSuccess) {
        set_error("kernel launch", e);
        return SS2D_ERR_CUDA;
    }
    if (ef != cudaSuccess) {
        set_error("cudaFreeAsync", ef);
        return SS2D_ERR_CUDA;
    }
    return SS2D_OK;
}

// Host path: copy in, run, copy out, synchronise.  A batch of more than one
// element is cut into slices of about kHostSliceBytes of input (at most
// kHostSlices, whole batch elements) that flow through three streams: the
// inputs of
// slice s + 1 are copied in (one copy stream) while slice s is computed on
// the caller's stream and slice s - 1 is copied out (a second copy stream),
// so that the two copy directions and the kernels overlap.  Every slice runs
// with the whole call's chunk plan: the result is bit for bit the device
// path's.
constexpr int kHostSlices = 8;
constexpr size_t kHostSliceBytes = 16u << 20;   // smaller slices scan too few sequences

struct HostStreams {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t ev[2 * kHostSlices + 2] = {};
    int nev = 0;
    cudaError_t create(int n)
    {
        cudaError_t e = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking);
        if (e == cudaSuccess)
            e = cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking);
        for (; nev < n && e == cudaSuccess; ++nev)
            e = cudaEventCreateWithFlags(&ev[nev], cudaEventDisableTiming);
        return e;
    }
    ~HostStreams()
    {
        for (int i = 0; i < nev; ++i)
            cudaEventDestroy(ev[i]);
        if (in)
            cudaStreamDestroy(in);
        if (out)
            cudaStreamDestroy(out);
    }
};

// one element: copy in, run, copy out on the caller's stream
int run_host_whole(const Problem &pr, cudaStream_t st, int variant, const size_t *sz,
                   const size_t *off, size_t total)
{
    void *buf = nullptr;
    int rc = pool_alloc(&buf, total, st);
    if (rc != SS2D_OK)
        return rc;
    char *base = static_cast<char *>(buf);
    const void *src[7] = {pr.x, pr.delta, pr.Bs, pr.Cs, pr.A_log, pr.Dskip, pr.delta_bias};
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < 7 && e == cudaSuccess; ++i)
        e = cudaMemcpyAsync(base + off[i], src[i], sz[i], cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) {
        set_error("cudaMemcpyAsync (host to device)", e);
        cudaFreeAsync(buf, st);
        cudaStreamSynchronize(st);
        return SS2D_ERR_CUDA;
    }
    Problem dp = pr;
    dp.x = base + off[0];
    dp.delta = base + off[1];
    dp.Bs = base + off[2];
    dp.Cs = base + off[3];
    dp.A_log = reinterpret_cast<const float *>(base + off[4]);
    dp.Dskip = reinterpret_cast<const float *>(base + off[5]);
    dp.delta_bias = reinterpret_cast<const float *>(base + off[6]);
    dp.y = reinterpret_cast<float *>(base + off[7]);
    rc = run_device(dp, st, variant, false);
    if (rc == SS2D_OK) {
        e = cudaMemcpyAsync(pr.y, dp.y, sz[7], cudaMemcpyDeviceToHost, st);
        if (e != cudaSuccess) {
            set_error("cudaMemcpyAsync (device to host)", e);
            rc = SS2D_ERR_CUDA;
        }
    }
    cudaFreeAsync(buf, st);
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess && rc == SS2D_OK) {
        set_error("cudaStreamSynchronize", e);
        rc = SS2D_ERR_CUDA;
    }
    return rc;
}

int run_host(const Problem &pr, cudaStream_t st, int variant)
{
    const size_t L = (size_t)pr.H * pr.W;
    const size_t esz = pr.dtype == SS2D_F32 ? 4 : 2;
    // per batch element: x, delta, Bs, Cs, y
    const size_t e_x = (size_t)pr.D * L, e_dl = (size_t)pr.K * pr.D * L;
    const size_t e_bc = (size_t)pr.K * pr.N * L;
    const size_t n_kd = (size_t)pr.K * pr.D;
    auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
    const size_t sz[8] = {pr.B * e_x * esz, pr.B * e_dl * esz, pr.B * e_bc * esz,
                          pr.B * e_bc * esz, n_kd * pr.N * 4, n_kd * 4, n_kd * 4,
                          pr.B * e_x * 4};
    const size_t per_b[8] = {e_x * esz, e_dl * esz, e_bc * esz, e_bc * esz, 0, 0, 0, e_x * 4};
    size_t off[8], total = 0;
    for (int i = 0; i < 8; ++i) {
        off[i] = total;
        total += up(sz[i]);
    }
    const size_t in_bytes = sz[0] + sz[1] + sz[2] + sz[3];
    long long want = (long long)((in_bytes + kHostSliceBytes - 1) / kHostSliceBytes);
    want = want < 1 ? 1 : (want > kHostSlices ? kHostSlices : want);
    const int nsl = pr.B < want ? pr.B : (int)want;
    if (nsl == 1)
        return run_host_whole(pr, st, variant, sz, off, total);
    HostStreams hs;
    cudaError_t e = hs.create(2 * nsl + 2);
    if (e != cudaSuccess) {
        set_error("cudaStreamCreate / cudaEventCreate", e);
        return SS2D_ERR_CUDA;
    }
    cudaEvent_t ready = hs.ev[0], copied_out = hs.ev[1];
    cudaEvent_t *in_done = hs.ev + 2, *computed = hs.ev + 2 + nsl;
    void *buf = nullptr;
    int rc = pool_alloc(&buf, total, st);
    if (rc != SS2D_OK)
        return rc;
    char *base = static_cast<char *>(buf);
    const void *src[7] = {pr.x, pr.delta, pr.Bs, pr.Cs, pr.A_log, pr.Dskip, pr.delta_bias};
    // the copy streams start after everything before this call on `st` (the
    // buffer's allocation included)
    e = cudaEventRecord(ready, st);
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(hs.in, ready, 0);
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(hs.out, ready, 0);
    for (int i = 4; i < 7 && e == cudaSuccess; ++i)   // the parameters, once
        e = cudaMemcpyAsync(base + off[i], src[i], sz[i], cudaMemcpyHostToDevice, hs.in);
    for (int s = 0; s < nsl && e == cudaSuccess && rc == SS2D_OK; ++s) {
        const int b0 = (int)((long long)pr.B * s / nsl), b1 = (int)((long long)pr.B * (s + 1) / nsl);
        for (int i = 0; i < 4 && e == cudaSuccess; ++i)
            e = cudaMemcpyAsync(base + off[i] + b0 * per_b[i],
                                static_cast<const char *>(src[i]) + b0 * per_b[i],
                                (size_t)(b1 - b0) * per_b[i], cudaMemcpyHostToDevice, hs.in);
        if (e == cudaSuccess)
            e = cudaEventRecord(in_done[s], hs.in);
        if (e == cudaSuccess)
            e = cudaStreamWaitEvent(st, in_done[s], 0);
        if (e != cudaSuccess)
            break;
        Problem dp = pr;
        dp.B = b1 - b0;
        dp.x = base + off[0] + b0 * per_b[0];
        dp.delta = base + off[1] + b0 * per_b[1];
        dp.Bs = base + off[2] + b0 * per_b[2];
        dp.Cs = base + off[3] + b0 * per_b[3];
        dp.A_log = reinterpret_cast<const float *>(base + off[4]);
        dp.Dskip = reinterpret_cast<const float *>(base + off[5]);
        dp.delta_bias = reinterpret_cast<const float *>(base + off[6]);
        dp.y = reinterpret_cast<float *>(base + off[7] + b0 * per_b[7]);
        rc = run_device(dp, st, variant, false, nullptr, pr.B);
        if (rc != SS2D_OK)
            break;
        e = cudaEventRecord(computed[s], st);
        if (e == cudaSuccess)
            e = cudaStreamWaitEvent(hs.out, computed[s], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(static_cast<char *>(static_cast<void *>(pr.y)) + b0 * per_b[7],
                                dp.y, (size_t)(b1 - b0) * per_b[7], cudaMemcpyDeviceToHost,
                                hs.out);
    }
    // `st` waits for both copy streams before the buffer goes back to the pool
    cudaError_t e2 = cudaEventRecord(copied_out, hs.out);
    if (e2 == cudaSuccess)
        e2 = cudaStreamWaitEvent(st, copied_out, 0);
    cudaError_t e3 = cudaEventRecord(ready, hs.in);
    if (e3 == cudaSuccess)
        e3 = cudaStreamWaitEvent(st, ready, 0);
    if (e2 == cudaSuccess && e3 == cudaSuccess)
        cudaFreeAsync(buf, st);
    const cudaError_t es = cudaStreamSynchronize(st);
    if (e2 != cudaSuccess || e3 != cudaSuccess) {
        // the streams could not be joined: wait for them before the buffer is freed
        cudaStreamSynchronize(hs.in);
        cudaStreamSynchronize(hs.out);
        cudaFree(buf);
    }
    if (rc != SS2D_OK)
        return rc;
    const cudaError_t ef = e != cudaSuccess ? e : e2 != cudaSuccess ? e2 : e3 != cudaSuccess ? e3 : es;
    if (ef != cudaSuccess) {
        set_error("host-buffer call (copies, stream order)", ef);
        return SS2D_ERR_CUDA;
    }
    return SS2D_OK;
}

int forward(const Problem &pr, void *stream, int variant, bool directions_only = false,
            bool gated = false, bool final_state = false)
{
    if ((gated && !pr.z) || (final_state && !pr.hlast))
        return SS2D_ERR_NULL;
    int rc = validate(pr);
    if (rc != SS2D_OK)
        return rc;
    if (variant < -1 || variant >= ss2d::num_variants())
        return SS2D_ERR_VARIANT;
    if (is_empty(pr))
        return SS2D_OK;
    rc = check_pointers(pr);
    if (rc != SS2D_OK)
        return rc;
    if (variant < 0)
        variant = ss2d::pick_variant(pr.two_d, pr.B, pr.D, pr.H, pr.W, pr.N, pr.K);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_error("cudaGetDevice", e);
        return SS2D_ERR_CUDA;
    }
    const void *ptrs[] = {pr.x, pr.delta, pr.Bs, pr.Cs, pr.A_log, pr.Dskip, pr.delta_bias, pr.y,
                          pr.z ? pr.z : pr.x, pr.hlast ? pr.hlast : pr.x};
    const PtrKind kind = pointer_kind(ptrs[0], dev);
    if (kind == kBadPtr)
        return SS2D_ERR_PTR;
    for (const void *q : ptrs)
        if (pointer_kind(q, dev) != kind)
            return SS2D_ERR_PTR;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (directions_only || gated || final_state)
        return kind == kDevicePtr ? run_device(pr, st, variant, directions_only) : SS2D_ERR_PTR;
    return kind == kDevicePtr ? run_device(pr, st, variant, false) : run_host(pr, st, variant);
}

// Backward: gradients of sum(dy * y).  Device pointers only.  Scratch from
// the pool: chunk entry states and adjoints (when L > 16), the per-direction
// du rows (K > 1) and the two reduction partials.
struct Grads {
    const float *dy;
    float *dx, *ddelta, *dA_log, *dBs, *dCs, *dDskip, *ddelta_bias;
};

int backward(const Problem &pr, const Grads &gr, void *stream)
{
    int rc = validate(pr);
    if (rc != SS2D_OK)
        return rc;
    if (pr.K * (long long)pr.D == 0)
        return SS2D_OK;
    // an empty batch or sequence reads nothing and writes only the parameter
    // gradients (zero); otherwise every pointer is used
    const bool empty = is_empty(pr);
    const void *all[] = {gr.dA_log, gr.dDskip, gr.ddelta_bias, pr.x, pr.delta, pr.Bs, pr.Cs,
                         pr.A_log, pr.Dskip, pr.delta_bias, gr.dy, gr.dx, gr.ddelta, gr.dBs,
                         gr.dCs};
    const int nptr = empty ? 3 : 15;
    for (int i = 0; i < nptr; ++i)
        if (!all[i])
            return SS2D_ERR_NULL;
    for (int i = 0; i < nptr; ++i)
        if (((uintptr_t)all[i] & 15u) != 0)
            return SS2D_ERR_ALIGN;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_error("cudaGetDevice", e);
        return SS2D_ERR_CUDA;
    }
    for (int i = 0; i < nptr; ++i)
        if (pointer_kind(all[i], dev) != kDevicePtr)
            return SS2D_ERR_PTR;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long L = (long long)pr.H * pr.W;
    if (empty) {
        // no step anywhere: the parameter gradients are zero
        const size_t kd = (size_t)pr.K * pr.D;
        e = cudaMemsetAsync(gr.dA_log, 0, sizeof(float) * kd * pr.N, st);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(gr.dDskip, 0, sizeof(float) * kd, st);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(gr.ddelta_bias, 0, sizeof(float) * kd, st);
        if (e != cudaSuccess) {
            set_error("cudaMemsetAsync", e);
            return SS2D_ERR_CUDA;
        }
        return SS2D_OK;
    }
    const ss2d::BwdShape sh = ss2d::backward_shape(pr.B, pr.D, (int)L, pr.K);
    if ((long long)sh.G * pr.B * pr.K > INT_MAX)
        return SS2D_ERR_SHAPE;
    const size_t rows = (size_t)pr.B * pr.K * pr.D;
    const size_t nc1 = (size_t)sh.NC - 1;
    const size_t hs_bytes = align256(sizeof(float) * rows * nc1 * ss2d::kNP);
    const size_t ds_bytes = align256(sizeof(float) * rows * nc1);
    // two directions, one state group: both add their du into dx (zeroed first)
    const bool add_merge = pr.K == 2 && pr.N <= ss2d::kNP;
    const size_t du_bytes = pr.K > 1 && !add_merge ? align256(sizeof(float) * rows * L) : 0;
    const size_t bc_bytes =
        align256(sizeof(float) * pr.B * pr.K * (size_t)sh.G * 2 * pr.N * L);
    const size_t pr_bytes = align256(sizeof(float) * rows * sh.CGN * (pr.N + 2));
    const size_t total = 2 * hs_bytes + 2 * ds_bytes + du_bytes + bc_bytes + pr_bytes;
    void *scratch = nullptr;
    rc = pool_alloc(&scratch, total, st);
    if (rc != SS2D_OK)
        return rc;
    char *base = static_cast<char *>(scratch);
    ss2d::BwdParams p{};
    p.x = pr.x;
    p.delta = pr.delta;
    p.Bs = pr.Bs;
    p.Cs = pr.Cs;
    p.A_log = pr.A_log;
    p.Dskip = pr.Dskip;
    p.delta_bias = pr.delta_bias;
    p.dy = gr.dy;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        float *q = bytes ? reinterpret_cast<float *>(base + off) : nullptr;
        off += bytes;
        return q;
    };
    p.hfwd = take(hs_bytes);
    p.hadj = take(hs_bytes);
    p.dtf = take(ds_bytes);
    p.dta = take(ds_bytes);
    p.du = pr.K > 1 && !add_merge ? take(du_bytes) : gr.dx;
    p.dxmerge = add_merge ? gr.dx : nullptr;
    p.bc_part = take(bc_bytes);
    p.prm_part = take(pr_bytes);
    p.ddelta = gr.ddelta;
    p.B = pr.B;
    p.D = pr.D;
    p.H = pr.H;
    p.W = pr.W;
    p.L = (int)L;
    p.N = pr.N;
    p.K = pr.K;
    p.two_d = pr.two_d;
    p.NC = sh.NC;
    p.G = sh.G;
    p.CPB = sh.CPB;
    p.CGN = sh.CGN;
    p.flip1 = pr.K > 1 ? 1 : 0;
    p.NS = pr.N;
    p.adj_chunks = sh.CGN > 1 ? 1 : 0;
    e = cudaSuccess;
    if (add_merge)
        e = cudaMemsetAsync(gr.dx, 0, sizeof(float) * (size_t)pr.B * pr.D * L, st);
    if (e == cudaSuccess)
        e = ss2d::launch_backward(p, pr.dtype, st);
    if (e == cudaSuccess && pr.K > 1 && !add_merge)
        e = ss2d::launch_merge(p.du, gr.dx, pr.B, pr.D, pr.H, pr.W, pr.K, pr.two_d, 1, st);
    if (e == cudaSuccess)
        e = ss2d::launch_backward_reduce(p, gr.dBs, gr.dCs, gr.dA_log, gr.dDskip,
                                         gr.ddelta_bias, st);
    const cudaError_t ef = cudaFreeAsync(scratch, st);
    if (e != cudaSuccess) {
        set_error("kernel launch", e);
        return SS2D_ERR_CUDA;
    }
    if (ef != cudaSuccess) {
        set_error("cudaFreeAsync", ef);
        return SS2D_ERR_CUDA;
    }
    return SS2D_OK;
}

}  // namespace

namespace ss2d {
int scratch_alloc(void **ptr, size_t bytes, cudaStream_t st) { return pool_alloc(ptr, bytes, st); }
void record_error(const char *what, cudaError_t e) { set_error(what, e); }
void record_message(const char *text) { snprintf(g_last_error, sizeof(g_last_error), "%s", text); }
}  // namespace ss2d

extern "C" {

int ss2d_forward_ex(const void *x, const void *delta, const float *A_log, const void *Bs,
                    const void *Cs, const float *Dskip, const float *delta_bias, float *y,
                    int B, int D, int H, int W, int N, int K, int dtype, void *stream,
                    int variant)
{
    Problem pr{x, delta, Bs, Cs, A_log, Dskip, delta_bias, y, B, D, H, W, N, K, dtype, 1};
    return forward(pr, stream, variant);
}

int ss2d_forward(const void *x, const void *delta, const float *A_log, const void *Bs,
                 const void *Cs, const float *Dskip, const float *delta_bias, float *y,
                 int B, int D, int H, int W, int N, int K, int dtype, void *stream)
{
    return ss2d_forward_ex(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y, B, D, H, W, N, K,
                           dtype, stream, -1);
}

int selective_scan_fwd_ex(const void *u, const void *delta, const float *A_log,
                          const void *Bs, const void *Cs, const float *Dskip,
                          const float *delta_bias, float *y, int B, int D, int L, int N,
                          int K, int dtype, void *stream, int variant)
{
    Problem pr{u, delta, Bs, Cs, A_log, Dskip, delta_bias, y, B, D, 1, L, N, K, dtype, 0};
    return forward(pr, stream, variant);
}

int selective_scan_fwd(const void *u, const void *delta, const float *A_log, const void *Bs,
                       const void *Cs, const float *Dskip, const float *delta_bias, float *y,
                       int B, int D, int L, int N, int K, int dtype, void *stream)
{
    return selective_scan_fwd_ex(u, delta, A_log, Bs, Cs, Dskip, delta_bias, y, B, D, L, N,
                                 K, dtype, stream, -1);
}

int ss2d_forward_gated(const void *x, const void *delta, const float *A_log, const void *Bs,
                       const void *Cs, const float *Dskip, const float *delta_bias,
                       const void *z, float *y, int B, int D, int H, int W, int N, int K,
                       int dtype, void *stream)
{
    Problem pr{x, delta, Bs, Cs, A_log, Dskip, delta_bias, y, B, D, H, W, N, K, dtype, 1, z};
    return forward(pr, stream, -1, false, true);
}

int selective_scan_fwd_gated(const void *u, const void *delta, const float *A_log,
                             const void *Bs, const void *Cs, const float *Dskip,
                             const float *delta_bias, const void *z, float *y, int B, int D,
                             int L, int N, int K, int dtype, void *stream)
{
    Problem pr{u, delta, Bs, Cs, A_log, Dskip, delta_bias, y, B, D, 1, L, N, K, dtype, 0, z};
    return forward(pr, stream, -1, false, true);
}

int ss2d_forward_final_state(const void *x, const void *delta, const float *A_log,
                             const void *Bs, const void *Cs, const float *Dskip,
                             const float *delta_bias, float *y, float *h_last, int B, int D,
                             int H, int W, int N, int K, int dtype, void *stream, int variant)
{
    Problem pr{x, delta, Bs, Cs, A_log, Dskip, delta_bias, y, B, D, H, W, N, K, dtype, 1};
    pr.hlast = h_last;
    return forward(pr, stream, variant, false, false, true);
}

int selective_scan_fwd_final_state(const void *u, const void *delta, const float *A_log,
                                   const void *Bs, const void *Cs, const float *Dskip,
                                   const float *delta_bias, float *y, float *h_last, int B,
                                   int D, int L, int N, int K, int dtype, void *stream,
                                   int variant)
{
    Problem pr{u, delta, Bs, Cs, A_log, Dskip, delta_bias, y, B, D, 1, L, N, K, dtype, 0};
    pr.hlast = h_last;
    return forward(pr, stream, variant, false, false, true);
}

int ss2d_backward(const void *x, const void *delta, const float *A_log, const void *Bs,
                  const void *Cs, const float *Dskip, const float *delta_bias, const float *dy,
                  float *dx, float *ddelta, float *dA_log, float *dBs, float *dCs,
                  float *dDskip, float *ddelta_bias, int B, int D, int H, int W, int N, int K,
                  int dtype, void *stream)
{
    Problem pr{x, delta, Bs, Cs, A_log, Dskip, delta_bias, dx, B, D, H, W, N, K, dtype, 1};
    return backward(pr, Grads{dy, dx, ddelta, dA_log, dBs, dCs, dDskip, ddelta_bias}, stream);
}

int selective_scan_bwd(const void *u, const void *delta, const float *A_log, const void *Bs,
                       const void *Cs, const float *Dskip, const float *delta_bias,
                       const float *dy, float *du, float *ddelta, float *dA_log, float *dBs,
                       float *dCs, float *dDskip, float *ddelta_bias, int B, int D, int L, int N,
                       int K, int dtype, void *stream)
{
    Problem pr{u, delta, Bs, Cs, A_log, Dskip, delta_bias, du, B, D, 1, L, N, K, dtype, 0};
    return backward(pr, Grads{dy, du, ddelta, dA_log, dBs, dCs, dDskip, ddelta_bias}, stream);
}

int ss2d_scan_directions(const void *x, const void *delta, const float *A_log,
                         const void *Bs, const void *Cs, const float *Dskip,
                         const float *delta_bias, float *y_dir, int B, int D, int H, int W,
                         int N, int K, int dtype, int two_d, void *stream, int variant)
{
    Problem pr{x, delta, Bs, Cs, A_log, Dskip, delta_bias, y_dir, B, D, H, W, N, K, dtype,
               two_d ? 1 : 0};
    return forward(pr, stream, variant, true);
}

int ss2d_plan(int two_d, int B, int D, int H, int W, int N, int K, int variant,
              int *chunk_len, int *num_chunks, int *launches)
{
    Problem pr{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
               B, D, H, W, N, K, SS2D_F32, two_d ? 1 : 0};
    int rc = validate(pr);
    if (rc != SS2D_OK)
        return rc;
    if (variant < -1 || variant >= ss2d::num_variants())
        return SS2D_ERR_VARIANT;
    if (variant < 0)
        variant = ss2d::pick_variant(pr.two_d, B, D, H, W, N, K);
    const ss2d::Plan pl = ss2d::make_plan(variant, B, D, H * W, K);
    if (chunk_len)
        *chunk_len = pl.LC;
    if (num_chunks)
        *num_chunks = pl.NC;
    if (launches)
        *launches = pl.launches + (pl.NC > 2 ? 3 : pl.NC > 1 ? 2 : 1) *
                                      ((N + ss2d::kNP - 1) / ss2d::kNP - 1) -
                    (K == 2 && N <= ss2d::kNP ? 1 : 0);   // merged in the scan pass
    return SS2D_OK;
}

int ss2d_forward_timed(const void *x, const void *delta, const float *A_log, const void *Bs,
                       const void *Cs, const float *Dskip, const float *delta_bias, float *y,
                       int B, int D, int H, int W, int N, int K, int dtype, int two_d,
                       void *stream, int variant, float *launch_ms)
{
    if (!launch_ms)
        return SS2D_ERR_NULL;
    Problem pr{x, delta, Bs, Cs, A_log, Dskip, delta_bias, y, B, D, H, W, N, K, dtype,
               two_d ? 1 : 0};
    int rc = validate(pr);
    if (rc != SS2D_OK)
        return rc;
    if (variant < -1 || variant >= ss2d::num_variants())
        return SS2D_ERR_VARIANT;
    if (is_empty(pr))
        return SS2D_OK;
    rc = check_pointers(pr);
    if (rc != SS2D_OK)
        return rc;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_error("cudaGetDevice", e);
        return SS2D_ERR_CUDA;
    }
    const void *ptrs[] = {x, delta, Bs, Cs, A_log, Dskip, delta_bias, y};
    for (const void *q : ptrs)
        if (pointer_kind(q, dev) != kDevicePtr)
            return SS2D_ERR_PTR;
    if (variant < 0)
        variant = ss2d::pick_variant(pr.two_d, B, D, H, W, N, K);
    cudaEvent_t ev[5];
    for (int i = 0; i < 5; ++i) {
        e = cudaEventCreate(&ev[i]);
        if (e != cudaSuccess) {
            for (int j = 0; j < i; ++j)
                cudaEventDestroy(ev[j]);
            set_error("cudaEventCreate", e);
            return SS2D_ERR_CUDA;
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const ss2d::Plan pl = ss2d::make_plan(variant, B, D, H * W, K);
    rc = run_device(pr, st, variant, false, ev);
    if (rc == SS2D_OK) {
        e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) {
            set_error("cudaStreamSynchronize", e);
            rc = SS2D_ERR_CUDA;
        }
    }
    for (int i = 0; i < 4; ++i)
        launch_ms[i] = -1.f;
    if (rc == SS2D_OK) {
        if (pl.NC > 1) {
            cudaEventElapsedTime(&launch_ms[0], ev[0], ev[1]);
            cudaEventElapsedTime(&launch_ms[1], ev[1], ev[2]);
        }
        cudaEventElapsedTime(&launch_ms[2], ev[2], ev[3]);
        if (K > 1)
            cudaEventElapsedTime(&launch_ms[3], ev[3], ev[4]);
    }
    for (int i = 0; i < 5; ++i)
        cudaEventDestroy(ev[i]);
    return rc;
}

int ss2d_num_variants(void) { return ss2d::num_variants(); }

const char *ss2d_variant_name(int i)
{
    const ss2d::VariantInfo *v = ss2d::variant(i);
    return v ? v->name : "";
}

int ss2d_pick_variant(int two_d, int B, int D, int H, int W, int N, int K)
{
    return ss2d::pick_variant(two_d, B, D, H, W, N, K);
}

const char *ss2d_status_string(int status)
{
    switch (status) {
    case SS2D_OK:
        return "ok";
    case SS2D_ERR_NULL:
        return "a required pointer is NULL";
    case SS2D_ERR_SHAPE:
        return "invalid size (negative, or beyond the supported range)";
    case SS2D_ERR_DTYPE:
        return "unsupported dtype";
    case SS2D_ERR_K:
        return "unsupported number of directions K";
    case SS2D_ERR_N:
        return "state size N must be in 1..64 (1..16 for ss2d_forward_timed)";
    case SS2D_ERR_ALIGN:
        return "a pointer is not 16-byte aligned";
    case SS2D_ERR_ALLOC:
        return "device memory allocation failed";
    case SS2D_ERR_CUDA:
        return "CUDA error (see ss2d_last_error)";
    case SS2D_ERR_PTR:
        return "pointers mix host and device memory, or name another device";
    case SS2D_ERR_VARIANT:
        return "unknown kernel variant";
    case SS2D_ERR_SCRATCH:
        return "problem needs more scratch than the fixed buffer of ss2d_forward_noalloc "
               "(SS2D_NOALLOC_SCRATCH_BYTES) holds";
    default:
        return "unknown status";
    }
}

const char *ss2d_last_error(void) { return g_last_error; }

}  // extern "C"
