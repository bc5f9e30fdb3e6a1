// ss2d_capi.cu -- the C ABI declared in include/ss2d.h: argument checks,
// scratch memory, the host-buffer path, and the launch of the scan kernel
// (per-direction pixel-order partials, merged in fixed order by the last CTA
// of each channel tile).
#include <cuda_runtime.h>
#include <limits.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "ss2d.h"
#include "ss2d_kernels.cuh"
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
};

int validate(const Problem &pr)
{
    if (pr.B < 0 || pr.D < 0 || pr.H < 0 || pr.W < 0)
        return SS2D_ERR_SHAPE;
    if (pr.dtype != SS2D_F32 && pr.dtype != SS2D_BF16)
        return SS2D_ERR_DTYPE;
    if (pr.two_d ? !(pr.K == 1 || pr.K == 2 || pr.K == 4) : !(pr.K == 1 || pr.K == 2))
        return SS2D_ERR_K;
    if (pr.N < 1 || pr.N > ss2d::kNP)
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
    const void *ptrs[] = {pr.x, pr.delta, pr.Bs, pr.Cs, pr.A_log, pr.Dskip, pr.delta_bias, pr.y};
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
    return p;
}

// Device path: every pointer is device memory of the current device.
// K = 1: the scan writes y directly.  K > 1: the scan writes per-direction
// partials to pool scratch, and the last CTA of each channel tile adds them
// into y (tickets zeroed here, on the stream, before the launch).
int run_device(const Problem &pr, cudaStream_t st, int variant)
{
    ss2d::ScanParams p = make_params(pr);
    const bool bf16 = pr.dtype == SS2D_BF16;
    const long long DL = (long long)pr.D * p.L;
    if (pr.K == 1) {
        p.out = pr.y;
        p.out_b_stride = DL;
        p.out_k_stride = 0;
        p.merge = 0;
        cudaError_t e = ss2d::launch_scan_variant(variant, bf16, p, st);
        if (e != cudaSuccess) {
            set_error("scan kernel launch", e);
            return SS2D_ERR_CUDA;
        }
        return SS2D_OK;
    }
    const ss2d::VariantInfo *vi = ss2d::variant(variant);
    const long long tiles = (pr.D + vi->channels_per_cta - 1) / vi->channels_per_cta;
    const size_t part_bytes = sizeof(float) * (size_t)pr.B * pr.K * DL;
    const size_t part_up = (part_bytes + 255) & ~(size_t)255;
    const size_t ticket_bytes = sizeof(unsigned int) * (size_t)pr.B * tiles;
    void *scratch = nullptr;
    int rc = pool_alloc(&scratch, part_up + ticket_bytes, st);
    if (rc != SS2D_OK)
        return rc;
    p.out = static_cast<float *>(scratch);
    p.out_b_stride = (long long)pr.K * DL;
    p.out_k_stride = DL;
    p.y = pr.y;
    p.tickets = reinterpret_cast<unsigned int *>(static_cast<char *>(scratch) + part_up);
    p.merge = 1;
    cudaError_t e = cudaMemsetAsync(p.tickets, 0, ticket_bytes, st);
    if (e == cudaSuccess)
        e = ss2d::launch_scan_variant(variant, bf16, p, st);
    cudaError_t ef = cudaFreeAsync(scratch, st);
    if (e != cudaSuccess) {
        set_error("scan kernel launch", e);
        return SS2D_ERR_CUDA;
    }
    if (ef != cudaSuccess) {
        set_error("cudaFreeAsync", ef);
        return SS2D_ERR_CUDA;
    }
    return SS2D_OK;
}

// Per-direction outputs only: the scan kernel writes straight into y_dir.
int run_directions(const Problem &pr, cudaStream_t st, int variant)
{
    ss2d::ScanParams p = make_params(pr);
    const long long DL = (long long)pr.D * p.L;
    p.out = pr.y;
    p.out_b_stride = (long long)pr.K * DL;
    p.out_k_stride = DL;
    p.merge = 0;
    cudaError_t e = ss2d::launch_scan_variant(variant, pr.dtype == SS2D_BF16, p, st);
    if (e != cudaSuccess) {
        set_error("scan kernel launch", e);
        return SS2D_ERR_CUDA;
    }
    return SS2D_OK;
}

// Host path: copy in, run, copy out, synchronise.
int run_host(const Problem &pr, cudaStream_t st, int variant)
{
    const size_t L = (size_t)pr.H * pr.W;
    const size_t esz = pr.dtype == SS2D_BF16 ? 2 : 4;
    const size_t n_x = (size_t)pr.B * pr.D * L;
    const size_t n_dl = (size_t)pr.B * pr.K * pr.D * L;
    const size_t n_bc = (size_t)pr.B * pr.K * pr.N * L;
    const size_t n_kd = (size_t)pr.K * pr.D;
    auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
    const size_t sz[8] = {n_x * esz, n_dl * esz, n_bc * esz, n_bc * esz,
                          n_kd * pr.N * 4, n_kd * 4, n_kd * 4, n_x * 4};
    size_t off[8], total = 0;
    for (int i = 0; i < 8; ++i) {
        off[i] = total;
        total += up(sz[i]);
    }
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
    rc = run_device(dp, st, variant);
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

int forward(const Problem &pr, void *stream, int variant, bool directions_only = false)
{
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
    const void *ptrs[] = {pr.x, pr.delta, pr.Bs, pr.Cs, pr.A_log, pr.Dskip, pr.delta_bias, pr.y};
    const PtrKind kind = pointer_kind(ptrs[0], dev);
    if (kind == kBadPtr)
        return SS2D_ERR_PTR;
    for (const void *q : ptrs)
        if (pointer_kind(q, dev) != kind)
            return SS2D_ERR_PTR;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (directions_only)
        return kind == kDevicePtr ? run_directions(pr, st, variant) : SS2D_ERR_PTR;
    return kind == kDevicePtr ? run_device(pr, st, variant) : run_host(pr, st, variant);
}

}  // namespace

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

int ss2d_scan_directions(const void *x, const void *delta, const float *A_log,
                         const void *Bs, const void *Cs, const float *Dskip,
                         const float *delta_bias, float *y_dir, int B, int D, int H, int W,
                         int N, int K, int dtype, int two_d, void *stream, int variant)
{
    Problem pr{x, delta, Bs, Cs, A_log, Dskip, delta_bias, y_dir, B, D, H, W, N, K, dtype,
               two_d ? 1 : 0};
    return forward(pr, stream, variant, true);
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
        return "state size N must be in 1..16";
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
    default:
        return "unknown status";
    }
}

const char *ss2d_last_error(void) { return g_last_error; }

}  // extern "C"
