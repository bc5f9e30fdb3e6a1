// ss2d_front.cu -- the C ABI of the fused front (include/ss2d.h): argument
// checks, scratch, and the launch sequence front kernel -> scan passes ->
// cross_merge; the bounded-wait fault word and its check.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <limits.h>
#include <stdint.h>
#include <stdio.h>

#include "ss2d.h"
#include "ss2d_front.cuh"
#include "ss2d_launch.h"
#include "ss2d_params.h"

// Set by a kernel whose bounded wait ran out (the code of the wait); read
// and cleared by ss2d_check_waits().
static __device__ int g_wait_fault;

namespace {

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

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

struct FrontCall {
    const void *x;
    const float *conv_w, *conv_b, *W_x, *w_dt, *A_log, *Dskip, *delta_bias;
    int B, D, L, N, K, dtype;
};

int front_validate(const FrontCall &c)
{
    if (c.B < 0 || c.D < 0 || c.L < 0)
        return SS2D_ERR_SHAPE;
    if (c.dtype != SS2D_F32 && c.dtype != SS2D_BF16 && c.dtype != SS2D_F16)
        return SS2D_ERR_DTYPE;
    if (c.K != 1 && c.K != 2)
        return SS2D_ERR_K;
    if (c.N < 1 || c.N > ss2d::kMaxN)
        return SS2D_ERR_N;
    // the conv kernel's CTAs (tiles x channel blocks x B x K) fit one grid dimension
    const long long conv_ctas = ((long long)c.L + ss2d::kFrontTile - 1) / ss2d::kFrontTile *
                                (((long long)c.D + ss2d::kFrontCh - 1) / ss2d::kFrontCh) * c.B *
                                c.K;
    if ((long long)c.L + 7 > INT_MAX || c.B > 65535 || (long long)c.K * c.D > INT_MAX ||
        conv_ctas > 0x7fffffffLL)
        return SS2D_ERR_SHAPE;
    return SS2D_OK;
}

int front_nm(int N) { return ((1 + 2 * N) + 15) / 16 * 16; }

// bytes of the bf16 B operands of every direction and channel block, and of
// the A operands of every (b, k, tile, channel block)
size_t front_wb_bytes(int K, int D, int N)
{
    const int nblk = (D + ss2d::kFrontCh - 1) / ss2d::kFrontCh;
    return (size_t)K * nblk * ss2d::front_bbytes(front_nm(N));
}
size_t front_ab_bytes(int B, int K, int D, int L)
{
    const long long nblk = (D + ss2d::kFrontCh - 1) / ss2d::kFrontCh;
    const long long ntiles = (L + ss2d::kFrontTile - 1) / ss2d::kFrontTile;
    return (size_t)B * K * ntiles * nblk * ss2d::kFrontABytes;
}
size_t up256_(size_t v) { return (v + 255) & ~(size_t)255; }
// scratch of the front kernels: Wb then Ab
size_t front_op_bytes(const FrontCall &c)
{
    return up256_(front_wb_bytes(c.K, c.D, c.N)) + up256_(front_ab_bytes(c.B, c.K, c.D, c.L));
}

// the A blocks within the scratch of front_op_bytes (after the B blocks)
void *front_ab(void *ops, const FrontCall &c)
{
    return static_cast<char *>(ops) + up256_(front_wb_bytes(c.K, c.D, c.N));
}

// the front kernels for one call (conv with the W_x conversion, x_proj); scratch
// rows of pitch LP, ops of front_op_bytes; utile: u only as the A blocks
cudaError_t launch_front(const FrontCall &c, int LP, void *u, float *dt_raw, float *Bs,
                         float *Cs, void *ops, cudaStream_t st, bool utile)
{
    void *Wb = ops;
    void *Ab = front_ab(ops, c);
    ss2d::FrontParams fp{};
    fp.Wb = Wb;
    fp.Ab = Ab;
    fp.utile = utile ? 1 : 0;
    fp.x = c.x;
    fp.conv_w = c.conv_w;
    fp.conv_b = c.conv_b;
    fp.W_x = c.W_x;
    fp.u = u;
    fp.dt_raw = dt_raw;
    fp.Bs = Bs;
    fp.Cs = Cs;
    int *fault = nullptr;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&fault), g_wait_fault);
    if (e != cudaSuccess)
        return e;
    fp.fault = fault;
    fp.B = c.B;
    fp.D = c.D;
    fp.L = c.L;
    fp.LP = LP;
    fp.N = c.N;
    fp.K = c.K;
    fp.NM = front_nm(c.N);
    int tc = 32;
    while (tc < fp.NM)
        tc <<= 1;
    fp.tcols = tc;
    const unsigned ntiles = (unsigned)((c.L + ss2d::kFrontTile - 1) / ss2d::kFrontTile);
    const unsigned nblk = (unsigned)((c.D + ss2d::kFrontCh - 1) / ss2d::kFrontCh);
    {
        const dim3 grid((unsigned)((long long)ntiles * nblk * c.B * c.K));
        switch (c.dtype) {
        case SS2D_BF16:
            ss2d::front_conv_kernel<__nv_bfloat16><<<grid, ss2d::kFrontConvThreads, 0, st>>>(fp);
            break;
        case SS2D_F16:
            ss2d::front_conv_kernel<__half><<<grid, ss2d::kFrontConvThreads, 0, st>>>(fp);
            break;
        default:
            ss2d::front_conv_kernel<float><<<grid, ss2d::kFrontConvThreads, 0, st>>>(fp);
            break;
        }
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    const int smem = ss2d::front_smem_bytes(fp.NM);
    cudaError_t r = cudaFuncSetAttribute(ss2d::front_proj_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (r != cudaSuccess)
        return r;
    return ss2d::launch_kernel(ss2d::front_proj_kernel, dim3(ntiles, (unsigned)c.K, (unsigned)c.B),
                               dim3(ss2d::kFrontProjThreads), (size_t)smem, st, false, fp);
}

int check_front_pointers(const FrontCall &c, const void *const *extra, int nextra, int dev)
{
    const void *ptrs[] = {c.x, c.conv_w, c.conv_b, c.W_x, c.w_dt, c.A_log, c.Dskip, c.delta_bias};
    const int np = c.A_log ? 8 : 5;   // the projection-only call has no scan parameters
    for (int i = 0; i < np; ++i)
        if (!ptrs[i])
            return SS2D_ERR_NULL;
    for (int i = 0; i < nextra; ++i)
        if (!extra[i])
            return SS2D_ERR_NULL;
    for (int i = 0; i < np; ++i)
        if (((uintptr_t)ptrs[i] & 15u) != 0)
            return SS2D_ERR_ALIGN;
    for (int i = 0; i < nextra; ++i)
        if (((uintptr_t)extra[i] & 15u) != 0)
            return SS2D_ERR_ALIGN;
    for (int i = 0; i < np; ++i)
        if (!on_device(ptrs[i], dev))
            return SS2D_ERR_PTR;
    for (int i = 0; i < nextra; ++i)
        if (!on_device(extra[i], dev))
            return SS2D_ERR_PTR;
    return SS2D_OK;
}

// The fused call; with ev (4 events), ev[0..3] are recorded before the front
// kernel, before the scan passes, before the merge and after it.
int front_forward(const FrontCall &c, float *y, cudaStream_t st, cudaEvent_t *ev)
{
    const int B = c.B, D = c.D, L = c.L, N = c.N, K = c.K, dtype = c.dtype;
    const float *w_dt = c.w_dt, *A_log = c.A_log, *Dskip = c.Dskip, *delta_bias = c.delta_bias;
    int rc = front_validate(c);
    if (rc != SS2D_OK)
        return rc;
    if (B == 0 || D == 0 || L == 0)
        return SS2D_OK;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        ss2d::record_error("cudaGetDevice", e);
        return SS2D_ERR_CUDA;
    }
    const void *extra[] = {y};
    rc = check_front_pointers(c, extra, 1, dev);
    if (rc != SS2D_OK)
        return rc;

    const int LP = (L + 7) / 8 * 8;
    const size_t esz = dtype == SS2D_F32 ? 4 : 2;
    // bf16 input: the x_proj A blocks are u itself (no rows of u)
    const bool utile = dtype == SS2D_BF16;
    // the lane kernel reads the front's scratch rows
    const int variant = ss2d::variant_index("lane2_wave");
    const ss2d::Plan pl = ss2d::make_plan(variant, B, D, L, K);
    const size_t rows = (size_t)B * K * D;
    const size_t u_bytes = utile ? 0 : up256(esz * rows * LP);
    const size_t dt_bytes = up256(sizeof(float) * (size_t)B * K * LP);
    const size_t bc_bytes = up256(sizeof(float) * (size_t)B * K * N * LP);
    // two directions, one state group: both add into y (zeroed first)
    // instead of writing rows for a merge kernel
    const bool pair_merge = K == 2 && N <= ss2d::kNP;
    const size_t part_bytes = K > 1 && !pair_merge ? up256(sizeof(float) * rows * L) : 0;
    const size_t hs_bytes = pl.NC > 1 ? up256(sizeof(float) * rows * (pl.NC - 1) * ss2d::kNP) : 0;
    const size_t ds_bytes = pl.NC > 1 ? up256(sizeof(float) * rows * (pl.NC - 1)) : 0;
    const size_t wb_bytes = up256(front_op_bytes(c));
    const size_t total = u_bytes + dt_bytes + 2 * bc_bytes + part_bytes + hs_bytes + ds_bytes +
                         wb_bytes;
    void *scratch = nullptr;
    rc = ss2d::scratch_alloc(&scratch, total, st);
    if (rc != SS2D_OK)
        return rc;
    char *base = static_cast<char *>(scratch);
    void *u = utile ? nullptr : static_cast<void *>(base);
    float *dt_raw = reinterpret_cast<float *>(base + u_bytes);
    float *Bs = reinterpret_cast<float *>(base + u_bytes + dt_bytes);
    float *Cs = reinterpret_cast<float *>(base + u_bytes + dt_bytes + bc_bytes);
    char *rest = base + u_bytes + dt_bytes + 2 * bc_bytes;

    if (ev)
        cudaEventRecord(ev[0], st);
    void *Wb = rest + part_bytes + hs_bytes + ds_bytes;
    e = launch_front(c, LP, u, dt_raw, Bs, Cs, Wb, st, utile);
    if (ev)
        cudaEventRecord(ev[1], st);
    if (e == cudaSuccess) {
        ss2d::ScanParams p{};
        p.x = utile ? front_ab(Wb, c) : u;
        p.utile = utile ? 1 : 0;
        p.delta = nullptr;
        p.A_log = A_log;
        p.Bs = Bs;
        p.Cs = Cs;
        p.Dskip = Dskip;
        p.delta_bias = delta_bias;
        p.B = B;
        p.D = D;
        p.H = 1;
        p.W = L;
        p.L = L;
        p.LP = LP;
        p.N = N;
        p.NS = N;
        p.K = K;
        p.two_d = 0;
        p.front = 1;
        p.dt_raw = dt_raw;
        p.w_dt = w_dt;
        p.out = K > 1 && !pair_merge ? reinterpret_cast<float *>(rest) : y;
        p.ymerge = pair_merge ? y : nullptr;
        p.hstate = pl.NC > 1 ? reinterpret_cast<float *>(rest + part_bytes) : nullptr;
        p.dtsum = pl.NC > 1 ? reinterpret_cast<float *>(rest + part_bytes + hs_bytes) : nullptr;
        p.vec = 16;   // scratch rows of pitch LP (a multiple of 8) start on 16-byte boundaries
        p.ovec = ((((uintptr_t)p.out) & 15) == 0 && ((size_t)L * 4) % 16 == 0) ? 1 : 0;
        if (pair_merge)
            e = cudaMemsetAsync(y, 0, sizeof(float) * (size_t)B * D * L, st);
        if (e == cudaSuccess)
            e = ss2d::launch_scan(pl, dtype, p, st, nullptr);
        if (ev)
            cudaEventRecord(ev[2], st);
        if (e == cudaSuccess && K > 1 && !pair_merge)
            e = ss2d::launch_merge(p.out, y, B, D, 1, L, K, 0, 1, st);
        if (ev)
            cudaEventRecord(ev[3], st);
    }
    const cudaError_t ef = cudaFreeAsync(scratch, st);
    if (e != cudaSuccess) {
        ss2d::record_error("kernel launch", e);
        return SS2D_ERR_CUDA;
    }
    if (ef != cudaSuccess) {
        ss2d::record_error("cudaFreeAsync", ef);
        return SS2D_ERR_CUDA;
    }
    return SS2D_OK;
}

}  // namespace

extern "C" {

int selective_scan_fwd_front(const void *x, const float *conv_w, const float *conv_b,
                             const float *W_x, const float *w_dt, const float *A_log,
                             const float *Dskip, const float *delta_bias, float *y, int B, int D,
                             int L, int N, int K, int dtype, void *stream)
{
    FrontCall c{x, conv_w, conv_b, W_x, w_dt, A_log, Dskip, delta_bias, B, D, L, N, K, dtype};
    return front_forward(c, y, static_cast<cudaStream_t>(stream), nullptr);
}

int selective_scan_fwd_front_timed(const void *x, const float *conv_w, const float *conv_b,
                                   const float *W_x, const float *w_dt, const float *A_log,
                                   const float *Dskip, const float *delta_bias, float *y, int B,
                                   int D, int L, int N, int K, int dtype, void *stream,
                                   float *launch_ms)
{
    if (!launch_ms)
        return SS2D_ERR_NULL;
    FrontCall c{x, conv_w, conv_b, W_x, w_dt, A_log, Dskip, delta_bias, B, D, L, N, K, dtype};
    cudaEvent_t ev[4];
    for (int i = 0; i < 4; ++i) {
        const cudaError_t e = cudaEventCreate(&ev[i]);
        if (e != cudaSuccess) {
            for (int j = 0; j < i; ++j)
                cudaEventDestroy(ev[j]);
            ss2d::record_error("cudaEventCreate", e);
            return SS2D_ERR_CUDA;
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = front_forward(c, y, st, ev);
    for (int i = 0; i < 3; ++i)
        launch_ms[i] = -1.f;
    if (rc == SS2D_OK && !(B == 0 || D == 0 || L == 0)) {
        const cudaError_t e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) {
            ss2d::record_error("cudaStreamSynchronize", e);
            rc = SS2D_ERR_CUDA;
        } else {
            cudaEventElapsedTime(&launch_ms[0], ev[0], ev[1]);
            cudaEventElapsedTime(&launch_ms[1], ev[1], ev[2]);
            if (K > 1)
                cudaEventElapsedTime(&launch_ms[2], ev[2], ev[3]);
        }
    }
    for (int i = 0; i < 4; ++i)
        cudaEventDestroy(ev[i]);
    return rc;
}

int ss2d_front_project(const void *x, const float *conv_w, const float *conv_b, const float *W_x,
                       void *u, float *dt_raw, float *Bs, float *Cs, int B, int D, int L, int N,
                       int K, int dtype, void *stream)
{
    // the w_dt slot of the shared checks is not used here: pass conv_w
    FrontCall c{x, conv_w, conv_b, W_x, conv_w, nullptr, nullptr, nullptr, B, D, L, N, K, dtype};
    int rc = front_validate(c);
    if (rc != SS2D_OK)
        return rc;
    if (B == 0 || D == 0 || L == 0)
        return SS2D_OK;
    if (L % 8 != 0)
        return SS2D_ERR_SHAPE;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        ss2d::record_error("cudaGetDevice", e);
        return SS2D_ERR_CUDA;
    }
    const void *extra[] = {u, dt_raw, Bs, Cs};
    rc = check_front_pointers(c, extra, 4, dev);
    if (rc != SS2D_OK)
        return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *Wb = nullptr;
    rc = ss2d::scratch_alloc(&Wb, front_op_bytes(c), st);
    if (rc != SS2D_OK)
        return rc;
    e = launch_front(c, L, u, dt_raw, Bs, Cs, Wb, st, false);
    const cudaError_t ef = cudaFreeAsync(Wb, st);
    if (e != cudaSuccess) {
        ss2d::record_error("kernel launch", e);
        return SS2D_ERR_CUDA;
    }
    if (ef != cudaSuccess) {
        ss2d::record_error("cudaFreeAsync", ef);
        return SS2D_ERR_CUDA;
    }
    return SS2D_OK;
}

int ss2d_check_waits(void)
{
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_wait_fault, sizeof(int));
    if (e != cudaSuccess) {
        ss2d::record_error("cudaMemcpyFromSymbol", e);
        return SS2D_ERR_CUDA;
    }
    if (v == 0)
        return SS2D_OK;
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_wait_fault, &zero, sizeof(int));
    char msg[160];
    snprintf(msg, sizeof(msg), "a bounded wait ran out of time (%s)",
             v == ss2d::kFaultFrontMma ? "front kernel, tensor-core completion"
                                       : "wait self-test");
    ss2d::record_message(msg);
    (void)e;   // the fault is reported either way
    return SS2D_ERR_CUDA;
}

int ss2d_wait_selftest(int limit_us, void *stream)
{
    if (limit_us < 1 || limit_us > 1000000)
        return SS2D_ERR_SHAPE;
    int *fault = nullptr;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&fault), g_wait_fault);
    if (e == cudaSuccess) {
        ss2d::wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
            fault, (unsigned long long)limit_us * 1000ull);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
        ss2d::record_error("wait self-test launch", e);
        return SS2D_ERR_CUDA;
    }
    return SS2D_OK;
}

}  // extern "C"
