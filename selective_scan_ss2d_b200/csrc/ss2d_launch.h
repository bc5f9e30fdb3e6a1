// ss2d_launch.h -- internal interface between the C ABI and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ss2d {

struct ScanParams;

constexpr int kMaxN = 64;   // states per channel a forward call accepts

// Launch kern on st; dependent = true launches it as a programmatic
// dependent of the previous kernel on the stream (it may start before that
// one finishes and waits in-kernel, with grid_dependency_wait, before it
// reads that kernel's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, bool dependent, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (dependent) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// A kernel variant: layout, CTA width (wc warps) and chunking policy
// (chunk = 0: chosen from the shape; chunk > 0: that many steps per chunk;
// chunk = -2: about 128 steps, fitted to the sequence length; chunk = -3:
// chunks for about one wave of CTAs; chunk = -1: never chunk).
struct VariantInfo {
    const char *name;
    int wc;
    int chunk;
    int regs;   // register cap per thread the kernels are compiled for
    int layout; // 0: one lane per channel (chunk_scan_kernel);
                // 2: one lane per channel, cp.async staging (lane_scan_kernel)
};

// How one call is executed.
struct Plan {
    int variant;
    int wc;
    int regs;
    int layout;
    int LC;        // steps per chunk (multiple of 32)
    int NC;        // chunks per sequence
    int launches;  // kernel launches of a forward call
};

int num_variants();
int variant_index(const char *name);   // -1 if there is no variant of that name
const VariantInfo *variant(int i);
int pick_variant(int two_d, int B, int D, int H, int W, int N, int K);
Plan make_plan(int variant, int B, int D, int L, int K);

// Launch the scan passes (state, carry, output) for a plan; the caller has
// set p.out (and p.hstate / p.dtsum when plan.NC > 1) and p.N to the call's
// state count (up to kMaxN; more than 16 states run as groups of 16).  If ev is not null,
// ev[0..3] are recorded on the stream before the state pass, the carry, the
// output pass and after it (the first two only when the plan is chunked).
cudaError_t launch_scan(const Plan &plan, int dtype, ScanParams &p, cudaStream_t st,
                        cudaEvent_t *ev = nullptr);
// the same for one input dtype (ss2d_scan_bf16.cu, ss2d_scan_f32.cu, ss2d_scan_f16.cu)
cudaError_t launch_scan_bf16(const Plan &plan, ScanParams &p, cudaStream_t st, cudaEvent_t *ev);
cudaError_t launch_scan_f32(const Plan &plan, ScanParams &p, cudaStream_t st, cudaEvent_t *ev);
cudaError_t launch_scan_f16(const Plan &plan, ScanParams &p, cudaStream_t st, cudaEvent_t *ev);
// cross_merge of the scan-order rows in `part` into y (sum = 1) or into the
// per-direction pixel-order copy (sum = 0); with z (sum = 1 only), y is
// multiplied by SiLU(z) (z in the layout of y; zt = the ss2d_dtype of z).
cudaError_t launch_merge(const float *part, float *y, int B, int D, int H, int W, int K,
                         int two_d, int sum, cudaStream_t st, const void *z = nullptr,
                         int zt = 0);

// Backward pass (ss2d_backward.cu): chunks of 16 steps, NC per sequence; G
// groups of 32 channels; CPB chunks per CTA in CGN groups.
struct BwdParams;
struct BwdShape {
    int NC, G, CPB, CGN;
};
BwdShape backward_shape(int B, int D, int L, int K);
// local pass, both carries and the final pass (the caller has filled every
// field of p, scratch included)
cudaError_t launch_backward(const BwdParams &p, int dtype, cudaStream_t st);
// dBs, dCs from the channel-group partials; dA_log, dDskip, ddelta_bias from
// the per-chunk-group partials
cudaError_t launch_backward_reduce(const BwdParams &p, float *dBs, float *dCs, float *dA_log,
                                   float *dDskip, float *ddelta_bias, cudaStream_t st);

// Scratch from the device's stream-ordered pool (ss2d_capi.cu), on st.
int scratch_alloc(void **ptr, size_t bytes, cudaStream_t st);

// Text that ss2d_last_error() returns on the calling thread.
void record_error(const char *what, cudaError_t e);
void record_message(const char *text);

}  // namespace ss2d
