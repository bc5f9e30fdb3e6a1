// ss2d_scan_bf16.cu -- scan passes for bfloat16 inputs.
#include "ss2d_scan_launch.cuh"

namespace ss2d {

cudaError_t launch_scan_bf16(const Plan &plan, ScanParams &p, cudaStream_t st, cudaEvent_t *ev)
{
    return launch_scan_t<__nv_bfloat16>(plan, p, st, ev);
}

}  // namespace ss2d
