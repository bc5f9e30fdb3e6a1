// ss2d_scan_f32.cu -- scan passes for float32 inputs.
#include "ss2d_scan_launch.cuh"

namespace ss2d {

cudaError_t launch_scan_f32(const Plan &plan, ScanParams &p, cudaStream_t st, cudaEvent_t *ev)
{
    return launch_scan_t<float>(plan, p, st, ev);
}

}  // namespace ss2d
