// ss2d_scan_f16.cu -- scan passes for float16 inputs.
#include <cuda_fp16.h>

#include "ss2d_scan_launch.cuh"

namespace ss2d {

cudaError_t launch_scan_f16(const Plan &plan, ScanParams &p, cudaStream_t st, cudaEvent_t *ev)
{
    return launch_scan_t<__half>(plan, p, st, ev);
}

}  // namespace ss2d
