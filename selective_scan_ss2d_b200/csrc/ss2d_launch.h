// ss2d_launch.h -- internal interface between the C ABI and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ss2d {

struct ScanParams;

struct VariantInfo {
    const char *name;
    int G, JW, J, WC, I;
    int channels_per_cta;
    int threads;
    int chunk;
    size_t smem_bytes;
    cudaError_t (*launch_f32)(const ScanParams &, cudaStream_t);
    cudaError_t (*launch_bf16)(const ScanParams &, cudaStream_t);
};

int num_variants();
const VariantInfo *variant(int i);
int pick_variant(int two_d, int B, int D, int H, int W, int N, int K);
cudaError_t launch_scan_variant(int v, bool bf16, const ScanParams &p, cudaStream_t st);
cudaError_t launch_merge(int K, const float *part, float *y, long long DL, long long total,
                         cudaStream_t st);

}  // namespace ss2d
