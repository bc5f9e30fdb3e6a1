// ss2d_launch.h -- internal interface between the C ABI and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ss2d {

struct ScanParams;

struct VariantInfo {
    const char *name;
    int split;             // 0: one lane per channel; 1: time-split, 4 lanes per channel
    int channels_per_cta;  // channel tile; one ticket per (batch, tile) when merging
    int threads;
    int chunk;             // steps staged per chunk
    int segments;          // time segments per chunk
    size_t smem_bytes;
    cudaError_t (*launch_f32)(const ScanParams &, cudaStream_t);
    cudaError_t (*launch_bf16)(const ScanParams &, cudaStream_t);
};

int num_variants();
const VariantInfo *variant(int i);
int pick_variant(int two_d, int B, int D, int H, int W, int N, int K);
cudaError_t launch_scan_variant(int v, bool bf16, const ScanParams &p, cudaStream_t st);

}  // namespace ss2d
