// ss2d_params.h -- launch parameters and constants shared by the C ABI and
// the kernels.
#pragma once

namespace ss2d {

constexpr int kNP = 16;     // states per channel held by the kernels (N <= 16)
constexpr int kT = 16;      // steps per sub-chunk
constexpr float kLog2e = 1.4426950408889634f;

struct ScanParams {
    const void *x;            // (B,D,H,W) / (B,D,L)
    const void *delta;        // (B,K,D,L) scan order
    const float *A_log;       // (K*D,N)
    const void *Bs;           // (B,K,N,L) scan order
    const void *Cs;           // (B,K,N,L) scan order
    const float *Dskip;       // (K*D)
    const float *delta_bias;  // (K*D)
    float *out;               // y_k in scan order, row (b,k,d) at out + ((b*K+k)*D+d)*L
                              // (K = 1: y itself)
    float *hstate;            // (B,K,D,NC-1,16): chunk end states, then entry states
    float *dtsum;             // (B,K,D,NC-1): sum of dt over every chunk but the last
    int B, D, H, W, L, N, K;
    int two_d;                // 1: SS2D scan orders; 0: 1D (k = 1 reversed)
    int LC;                   // steps per chunk (multiple of kT)
    int NC;                   // chunks per sequence
    int vec;                  // 16 / 8: byte width of vector loads of delta and x rows; 0: none
    int ovec;                 // 1: rows of out allow 16-byte vector stores
    float *hlast;             // (B,K,D,NS): state after each direction's last step, or null
    // state groups: a call with more than 16 states runs the passes once per
    // group of at most 16 (the states of a channel never interact)
    int n0;                   // first state of this group
    int NS;                   // states per row of A_log, Bs, Cs, hlast (N is this group's count)
    int accum;                // 1: add this group's output to `out` (skip term left out)
    // row pitch (elements) of the rows of x / u, delta, Bs and Cs: L for the
    // caller's arrays, L rounded up to 8 for the fused front's scratch
    int LP;
    // fused front: u per direction (B,K,D,LP) in scan order in x, no delta;
    // delta = w_dt[k*D+d] * dt_raw[b,k,l]; Bs, Cs float32 (B,K,N,LP)
    int front;
    // fused front with bf16 input: u only as the x_proj A blocks, x of
    // ((b*K+k)*tiles + l/128)*blocks + d/64 blocks of 16 KB, element (l, d)
    // at (l%128/8)*1024 + (d%64)*16 + (l%8)*2 bytes (blocks of 64 channels)
    int utile;
    const float *dt_raw;      // (B,K,LP)
    const float *w_dt;        // (K*D)
    // K = 2 (no column-major direction), one state group: both directions
    // add their outputs into ymerge (B,D,L), zero on entry, with float
    // atomic adds; the two terms meet in either order and a + b = b + a
    // exactly, so ymerge ends as y_0 + y_1 bit for bit, cross_merge's sum.
    // Null: the output pass writes out and a merge kernel sums.
    float *ymerge;
};

}  // namespace ss2d
