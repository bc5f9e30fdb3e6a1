// ss2d_bwd_params.h -- launch parameters of the backward pass, shared by the
// C ABI and the kernels (ss2d_backward.cuh).
#pragma once

#include "ss2d_params.h"

namespace ss2d {

struct BwdParams {
    const void *x, *delta, *Bs, *Cs;   // forward inputs (dtype)
    const float *A_log, *Dskip, *delta_bias;
    const float *dy;                   // (B,D,H,W) / (B,D,L) float32
    float *hfwd;       // (B,K,D,NC-1,16): chunk end states -> entry states of chunks 1..NC-1
    float *dtf;        // (B,K,D,NC-1): sum of dt of chunks 0..NC-2
    float *hadj;       // (B,K,D,NC-1,16): Q in reversed chunk order -> G of chunks NC-2..0
    float *dta;        // (B,K,D,NC-1): sum of dt of chunks NC-1..1
    float *du;         // du rows (direction 1 in pixel order when flip1); dx itself when K = 1
    float *ddelta;     // (B,K,D,L) float32, scan order
    float *bc_part;    // (B,K,G,2,NS,L): dB | dC summed over one group of 32 channels
    float *prm_part;   // (B,K,D,CGN,NS+2): dA (natural A), dDskip, dbias per chunk group
    int B, D, H, W, L, N, K, two_d;
    int NC;            // chunks of kT steps
    int G;             // channel groups of 32
    int CPB;           // chunks per CTA
    int CGN;           // chunk groups (gridDim.y)
    int flip1;         // store direction 1's du in pixel order (the merge's layout)
    // state groups (more than 16 states): N is this group's count
    int n0;            // first state of this group
    int NS;            // states per row of A_log, Bs, Cs (the call's N)
    int accum;         // 1: add ddelta, du to the rows (no skip term, no dDskip)
    int adj_chunks;    // 1: local adjoints and their carry are needed (CGN > 1)
    // K = 2, one state group: both directions add their du into dxmerge
    // (B,D,H,W) / (B,D,L), zero on entry, with float atomic adds (two terms:
    // the same bits in either order, the merge kernel's sum); du unused.
    // Null: du rows and a merge kernel.
    float *dxmerge;
};

constexpr int kBwdLanes = 32;
}  // namespace ss2d
