"""B200-native (sm_100a) SS2D path: cross_scan -> selective scan ->
cross_merge, and the 1D one- or two-direction selective scan of Vision Mamba;
forward (plain, gated by SiLU(z), or returning the final states) and backward
(every input's gradient).

The computation lives in the CUDA library built from ``csrc/`` (C ABI in
``include/ss2d.h``); :mod:`.binding` marshals torch tensors into it.
:mod:`.workloads` draws the seeded synthetic inputs.
"""
from .binding import (SS2DError, forward_final_state, selective_scan_bwd, selective_scan_fwd,
                      selective_scan_fwd_gated, ss2d_backward, ss2d_forward, ss2d_forward_gated,
                      ss2d_forward_noalloc, ss2d_num_variants, ss2d_pick_variant,
                      ss2d_scan_directions, ss2d_status_string, ss2d_variant_name)

__all__ = ["ss2d_forward", "ss2d_forward_gated", "ss2d_forward_noalloc", "selective_scan_fwd",
           "selective_scan_fwd_gated", "ss2d_backward", "forward_final_state", "selective_scan_bwd", "ss2d_status_string",
           "ss2d_num_variants", "ss2d_variant_name", "ss2d_pick_variant", "ss2d_scan_directions",
           "SS2DError"]
