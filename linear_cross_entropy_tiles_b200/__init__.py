"""B200-native fused linear cross-entropy (FLCE).

``binding`` exposes the C ABI of ``_build/libflce.so`` (include/flce.h) under
the same names (the fused LM-head loss, and the cross-entropy path for callers
that already hold the logits); ``dp`` runs it data-parallel over torch.distributed ranks;
``inputs`` holds the seeded synthetic workloads.
"""
from .binding import (ce_backward, ce_forward, ce_fused, ce_workspace, flce_ce_backward,
                      flce_ce_fused,
                      flce_ce_forward, flce_ce_problem_t, flce_ce_workspace_size,
                      make_ce_problem)
from .binding import (FLCE_BF16, FLCE_FP32, FLCE_SCHEDULE_AUTO, FLCE_SCHEDULE_FUSED_FORWARD,
                      FLCE_SCHEDULE_RECOMPUTE, FLCE_OP_BACKWARD, FLCE_OP_FORWARD, FLCE_OP_FUSED,
                      FlceError, backward, count_valid, flce_backward, flce_count_valid,
                      dw_slice_bounds, flce_dw_slice_rows, flce_forward, flce_fused,
                      flce_fused_global, flce_fused_global_sliced,
                      flce_get_device_status, flce_kernel_name, flce_last_launch_count,
                      flce_profile_start, flce_profile_stop, flce_selftest_wait_timeout, flce_problem_t,
                      flce_set_schedule, flce_set_wait_limit_ns, flce_set_workspace_limit, flce_status_string, flce_workspace_size, forward,
                      fused, make_problem, workspace)
