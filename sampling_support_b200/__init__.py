"""B200 (sm_100a) vocabulary scoring over the full vocabulary and a sampling
support: C-ABI library libvs.so (hand-written CUDA kernels) plus a thin
ctypes binding.  PyTorch is used only for device memory and streams."""

from ._binding import (  # noqa: F401
    LIB_PATH,
    VsError,
    fused_lmhead_bwd,
    fused_lmhead_merge,
    fused_lmhead_partial,
    fused_lmhead_score,
    l1_distance,
    l1_weight_sum,
    load,
    score_bwd,
    score_fwd,
    support_lmhead_score,
)
from ._binding import (  # noqa: F401
    ROW_BAD_SUPPORT_ID,
    ROW_DEVICE_TIMEOUT,
    ROW_DUP_SUPPORT_ID,
    ROW_EMPTY_SUPPORT,
    ROW_NONFINITE_INPUT,
    ROW_TARGET_NOT_IN_SUPPORT,
    ROW_TARGET_OUT_OF_RANGE,
    VS_GRAD_ACCUMULATE,
    VS_GRAD_DENSE,
    VS_GRAD_SPARSE,
)
