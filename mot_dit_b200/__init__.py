"""mot_dit_b200 -- B200 (sm_100a) MoT world-action-model forward behind a C ABI.

The package is a thin ctypes binding over ``libmotdit.so`` (built in-tree by
``mot_dit_b200.build``): every step of the forward runs in the library's CUDA
kernels; this module only marshals arguments (device pointers of torch
tensors, CUDA stream handles, host arrays).  Importing works without a GPU;
calling anything that needs the library raises if it is missing -- there is
no CPU fallback.
"""
from ._binding import (  # noqa: F401
    BF16,
    CEWP,
    FP32,
    PROF_CLASSES,
    SEQUENTIAL,
    TRACE_KINDS,
    Wam,
    WamConfig,
    WamError,
    lib,
    library_path,
    op_attention,
    op_attention_noalloc,
    op_linear,
    op_linear_tiled,
    op_attention_joint,
    op_norm_mod,
    patchify,
    preset,
)
