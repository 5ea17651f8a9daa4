"""SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).

    Y = Xh L1 L2 + Q(Xh) Q(R) + bias,   Xh = X diag(lambda)^-1

The product is the C-ABI library ``libsvdq.so`` (include/svdq.h); this
package is a thin ctypes binding with the same call names.  Every step of the
layer runs in the library's CUDA kernels; there is no CPU fallback, and the
binding raises if the library is missing.
"""

from .binding import (  # noqa: F401
    SvdqError,
    attach_lora,
    channel_absmax,
    lib_path,
    linear,
    load,
    pack_residual,
    packed_sizes,
    quantize_act,
    selftest_wait_timeout,
    set_launch_overlap,
    set_linear_path,
    set_wait_timeout,
    status_string,
    sync_status,
)
