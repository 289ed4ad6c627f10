"""B200 (sm_100a) FLARE / FLARE++ mixer, forward and backward.

The compute lives in ``libflare.so`` (hand-written CUDA kernels behind the C
ABI of ``include/flare.h``).  This package is a thin ctypes binding: it checks
tensor types, passes device pointers and sizes, and raises ``FlareError`` on a
non-OK status.  PyTorch only provides device memory and streams.  There is no
CPU fallback: if the library cannot be loaded, every call raises.
"""
from ._binding import (  # noqa: F401
    FLARE_VARIANT_FLARE,
    FLARE_VARIANT_FLAREPP,
    FLARE_VARIANT_FLAREPP_OUT,
    FLARE_VARIANT_FLARE_BWD,
    FLARE_VARIANT_FLAREPP_BWD,
    FlareError,
    Status,
    flare_last_device_status,
    flare_mixer_bwd,
    flare_mixer_bwd_train,
    flare_mixer_fwd,
    flare_mixer_fwd_train,
    flare_mixer_fwd_static,
    flare_probe_pipe_rates,
    flare_selftest_wait_timeout,
    flare_static_last_device_status,
    flare_status_string,
    flare_workspace_bytes,
    flarepp_mixer_bwd,
    flarepp_mixer_bwd_train,
    flarepp_mixer_fwd,
    flarepp_mixer_fwd_train,
    flarepp_mixer_out_fwd,
    library_path,
    load_library,
)
from . import cp  # noqa: F401,E402  (context-parallel forward and backward over torch.distributed)
from .autograd import flare_mixer, flarepp_mixer  # noqa: F401,E402  (torch.autograd wrappers)
