"""FLARE++ token-mixer forward for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libflarepp.so`` (C ABI in
include/flarepp.h); ``binding`` is its thin Python binding.  ``workloads``
draws the seeded synthetic inputs.  Importing the binding raises if the
library has not been built: there is no CPU fallback.
"""
from . import workloads  # noqa: F401

_BINDING_NAMES = {"mixer_fwd", "mixer_fwd_plain", "flare_fwd", "mixer_fwd_host", "workspace_bytes",
                  "selected_path", "check_device_status", "FlareppError", "PATH_AUTO", "PATH_SIMT",
                  "PATH_TCGEN05"}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
