"""B200-native (sm_100a) Mesa layer: chunkwise-parallel forward and recurrent decode.

The computation lives in the CUDA library ``libmesa_b200.so`` (C ABI in
``include/mesa.h``); ``mesa`` is a thin ctypes binding that only marshals
torch tensors (device memory, streams) into that ABI.
"""
from . import mesa  # noqa: F401
from .mesa import (forward, forward_host, get_error, library_path, step,  # noqa: F401
                   timing_enable, timing_read, workspace_size, MesaError)
