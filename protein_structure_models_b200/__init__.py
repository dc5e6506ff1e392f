"""Fused Invariant Point Attention forward for B200 (sm_100a).

The compute lives in libfipa.so (C ABI in include/fipa.h); this package is
its thin Python binding and build step."""
from .fipa import (Fipa, FipaError, FipaDims, invariant_point_attention, load_library,  # noqa: F401
                   library_path, make_dims)
