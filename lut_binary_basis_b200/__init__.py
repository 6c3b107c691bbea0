"""FluxBin LUT GEMV for B200 (sm_100a).

The compute path is libfluxbin.so (CUDA kernels behind a C-ABI declared in
include/fluxbin.h); ``fluxbin`` is its ctypes binding and ``synth`` the
seeded synthetic-workload generator.  Importing the package does not load
the shared library; the first call into ``fluxbin`` does, and fails loudly if
it has not been built.
"""
from . import synth  # noqa: F401
from .fluxbin import (FLAG_ACCUMULATE, FLAG_EARLY_WEIGHTS, FLAG_Y_FP32, DeviceLayer, FluxbinError,  # noqa: F401
                      FluxbinLibraryMissing, LayerDesc, fluxbin_linear, fluxbin_linear_static_scratch,
                      fluxbin_lut_gemv, fluxbin_pack, fluxbin_packed_sizes, fluxbin_status_string, fluxbin_version, fluxbin_workspace_bytes,
                      new_workspace)
