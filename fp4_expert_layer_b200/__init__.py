"""B200 (sm_100a) sparse MoE layer over MXFP4 / NVFP4 experts with a resident-slot table.

The compute path is the CUDA library ``libfp4moe.so`` (C ABI in
``include/moe_layer.h``); this package is its Python binding.  Importing the
package does not load the library; creating a layer does, and fails loudly if
the library is missing.
"""
from ._lib import (MoEError, MoELayer, admit, lib, make_config, plan,  # noqa: F401
                   weights_from_layer)

__all__ = ["MoELayer", "MoEError", "make_config", "plan", "admit", "weights_from_layer", "lib"]
