"""Level-of-Detail (LoD) attention for NVIDIA B200 (sm_100a).

The compute path is the CUDA library liblod.so (C ABI in include/lod.h); this
package is its Python binding.  `synth` draws the seeded synthetic inputs.
"""
from ._lib import (LOD_DTYPE_BF16, LOD_DTYPE_F32, LOD_EDEVICE, LOD_EINVAL, LOD_EUNSUPPORTED,
                   LOD_OK, LOD_OP_BUILD, LOD_OP_DECODE, LOD_OP_PREFILL, LodError, load)
from .api import (Index, Params, lod_build_index, lod_decode, lod_get_status, lod_prefill,
                  workspace, workspace_bytes)

__all__ = [
    "Params", "Index", "lod_build_index", "lod_decode", "lod_prefill", "lod_get_status",
    "workspace", "workspace_bytes", "load", "LodError", "LOD_OK", "LOD_EINVAL", "LOD_EUNSUPPORTED",
    "LOD_EDEVICE", "LOD_OP_BUILD", "LOD_OP_DECODE", "LOD_OP_PREFILL", "LOD_DTYPE_F32",
    "LOD_DTYPE_BF16",
]
