"""DynamicRad block-sparse attention hot path for NVIDIA B200 (sm_100a).

Three stages behind a C ABI (include/dynrad.h, libdynrad.so), bound here by
ctypes with the same names:

* ``dynrad_build_candidates`` -- radial candidate block set (Sec. 3.1, Eqs. 1-7);
* ``dynrad_select_blocks``    -- pooled block scores, static-ratio or
  dynamic-threshold selection into CSR (Sec. 3.2);
* ``dynrad_sparse_attn``      -- block-sparse attention forward, O and LSE
  (Sec. 3.3, Eq. 13); ``dynrad_attn_backward`` is its gradient under the
  same mask.

``workloads`` holds the seeded synthetic inputs.  The binding is imported
lazily so that the workload generator can be used without a GPU.
"""

_ABI_NAMES = ("dynrad_num_blocks", "dynrad_build_candidates", "dynrad_build_candidates_into", "dynrad_select_blocks",
              "dynrad_sparse_attn", "dynrad_attn_backward", "dynrad_device_status", "dynrad_select_workspace_bytes",
              "SelectBuffers", "DynradError", "make_geom", "lib")


def __getattr__(name):
    if name in _ABI_NAMES:
        from . import abi
        return getattr(abi, name)
    raise AttributeError(name)
