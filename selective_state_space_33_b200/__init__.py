"""B200-native selective state-space scan (Mamba S6): a C-ABI CUDA library
(``libsscan.so``) with a thin Python binding.

The binding is imported lazily so that ``selective_state_space_33_b200.workloads``
(seeded inputs) can be used without loading the CUDA library.
"""
_BINDING_NAMES = ("sscan_fwd", "sscan_last_state", "sscan_bwd", "sscan_step", "sscan_chunk_summary", "sscan_carry", "sscan_workspace_size",
                  "SscanError", "load_library", "make_problem", "Problem")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
