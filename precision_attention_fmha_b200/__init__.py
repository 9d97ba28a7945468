"""B200-native mixed-precision fused multi-head attention forward (sm_100a).

The compute path is the C-ABI library ``libfmha.so`` built from ``csrc/``
(hand-written tcgen05 / TMA kernels); ``precision_attention_fmha_b200.fmha``
is its thin ctypes binding. Importing this package is cheap: the library is
loaded on first use of a binding name, and that load fails loudly when the
library is missing -- there is no fallback implementation.
"""

_BINDING_NAMES = (
    "fmha_fwd", "fmha_fwd_block_sparse", "fmha_fwd_paged", "fmha_quantize_blockwise",
    "quantize_workspace_bytes", "get_device_error", "FmhaError", "load_library",
)


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import fmha

        return getattr(fmha, name)
    raise AttributeError(name)
