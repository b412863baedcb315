"""B200-native (sm_100a) Kimi Delta Attention hot path.

The product is the C-ABI library ``libkda_b200.so`` (declared in
``include/kda.h``); this package holds its CUDA sources (``csrc/``), the
in-tree build (``build.py``) and a thin ctypes binding (``kda.py``).  The
binding is loaded on first attribute access, so ``build`` can run before the
library exists.
"""
_EXPORTS = (
    "KDA_BF16", "KDA_F32", "KDA_QK_L2NORM", "KDA_COMPLEX", "KDA_FUSED", "KDA_SPLIT", "KdaError",
    "kda_opts", "make_opts",
    "kda_chunk_fwd", "kda_chunk_fwd_noalloc", "kda_recurrent_step", "kda_chunk_fwd_prologue",
    "kda_recurrent_step_prologue", "kda_conv_state_from_prefill", "kda_chunk_fwd_gated",
    "kda_chunk_workspace_bytes", "kda_prologue_workspace_bytes", "kda_abi_version",
    "kda_chunk_bwd", "kda_chunk_bwd_workspace_bytes", "chunk_bwd", "KDA_UNBOUNDED_DECAY",
    "KDA_GATE_SOFTPLUS", "kda_segment_pair", "kda_segment_pair_workspace_bytes",
    "kda_affine_combine", "segment_pair", "affine_combine", "kda_selftest_bounded_wait",
    "kda_segment_forward", "segment_forward",
    "kda_device_status", "kda_set_wait_limit", "KDA_WAIT_LIMIT_DEFAULT",
    "status_string", "chunk_fwd", "recurrent_step", "chunk_fwd_prologue",
    "recurrent_step_prologue", "conv_state_from_prefill", "chunk_fwd_gated", "LIB_PATH",
)


def __getattr__(name):
    if name in _EXPORTS or name == "kda":
        import importlib
        mod = importlib.import_module(".kda", __name__)
        return mod if name == "kda" else getattr(mod, name)
    raise AttributeError(name)


__all__ = list(_EXPORTS)
