"""B200-native Parallax (parameterized Local Linear Attention) decode.

The compute path is libparallax.so (hand-written sm_100a CUDA behind a C ABI,
declared in include/parallax.h); `binding` marshals torch tensors into it.
The binding is imported lazily so that `inputs` can be used without a GPU;
calling any entry point without the built library or a CUDA device raises.
"""
__all__ = ["parallax_decode", "parallax_softmax_decode", "parallax_decode_phase", "parallax_decode_ex",
           "parallax_prefill", "parallax_varlen_prefill", "parallax_decode_paged",
           "parallax_decode_block_sparse", "parallax_copy",
           "parallax_decode_workspace_bytes", "parallax_choose_splits", "parallax_default_splits",
           "parallax_status_string", "parallax_workspace_status", "Workspace"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
