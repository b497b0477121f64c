"""libssd: the Mamba-2 SSD layer forward pass (chunked algorithm) and its
speculative-decoding verify step, as hand-written CUDA kernels for B200 (sm_100a)
behind a C ABI (include/ssd.h). This package is the thin Python binding."""

__all__ = ["ssd_fwd", "ssd_verify", "ssd_select_state", "fwd_workspace_bytes", "SSDError", "build"]


def __getattr__(name):
    # The binding imports torch; keep `import state_space_sequence_chunked_b200.inputs` light.
    if name in ("ssd_fwd", "ssd_verify", "ssd_select_state", "fwd_workspace_bytes", "SSDError", "lib"):
        from . import _binding

        return getattr(_binding, name)
    if name == "build":
        from .build import build

        return build
    raise AttributeError(name)
