"""RainFusion v2 block-sparse video attention for B200 (sm_100a).

The compute path lives in the CUDA library `librf.so` (built from `csrc/`),
reached through `block_sparse_video_rearrange_b200.rf` (ctypes binding).
`ulysses` shards one layer over a process group by heads (sequence <-> head
all-to-all around the path); `pipeline` runs host tensors in head chunks
whose copies overlap the compute.  `synth` holds the seeded synthetic input
generator.
"""
import importlib

__all__ = ["rf", "synth", "ulysses", "pipeline"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
