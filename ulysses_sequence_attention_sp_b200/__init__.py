"""Ulysses sequence-parallel attention block on one B200 (sm_100a).

P sequence-parallel ranks are P virtual-rank buffers in one GPU's memory. The
compute path is the C-ABI library ``libusp.so`` (hand-written CUDA kernels for
sm_100a); :mod:`.usp` is a thin ctypes binding over it and uses PyTorch only
for device memory and streams.

The binding loads lazily: ``ulysses_sequence_attention_sp_b200.usp`` (or any
API name accessed on this package) loads ``libusp.so`` and raises if it is
missing. There is no CPU fallback.
"""

_API = (
    "sp_seq_split", "Plan", "scatter_sequence", "gather_sequence", "sp_head_slice",
    "sp_head_gather", "ulysses_seq_to_head", "ulysses_head_to_seq", "head_attention",
    "ulysses_attention", "UspError", "library_path",
)


def __getattr__(name):
    if name in _API:
        from . import usp
        return getattr(usp, name)
    raise AttributeError(name)
