"""Helpers shared by the GPU tests: numpy storage <-> CUDA tensors, error stats."""

import numpy as np
import torch

from ulysses_sequence_attention_sp_b200.synth import storage_to_f64

TORCH_DTYPE = {"bf16": torch.bfloat16, "fp32": torch.float32, "fp16": torch.float16}


def to_device(storage: np.ndarray, dtype: str) -> torch.Tensor:
    """Storage (uint16 bf16 bits, or float32) -> CUDA tensor with the same bits."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(storage).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(storage, dtype=np.float32)).cuda()


def bits_to_device(bits: np.ndarray) -> torch.Tensor:
    dt = {2: np.int16, 4: np.int32}[bits.dtype.itemsize]
    return torch.from_numpy(np.ascontiguousarray(bits).view(dt)).cuda()


def device_bits(t: torch.Tensor) -> np.ndarray:
    if t.element_size() == 2:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.view(torch.int32).cpu().numpy().view(np.uint32)


def to_f64(t: torch.Tensor, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return storage_to_f64(device_bits(t), "bf16")
    return t.double().cpu().numpy()


def error_stats(got: np.ndarray, ref: np.ndarray) -> dict:
    diff = np.abs(got - ref)
    return {
        "max_abs": float(diff.max()) if diff.size else 0.0,
        "mean_abs": float(diff.mean()) if diff.size else 0.0,
        "rel_l2": float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)),
        "nan": int(np.isnan(got).sum()),
    }


# Tolerances of the block against the float64 oracle: bf16 inputs max-abs
# 2e-2 and mean-abs 2e-3 (plus relative L2 1e-2, so a near-zero output cannot
# pass on absolute error alone); fp32 inputs max-abs 1e-4.
def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = "") -> dict:
    st = error_stats(got, ref)
    assert st["nan"] == 0, (what, st)
    if dtype == "fp32":
        assert st["max_abs"] <= 1e-4, (what, st)
    else:
        assert st["max_abs"] <= 2e-2, (what, st)
        assert st["mean_abs"] <= 2e-3, (what, st)
        assert st["rel_l2"] <= 1e-2, (what, st)
    return st
