"""Helpers for the GPU parity tests: device tensors from seeded numpy inputs."""
import numpy as np

try:
    import torch
except ImportError:  # pragma: no cover
    torch = None


def require_gpu():
    import pytest
    if torch is None or not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gpt_step_b200 import build
    build.build()


def bf16(a: np.ndarray):
    """numpy -> device bf16 tensor."""
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16).cuda()


def f32(a: np.ndarray):
    return torch.tensor(np.asarray(a, np.float32)).cuda()


def i32(a: np.ndarray):
    return torch.tensor(np.asarray(a, np.int32)).cuda()


def host(t) -> np.ndarray:
    """device tensor (any float dtype) -> numpy fp64."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def rounded(a: np.ndarray) -> np.ndarray:
    """The fp64 value of `a` after rounding to bf16 (what the device actually sees)."""
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    d = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (d if d > 0 else 1.0))


def err_word():
    return torch.zeros(4, dtype=torch.int32, device="cuda")
