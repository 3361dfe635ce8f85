"""Test helpers: numpy <-> torch transfer of stored values and error metrics."""
import numpy as np

import workloads as WL


def rel_fro(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    d = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (d if d > 0 else 1.0))


def to_dev(a: np.ndarray, dtype: str):
    """Upload a stored array (bf16 bits or float32) as a CUDA tensor of that dtype."""
    import torch
    if dtype == WL.BF16:
        t = torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a, np.float32))
    return t.cuda()


def f64(t) -> np.ndarray:
    """Exact float64 value of a CUDA tensor (bf16 or fp32)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |x| (the RNE rounding budget)."""
    ax = np.maximum(np.abs(x), 1e-38)
    e = np.floor(np.log2(ax))
    return 2.0 ** (e - 8)


def dtype_name(code: int) -> str:
    return WL.BF16 if code == 1 else WL.F32
