"""Helpers for the GPU tests: moving the synthetic inputs to the device and
choosing the rows the oracle checks."""
from __future__ import annotations

import numpy as np
import torch

import synthetic


def to_device(raw: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """bf16 bit patterns (uint16) or fp32 values -> a CUDA tensor of that dtype."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(raw, dtype=np.float32))
    return t.to(device)


def device_activations(w: synthetic.Workload, device="cuda") -> torch.Tensor:
    """The whole workload on the device, uploaded chunk by chunk."""
    tdtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    x = torch.empty((w.M, w.d), dtype=tdtype, device=device)
    step = synthetic.ROW_CHUNK * 8
    for r0 in range(0, w.M, step):
        rows = np.arange(r0, min(w.M, r0 + step))
        x[r0:r0 + rows.size] = to_device(synthetic.make_activations(w, rows), w.dtype, device)
    return x


def sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    """All rows when M <= n, else n seeded random rows plus the first and last."""
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng([seed, M, 99])
    rows = set(rng.choice(M, size=n, replace=False).tolist()) | {0, M - 1}
    return np.array(sorted(rows))


def f64(raw: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return synthetic.f32_from_bf16_bits(raw).astype(np.float64)
    return np.asarray(raw, dtype=np.float64)


def padded_u8(shape, device="cuda", pad=256, fill=0xA5):
    """A uint8 output with guard bytes before and after; returns (view, whole)."""
    n = int(np.prod(shape))
    whole = torch.full((n + 2 * pad,), fill, dtype=torch.uint8, device=device)
    return whole[pad:pad + n].view(*shape), whole


def guards_intact(whole: torch.Tensor, n: int, pad=256, fill=0xA5) -> bool:
    h = whole.cpu().numpy()
    return bool(np.all(h[:pad] == fill) and np.all(h[pad + n:] == fill))
