"""Offline fitting of the LU parameters on calibration activations.

The pages learn the 15 parameters of every block but give no objective.  The
plain reading used here: choose them to minimise the error of the quantised
linear layer itself, ||Q(T X) Q(W T^-1)^T - X W^T||_F over calibration
tokens, where Q is MXFP4 and T = blockdiag(T_j).  The search is coordinate
descent over blocks.  For block j it tries:
  - the identity (plain MXFP4);
  - five 45-degree rotations, whose Kronecker product is an orthonormal
    Walsh-Hadamard transform that spreads an outlier channel over the block;
  - random perturbations of the block's best parameters so far.
It keeps whichever gives the lowest layer error, with every other block
fixed.  Every candidate is scored by the library's own kernels (activation
and weight quantizers, block-scaled FP4 GEMM) on the GPU; torch only holds
the buffers, computes the unquantised reference product once and takes the
norm of the difference.

This is calibration, run once per layer, not part of the per-step path.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import (kq_gemm_mxfp4, kq_quantize_sf_tiled, kq_quantize_weights, kq_sf_tile)

__all__ = ["identity_block", "hadamard_block", "layer_error", "fit_params"]


def identity_block() -> np.ndarray:
    """a = b = 0, u = 1 for all five factors: T_j = I."""
    return np.array([0.0, 0.0, 1.0] * 5, dtype=np.float32)


def hadamard_block() -> np.ndarray:
    """a = -1, b = u = 1/sqrt(2): each factor is the rotation [[c, c], [-c, c]]
    (c = 1/sqrt(2)), so T_j is an orthonormal Walsh-Hadamard transform up to
    signs."""
    c = 1.0 / math.sqrt(2.0)
    return np.array([-1.0, c, c] * 5, dtype=np.float32)


class _Layer:
    """Calibration activations and weights on the device, with the reusable
    output buffers of one scoring pass."""

    def __init__(self, x: torch.Tensor, W: torch.Tensor):
        if x.dim() != 2 or W.dim() != 2 or x.shape[1] != W.shape[1]:
            raise ValueError("x [M, d] and W [N, d] must share d")
        M, d = x.shape
        if d % 128:
            raise ValueError("d must be a multiple of 128 (the FP4 GEMM's K step)")
        self.x, self.W = x, W.float().contiguous()
        self.M, self.N, self.d = M, W.shape[0], d
        dev = x.device
        self.codes = torch.empty((M, d // 2), dtype=torch.uint8, device=dev)
        self.tiled = torch.empty(((M + 127) // 128, d // 128, 512), dtype=torch.uint8, device=dev)
        self.Y = torch.empty((M, self.N), dtype=torch.float32, device=dev)
        ref = x.float() @ self.W.t()
        self.ref = ref
        self.ref_norm = float(torch.linalg.norm(ref))

    def error(self, params: torch.Tensor) -> float:
        kq_quantize_sf_tiled(self.x, params, self.codes, self.tiled)
        cw, sw = kq_quantize_weights(self.W, params)
        kq_gemm_mxfp4(self.codes, self.tiled, cw, kq_sf_tile(sw), self.Y)
        return float(torch.linalg.norm(self.Y - self.ref)) / self.ref_norm


def layer_error(x: torch.Tensor, W: torch.Tensor, params: torch.Tensor) -> float:
    """Relative Frobenius error of the quantised layer against x W^T."""
    return _Layer(x, W).error(params)


def fit_params(x: torch.Tensor, W: torch.Tensor, params0: np.ndarray | None = None,
               sweeps: int = 2, n_perturb: int = 4, sigma: float = 0.15, seed: int = 0):
    """Coordinate descent over blocks (see the module docstring).

    x: bf16 or fp32 [M, d] calibration activations on the GPU; W: fp32 [N, d]
    weights of the layer.  Returns (params fp32 [d/32, 15] on x's device,
    list of the layer error after each sweep, starting with params0's)."""
    layer = _Layer(x, W)
    nb = layer.d // 32
    rng = np.random.default_rng(seed)
    P = np.tile(identity_block(), (nb, 1)) if params0 is None else np.array(params0, dtype=np.float32)
    Pd = torch.from_numpy(P).to(x.device)
    best = layer.error(Pd)
    history = [best]
    for _ in range(sweeps):
        for j in range(nb):
            cands = [identity_block(), hadamard_block()]
            for _ in range(n_perturb):
                c = P[j].astype(np.float64).reshape(5, 3).copy()
                c[:, 0] += rng.normal(0.0, sigma, 5)
                c[:, 1] += rng.normal(0.0, sigma, 5)
                c[:, 2] *= np.exp(rng.normal(0.0, sigma, 5))
                cands.append(c.reshape(15).astype(np.float32))
            keep = P[j].copy()
            for c in cands:
                Pd[j] = torch.from_numpy(c).to(x.device)
                e = layer.error(Pd)
                if e < best:
                    best, keep = e, c
            P[j] = keep
            Pd[j] = torch.from_numpy(keep).to(x.device)
        history.append(best)
    return Pd, history
