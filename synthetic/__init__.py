"""Seeded synthetic inputs for the KroQuant activation quantizer.

This module is the only code shared by the CPU oracle (``oracle/``), the tests
and ``bench.py``.  It draws inputs and does nothing else: it holds none of the
quantizer's arithmetic (no transform, no scale rule, no rounding onto the
E2M1 grid).  The one numeric step here, rounding fp32 samples to bf16, belongs
to making the input: the quantizer's input *is* the rounded bf16 tensor, and
both sides read the same bits.

Workloads.  The pages measure on real DiT activations (PixArt-Sigma, SANA,
FLUX.1-schnell on MJHQ-30K / SDCI; KroQuant abstract).  Neither the models nor
the datasets are available, so these generators stand in for the inputs of a
DiT linear layer: a base distribution, a few outlier channels scaled up, and
a per-token mean shift of the kind adaptive layer-norm adds.  Order of draws
for one (config, M, d): outlier channel set, outlier-free noise chunk by
chunk, per-token mean, then LU parameters from a separate stream.

"N(mu, s)" means mean mu, standard deviation s.
"""
from __future__ import annotations

import dataclasses
from typing import Iterable, Sequence

import numpy as np

__all__ = [
    "Workload", "CONFIGS", "workloads", "bf16_bits_from_f32", "f32_from_bf16_bits",
    "make_activations", "make_params", "identity_params", "make_weights",
    "smoothquant_inv_scales", "ROW_CHUNK",
]

# Rows are drawn in chunks, each from its own seeded stream, so any subset of
# rows can be regenerated without drawing the whole tensor (the oracle checks
# sampled rows of the largest workloads).
ROW_CHUNK = 1024


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str          # e.g. "flux"
    M: int             # tokens (rows)
    d: int             # channels (columns); a multiple of 32
    dtype: str         # "bf16" or "f32"
    base: str          # "normal" or "student_t3"
    outlier_frac: float | None   # fraction of channels made outliers
    outlier_count: int | None    # or an explicit count (tiny config)
    outlier_gain: float
    token_mean_std: float        # 0 = no per-token mean shift
    seed: int

    @property
    def nb(self) -> int:
        return self.d // 32

    @property
    def n_outliers(self) -> int:
        if self.outlier_count is not None:
            return self.outlier_count
        return int(round(self.outlier_frac * self.d))

    @property
    def key(self) -> str:
        return f"{self.name}_{self.M}x{self.d}"


def _w(name, M, d, dtype, base, frac, count, gain, mstd, seed):
    return Workload(name, M, d, dtype, base, frac, count, gain, mstd, seed)


def _build_configs() -> dict[str, list[Workload]]:
    cfg: dict[str, list[Workload]] = {}
    # tiny: fp32, N(0,1), 8 outlier channels x30, per-token mean N(0,2).
    cfg["tiny"] = [_w("tiny", 256, 1152, "f32", "normal", None, 8, 30.0, 2.0, 0)]
    # PixArt-Sigma: CFG batch 2 x 4096 tokens, d=1152 and MLP-in 4608.
    cfg["pixart"] = [_w("pixart", 8192, d, "bf16", "normal", 0.01, None, 50.0, 3.0, 1)
                     for d in (1152, 4608)]
    # SANA: 2 x 1024 tokens, heavy-tailed Student-t(3), 0.5 % channels x80.
    cfg["sana"] = [_w("sana", 2048, d, "bf16", "student_t3", 0.005, None, 80.0, 0.0, 2)
                   for d in (2240, 5600)]
    # FLUX.1-schnell: 4096 image + 512 text tokens, d=3072 and MLP 12288.
    cfg["flux"] = [_w("flux", 4608, d, "bf16", "normal", 0.01, None, 100.0, 4.0, 3)
                   for d in (3072, 12288)]
    sweep = []
    i = 0
    for M in (1024, 4096, 16384, 65536):
        for d in (1152, 3072, 12288):
            sweep.append(_w("sweep", M, d, "bf16", "normal", 0.01, None, 50.0, 0.0, 100 + i))
            i += 1
    cfg["sweep"] = sweep
    return cfg


CONFIGS: dict[str, list[Workload]] = _build_configs()


def workloads(names: Iterable[str] | None = None) -> list[Workload]:
    names = list(CONFIGS) if names is None else list(names)
    return [w for n in names for w in CONFIGS[n]]


# --------------------------------------------------------------------------
# bf16 bits <-> fp32
# --------------------------------------------------------------------------
def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even) and return the
    16-bit patterns as uint16.  Inputs here are finite."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# activations
# --------------------------------------------------------------------------
def _layout_rng(w: Workload) -> np.random.Generator:
    return np.random.default_rng([w.seed, w.M, w.d, 0])


def _outlier_channels(w: Workload) -> np.ndarray:
    rng = _layout_rng(w)
    return np.sort(rng.choice(w.d, size=w.n_outliers, replace=False))


def _token_means(w: Workload) -> np.ndarray:
    if w.token_mean_std == 0.0:
        return np.zeros(w.M, dtype=np.float64)
    rng = np.random.default_rng([w.seed, w.M, w.d, 1])
    return rng.normal(0.0, w.token_mean_std, size=w.M)


def _chunk(w: Workload, c: int, ch: np.ndarray, means: np.ndarray) -> np.ndarray:
    r0 = c * ROW_CHUNK
    r1 = min(w.M, r0 + ROW_CHUNK)
    rng = np.random.default_rng([w.seed, w.M, w.d, 2, c])
    if w.base == "normal":
        x = rng.standard_normal((r1 - r0, w.d), dtype=np.float32)
    elif w.base == "student_t3":
        x = rng.standard_t(3.0, size=(r1 - r0, w.d)).astype(np.float32)
    else:
        raise ValueError(w.base)
    if ch.size:
        x[:, ch] *= np.float32(w.outlier_gain)
    x += means[r0:r1, None].astype(np.float32)
    return x


def make_activations(w: Workload, rows: Sequence[int] | np.ndarray | None = None) -> np.ndarray:
    """The workload's activations as stored in HBM.

    Returns uint16 bf16 bit patterns [len(rows), d] for bf16 workloads, or
    float32 [len(rows), d] for fp32 workloads.  ``rows=None`` means all rows.
    Any subset of rows is bit-identical to the same rows of the full tensor.
    """
    ch = _outlier_channels(w)
    means = _token_means(w)
    if rows is None:
        rows = np.arange(w.M)
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= w.M):
        raise IndexError("row out of range")
    out_dtype = np.uint16 if w.dtype == "bf16" else np.float32
    out = np.empty((rows.size, w.d), dtype=out_dtype)
    chunks = rows // ROW_CHUNK
    for c in np.unique(chunks):
        sel = np.nonzero(chunks == c)[0]
        x = _chunk(w, int(c), ch, means)
        xs = x[rows[sel] - c * ROW_CHUNK]
        out[sel] = bf16_bits_from_f32(xs) if w.dtype == "bf16" else xs
    return out


def activations_f64(w: Workload, raw: np.ndarray) -> np.ndarray:
    """Exact fp64 view of what ``make_activations`` returned."""
    if w.dtype == "bf16":
        return f32_from_bf16_bits(raw).astype(np.float64)
    return raw.astype(np.float64)


# --------------------------------------------------------------------------
# LU parameters, weights, SmoothQuant scales
# --------------------------------------------------------------------------
def make_params(nb: int, seed: int, a_std: float = 0.5, b_std: float = 0.5,
                logu_std: float = 0.3) -> np.ndarray:
    """fp32 [nb, 15]: per block, five factors m = 0..4 stored as
    (a, b, u) at [3m], [3m+1], [3m+2].  a, b ~ N(0, a_std / b_std),
    u = exp(N(0, logu_std))."""
    rng = np.random.default_rng([seed, nb, 7])
    a = rng.normal(0.0, a_std, size=(nb, 5))
    b = rng.normal(0.0, b_std, size=(nb, 5))
    u = np.exp(rng.normal(0.0, logu_std, size=(nb, 5)))
    p = np.stack([a, b, u], axis=-1).reshape(nb, 15)
    return p.astype(np.float32)


def identity_params(nb: int) -> np.ndarray:
    p = np.zeros((nb, 5, 3), dtype=np.float32)
    p[:, :, 2] = 1.0
    return p.reshape(nb, 15)


def make_weights(n_out: int, d: int, seed: int) -> np.ndarray:
    """fp32 [n_out, d] ~ N(0, 1/sqrt(d)) (nn.Linear layout, y = W x)."""
    rng = np.random.default_rng([seed, n_out, d, 9])
    return (rng.standard_normal((n_out, d), dtype=np.float32) / np.float32(np.sqrt(d)))


def smoothquant_inv_scales(x_f32: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """Synthetic SmoothQuant calibration: s_c = max_m |x_mc| ** alpha (unit
    weight range), returned as fp32 1/s_c.  The pages name SmoothQuant's
    per-channel scaling but give no formula for s; this input only feeds the
    comparison kernel, whose cost does not depend on the values."""
    amax = np.abs(x_f32.astype(np.float64)).max(axis=0)
    s = np.maximum(amax, 1e-5) ** alpha
    return (1.0 / s).astype(np.float32)
