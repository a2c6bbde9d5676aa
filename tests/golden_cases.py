"""Reader for the hand-worked blocks in tests/golden/kq_hand_blocks.txt (the
file states where each expected value comes from)."""
from __future__ import annotations

import os
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HAND_BLOCKS = os.path.join(HERE, "golden", "kq_hand_blocks.txt")


@dataclass
class HandBlock:
    name: str
    params: np.ndarray     # [1][15] float32
    x: np.ndarray          # [1][32] float64, exactly representable in fp32
    scale: int
    codes: np.ndarray      # [1][16] uint8


def _number(tok: str) -> float:
    if tok.startswith("2^"):
        return float(np.ldexp(1.0, int(tok[2:])))
    return float(tok)


def hand_blocks(path: str = HAND_BLOCKS) -> list[HandBlock]:
    out, cur = [], {}
    with open(path) as f:
        for raw in f:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            if key == "case":
                cur = {"name": rest[0]}
            elif key == "params":
                if rest == ["identity"]:
                    p = np.tile(np.array([0.0, 0.0, 1.0], dtype=np.float32), 5)
                else:
                    p = np.array([float(t) for t in rest], dtype=np.float32)
                assert p.size == 15, cur
                cur["params"] = p.reshape(1, 15)
            elif key == "x":
                # the values are used as rounded to fp32 (and to bf16 on the
                # bf16 path); the expected results do not depend on that rounding
                x = np.array([_number(t) for t in rest], dtype=np.float64)
                assert x.size == 32, cur
                cur["x"] = x.reshape(1, 32)
            elif key == "scale":
                cur["scale"] = int(rest[0])
            elif key == "codes":
                cur["codes"] = np.array([int(t, 16) for t in rest], dtype=np.uint8).reshape(1, 16)
                out.append(HandBlock(**cur))
            else:
                raise ValueError(f"unknown line: {line}")
    return out
