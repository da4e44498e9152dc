"""Readers for the hand-derived text fixtures in tests/golden/."""
from __future__ import annotations

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _parse_float(tok: str) -> float:
    if "0x" in tok.lower() and "p" in tok.lower():
        return float.fromhex(tok)
    return float(tok)


def binary16_cases():
    """[(value, bits, note)] from binary16_rounding.txt."""
    out = []
    with open(os.path.join(GOLDEN, "binary16_rounding.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split(None, 2)
            out.append((_parse_float(parts[0]), int(parts[1], 16), parts[2] if len(parts) > 2 else ""))
    return out


def worked_examples():
    """{name: dict(K, N, group, qweight, scales, codes?, W?, xy=[(x, y), ...])}."""
    examples = {}
    cur = None
    pending_x = None
    with open(os.path.join(GOLDEN, "worked_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(" ")
            if key == "example":
                cur = {"xy": []}
                examples[rest.strip()] = cur
            elif key == "end":
                cur = None
            elif key in ("K", "N", "group"):
                cur[key] = int(rest)
            elif key == "qweight":
                cur["qweight"] = np.array([int(t) for t in rest.split()], dtype=np.int64)
            elif key in ("scales", "W"):
                cur[key] = np.array([float(t) for t in rest.split()], dtype=np.float64)
            elif key == "codes":
                cur["codes"] = np.array([int(t) for t in rest.split()], dtype=np.int64)
            elif key == "x":
                pending_x = np.array([float(t) for t in rest.split()], dtype=np.float64)
            elif key == "y":
                cur["xy"].append((pending_x, np.array([float(t) for t in rest.split()])))
                pending_x = None
            else:
                raise ValueError(f"unknown fixture key {key!r}")
    for ex in examples.values():
        K, N = ex["K"], ex["N"]
        ex["qweight"] = ex["qweight"].astype(np.int32).reshape(K // 8, N)
        ex["scales"] = ex["scales"].astype(np.float16).reshape(-1, N)
        if "codes" in ex:
            ex["codes"] = ex["codes"].reshape(K, N)
        if "W" in ex:
            ex["W"] = ex["W"].reshape(K, N)
        ex["xy"] = [(x.astype(np.float16).reshape(1, K), y.reshape(1, N)) for x, y in ex["xy"]]
    return examples
