"""Builds the hand-worked fixture under tests/golden/ into tensors.

The fixture's expected values are closed forms written in the JSON file;
``closed_form`` evaluates them with ``math.exp`` only.
"""
import json
import math
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HANDWORKED = os.path.join(HERE, "golden", "handworked_n4_d64.json")


def load(path=HANDWORKED):
    with open(path) as f:
        return json.load(f)


def closed_form(expr: str) -> float:
    allowed = set("0123456789.+-*/() expEXP")
    if not set(expr) <= allowed:
        raise ValueError(expr)
    return float(eval(expr, {"__builtins__": {}}, {"exp": math.exp}))


def tensors(case):
    """(q, k, v, sigma_q, sigma_k) as float32 numpy arrays [B,H,n,d]."""
    B, H, n, d = case["B"], case["H"], case["n"], case["d"]
    q = np.zeros((B, H, n, d), np.float32)
    k = np.zeros((B, H, n, d), np.float32)
    for r, spec in case["q_rows"].items():
        row = np.full(d, spec["fill"], np.float32)
        for c, val in spec.get("set", {}).items():
            row[int(c)] = val
        if spec.get("set_negative_every_other"):
            row[1::2] = -row[1::2]
        q[0, 0, int(r)] = row
    for r, spec in case["k_rows"].items():
        row = np.full(d, spec["fill"], np.float32)
        for a, b in spec["negative_ranges"]:
            row[a:b] = -row[a:b]
        k[0, 0, int(r)] = row
    v = np.zeros((B, H, n, d), np.float32)
    for j in range(n):
        v[0, 0, j, j] = 1.0
    return (q, k, v, np.asarray(case["sigma_q"], np.float32),
            np.asarray(case["sigma_k"], np.float32))
