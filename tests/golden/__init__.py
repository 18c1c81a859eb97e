"""Hand-worked fixtures (text files beside this module), each citing the passage it follows."""

import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def load(name: str) -> dict:
    """Parse a fixture: '#' lines are comments, every other line is `key value value ...`.
    q, k are returned as [1, 1, N, D] and v as [1, 1, N, E] float64 arrays; S_in / z_in (when present)
    as [1, 1, D, E] and [1, 1, D]."""
    vals = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = np.array([float(x) for x in rest])
    D, E = int(vals["D"][0]), int(vals["E"][0])
    out = {"D": D, "E": E, "block_len": int(vals["block_len"][0]), "eps": float(vals["eps"][0])}
    out["q"] = vals["q"].reshape(1, 1, -1, D)
    out["k"] = vals["k"].reshape(1, 1, -1, D)
    out["v"] = vals["v"].reshape(1, 1, -1, E)
    for key in ("o_block_causal", "o_bidirectional"):
        out[key] = vals[key].reshape(1, 1, -1, E)
    if "S_in" in vals:
        out["S_in"] = vals["S_in"].reshape(1, 1, D, E)
        out["z_in"] = vals["z_in"].reshape(1, 1, D)
        out["S_out"] = vals["S_out"].reshape(1, 1, D, E)
        out["z_out"] = vals["z_out"].reshape(1, 1, D)
    return out


FIXTURES = ["hand_worked_d2_n4.txt", "hand_worked_cache_d1_n3.txt"]


def load_values(name: str) -> dict:
    """Parse any fixture into {key: float64 array} ('#' lines are comments)."""
    vals = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = np.array([float(x) for x in rest])
    return vals
