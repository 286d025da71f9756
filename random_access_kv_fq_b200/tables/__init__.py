"""Rotation matrices and codebooks used as input data (float32 .npy files in this folder).

They were produced offline by the repository's table script from the method's description
(Haar rotation from a sign-corrected QR; Beta-quantile radii, Fibonacci / Roberts-Kronecker
directions and multi-restart Lloyd-Max refinement) and are plain data here: the product path
only reads them.  ``manifest.json`` records how each one was made.
"""
from __future__ import annotations

import json
import os

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))


def rotation(dp: int, seed: int) -> np.ndarray:
    return np.load(os.path.join(_DIR, f"rot_d{dp}_s{seed}.npy"))


def codebook(dp: int, k: int, N: int) -> np.ndarray:
    return np.load(os.path.join(_DIR, f"cb_d{dp}_k{k}_N{N}.npy"))


def manifest() -> dict:
    with open(os.path.join(_DIR, "manifest.json")) as f:
        return json.load(f)


def have(name: str) -> bool:
    return os.path.exists(os.path.join(_DIR, name + ".npy"))
