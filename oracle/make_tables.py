"""Write the rotation matrices and codebooks that both sides use as data (TEST INFRASTRUCTURE).

FibQuant's codebook is built once offline and shared by every layer, head and model
(FibQuant summary, sec. 2.1 and 2.2); the rotation is one shared Haar matrix.  This script
builds them with the oracle, rounds them to float32 and stores them under
``random_access_kv_fq_b200/tables/`` as .npy files plus ``manifest.json``.  The CUDA path
reads these files as plain input data; it never runs this script or the oracle.

Usage:  python -m oracle.make_tables [--only NAME ...]
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
from oracle import fq_oracle as fo  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "random_access_kv_fq_b200", "tables")

ROTATIONS = [(64, 17), (64, 18), (66, 17), (66, 18), (128, 17), (128, 18)]
# (d', k, N, restarts, max_iter[, training draws]): large codebooks get fewer restarts and
# iterations (cost).  The half- and full-vector codes at N = 2^15 (the extreme-compression end of
# the frontier) train on 4N draws for 20 iterations from the deterministic start only.
CODEBOOKS = [
    (64, 2, 16, 8, 300),
    (64, 2, 8, 8, 300),
    (64, 2, 256, 8, 300),
    (66, 3, 64, 8, 300),
    (64, 4, 8, 8, 300),
    (128, 4, 4096, 2, 100),
    (64, 32, 32768, 1, 20, 4 * 32768),
    (64, 64, 32768, 1, 20, 4 * 32768),
]
CODEBOOK_SEED = 101
# scalar Lloyd-Max levels of the coordinate law (k = 1, TurboQuant notes sec. 3.1): (d, N1)
SCALAR = [(64, 2), (64, 4), (64, 16)]


def rot_name(dp, seed):
    return f"rot_d{dp}_s{seed}"


def cb_name(dp, k, N):
    return f"cb_d{dp}_k{k}_N{N}"


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", nargs="*", default=None)
    args = ap.parse_args(argv)
    os.makedirs(OUT, exist_ok=True)
    man_path = os.path.join(OUT, "manifest.json")
    manifest = json.load(open(man_path)) if os.path.exists(man_path) else {}
    for dp, seed in ROTATIONS:
        name = rot_name(dp, seed)
        if args.only is not None and name not in args.only:
            continue
        R = fo.haar_rotation(dp, seed).astype(np.float32)
        np.save(os.path.join(OUT, name + ".npy"), R)
        manifest[name] = {"kind": "rotation", "dp": dp, "seed": seed,
                          "orth_err_f32": float(np.abs(R.astype(np.float64) @ R.T.astype(np.float64)
                                                       - np.eye(dp)).max())}
        print(name, manifest[name], flush=True)
    for dp, k, N, restarts, max_iter, *draws in CODEBOOKS:
        name = cb_name(dp, k, N)
        if args.only is not None and name not in args.only:
            continue
        t0 = time.time()
        C, info = fo.build_codebook(dp, k, N, seed=CODEBOOK_SEED, restarts=restarts,
                                    max_iter=max_iter, M=draws[0] if draws else None)
        np.save(os.path.join(OUT, name + ".npy"), C.astype(np.float32))
        manifest[name] = {"kind": "codebook", "dp": dp, "k": k, "N": N, "seed": CODEBOOK_SEED,
                          "restarts": restarts, "max_iter": max_iter, "train_samples": info.M,
                          "train_mse_per_restart": info.train_mse, "iters": info.iters,
                          "best_restart": info.best,
                          "unit_vector_mse": (dp // k) * min(info.train_mse),
                          "seconds": round(time.time() - t0, 1)}
        print(name, manifest[name], flush=True)
        json.dump(manifest, open(man_path, "w"), indent=1, sort_keys=True)
    for d, N1 in SCALAR:
        name = cb_name(d, 1, N1)
        if args.only is not None and name not in args.only:
            continue
        c1 = np.sort(fo.scalar_lloyd(d, N1))
        np.save(os.path.join(OUT, name + ".npy"), c1.astype(np.float32)[:, None])
        manifest[name] = {"kind": "scalar codebook", "d": d, "N": N1,
                          "mse_per_coord": fo.scalar_mse_per_coord(c1, d)}
        print(name, manifest[name], flush=True)
    json.dump(manifest, open(man_path, "w"), indent=1, sort_keys=True)


if __name__ == "__main__":
    main()
