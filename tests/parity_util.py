"""Helpers shared by the GPU parity tests: build a seeded case, put it on the
GPU, evaluate the oracle (optionally in a spawn process pool), compare."""
from __future__ import annotations

import json
import multiprocessing as mp
import os

import numpy as np
import torch

import oracle as O
from synth import CONFIGS, LayerShape, make_layer

TOL = {"f32": 1e-4, "bf16": 2e-2}    # max|err| <= TOL * RMS(oracle output)

_POOL = None


def pool():
    """A process pool for the oracle, started with 'spawn' (safe after CUDA init)."""
    global _POOL
    if _POOL is None:
        n = max(1, min(32, (os.cpu_count() or 2) - 1))
        _POOL = mp.get_context("spawn").Pool(n)
    return _POOL


def _route_rows(args):
    x, W_r, b_r = args
    return O.route(x, W_r, b_r)[0]


def oracle_logits(x64, W_r64, b_r64, parallel=True):
    """Exact-sign router logits [T,E] (in chunks across the pool for big T)."""
    T = x64.shape[0]
    if not parallel or T * W_r64.shape[0] * x64.shape[1] < 2_000_000:
        return O.route(x64, W_r64, b_r64)[0]
    chunks = np.array_split(np.arange(T), min(T, 8 * (os.cpu_count() or 1)))
    parts = pool().map(_route_rows, [(x64[c], W_r64, b_r64) for c in chunks if len(c)])
    return np.concatenate(parts, axis=0)


def _layer_tokens(args):
    x64, L64, eps, toks = args
    return O.layer_forward_tokens(x64, L64, eps, toks)[0]


def oracle_forward(x64, L64, eps, tokens, parallel=True):
    tokens = list(tokens)
    if not parallel or len(tokens) < 8:
        return O.layer_forward_tokens(x64, L64, eps, tokens)[0]
    chunks = [c.tolist() for c in np.array_split(np.array(tokens), min(len(tokens), 4 * (os.cpu_count() or 1))) if len(c)]
    parts = pool().map(_layer_tokens, [(x64, L64, eps, c) for c in chunks])
    return np.concatenate(parts, axis=0)


def case(name: str, **over):
    cfg = dict(CONFIGS[name])
    shape = cfg.pop("shape")
    if "T" in over:
        shape = LayerShape(over.pop("T"), shape.D, shape.E, shape.d_e, shape.d_s, shape.dtype, shape.eps)
    cfg.update(over)
    seed = cfg.pop("seed")
    return shape, make_layer(shape, seed, **cfg)


def to_gpu(L: dict, deco) -> dict:
    G = {k: v.cuda() for k, v in L.items()}
    G["W_bar_up"] = deco.mean_up(G["W_up"])
    return G


def to_oracle(L: dict, dtype: str) -> dict:
    L64 = {k: O.to_f64(v) for k, v in L.items()}
    L64["W_bar_up"] = O.mean_up(L64["W_up"], dtype)
    return L64


def half_ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    """Half the spacing of the storage format at |ref|: the rounding error that
    storing the exact output in that format makes by itself."""
    mant = 8 if dtype == "bf16" else 24
    _, e = np.frexp(np.abs(ref))
    return np.ldexp(1.0, np.maximum(e, -125) - mant - 1)


def check_close(got: np.ndarray, ref: np.ndarray, dtype: str, what=""):
    """max|got - ref| <= TOL * RMS(ref), beyond the storage rounding of the
    output itself (ref is the oracle's unrounded fp64 value; got was stored in
    `dtype`, which alone moves it by up to half a unit in the last place)."""
    rms = float(np.sqrt(np.mean(ref * ref)))
    if not got.size:
        return 0.0
    excess = np.abs(got - ref) - half_ulp(ref, dtype)
    err = float(max(excess.max(), 0.0))
    log = os.environ.get("DECO_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"what": what, "dtype": dtype, "err_over_rms": err / rms if rms else 0.0,
                                "raw_max_over_rms": float(np.abs(got - ref).max()) / rms if rms else 0.0})
                    + "\n")
    assert err <= TOL[dtype] * rms, f"{what}: max|err| {err:.3e} > {TOL[dtype]} * RMS {rms:.3e}"
    return err / rms if rms else 0.0
