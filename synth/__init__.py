"""Seeded synthetic inputs for the DECO MoE FFN layer.

This module is shared by the CPU oracle's tests and by the CUDA path's tests
and benchmark.  It draws random tensors and nothing else: it holds none of the
layer's arithmetic (no routing, no normalisation, no projection).  The one
derived weight of the layer, the mean up-projection, is NOT made here; each
side computes it with its own code.

Recipe (the pages give no trained weights, so every tensor is synthetic):

* x ~ N(0, 1); every weight matrix ~ N(0, 1/fan_in) with fan_in the size of
  the contracted axis (d_model for the router, the up-projections and the
  shared up-projection; d_e for the routed down-projections; d_s for the
  shared down-projection; d_model and d_ff for the dense FFN).
* s_e ~ U(0.5, 2).
* Router bias b_r[e] = q * sigma_e with sigma_e = ||W_r[e]||_2, the exact
  standard deviation of the logit x.W_r[e] when x ~ N(0, I), and q the
  standard-normal quantile of the wanted mean activation ratio (20 % is the
  ratio the DECO pages train and benchmark at); "100 %" uses q = +8.
* Optional per-token jitter: x_t = g_t + c_t v with v the minimum-norm vector
  whose router logits are exactly sigma (W_r v = sigma), c_t ~ N(0, jitter^2).
  The bias then uses q * sqrt(1 + jitter^2) so the mean ratio is kept; every
  `zero_every`-th token gets c_t = -8 so that it activates no routed expert.

Everything is drawn in fp32 on the CPU from `torch.Generator` seeded with
seed*1000 + layer*10 + tensor_id, then rounded once to the storage dtype.
"""
from __future__ import annotations

import dataclasses
import math
import statistics

import torch

# Storage dtypes by name.
DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}

# tensor ids used in the seed formula
_TID = dict(x=0, W_r=1, W_up=2, W_down=3, s=4, W_s_up=5, W_s_down=6, jitter=7,
            W1=8, W2=9, W_val=10)


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Sizes of one DECO MoE FFN layer and of the token batch fed to it."""
    T: int          # tokens
    D: int          # d_model
    E: int          # routed experts
    d_e: int        # routed expert hidden width
    d_s: int        # shared expert hidden width
    dtype: str = "bf16"   # storage dtype of x, weights and out ("f32" | "bf16")
    eps: float = 1e-6     # RMS normalisation epsilon (a documented choice)

    @property
    def torch_dtype(self) -> torch.dtype:
        return DTYPES[self.dtype]


def _gen(seed: int, layer: int, tid: str) -> torch.Generator:
    g = torch.Generator()
    i = _TID[tid]
    # ids 0..9: seed*1000 + layer*10 + id; later ids (the gated value branch)
    # start a second block, seed*1000 + 500 + layer*10 + (id - 10), layer < 50
    g.manual_seed(seed * 1000 + layer * 10 + i if i < 10 else seed * 1000 + 500 + layer * 10 + (i - 10))
    return g


def _normal(shape, std, seed, layer, tid):
    return torch.randn(shape, generator=_gen(seed, layer, tid), dtype=torch.float32) * std


def ratio_quantile(ratio: float) -> float:
    """Standard-normal quantile giving an expected activation `ratio`."""
    if ratio >= 1.0:
        return 8.0
    return statistics.NormalDist().inv_cdf(ratio)


def make_x(T: int, D: int, dtype: str, seed: int, layer: int = 0) -> torch.Tensor:
    return _normal((T, D), 1.0, seed, layer, "x").to(DTYPES[dtype])


def make_layer(shape: LayerShape, seed: int, layer: int = 0, ratio: float = 0.2,
               jitter: float = 0.0, zero_every: int = 0, with_x: bool = True,
               gated: bool = False) -> dict:
    """Draw one layer's weights (and its input batch) on the CPU.

    Returns a dict of CPU tensors in the storage dtype (b_r and s are always
    fp32): x [T,D], W_r [E,D], b_r [E], W_up [E,d_e,D], W_down [E,D,d_e],
    s [E], W_s_up [d_s,D], W_s_down [D,d_s], and with gated=True the gated
    experts' value branch W_val [E,d_e,D] ~ N(0, 1/D).
    """
    T, D, E, d_e, d_s = shape.T, shape.D, shape.E, shape.d_e, shape.d_s
    td = shape.torch_dtype
    W_r = _normal((E, D), 1.0 / math.sqrt(D), seed, layer, "W_r").to(td)
    W_up = _normal((E, d_e, D), 1.0 / math.sqrt(D), seed, layer, "W_up").to(td)
    W_down = _normal((E, D, d_e), 1.0 / math.sqrt(d_e), seed, layer, "W_down").to(td)
    s = torch.rand((E,), generator=_gen(seed, layer, "s"), dtype=torch.float32) * 1.5 + 0.5
    W_s_up = _normal((d_s, D), 1.0 / math.sqrt(D), seed, layer, "W_s_up").to(td)
    W_s_down = _normal((D, d_s), 1.0 / math.sqrt(d_s), seed, layer, "W_s_down").to(td)

    Wr64 = W_r.to(torch.float64)
    sigma = Wr64.norm(dim=1)                       # exact logit std per expert
    q = ratio_quantile(ratio)
    if jitter > 0.0 and ratio < 1.0:
        q = q * math.sqrt(1.0 + jitter * jitter)
    b_r = (q * sigma).to(torch.float32)

    out = dict(W_r=W_r, b_r=b_r, W_up=W_up, W_down=W_down, s=s,
               W_s_up=W_s_up, W_s_down=W_s_down)
    if gated:
        out["W_val"] = _normal((E, d_e, D), 1.0 / math.sqrt(D), seed, layer, "W_val").to(td)
    if with_x:
        g = _normal((T, D), 1.0, seed, layer, "x")
        if jitter > 0.0:
            # minimum-norm v with W_r v = sigma (least squares on the rows)
            v = Wr64.T @ torch.linalg.solve(Wr64 @ Wr64.T, sigma)
            c = torch.randn((T,), generator=_gen(seed, layer, "jitter"),
                            dtype=torch.float64) * jitter
            if zero_every:
                c[::zero_every] = -8.0
            g = (g.to(torch.float64) + c[:, None] * v[None, :]).to(torch.float32)
        out["x"] = g.to(td)
    return out


def make_dense(T: int, D: int, d_ff: int, dtype: str, seed: int) -> dict:
    """Equal-parameter dense non-gated FFN: W1 [d_ff,D], W2 [D,d_ff], x [T,D]."""
    td = DTYPES[dtype]
    return dict(
        x=make_x(T, D, dtype, seed),
        W1=_normal((d_ff, D), 1.0 / math.sqrt(D), seed, 0, "W1").to(td),
        W2=_normal((D, d_ff), 1.0 / math.sqrt(d_ff), seed, 0, "W2").to(td),
    )


# The workloads: single layers shaped like the DECO pages' edge deployments.
CONFIGS = {
    # tiny fp32 layer, the case the oracle finishes in seconds
    "tiny_f32": dict(shape=LayerShape(64, 256, 8, 128, 128, "f32"), seed=0),
    # edge-scale layer, decode batches
    "edge_decode_t1": dict(shape=LayerShape(1, 2048, 64, 256, 1024, "bf16"), seed=1),
    "edge_decode_t4": dict(shape=LayerShape(4, 2048, 64, 256, 1024, "bf16"), seed=1),
    "edge_decode_t16": dict(shape=LayerShape(16, 2048, 64, 256, 1024, "bf16"), seed=1),
    # same layer, prefill with per-token activation jitter and zero-expert tokens
    "edge_prefill_t4096": dict(shape=LayerShape(4096, 2048, 64, 256, 1024, "bf16"),
                               seed=2, jitter=0.5, zero_every=64),
    # one layer of the larger 8-layer stack
    "large_t16": dict(shape=LayerShape(16, 4096, 128, 256, 2048, "bf16"), seed=3),
    "large_t16384": dict(shape=LayerShape(16384, 4096, 128, 256, 2048, "bf16"), seed=3),
}
