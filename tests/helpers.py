"""Shared test helpers: near-tie screening of router inputs and tolerances."""
from __future__ import annotations

import numpy as np

import oracle
import synth

# Feed-forward outputs: max |y - y_ref| / max |y_ref| over the output tensor.
FFN_TOL = 2e-3
# Router weights: the library accumulates logits in fp32 (error ~ sqrt(H) * 2^-24
# * max partial sum ~ 2e-5 at H = 7168 with these inputs); |dw| <= 2 max |dl|.
TOPK_W_TOL = 1e-4
# Minimum gap between adjacent logits among the top k+1 of every token.
TAU = 1e-3


def near_tie_tokens(logits: np.ndarray, k: int, tau: float = TAU) -> np.ndarray:
    """Tokens whose top-(k+1) logits (double) have an adjacent gap below tau."""
    E = logits.shape[1]
    m = min(k + 1, E)
    top = -np.sort(-logits, axis=1)[:, :m]
    gaps = top[:, :-1] - top[:, 1:]
    return np.nonzero((gaps < tau).any(axis=1))[0] if m > 1 else np.zeros(0, np.int64)


def screened_x(cfg: synth.Config, lw: synth.LayerWeights, T: int | None = None, layer: int = 0):
    """Activations with no near-tie in the router: a rejected token is redrawn
    from its next stream (attempt + 1), as the input recipe prescribes."""
    T = cfg.T if T is None else T
    xs = [synth.make_token(cfg, t, 0, layer) for t in range(T)]
    attempts = [0] * T
    todo = list(range(T))
    while todo:
        x = np.stack([xs[t] for t in todo])
        _, _, logits = oracle.route(lw.router_w, lw.router_bias, x, cfg.k, want_logits=True)
        bad = near_tie_tokens(logits, cfg.k)
        nxt = []
        for i in bad:
            t = todo[i]
            attempts[t] += 1
            xs[t] = synth.make_token(cfg, t, attempts[t], layer)
            nxt.append(t)
        todo = nxt
    return np.stack(xs) if T else synth.make_x(cfg, 0)


def normwise(a: np.ndarray, ref: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    return float(np.max(np.abs(a - ref)) / den) if den > 0 else float(np.max(np.abs(a - ref), initial=0.0))
