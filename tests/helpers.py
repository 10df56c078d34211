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


def with_outliers(x_tok: np.ndarray, seed: int, value: float = 64.0) -> np.ndarray:
    """One large element (+-value) per 256-element block, at a seeded position,
    among the token's ordinary values (a layout change of the input, no layer
    arithmetic). Works on fp32 values and on bf16 bit patterns."""
    x = x_tok.copy()
    nblk = x.shape[0] // 256
    pos = synth.rand_bytes(seed, (nblk, 2))
    for b in range(nblk):
        i = b * 256 + int(pos[b, 0])
        v = value if pos[b, 1] & 1 else -value
        if x.dtype == np.uint16:
            x[i] = np.float32(v).view(np.uint32) >> 16  # +-64 is exact in bf16
        else:
            x[i] = np.float32(v)
    return x


def screened_x(cfg: synth.Config, lw: synth.LayerWeights, T: int | None = None, layer: int = 0,
               outliers: bool = False):
    """Activations with no near-tie in the router: a rejected token is redrawn
    from its next stream (attempt + 1), as the input recipe prescribes. With
    ``outliers`` every drawn token gets one large element per 256-block."""
    T = cfg.T if T is None else T

    def draw(t, attempt):
        v = synth.make_token(cfg, t, attempt, layer)
        return with_outliers(v, synth.seed(cfg.seed, layer, 99, t + (attempt << 24))) if outliers else v

    xs = [draw(t, 0) for t in range(T)]
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
            xs[t] = draw(t, attempts[t])
            nxt.append(t)
        todo = nxt
    return np.stack(xs) if T else synth.make_x(cfg, 0)


def normwise(a: np.ndarray, ref: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    return float(np.max(np.abs(a - ref)) / den) if den > 0 else float(np.max(np.abs(a - ref), initial=0.0))


def elementwise(a: np.ndarray, ref: np.ndarray, floor_frac: float = 1e-3) -> float:
    """max |a - ref| / (|ref| + floor_frac * max |ref|): the element-wise relative
    error with a small absolute floor (reported beside the normwise figure)."""
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    if not ref.size:
        return 0.0
    fl = floor_frac * float(np.max(np.abs(ref)))
    return float(np.max(np.abs(a - ref) / (np.abs(ref) + fl))) if fl > 0 else float(np.max(np.abs(a - ref)))


def bf16_rne_bits(y: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of finite fp32 values, rounded to nearest with ties to even: add 0x7FFF plus the
    lowest kept bit to the fp32 bits, then drop the low 16 bits (a carry into the exponent is the correct
    rounding up to the next binade, or to infinity)."""
    assert np.all(np.isfinite(y))
    u = np.ascontiguousarray(y, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
