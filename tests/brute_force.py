"""Independent numpy forms used to pin the oracle (tests only).

`quadratic_form` evaluates the scan as one masked matrix product per head,
y = (L o C B^T o dt) x + D x (+ the initial-state term), the "dense" form of
the selective SSM, which shares no loop structure with the oracle's token-by-
token recurrence.  The two agree only if the decay products, the document
masks, the dt/B/C/x indexing and the state carry are all right.
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit


def silu(v):
    return v * expit(v)


def softplus(v):
    return np.logaddexp(0.0, v)


def head_inputs(inp: dict, dims: dict, b: int, h: int):
    """Slice row b / head h out of a workload's inputs (no conv, no B/C norm)."""
    H, P, N, G = dims["nheads"], dims["headdim"], dims["dstate"], dims["ngroups"]
    g = h // (H // G)
    x = inp["x"][b, :, h * P:(h + 1) * P].astype(np.float64)
    z = inp["z"][b, :, h * P:(h + 1) * P].astype(np.float64)
    Bm = inp["B"][b, :, g * N:(g + 1) * N].astype(np.float64)
    Cm = inp["C"][b, :, g * N:(g + 1) * N].astype(np.float64)
    dt = softplus(inp["dt_raw"][b, :, h].astype(np.float64) + float(inp["dt_bias"][h]))
    if dims.get("a_per_token"):
        a = np.minimum(inp["A"][b, :, h].astype(np.float64), -1e-4)
    else:
        a = np.full(x.shape[0], float(inp["A"][h]))
    seq = None if inp.get("seq_idx") is None else np.asarray(inp["seq_idx"][b])
    h0 = None if inp.get("init_ssm") is None else inp["init_ssm"][b, h].astype(np.float64)
    return x, z, Bm, Cm, dt, a, float(inp["D"][h]), seq, h0


def quadratic_form(x, z, Bm, Cm, dt, a, D, seq=None, h0=None):
    """Gated outputs (L, P) and final state (P, N) of one head, by the matrix form."""
    L = x.shape[0]
    cs = np.cumsum(dt * a)
    doc = np.zeros(L, dtype=np.int64) if seq is None else np.asarray(seq)
    t = np.arange(L)
    same = doc[:, None] == doc[None, :]
    causal = t[:, None] >= t[None, :]
    seg = np.where(causal, cs[:, None] - cs[None, :], 0.0)
    decay = np.where(causal & same, np.exp(seg), 0.0)
    M = (Cm @ Bm.T) * decay * dt[None, :]
    y = M @ x + D * x
    if h0 is not None:
        first = (doc == doc[0]).astype(np.float64)
        y = y + (first * np.exp(cs))[:, None] * (Cm @ h0.T)
    out = y * silu(z)
    w = np.where(doc == doc[-1], np.exp(cs[-1] - cs) * dt, 0.0)
    hf = (x * w[:, None]).T @ Bm
    if h0 is not None and doc[-1] == doc[0]:
        hf = hf + np.exp(cs[-1]) * h0
    return out, hf
