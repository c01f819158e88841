"""Pins of the Mamba-1 selective-scan (S6) oracle (no GPU needed).

The S6 scan (falcon_mamba.ts header: Falcon-Mamba is a Mamba-1 / S6 model;
A = -exp(clamp(A_log, -10, 5)) as selective_scan.ts computes it; dt =
softplus(dt + bias)) is pinned against things other than itself: its matrix
form written independently in numpy, the SSD oracle (itself pinned) in the
special case where every state of a channel shares one decay, the clamp
bounds of A_log, and closed forms at strong decay and at dt -> 0.
"""
import numpy as np
import pytest

import oracle


def _inputs(B=2, L=40, DI=5, N=6, seed=0, gate=True, init=True):
    rng = np.random.Generator(np.random.PCG64(seed))
    f = np.float32
    return dict(u=rng.standard_normal((B, L, DI)).astype(f),
                delta=(rng.standard_normal((B, L, DI)) - 1.0).astype(f),
                z=rng.standard_normal((B, L, DI)).astype(f) if gate else None,
                B=rng.standard_normal((B, L, N)).astype(f),
                C=rng.standard_normal((B, L, N)).astype(f),
                A_log=rng.uniform(-1.0, 2.5, (DI, N)).astype(f),
                delta_bias=rng.uniform(-1.0, 0.5, DI).astype(f),
                D=rng.uniform(0.0, 1.0, DI).astype(f),
                init=(0.1 * rng.standard_normal((B, DI, N))).astype(f) if init else None)


def _matrix_form(inp):
    """y_t = sum_{s<=t} sum_n C_t[n] B_s[n] e^{A[n](T_t - T_s)} dt_s u_s
             + sum_n C_t[n] e^{A[n] T_t} h0[n] + D u_t,  T_t = sum_{r<=t} dt_r."""
    u = inp["u"].astype(np.float64)
    Bm, Cm = inp["B"].astype(np.float64), inp["C"].astype(np.float64)
    Bb, L, DI = u.shape
    A = -np.exp(np.clip(inp["A_log"].astype(np.float64), -10.0, 5.0))          # (DI, N)
    dt = np.logaddexp(0.0, inp["delta"].astype(np.float64) + inp["delta_bias"].astype(np.float64))
    T = np.cumsum(dt, axis=1)                                                    # (B, L, DI)
    out = np.zeros((Bb, L, DI))
    fin = np.zeros((Bb, DI, A.shape[1]))
    for b in range(Bb):
        for d in range(DI):
            Td = T[b, :, d]
            gap = Td[:, None] - Td[None, :]                                      # (t, s)
            causal = np.tril(np.ones((L, L), dtype=bool))
            w = dt[b, :, d] * u[b, :, d]                                         # (s,)
            # decay[t, s, n]
            decay = np.where(causal[:, :, None],
                             np.exp(np.maximum(gap, 0.0)[:, :, None] * A[d][None, None, :]), 0.0)
            cb = Cm[b][:, None, :] * Bm[b][None, :, :]                          # (t, s, n)
            y = np.einsum("tsn,s->t", cb * decay, w)
            h0 = inp["init"][b, d].astype(np.float64) if inp.get("init") is not None else 0.0
            y += (Cm[b] * np.exp(Td[:, None] * A[d][None, :]) * h0).sum(axis=1)
            y += inp["D"][d] * u[b, :, d]
            if inp.get("z") is not None:
                zz = inp["z"][b, :, d].astype(np.float64)
                y = y * zz / (1.0 + np.exp(-zz))
            out[b, :, d] = y
            fin[b, d] = np.exp(A[d] * Td[-1]) * h0 + (np.exp(A[d][None, :] * (Td[-1] - Td)[:, None])
                                                       * (w[:, None] * Bm[b])).sum(axis=0)
    return out, fin


@pytest.mark.parametrize("gate,init", [(True, True), (False, False)])
def test_s6_equals_its_matrix_form(oracle_mod, gate, init):
    inp = _inputs(gate=gate, init=init)
    r = oracle.s6_forward(inp)
    y, hf = _matrix_form(inp)
    assert np.max(np.abs(r["out"] - y)) <= 1e-11 * np.max(np.abs(y))
    assert np.max(np.abs(r["final"] - hf)) <= 1e-11 * np.max(np.abs(hf))


def test_s6_with_one_decay_per_channel_is_the_ssd_scan(oracle_mod):
    """A[d, n] = A_d for every n: the S6 scan is the SSD scan with one head per
    channel, head dim 1, one B/C group and no conv."""
    inp = _inputs(B=2, L=70, DI=4, N=5, seed=3)
    inp["A_log"] = np.repeat(inp["A_log"][:, :1], 5, axis=1)
    r = oracle.s6_forward(inp)
    Bb, L, DI = inp["u"].shape
    dims = dict(batch=Bb, seqlen=L, nheads=DI, headdim=1, dstate=5, ngroups=1, dconv=1,
                a_per_token=0, bc_norm=0)
    A = (-np.exp(np.clip(inp["A_log"][:, 0].astype(np.float64), -10, 5))).astype(np.float32)
    ssd = oracle.forward(dims, dict(x=inp["u"], z=inp["z"], B=inp["B"], C=inp["C"],
                                    dt_raw=inp["delta"], dt_bias=inp["delta_bias"], A=A,
                                    D=inp["D"], conv_w=None, conv_b=None, seq_idx=None,
                                    init_ssm=inp["init"].reshape(Bb, DI, 1, 5)))
    # the S6 oracle applies the exponential to the fp32 A_log, the SSD one receives
    # A rounded to fp32: agreement to fp32 rounding of A
    assert np.max(np.abs(r["out"] - ssd["out"])) <= 1e-5 * np.max(np.abs(ssd["out"]))
    assert np.max(np.abs(r["final"] - ssd["final_ssm"][:, :, 0, :])) <= 1e-5 * np.max(np.abs(r["final"]))


def test_s6_a_log_is_clamped_to_minus_10_and_5(oracle_mod):
    inp = _inputs(seed=4)
    base = oracle.s6_forward(inp)
    far = dict(inp, A_log=np.where(inp["A_log"] > 1.0, np.float32(9.0), np.float32(-30.0)))
    near = dict(inp, A_log=np.where(inp["A_log"] > 1.0, np.float32(5.0), np.float32(-10.0)))
    a, b = oracle.s6_forward(far), oracle.s6_forward(near)
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["final"], b["final"])
    assert not np.array_equal(a["out"], base["out"])


def test_s6_strong_decay_forgets_the_past(oracle_mod):
    """A = -e^5 and dt ~ 20: e^{dt A} underflows to 0, so h_t = dt_t u_t B_t and
    y_t = dt_t u_t (C_t . B_t) + D u_t exactly (no gate)."""
    inp = _inputs(seed=5, gate=False)
    inp["A_log"] = np.full_like(inp["A_log"], 5.0)
    inp["delta"] = np.full_like(inp["delta"], 20.0)
    inp["delta_bias"] = np.zeros_like(inp["delta_bias"])
    r = oracle.s6_forward(inp)
    dt = 20.0 + np.log1p(np.exp(-20.0))
    u = inp["u"].astype(np.float64)
    cb = np.sum(inp["C"].astype(np.float64) * inp["B"].astype(np.float64), axis=2)   # (B, L)
    want = dt * u * cb[:, :, None] + inp["D"][None, None, :] * u
    assert np.max(np.abs(r["out"] - want)) <= 1e-12 * np.max(np.abs(want))


def test_s6_vanishing_dt_keeps_the_initial_state(oracle_mod):
    """dt -> 0 (delta = -60): the state stays h0 and y_t = C_t . h0 + D u_t."""
    inp = _inputs(seed=6, gate=False)
    inp["delta"] = np.full_like(inp["delta"], -60.0)
    inp["delta_bias"] = np.zeros_like(inp["delta_bias"])
    r = oracle.s6_forward(inp)
    h0 = inp["init"].astype(np.float64)                                       # (B, DI, N)
    want = (np.einsum("bln,bdn->bld", inp["C"].astype(np.float64), h0)
            + inp["D"].astype(np.float64) * inp["u"].astype(np.float64))
    assert np.max(np.abs(r["out"] - want)) <= 1e-12 * np.max(np.abs(want))
    assert np.max(np.abs(r["final"] - h0)) <= 1e-20 + 1e-12 * np.max(np.abs(h0))
