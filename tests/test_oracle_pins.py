"""Pins of the CPU oracle against facts fixed outside it (no GPU needed).

Every test here checks the fp64 oracle against something other than itself:
the SSD matrix (quadratic) form computed independently in numpy, closed forms
(dt*A = 0 cumulative sum, one-token documents, delta conv taps, the RMSNorm
norm identity, the inverse-softplus identity of the transplant article), a
hand-worked example, and invariants (document isolation, continuation).
"""
import json
import os

import numpy as np
import pytest

from brute_force import head_inputs, quadratic_form, silu, softplus
from selective_state_space_forward_b200.synthetic import (Workload, make_inputs, round_bf16,
                                                          softplus_inverse)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _small(**kw):
    base = dict(name="pin", batch=2, seqlen=200, nheads=4, headdim=8, dstate=6, ngroups=2,
                dconv=1, act_dtype="f32", seed=11)
    base.update(kw)
    return Workload(**base)


def _rel_err(got, want):
    return float(np.max(np.abs(got - want)) / max(np.max(np.abs(want)), 1e-300))


def _check_quadratic(oracle_mod, w, inp, tol=1e-11):
    dims = w.dims()
    res = oracle_mod.forward(dims, inp)
    for b in range(w.batch):
        for h in range(w.nheads):
            x, z, Bm, Cm, dt, a, D, seq, h0 = head_inputs(inp, dims, b, h)
            y, hf = quadratic_form(x, z, Bm, Cm, dt, a, D, seq, h0)
            got = res["out"][b, :, h * w.headdim:(h + 1) * w.headdim]
            assert _rel_err(got, y) < tol, (b, h)
            assert _rel_err(res["final_ssm"][b, h], hf) < tol, (b, h)


def _docs_with_boundaries(L, cuts):
    seq = np.zeros(L, dtype=np.int32)
    for c in sorted(cuts):
        seq[c:] += 1
    return seq


@pytest.mark.parametrize("init", [False, True])
def test_recurrence_equals_quadratic_form(oracle_mod, init):
    w = _small(init_state=init)
    inp = make_inputs(w)
    seq = np.stack([_docs_with_boundaries(w.seqlen, [1, 63, 64, 65, 120, 199]),
                    _docs_with_boundaries(w.seqlen, [])])
    inp["seq_idx"] = seq
    _check_quadratic(oracle_mod, w, inp)


def test_quadratic_form_per_token_a_with_floor(oracle_mod):
    w = _small(a_per_token=True, init_state=True, seqlen=130)
    inp = make_inputs(w)
    # a few rates at and inside the 1e-4 floor
    inp["A"][0, 5:9, 1] = np.array([0.0, -1e-6, -1e-4, -0.5], dtype=np.float32)
    inp["seq_idx"] = np.stack([_docs_with_boundaries(w.seqlen, [64]),
                               _docs_with_boundaries(w.seqlen, [0 + 1, 100])])
    _check_quadratic(oracle_mod, w, inp)


def test_quadratic_form_strong_decay_and_tiny_dt(oracle_mod):
    # decays that underflow (dt*A ~ -40 per token) and dt ~ 1e-7
    w = _small(seqlen=96, init_state=True)
    inp = make_inputs(w)
    inp["dt_raw"][0, :, 0] = 40.0
    inp["dt_raw"][1, :, 2] = -16.0
    _check_quadratic(oracle_mod, w, inp)


def test_decay_free_closed_form(oracle_mod):
    """A = 0: h_t = h0 + sum_{s<=t} dt_s x_s (x) B_s, a plain cumulative sum."""
    w = _small(init_state=True, seqlen=150)
    inp = make_inputs(w)
    inp["A"][:] = 0.0
    dims = w.dims()
    res = oracle_mod.forward(dims, inp)
    P, N, G, H = w.headdim, w.dstate, w.ngroups, w.nheads
    for b in range(w.batch):
        for h in range(H):
            g = h // (H // G)
            x = inp["x"][b, :, h * P:(h + 1) * P].astype(np.float64)
            Bm = inp["B"][b, :, g * N:(g + 1) * N].astype(np.float64)
            Cm = inp["C"][b, :, g * N:(g + 1) * N].astype(np.float64)
            z = inp["z"][b, :, h * P:(h + 1) * P].astype(np.float64)
            dt = softplus(inp["dt_raw"][b, :, h].astype(np.float64) + float(inp["dt_bias"][h]))
            Hs = inp["init_ssm"][b, h].astype(np.float64)[None] + np.cumsum(
                np.einsum("t,tp,tn->tpn", dt, x, Bm), axis=0)
            y = np.einsum("tpn,tn->tp", Hs, Cm) + float(inp["D"][h]) * x
            assert _rel_err(res["out"][b, :, h * P:(h + 1) * P], y * silu(z)) < 1e-12
            assert _rel_err(res["final_ssm"][b, h], Hs[-1]) < 1e-12


def test_every_token_its_own_document(oracle_mod):
    """seq_idx[t] = t: y_t = dt_t (B_t.C_t) x_t + D x_t, and the conv sees only
    the current token (plus, at t = 0, the initial conv history)."""
    w = _small(dconv=4, seqlen=40, init_state=True)
    inp = make_inputs(w)
    rng = np.random.default_rng(5)
    inp["init_conv"] = rng.standard_normal((w.batch, 3, w.conv_dim)).astype(np.float32)
    inp["seq_idx"] = np.tile(np.arange(w.seqlen, dtype=np.int32), (w.batch, 1))
    dims = w.dims()
    res = oracle_mod.forward(dims, inp)
    H, P, N, G = w.nheads, w.headdim, w.dstate, w.ngroups
    wc, bc = inp["conv_w"].astype(np.float64), inp["conv_b"].astype(np.float64)
    for b in range(w.batch):
        raw = np.concatenate([inp["x"][b], inp["B"][b], inp["C"][b]], axis=1).astype(np.float64)
        u = silu(bc[None, :] + wc[None, :, 3] * raw)
        u[0] = silu(bc + wc[:, 3] * raw[0] + np.einsum("kc,ck->c", inp["init_conv"][b, :3],
                                                       wc[:, :3]))
        for h in range(H):
            g = h // (H // G)
            x = u[:, h * P:(h + 1) * P]
            Bm = u[:, H * P + g * N:H * P + (g + 1) * N]
            Cm = u[:, H * P + G * N + g * N:H * P + G * N + (g + 1) * N]
            z = inp["z"][b, :, h * P:(h + 1) * P].astype(np.float64)
            dt = softplus(inp["dt_raw"][b, :, h].astype(np.float64) + float(inp["dt_bias"][h]))
            D = float(inp["D"][h])
            y = (dt * np.sum(Bm * Cm, axis=1))[:, None] * x + D * x
            h0 = inp["init_ssm"][b, h].astype(np.float64)
            y[0] += np.exp(dt[0] * float(inp["A"][h])) * (h0 @ Cm[0])
            assert _rel_err(res["out"][b, :, h * P:(h + 1) * P], y * silu(z)) < 1e-12
            last = dt[-1] * np.outer(x[-1], Bm[-1])
            assert _rel_err(res["final_ssm"][b, h], last) < 1e-12
        # final conv history: only the last token is in the last document
        fc = res["final_conv"][b]
        assert np.all(fc[:2] == 0.0) and np.array_equal(fc[2], raw[-1])


def test_conv_delta_taps_fix_tap_order(oracle_mod):
    """w[:,3] = 1 is identity+SiLU; w[:,0] = 1 delays by 3 tokens, reaching into
    the initial history -- this fixes which tap multiplies the current token."""
    w = _small(dconv=4, seqlen=20, batch=1)
    inp = make_inputs(w)
    rng = np.random.default_rng(3)
    hist = rng.standard_normal((1, 3, w.conv_dim)).astype(np.float32)
    inp["init_conv"] = hist
    raw = np.concatenate([inp["x"][0], inp["B"][0], inp["C"][0]], axis=1).astype(np.float64)
    dims = w.dims()
    for tap in (3, 0, 1):
        cw = np.zeros((w.conv_dim, 4), dtype=np.float32)
        cw[:, tap] = 1.0
        inp["conv_w"], inp["conv_b"] = cw, np.zeros(w.conv_dim, dtype=np.float32)
        u = oracle_mod.conv_stage(dims, inp)[0]
        padded = np.concatenate([hist[0].astype(np.float64), raw], axis=0)
        delay = 3 - tap
        want = silu(padded[3 - delay:3 - delay + w.seqlen])
        assert np.allclose(u, want, rtol=1e-14, atol=1e-300), tap


def test_conv_matches_padded_correlation(oracle_mod):
    w = _small(dconv=4, seqlen=50, batch=2)
    inp = make_inputs(w)
    rng = np.random.default_rng(4)
    inp["init_conv"] = rng.standard_normal((2, 3, w.conv_dim)).astype(np.float32)
    inp["seq_idx"] = np.stack([_docs_with_boundaries(50, [2, 3, 30]), np.zeros(50, np.int32)])
    u = oracle_mod.conv_stage(w.dims(), inp)
    for b in range(2):
        raw = np.concatenate([inp["x"][b], inp["B"][b], inp["C"][b]], axis=1).astype(np.float64)
        seq = inp["seq_idx"][b]
        for t in range(50):
            acc = inp["conv_b"].astype(np.float64).copy()
            for k in range(4):
                tau = t - 3 + k
                if tau >= 0:
                    v = raw[tau] if seq[tau] == seq[t] else 0.0
                else:
                    v = inp["init_conv"][b, tau + 3].astype(np.float64) if seq[t] == seq[0] else 0.0
                acc = acc + inp["conv_w"][:, k].astype(np.float64) * v
            assert np.allclose(u[b, t], silu(acc), rtol=1e-14, atol=1e-14)


def test_documents_are_isolated_bitwise(oracle_mod):
    """Changing one packed document changes no output of any other document
    (model card, 'Checkpoint and training': zero influence across documents)."""
    w = _small(dconv=4, seqlen=160, batch=1, init_state=True, a_per_token=True)
    inp = make_inputs(w)
    cuts = [1, 40, 64, 65, 100]
    seq = _docs_with_boundaries(w.seqlen, cuts)[None]
    inp["seq_idx"] = seq
    dims = w.dims()
    base = oracle_mod.forward(dims, inp)
    rng = np.random.default_rng(9)
    ndoc = int(seq.max()) + 1
    for k in range(ndoc):
        sel = seq[0] == k
        pert = {key: (None if v is None else np.array(v)) for key, v in inp.items()}
        for key in ("x", "z", "B", "C", "dt_raw", "A"):
            pert[key][0, sel] += rng.standard_normal(pert[key][0, sel].shape).astype(np.float32)
        pert["A"] = -np.abs(pert["A"])
        res = oracle_mod.forward(dims, pert)
        other = ~sel
        assert np.array_equal(res["out"][0, other], base["out"][0, other]), k
        assert not np.array_equal(res["out"][0, sel], base["out"][0, sel]), k
        if k != ndoc - 1:
            assert np.array_equal(res["final_ssm"], base["final_ssm"]), k
            assert np.array_equal(res["final_conv"], base["final_conv"]), k


def test_packed_documents_equal_separate_calls(oracle_mod):
    """A document packed in a row gives the outputs of the same document run as
    its own call, bit for bit (model card, Checkpoint and training: packed and
    separately launched documents differ only by the GPU's reduction order;
    the sequential oracle has none).  The first document also carries the
    row's initial state, and the last one hands its state out."""
    w = _small(dconv=4, seqlen=160, batch=1, init_state=True, a_per_token=True)
    inp = make_inputs(w)
    rng = np.random.default_rng(4)
    inp["init_conv"] = rng.standard_normal((1, 3, w.conv_dim)).astype(np.float32)
    seq = _docs_with_boundaries(w.seqlen, [1, 40, 64, 65, 100])[None]
    inp["seq_idx"] = seq
    packed = oracle_mod.forward(w.dims(), inp)
    ndoc = int(seq.max()) + 1
    for k in range(ndoc):
        idx = np.flatnonzero(seq[0] == k)
        lo, hi = int(idx[0]), int(idx[-1]) + 1
        alone = dict(inp, seq_idx=None)
        for key in ("x", "z", "B", "C", "dt_raw", "A"):
            alone[key] = np.ascontiguousarray(inp[key][:, lo:hi])
        if k > 0:
            alone["init_ssm"] = alone["init_conv"] = None
        r = oracle_mod.forward(dict(w.dims(), seqlen=hi - lo), alone)
        assert np.array_equal(r["out"][0], packed["out"][0, lo:hi]), k
        if k == ndoc - 1:
            assert np.array_equal(r["final_ssm"], packed["final_ssm"])
            assert np.array_equal(r["final_conv"], packed["final_conv"])


def test_prefill_then_steps_continues_the_sequence(oracle_mod):
    """forward(L1) -> state -> steps == forward(L1 + M) (Mamba3Block.step: decoding
    continues a prefill).  The state crosses the call boundary as fp32."""
    w = _small(dconv=4, seqlen=70, batch=2, init_state=True)
    inp = make_inputs(w)
    dims = w.dims()
    full = oracle_mod.forward(dims, inp)
    L1 = 61
    part = {k: (v[:, :L1] if (v is not None and k in ("x", "z", "B", "C", "dt_raw")) else v)
            for k, v in inp.items()}
    d1 = dict(dims, seqlen=L1)
    r1 = oracle_mod.forward(d1, part)
    ssm = r1["final_ssm"].astype(np.float32)
    conv = r1["final_conv"].astype(np.float32)
    assert _rel_err(r1["out"], full["out"][:, :L1]) == 0.0
    for t in range(L1, w.seqlen):
        tok = {k: (v[:, t:t + 1] if (v is not None and k in ("x", "z", "B", "C", "dt_raw")) else v)
               for k, v in inp.items()}
        r = oracle_mod.step(dims, tok, ssm, conv)
        assert _rel_err(r["out"][:, 0], full["out"][:, t]) < 1e-6, t
        ssm, conv = r["final_ssm"].astype(np.float32), r["final_conv"].astype(np.float32)
    assert _rel_err(ssm, full["final_ssm"]) < 1e-6
    assert np.array_equal(conv, full["final_conv"].astype(np.float32))


def test_split_prefill_equals_one_prefill(oracle_mod):
    w = _small(dconv=4, seqlen=150, batch=1, init_state=True)
    inp = make_inputs(w)
    inp["seq_idx"] = _docs_with_boundaries(150, [90])[None]
    dims = w.dims()
    full = oracle_mod.forward(dims, inp)
    for L1 in (1, 2, 64, 100):
        a = {k: (v[:, :L1] if (v is not None and k in ("x", "z", "B", "C", "dt_raw", "seq_idx"))
                 else v) for k, v in inp.items()}
        r1 = oracle_mod.forward(dict(dims, seqlen=L1), a)
        b = {k: (v[:, L1:] if (v is not None and k in ("x", "z", "B", "C", "dt_raw", "seq_idx"))
                 else v) for k, v in inp.items()}
        b["init_ssm"] = r1["final_ssm"].astype(np.float32)
        b["init_conv"] = r1["final_conv"].astype(np.float32)
        r2 = oracle_mod.forward(dict(dims, seqlen=150 - L1), b)
        got = np.concatenate([r1["out"], r2["out"]], axis=1)
        assert _rel_err(got, full["out"]) < 1e-6, L1
        assert _rel_err(r2["final_ssm"], full["final_ssm"]) < 1e-6, L1


def test_inverse_softplus_identity(oracle_mod):
    """softplus(log(exp(u) - 1)) = u (transplant article, inverse-softplus
    reparameterisation): with dt_raw = 0 the oracle's dt returns u."""
    rng = np.random.default_rng(0)
    u = np.concatenate([np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), 500)),
                        np.exp(rng.uniform(np.log(1e-4), np.log(20.0), 500))])
    H = u.size
    bias = softplus_inverse(u).astype(np.float32)
    inp = dict(x=np.zeros((1, 1, H)), z=np.zeros((1, 1, H)), B=np.zeros((1, 1, 1)),
               C=np.zeros((1, 1, 1)), dt_raw=np.zeros((1, 1, H)), dt_bias=bias,
               A=-np.ones(H), D=np.zeros(H))
    dims = dict(batch=1, seqlen=1, nheads=H, headdim=1, dstate=1, ngroups=1, dconv=1)
    dt, a = oracle_mod.dt_stage(dims, inp)
    # the only error is bias's rounding to fp32, scaled by softplus' <= 1 slope
    tol = np.abs(bias.astype(np.float64)) * 2.0 ** -24 + 1e-300
    assert np.all(np.abs(dt[0, 0] - u) <= tol + 2e-16 * u)
    # softplus of large arguments is the argument itself to within e^-v
    big = np.array([20.5, 30.0, 60.0], dtype=np.float32)
    d2 = dict(dims, nheads=3)
    inp2 = dict(inp, x=np.zeros((1, 1, 3)), z=np.zeros((1, 1, 3)), dt_raw=np.zeros((1, 1, 3)),
                dt_bias=big, A=-np.ones(3), D=np.zeros(3))
    dt2, _ = oracle_mod.dt_stage(d2, inp2)
    assert np.allclose(dt2[0, 0], big.astype(np.float64) + np.exp(-big.astype(np.float64)),
                       rtol=1e-15, atol=0)


def test_a_floor(oracle_mod):
    """Per-token A is clamped to |A| >= 1e-4 (Mamba3Block, 'A floor 1e-4'); a
    per-token A equal to the per-head A everywhere gives the per-head result."""
    H = 6
    A = np.array([[[0.0, -1e-6, -1e-4, -0.5, -3.0, -1e-5]]], dtype=np.float32)
    inp = dict(x=np.zeros((1, 1, H)), z=np.zeros((1, 1, H)), B=np.zeros((1, 1, 1)),
               C=np.zeros((1, 1, 1)), dt_raw=np.zeros((1, 1, H)), dt_bias=np.zeros(H),
               A=A, D=np.zeros(H))
    dims = dict(batch=1, seqlen=1, nheads=H, headdim=1, dstate=1, ngroups=1, dconv=1,
                a_per_token=1)
    _, a = oracle_mod.dt_stage(dims, inp)
    want = np.array([-1e-4, -1e-4, -1e-4, float(np.float32(-0.5)), -3.0, -1e-4])
    assert np.array_equal(a[0, 0], want)

    w = _small(init_state=True, seqlen=80)
    base = make_inputs(w)
    tok = dict(base)
    tok["A"] = np.broadcast_to(base["A"], (w.batch, w.seqlen, w.nheads)).copy()
    r_head = oracle_mod.forward(w.dims(), base)
    r_tok = oracle_mod.forward(dict(w.dims(), a_per_token=1), tok)
    assert np.array_equal(r_head["out"], r_tok["out"])
    assert np.array_equal(r_head["final_ssm"], r_tok["final_ssm"])


def test_bc_norm_closed_forms(oracle_mod):
    """With unit weight and zero bias, |B_hat|^2 = N * m / (m + 1e-5), m = mean(B^2);
    with B = 0 the normalised B is the head's bias (Mamba3Block Parameters)."""
    w = _small(bc_norm=True, ngroups=1, seqlen=30, batch=1, dstate=16)
    inp = make_inputs(w)
    N = w.dstate
    inp["B_norm_w"] = np.ones(N, np.float32)
    inp["C_norm_w"] = np.ones(N, np.float32)
    bias_b = inp["B_bias"].copy()
    inp["B_bias"] = np.zeros_like(bias_b)
    inp["B"][0, 7] = 0.0
    bh, ch = oracle_mod.bcnorm_stage(w.dims(), inp)
    m = np.mean(inp["B"][0].astype(np.float64) ** 2, axis=1)
    norm2 = np.sum(bh[0] ** 2, axis=2)
    assert np.allclose(norm2, (N * m / (m + 1e-5))[:, None], rtol=1e-13, atol=1e-300)
    inp["B_bias"] = bias_b
    bh, ch = oracle_mod.bcnorm_stage(w.dims(), inp)
    assert np.array_equal(bh[0, 7], bias_b.astype(np.float64))


def test_bc_norm_is_applied_per_head_in_the_scan(oracle_mod):
    """A normed G=1 scan equals an un-normed G=H scan fed each head's B_hat, C_hat."""
    w = _small(bc_norm=True, ngroups=1, seqlen=70, batch=2, dstate=16, init_state=True)
    inp = make_inputs(w)
    inp["B_norm_w"] = (1.0 + 0.1 * np.arange(16)).astype(np.float32)
    dims = w.dims()
    res = oracle_mod.forward(dims, inp)
    bh, ch = oracle_mod.bcnorm_stage(dims, inp)
    H, N = w.nheads, w.dstate
    flat = dict(inp)
    flat["B"] = bh.reshape(w.batch, w.seqlen, H * N).astype(np.float32)
    flat["C"] = ch.reshape(w.batch, w.seqlen, H * N).astype(np.float32)
    res2 = oracle_mod.forward(dict(dims, ngroups=H, bc_norm=0), flat)
    assert _rel_err(res2["out"], res["out"]) < 1e-6
    assert _rel_err(res2["final_ssm"], res["final_ssm"]) < 1e-6


def test_heads_share_groups_contiguously(oracle_mod):
    """Head h reads group h // (H / G): a 4-head, 2-group scan's head 3 equals a
    1-head scan given group 1's B and C."""
    w = _small(seqlen=64, batch=1)
    inp = make_inputs(w)
    dims = w.dims()
    res = oracle_mod.forward(dims, inp)
    P, N = w.headdim, w.dstate
    for h in range(4):
        g = h // 2
        one = dict(x=inp["x"][:, :, h * P:(h + 1) * P], z=inp["z"][:, :, h * P:(h + 1) * P],
                   B=inp["B"][:, :, g * N:(g + 1) * N], C=inp["C"][:, :, g * N:(g + 1) * N],
                   dt_raw=inp["dt_raw"][:, :, h:h + 1], dt_bias=inp["dt_bias"][h:h + 1],
                   A=inp["A"][h:h + 1], D=inp["D"][h:h + 1])
        r1 = oracle_mod.forward(dict(dims, nheads=1, ngroups=1), one)
        assert np.array_equal(r1["out"][0], res["out"][0, :, h * P:(h + 1) * P])


def test_hand_worked_scalar_example(oracle_mod):
    with open(os.path.join(GOLDEN, "scalar_decay_half.json")) as f:
        g = json.load(f)
    i = g["inputs"]
    L = len(i["x"])
    ln2 = np.log(2.0)
    for case in g["cases"]:
        inp = dict(x=np.array(i["x"]).reshape(1, L, 1), z=np.array(i["z"]).reshape(1, L, 1),
                   B=np.array(i["B"]).reshape(1, L, 1), C=np.array(i["C"]).reshape(1, L, 1),
                   dt_raw=np.array(i["dt_raw"]).reshape(1, L, 1),
                   dt_bias=np.array([i["dt_bias"]]), A=np.array([i["A"]]), D=np.array([i["D"]]),
                   init_ssm=np.full((1, 1, 1, 1), i["init_ssm"]),
                   seq_idx=None if case["seq_idx"] is None else np.array([case["seq_idx"]]))
        dims = dict(batch=1, seqlen=L, nheads=1, headdim=1, dstate=1, ngroups=1, dconv=1)
        res = oracle_mod.forward(dims, inp)
        y = np.array([r + k * ln2 for r, k in case["y_before_gate"]])
        zv = np.array(i["z"])
        assert np.allclose(res["out"][0, :, 0], y * silu(zv), rtol=1e-14, atol=1e-15)
        r, k = case["final_ssm"]
        assert abs(res["final_ssm"][0, 0, 0, 0] - (r + k * ln2)) < 1e-14


def test_generator_rounds_to_bf16_and_is_seeded():
    w = _small(act_dtype="bf16")
    a, b = make_inputs(w), make_inputs(w)
    for k in ("x", "z", "B", "C"):
        assert np.array_equal(a[k], b[k])
        assert np.all((a[k].view(np.uint32) & 0xFFFF) == 0)
    assert np.array_equal(round_bf16(np.float32(1.0 + 2 ** -8)), np.float32(1.0))  # tie -> even
    assert np.array_equal(round_bf16(np.float32(1.0 + 3 * 2 ** -8)), np.float32(1.0 + 2 ** -6))


def test_document_ids_are_compared_between_neighbours(oracle_mod):
    """A boundary is where the id changes from one token to the next, so an id
    that recurs later still starts a new document: [0,0,1,1,0,0] behaves like
    [0,0,1,1,2,2] in both the conv and the scan."""
    w = _small(dconv=4, seqlen=48, batch=1, init_state=True)
    inp = make_inputs(w)
    rng = np.random.default_rng(8)
    inp["init_conv"] = rng.standard_normal((1, 3, w.conv_dim)).astype(np.float32)
    a = _docs_with_boundaries(48, [10, 11, 30])
    recur = np.where(a == 2, 0, a).astype(np.int32)    # [0..,1,2(->0)..,3]
    inp["seq_idx"] = recur[None]
    r1 = oracle_mod.forward(w.dims(), inp)
    inp["seq_idx"] = a[None]
    r2 = oracle_mod.forward(w.dims(), inp)
    assert np.array_equal(r1["out"], r2["out"])
    assert np.array_equal(r1["final_ssm"], r2["final_ssm"])
    assert np.array_equal(r1["final_conv"], r2["final_conv"])


def _row_slice(inp, b, L):
    """Row b of a batch, truncated to its first L tokens, as a batch of one."""
    per_tok = ("x", "z", "B", "C", "dt_raw", "seq_idx")
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif k in per_tok or (k == "A" and v.ndim == 3):
            out[k] = np.ascontiguousarray(v[b:b + 1, :L])
        elif k in ("init_ssm", "init_conv"):
            out[k] = np.ascontiguousarray(v[b:b + 1])
        else:
            out[k] = v
    return out


@pytest.mark.parametrize("a_per_token", [False, True])
def test_ragged_rows_equal_truncated_rows(oracle_mod, a_per_token):
    """Ragged lengths: each row equals the same row run alone over its real
    tokens, padding outputs are exactly +0.0, and a zero-length row hands its
    initial state and conv history through unchanged."""
    w = _small(batch=4, seqlen=150, dconv=4, init_state=True, a_per_token=a_per_token,
               documents="geometric", mean_doc_len=40)
    inp = make_inputs(w)
    rng = np.random.Generator(np.random.PCG64(5))
    inp["init_conv"] = (0.5 * rng.standard_normal((w.batch, 3, w.conv_dim))).astype(np.float32)
    lengths = np.array([150, 77, 0, 1], dtype=np.int32)
    res = oracle_mod.forward(w.dims(), dict(inp, lengths=lengths))
    for b, L in enumerate(lengths):
        pad = res["out"][b, L:]
        assert np.all(pad == 0.0) and not np.any(np.signbit(pad)), "padding must be +0.0"
        if L == 0:
            assert np.array_equal(res["final_ssm"][b], inp["init_ssm"][b].astype(np.float64))
            assert np.array_equal(res["final_conv"][b], inp["init_conv"][b].astype(np.float64))
            continue
        one = oracle_mod.forward(w.with_(batch=1, seqlen=int(L)).dims(), _row_slice(inp, b, int(L)))
        assert np.array_equal(res["out"][b, :L], one["out"][0])
        assert np.array_equal(res["final_ssm"][b], one["final_ssm"][0])
        assert np.array_equal(res["final_conv"][b], one["final_conv"][0])


def test_full_lengths_equal_no_lengths(oracle_mod):
    w = _small(batch=2, seqlen=90, dconv=4, documents="geometric", mean_doc_len=30)
    inp = make_inputs(w)
    a = oracle_mod.forward(w.dims(), inp)
    b = oracle_mod.forward(w.dims(), dict(inp, lengths=np.full(w.batch, w.seqlen, np.int32)))
    for k in ("out", "final_ssm", "final_conv"):
        assert np.array_equal(a[k], b[k])
