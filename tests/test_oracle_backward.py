"""Pins of the oracle's backward (the gradients of a zero-state prefill).

The backward is checked against the forward oracle itself, by numerical
differentiation, which shares nothing with the hand-written reverse sweep:

  * directional derivatives: for every input and weight T and an integer
    direction v, <dL/dT, v> must equal d/de <gout, out(T + e v)> at e = 0,
    taken by central differences at two step sizes and Richardson
    extrapolation (error O(e^4));
  * brute force on a tiny case: the same, one element at a time, for every
    element of every input and weight;
  * the document gate of the Mini-K3-1H model card (Checkpoint and training:
    a loss on a later document gives exactly zero gradient on earlier
    documents' inputs), and packed-versus-alone equality of a document's
    gradients;
  * ragged rows: padding takes no gradient, and a row's gradients equal the
    same row run alone over its real tokens;
  * autograd (torch, float64, CPU) of an independent implementation: the SSD
    matrix form of the whole forward, conv and B/C norm included.

Inputs are put on a coarse binary grid (multiples of 2^-8) so that every
perturbed value x +- e v (e = 2^-12, 2^-13, |v| <= 4) is exactly a float32: the
difference quotients then see exactly the step they divide by.
"""
import numpy as np
import pytest

from selective_state_space_forward_b200.synthetic import Workload, make_inputs

import oracle

E = 2.0 ** -12
GRID = 8


def grid(a, q=GRID):
    if a is None:
        return None
    return (np.round(np.asarray(a, np.float64) * 2.0 ** q) / 2.0 ** q).astype(np.float32)


def docs(L, cuts):
    seq = np.zeros(L, dtype=np.int32)
    for c in cuts:
        seq[c:] += 1
    return seq


def case(conv: bool, seed: int, batch=2, L=70, H=4, P=3, N=5, G=2):
    """A small problem on the grid.  With conv: documents (a 1-token one
    included), per-head A, G groups.  Without: the B/C norm with non-unit
    weights and biases, per-token A with entries the floor replaces."""
    if conv:
        w = Workload("bw", batch, L, H, P, N, G, 4, "f32", seed=seed)
    else:
        w = Workload("bn", batch, L, H, P, N, 1, 1, "f32", a_per_token=True, bc_norm=True,
                     seed=seed)
    inp = {k: (grid(v) if isinstance(v, np.ndarray) and v.dtype == np.float32 else v)
           for k, v in make_inputs(w).items()}
    rng = np.random.default_rng(seed + 100)
    if conv:
        seq = np.stack([docs(L, [9, 10, 40]) for _ in range(batch)])
        seq[-1] = docs(L, [L // 2])
        inp["seq_idx"] = seq
    else:
        inp["B_norm_w"] = grid(1 + 0.3 * rng.standard_normal(N))
        inp["C_norm_w"] = grid(1 + 0.3 * rng.standard_normal(N))
        inp["B_bias"] = grid(0.3 * rng.standard_normal((H, N)))
        inp["C_bias"] = grid(0.3 * rng.standard_normal((H, N)))
        # replaced by the floor -1e-4, and still so after any perturbation below
        inp["A"][0, 3, 1] = 0.25
        inp["A"][-1, L - 1, 0] = 0.5
    gout = grid(rng.standard_normal((batch, L, H * P)))
    return w.dims(), inp, gout


def objective(dims, inp, gout, lib=None):
    out = oracle.forward(dims, inp, final=False, lib=lib)["out"]
    return float(np.dot(out.ravel(), gout.astype(np.float64).ravel()))


def directional_fd(dims, inp, gout, name, v, lib=None):
    """d/de <gout, out(inp[name] + e v)> at 0, Richardson-extrapolated."""
    base = inp[name].astype(np.float64)

    def central(e):
        plus, minus = base + e * v, base - e * v
        assert np.array_equal(plus.astype(np.float32).astype(np.float64), plus)
        assert np.array_equal(minus.astype(np.float32).astype(np.float64), minus)
        fp = objective(dims, dict(inp, **{name: plus.astype(np.float32)}), gout, lib)
        fm = objective(dims, dict(inp, **{name: minus.astype(np.float32)}), gout, lib)
        return (fp - fm) / (2 * e)

    return (4 * central(E / 2) - central(E)) / 3


def check_directional(dims, inp, gout, seed, lib=None, grads=None):
    """Names of the gradients whose directional derivative disagrees."""
    g = grads if grads is not None else oracle.backward(dims, inp, gout, lib=lib)
    rng = np.random.default_rng(seed)
    bad = []
    for name in sorted(k for k, val in g.items() if val is not None):
        v = rng.integers(-4, 5, size=np.shape(inp[name])).astype(np.float64)
        an = float(np.sum(g[name] * v))
        # the reference derivative comes from the unmodified forward
        fd = directional_fd(dims, inp, gout, name, v)
        scale = np.linalg.norm(g[name]) * np.linalg.norm(v) + 1e-300
        if not abs(an - fd) <= 1e-8 * scale:
            bad.append(name)
    return bad


@pytest.mark.parametrize("conv", [True, False], ids=["conv_docs_groups", "bcnorm_per_token_A"])
def test_every_gradient_matches_directional_differences(oracle_mod, conv):
    dims, inp, gout = case(conv, seed=31 if conv else 32)
    assert check_directional(dims, inp, gout, seed=7) == []


@pytest.mark.parametrize("conv", [True, False], ids=["conv_docs", "bcnorm_per_token_A"])
def test_every_element_matches_central_differences(oracle_mod, conv):
    dims, inp, gout = case(conv, seed=41, batch=1, L=7, H=2, P=2, N=3, G=1)
    if conv:
        inp["seq_idx"] = docs(7, [3, 4])[None]
    else:
        inp["A"][0, 2, 0] = 0.25
    g = oracle.backward(dims, inp, gout)
    for name, gv in g.items():
        if gv is None:
            continue
        flat = gv.reshape(-1)
        for i in range(flat.size):
            v = np.zeros(flat.size)
            v[i] = 1.0
            fd = directional_fd(dims, inp, gout, name, v.reshape(gv.shape))
            assert abs(flat[i] - fd) <= 1e-9 * max(1.0, abs(fd)), (name, i, flat[i], fd)


def test_floored_A_takes_no_gradient(oracle_mod):
    dims, inp, gout = case(False, seed=33)
    g = oracle.backward(dims, inp, gout)
    assert g["A"][0, 3, 1] == 0.0 and g["A"][-1, -1, 0] == 0.0
    # the decay of a document's first token multiplies the zero state: no
    # gradient there either; every other token's decay rate has one
    assert np.all(g["A"][:, 0, :] == 0.0)
    assert np.count_nonzero(g["A"]) == g["A"].size - 2 - g["A"].shape[0] * g["A"].shape[2]


def test_later_document_loss_gives_zero_gradient_elsewhere(oracle_mod):
    """Only document 2 of row 0 carries a loss: every per-token gradient of
    every other document is exactly zero, and document 2's gradients are
    those of document 2 run alone (bit for bit)."""
    dims, inp, gout = case(True, seed=34, batch=1)
    seq = docs(70, [9, 10, 40])[None]            # documents [0,9) [9,10) [10,40) [40,70)
    inp["seq_idx"] = seq
    lo, hi = 10, 40
    g_only = np.zeros_like(gout)
    g_only[:, lo:hi] = gout[:, lo:hi]
    g = oracle.backward(dims, inp, g_only)
    for name in ("x", "z", "B", "C", "dt_raw"):
        outside = np.concatenate([g[name][0, :lo], g[name][0, hi:]])
        assert np.all(outside == 0.0), name
        assert np.any(g[name][0, lo:hi] != 0.0), name

    alone = {k: v for k, v in inp.items()}
    for k in ("x", "z", "B", "C", "dt_raw"):
        alone[k] = np.ascontiguousarray(inp[k][:, lo:hi])
    alone["seq_idx"] = None
    ga = oracle.backward(dict(dims, seqlen=hi - lo), alone, np.ascontiguousarray(g_only[:, lo:hi]))
    for name in ("x", "z", "B", "C", "dt_raw"):
        assert np.array_equal(g[name][0, lo:hi], ga[name][0]), name
    for name in ("dt_bias", "A", "D", "conv_w", "conv_b"):
        assert np.array_equal(g[name], ga[name]), name


def test_ragged_rows_equal_rows_run_alone(oracle_mod):
    dims, inp, gout = case(True, seed=35, batch=3)
    inp["seq_idx"] = None
    lens = np.array([70, 23, 0], np.int32)
    g = oracle.backward(dims, dict(inp, lengths=lens), gout)
    for name in ("x", "z", "B", "C", "dt_raw"):
        for b in range(3):
            assert np.all(g[name][b, lens[b]:] == 0.0), (name, b)
    # weight gradients of the ragged batch = the sum over rows run alone
    wsum = {k: 0.0 for k in ("dt_bias", "A", "D", "conv_w", "conv_b")}
    for b in range(3):
        L = int(lens[b])
        if L == 0:
            continue
        row = dict(inp)
        for k in ("x", "z", "B", "C", "dt_raw"):
            row[k] = np.ascontiguousarray(inp[k][b:b + 1, :L])
        gb = oracle.backward(dict(dims, batch=1, seqlen=L), row,
                             np.ascontiguousarray(gout[b:b + 1, :L]))
        for name in ("x", "z", "B", "C", "dt_raw"):
            assert np.array_equal(g[name][b, :L], gb[name][0]), (name, b)
        for k in wsum:
            wsum[k] = wsum[k] + gb[k]
    for k, v in wsum.items():
        np.testing.assert_allclose(g[k], v, rtol=1e-13, atol=1e-13 * np.max(np.abs(v)), err_msg=k)


def test_backward_refuses_a_carried_state(oracle_mod):
    dims, inp, gout = case(True, seed=36, batch=1, L=8)
    with pytest.raises(ValueError):
        oracle.backward(dims, dict(inp, init_ssm=np.zeros((1, 4, 3, 5), np.float32)), gout)
    with pytest.raises(ValueError):
        oracle.backward(dims, dict(inp, init_conv=np.zeros((1, 3, 22), np.float32)), gout)


def _torch_matrix_form(dims, inp):
    """The whole forward in the SSD matrix form, in float64 torch ops on the CPU:
    conv (document-masked taps) + SiLU, the B/C norm, softplus dt, the floored
    per-token A, y = (L o C B^T o dt) x + D x, out = y SiLU(z).  It shares no
    loop with the oracle's token-by-token recurrence; autograd gives its
    gradients.  Returns (out, leaves) with leaves the inputs requiring grad."""
    import torch
    Bb, L, H, P, N, G, K = (dims["batch"], dims["seqlen"], dims["nheads"], dims["headdim"],
                            dims["dstate"], dims["ngroups"], dims["dconv"])
    leaves = {k: torch.tensor(np.asarray(v, np.float64), requires_grad=True)
              for k, v in inp.items() if isinstance(v, np.ndarray) and v.dtype == np.float32}
    seq = np.zeros((Bb, L), np.int64) if inp.get("seq_idx") is None else np.asarray(inp["seq_idx"])
    # doc[b, t]: the document ordinal (boundaries where neighbours differ)
    doc = np.concatenate([np.zeros((Bb, 1), np.int64),
                          np.cumsum(seq[:, 1:] != seq[:, :-1], axis=1)], axis=1)
    raw = torch.cat([leaves["x"], leaves["B"], leaves["C"]], dim=-1)
    if K == 4:
        pre = leaves["conv_b"].expand_as(raw)
        for k in range(4):
            sh = 3 - k
            shifted = torch.zeros_like(raw)
            shifted[:, sh:] = raw[:, :L - sh]
            ok = np.zeros((Bb, L), bool)
            ok[:, sh:] = doc[:, sh:] == doc[:, :L - sh]
            pre = pre + leaves["conv_w"][:, k] * shifted * torch.tensor(ok, dtype=torch.float64)[..., None]
        u = pre * torch.sigmoid(pre)
    else:
        u = raw
    HP, GN = H * P, G * N
    ux = u[..., :HP].reshape(Bb, L, H, P)
    gmap = torch.tensor([h // (H // G) for h in range(H)])
    ub = u[..., HP:HP + GN].reshape(Bb, L, G, N)[:, :, gmap]
    uc = u[..., HP + GN:].reshape(Bb, L, G, N)[:, :, gmap]
    if dims.get("bc_norm"):
        ub = ub * torch.rsqrt((ub ** 2).mean(-1, keepdim=True) + 1e-5) * leaves["B_norm_w"] + leaves["B_bias"]
        uc = uc * torch.rsqrt((uc ** 2).mean(-1, keepdim=True) + 1e-5) * leaves["C_norm_w"] + leaves["C_bias"]
    dt = torch.nn.functional.softplus(leaves["dt_raw"] + leaves["dt_bias"])          # (Bb, L, H)
    a = torch.clamp(leaves["A"], max=-1e-4) if dims.get("a_per_token") else leaves["A"].expand(Bb, L, H)
    cs = torch.cumsum(dt * a, dim=1)
    t = np.arange(L)
    keep = torch.tensor((t[:, None] >= t[None, :])[None] & (doc[:, :, None] == doc[:, None, :]))
    diff = cs[:, :, None, :] - cs[:, None, :, :]                                   # (Bb, t, s, H)
    decay = torch.exp(torch.where(keep[..., None], diff, torch.full_like(diff, -torch.inf)))
    cb = torch.einsum("btgn,bsgn->btsg", uc, ub)                                   # per head
    M = cb * decay * dt[:, None, :, :]
    y = torch.einsum("btsh,bshp->bthp", M, ux) + leaves["D"][:, None] * ux
    z = leaves["z"].reshape(Bb, L, H, P)
    out = (y * z * torch.sigmoid(z)).reshape(Bb, L, HP)
    return out, leaves


@pytest.mark.parametrize("conv", [True, False], ids=["conv_docs_groups", "bcnorm_per_token_A"])
def test_gradients_equal_autograd_of_the_matrix_form(oracle_mod, conv):
    import torch
    dims, inp, gout = case(conv, seed=51 if conv else 52)
    out, leaves = _torch_matrix_form(dims, inp)
    ref = oracle.forward(dims, inp, final=False)["out"]
    assert np.max(np.abs(out.detach().numpy() - ref)) <= 1e-11 * np.max(np.abs(ref))
    names = sorted(k for k, v in oracle.backward(dims, inp, gout).items() if v is not None)
    want = torch.autograd.grad((out * torch.tensor(gout, dtype=torch.float64)).sum(),
                               [leaves[k] for k in names])
    got = oracle.backward(dims, inp, gout)
    for k, wv in zip(names, want):
        wv = wv.numpy()
        assert np.max(np.abs(got[k] - wv)) <= 1e-10 * max(np.max(np.abs(wv)), 1e-300), k
