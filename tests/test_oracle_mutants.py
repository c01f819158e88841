"""The oracle's pins catch plausible mistakes (no GPU needed).

Each case plants one mistake in a temporary copy of oracle/ssd_oracle.c (a
dropped term, a wrong sign, a wrong index, a missing reset ...), builds it,
and checks that the pin battery below -- the same independent forms the
oracle pin tests use -- rejects it, while the unmodified oracle passes.
"""
import os
import shutil

import numpy as np
import pytest

from brute_force import head_inputs, quadratic_form, silu
from test_oracle_backward import case as _bwd_case, check_directional as _bwd_directional
from test_oracle_gated_norm import check_gated_norm as _gated_norm_checks
from test_oracle_s6 import _inputs as _s6_inputs, _matrix_form as _s6_matrix_form
from selective_state_space_forward_b200.synthetic import Workload, make_inputs

import oracle

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "ssd_oracle.c")

MUTANTS = {
    "drop_D_skip": ("y += in->D[h] * ux[p];", "y += 0.0 * ux[p];"),
    "decay_sign": ("const double decay = exp(dt * a);", "const double decay = exp(-dt * a);"),
    "no_document_reset": ("memset(hs, 0, sizeof(double) * P * N);", "(void)0;"),
    "conv_taps_reversed": ("in->conv_w[(size_t)ch * K + k] * v;", "in->conv_w[(size_t)ch * K + (K - 1 - k)] * v;"),
    "update_with_C": ("hp[n] = decay * hp[n] + dxp * ub[n];", "hp[n] = decay * hp[n] + dxp * uc[n];"),
    "no_gate_silu": ("out[tok * dx + h * P + p] = y * silu(zv);", "out[tok * dx + h * P + p] = y * zv;"),
    "groups_interleaved": ("const int g = h / (H / d->ngroups);\n    const int dx = H * P, gn = d->ngroups * N;\n    double *hs",
                           "const int g = h % d->ngroups;\n    const int dx = H * P, gn = d->ngroups * N;\n    double *hs"),
    "dt_bias_dropped": ("softplus_exact((double)in->dt_raw[tok * H + h] + in->dt_bias[h])",
                        "softplus_exact((double)in->dt_raw[tok * H + h])"),
    "a_floor_inverted": ("if (a > -1e-4) a = -1e-4;", "if (a < -1e-4) a = -1e-4;"),
    "init_history_crosses_documents": ("} else if (in->init_conv && same_doc(in, d, b, 0, t)) {",
                                       "} else if (in->init_conv) {"),
    "norm_uses_C_bias_for_B": ("ub[n] = ub[n] * rb * wb + bb;", "ub[n] = ub[n] * rb * wb + bc;"),
    "output_before_update": ("hp[n] = decay * hp[n] + dxp * ub[n];\n                y += uc[n] * hp[n];",
                             "y += uc[n] * hp[n];\n                hp[n] = decay * hp[n] + dxp * ub[n];"),
    "padding_runs_the_recurrence": ("= 0.0;\n    for (int t = 0; t < Lb; t++) {", "= 0.0;\n    for (int t = 0; t < L; t++) {"),
    "final_history_ignores_length": ("const int L = row_len(d, in, b);   /* the row's last real token is L - 1 */",
                                     "const int L = d->seqlen;"),
    "s6_no_clamp": ("            if (al < -10.0) al = -10.0;\n            if (al > 5.0) al = 5.0;\n", ""),
    "s6_decay_sign": ("hc[n] = exp(dt * a[(size_t)c * N + n]) * hc[n] + dt * uv * Bt[n];",
                      "hc[n] = exp(-dt * a[(size_t)c * N + n]) * hc[n] + dt * uv * Bt[n];"),
    "s6_output_with_B": ("                y += Ct[n] * hc[n];", "                y += Bt[n] * hc[n];"),
    "s6_drop_D": ("            y += in->D[c] * uv;", "            y += 0.0 * uv;"),
    "s6_no_gate": ("out[tok * DI + c] = in->z ? y * silu(in->z[tok * DI + c]) : y;",
                   "out[tok * DI + c] = y;"),
    "bwd_drop_decay_term_of_dt": ("gdt += gdecay * k.decay * k.a;", "(void)gdecay;"),
    "bwd_no_adjoint_reset": ("            else\n                memset(gh, 0, sizeof(double) * (size_t)P * N);",
                             "            else\n                (void)0;"),
    "bwd_norm_cross_term_sign": ("gub[n] += k.rb * wb * gbh[n] - k.rb * k.rb * k.rb / N * k.ub[n] * sb;",
                                 "gub[n] += k.rb * wb * gbh[n] + k.rb * k.rb * k.rb / N * k.ub[n] * sb;"),
    "bwd_conv_taps_reversed": ("graw[(size_t)tau * cd + ch] += gpre * in->conv_w[(size_t)ch * K + kk];",
                               "graw[(size_t)tau * cd + ch] += gpre * in->conv_w[(size_t)ch * K + (K - 1 - kk)];"),
    "bwd_conv_without_silu_grad": ("const double gpre = gv * silu_grad(conv_pre(d, in, b, t, ch));",
                                   "const double gpre = gv;"),
    "bwd_floored_A_passes": ("gr->A[tok * H + h] = k.floored ? 0.0 : ga;", "gr->A[tok * H + h] = ga;"),
    "bwd_gate_uses_silu": ("go * y * silu_grad(zv);", "go * y * silu(zv);"),
    "bwd_softplus_grad_at_dt": ("const double gv = gdt * sigmoid(k.v);", "const double gv = gdt * sigmoid(k.dt);"),
    "bwd_group_gradient_overwritten": ("for (int n = 0; n < N; n++) { gub[n] += gbh[n]; guc[n] += gch[n]; }",
                                       "for (int n = 0; n < N; n++) { gub[n] = gbh[n]; guc[n] = gch[n]; }"),
    "norm_mean_over_the_row": ("const double rs = 1.0 / sqrt(ss / group + eps);",
                               "const double rs = 1.0 / sqrt(ss / d_inner + eps);"),
    "norm_eps_outside_the_root": ("const double rs = 1.0 / sqrt(ss / group + eps);",
                                  "const double rs = 1.0 / (sqrt(ss / group) + eps);"),
    "norm_weight_by_group_position": ("gv[c] * rs * (w ? w[c0 + c] : 1.0);", "gv[c] * rs * (w ? w[c] : 1.0);"),
    "bwd_decay_grad_with_new_state": ("if (hprev) gdecay += ghv * hprev[p * N + n];",
                                      "if (hprev) gdecay += ghv * ht[p * N + n];"),
}


def _docs(L, cuts):
    seq = np.zeros(L, dtype=np.int32)
    for c in cuts:
        seq[c:] += 1
    return seq


def _battery(lib) -> list:
    """Run the independent checks; return the names of those that fail."""
    failed = []
    # 1. matrix form, with documents, initial state and per-token A
    w = Workload("m", 2, 90, 4, 4, 5, 2, 1, "f32", a_per_token=True, init_state=True, seed=21)
    inp = make_inputs(w)
    inp["seq_idx"] = np.stack([_docs(90, [1, 64, 65]), _docs(90, [])])
    inp["A"][0, 3:6, 0] = np.array([0.0, -1e-6, -0.3], dtype=np.float32)
    dims = w.dims()
    res = oracle.forward(dims, inp, lib=lib)
    ok = True
    for b in range(2):
        for h in range(4):
            x, z, Bm, Cm, dt, a, D, seq, h0 = head_inputs(inp, dims, b, h)
            y, hf = quadratic_form(x, z, Bm, Cm, dt, a, D, seq, h0)
            got = res["out"][b, :, h * 4:(h + 1) * 4]
            ok &= bool(np.max(np.abs(got - y)) <= 1e-10 * np.max(np.abs(y)))
            ok &= bool(np.max(np.abs(res["final_ssm"][b, h] - hf)) <= 1e-10 * np.max(np.abs(hf)))
    if not ok:
        failed.append("quadratic_form")
    # 2. conv against a padded correlation, with documents and an initial history
    w = Workload("c", 1, 30, 2, 4, 3, 1, 4, "f32", seed=22)
    inp = make_inputs(w)
    rng = np.random.default_rng(1)
    inp["init_conv"] = rng.standard_normal((1, 3, w.conv_dim)).astype(np.float32)
    inp["seq_idx"] = _docs(30, [2, 17])[None]
    u = oracle.conv_stage(w.dims(), inp, lib=lib)[0]
    raw = np.concatenate([inp["x"][0], inp["B"][0], inp["C"][0]], axis=1).astype(np.float64)
    seq = inp["seq_idx"][0]
    want = np.empty_like(u)
    for t in range(30):
        acc = inp["conv_b"].astype(np.float64).copy()
        for k in range(4):
            tau = t - 3 + k
            if tau >= 0:
                v = raw[tau] if seq[tau] == seq[t] else 0.0
            else:
                v = inp["init_conv"][0, tau + 3].astype(np.float64) if seq[t] == seq[0] else 0.0
            acc = acc + inp["conv_w"][:, k].astype(np.float64) * v
        want[t] = silu(acc)
    if not np.allclose(u, want, rtol=1e-13, atol=1e-300):
        failed.append("conv")
    # 3. B/C norm closed form: zero bias, unit weight
    w = Workload("n", 1, 8, 2, 4, 8, 1, 1, "f32", bc_norm=True, seed=23)
    inp = make_inputs(w)
    inp["B_bias"] = np.zeros_like(inp["B_bias"])
    bh, ch = oracle.bcnorm_stage(w.dims(), inp, lib=lib)
    m = np.mean(inp["B"][0].astype(np.float64) ** 2, axis=1)
    if not np.allclose(np.sum(bh[0] ** 2, axis=2), (8 * m / (m + 1e-5))[:, None], rtol=1e-12):
        failed.append("bcnorm_closed_form")
    # 4. normed scan == un-normed scan fed per-head B_hat / C_hat (G = H)
    w = Workload("nw", 1, 40, 2, 4, 8, 1, 1, "f32", bc_norm=True, seed=24)
    inp = make_inputs(w)
    r = oracle.forward(w.dims(), inp, lib=lib)
    bh, ch = oracle.bcnorm_stage(w.dims(), inp)   # the unmodified oracle's norm stage
    flat = dict(inp, B=bh.reshape(1, 40, 16).astype(np.float32),
                C=ch.reshape(1, 40, 16).astype(np.float32))
    r2 = oracle.forward(dict(w.dims(), ngroups=2, bc_norm=0), flat)
    if not np.max(np.abs(r["out"] - r2["out"])) <= 1e-5 * np.max(np.abs(r2["out"])):
        failed.append("bcnorm_wiring")
    # 5. ragged lengths: a row equals the matrix form over its real tokens, padding is +0.0,
    #    and the final conv history holds the last real raw inputs
    w = Workload("r", 3, 70, 2, 4, 5, 1, 4, "f32", init_state=True, seed=25)
    inp = make_inputs(w)
    rng = np.random.default_rng(2)
    inp["init_conv"] = rng.standard_normal((3, 3, w.conv_dim)).astype(np.float32)
    lens = np.array([70, 33, 2], np.int32)
    res = oracle.forward(w.dims(), dict(inp, lengths=lens), lib=lib)
    ok = True
    for b in range(3):
        L = int(lens[b])
        pad = res["out"][b, L:]
        ok &= bool(np.all(pad == 0.0) and not np.any(np.signbit(pad)))
        # the conv'd x|B|C of the row's real tokens, then the matrix form on them
        row = {k: (None if v is None else (v[b:b + 1, :L] if k in ("x", "z", "B", "C", "dt_raw")
                                           else (v[b:b + 1] if k in ("init_ssm", "init_conv") else v)))
               for k, v in inp.items()}
        wr = w.with_(batch=1, seqlen=L)
        u = oracle.conv_stage(wr.dims(), row)[0]   # the unmodified oracle's conv stage
        HP, GN = 8, 5
        flat = dict(row, x=u[None, :, :HP].astype(np.float32), B=u[None, :, HP:HP + GN].astype(np.float32),
                    C=u[None, :, HP + GN:].astype(np.float32), conv_w=None, conv_b=None)
        dims1 = dict(wr.dims(), dconv=1)
        for h in range(2):
            x, z, Bm, Cm, dt, a, D, seq, h0 = head_inputs(flat, dims1, 0, h)
            y, hf = quadratic_form(x, z, Bm, Cm, dt, a, D, seq, h0)
            got = res["out"][b, :L, h * 4:(h + 1) * 4]
            ok &= bool(np.max(np.abs(got - y)) <= 1e-6 * np.max(np.abs(y)))
            ok &= bool(np.max(np.abs(res["final_ssm"][b, h] - hf)) <= 1e-6 * np.max(np.abs(hf)))
        raw = np.concatenate([inp["init_conv"][b].astype(np.float64),
                              np.concatenate([inp["x"][b, :L], inp["B"][b, :L], inp["C"][b, :L]], axis=1)])
        ok &= bool(np.array_equal(res["final_conv"][b], raw[-3:]))
    if not ok:
        failed.append("ragged")
    # 6. S6: the matrix form, with A_log values beyond both clamp bounds
    inp = _s6_inputs(B=1, L=30, DI=3, N=4, seed=26)
    inp["A_log"][0, 0] = 7.0
    inp["A_log"][1, 2] = -12.0
    r = oracle.s6_forward(inp, lib=lib)
    y, hf = _s6_matrix_form(inp)
    if not (np.max(np.abs(r["out"] - y)) <= 1e-10 * np.max(np.abs(y)) and
            np.max(np.abs(r["final"] - hf)) <= 1e-10 * np.max(np.abs(hf))):
        failed.append("s6_matrix_form")
    # 7. backward: directional derivatives of the unmodified forward, with and without
    #    conv / documents / the B/C norm / per-token A
    for conv, seed in ((True, 27), (False, 28)):
        dims, inp, gout = _bwd_case(conv, seed=seed)
        if _bwd_directional(dims, inp, gout, seed=seed, lib=lib):
            failed.append("backward_%s" % ("conv" if conv else "norm"))
    # 8. the gated RMSNorm after the scan
    failed += ["gated_norm_" + n for n in _gated_norm_checks(lib)]
    return failed


def _build_variant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path = tmp_path / (name + ".c")
    path.write_text(src.replace(old, new))
    so = str(tmp_path / (name + ".so"))
    oracle.build(force=True, src=str(path), out=so)
    return oracle.load_variant(so)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_unmodified_oracle_passes_the_battery(oracle_mod):
    assert _battery(None) == []


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(oracle_mod, tmp_path, name):
    old, new = MUTANTS[name]
    lib = _build_variant(tmp_path, name, old, new)
    assert _battery(lib), f"mutant {name} passed every pin"
