"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small cases compare every output element and the final state; the full-size
workloads (the launch configuration the bench times) compare sampled
(row, head) pairs that the oracle computes one by one.  Tolerances: bf16
activations rel-L2 <= 5e-3 and max-abs <= 2e-2 * max|ref|; fp32 rel-L2 <= 1e-5.
Document and chunk-boundary indexing is checked bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_close, init_state_of, make_handle, run_forward, state_from_numpy,
                      state_to_numpy, to_device)
from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs, make_step_inputs

pytestmark = pytest.mark.gpu

PATHS = ["staged", "auto"]


def _docs_row(L, cuts):
    s = np.zeros(L, dtype=np.int32)
    for c in cuts:
        if 0 < c < L:
            s[c:] += 1
    return s


def _small(name, **kw):
    return WORKLOADS[name].with_(**kw)


SMALL = {
    "tiny_fp32": _small("tiny_fp32"),
    "mini_k3_mixer": _small("mini_k3_mixer", batch=2, seqlen=300, mean_doc_len=90),
    "mamba3_siso": _small("mamba3_siso", batch=2, seqlen=200),
    "long_7b": _small("long_7b", batch=1, seqlen=330),
}


def _compare_all(w, inp, res, out, fs, fc, what):
    assert_close(out, res["out"], w.act_dtype, what + " out")
    assert_close(fs, res["final_ssm"], w.act_dtype, what + " final ssm")
    if fc is not None:
        # the conv history is copied raw inputs: exact
        assert np.array_equal(fc, res["final_conv"]), what + " final conv history"


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_full_parity(name, path):
    w = SMALL[name]
    inp = make_inputs(w)
    if w.documents == "geometric":
        inp["seq_idx"][0] = _docs_row(w.seqlen, [1, 63, 64, 65, 150, w.seqlen - 1])
    res = oracle.forward(w.dims(), inp)
    h = make_handle(w, path)
    dev = to_device(inp, w)
    out, fs, fc, _ = run_forward(h, w, dev, init_state_of(h, w, inp))
    _compare_all(w, inp, res, out, fs, fc, f"{name}/{h.path}")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("L", [1, 2, 3, 63, 64, 65, 127, 129])
def test_ragged_lengths(L, path):
    w = _small("mini_k3_mixer", batch=2, seqlen=L, nheads=8, ngroups=2, documents="none",
               init_state=True)
    inp = make_inputs(w)
    rng = np.random.default_rng(L)
    inp["init_conv"] = np.asarray(
        np.round(rng.standard_normal((2, 3, w.conv_dim)) * 64) / 64, dtype=np.float32)
    res = oracle.forward(w.dims(), inp)
    h = make_handle(w, path)
    out, fs, fc, _ = run_forward(h, w, to_device(inp, w), init_state_of(h, w, inp))
    _compare_all(w, inp, res, out, fs, fc, f"L={L}/{h.path}")


@pytest.mark.parametrize("path", PATHS)
def test_one_head_one_group(path):
    w = _small("long_7b", batch=1, seqlen=100, nheads=1, ngroups=1)
    inp = make_inputs(w)
    res = oracle.forward(w.dims(), inp)
    h = make_handle(w, path)
    out, fs, fc, _ = run_forward(h, w, to_device(inp, w), init_state_of(h, w, inp))
    _compare_all(w, inp, res, out, fs, fc, f"H=1/{h.path}")


@pytest.mark.parametrize("path", PATHS)
def test_one_token_documents(path):
    w = _small("mini_k3_mixer", batch=1, seqlen=80, documents="none", init_state=True)
    inp = make_inputs(w)
    inp["seq_idx"] = np.arange(80, dtype=np.int32)[None]
    res = oracle.forward(w.dims(), inp)
    h = make_handle(w, path)
    out, fs, fc, _ = run_forward(h, w, to_device(inp, w), init_state_of(h, w, inp))
    _compare_all(w, inp, res, out, fs, fc, f"1-token docs/{h.path}")


def _sampled_pairs(w, k=4):
    hs = sorted({0, w.nheads - 1, w.nheads // 2 + 1, (w.nheads * 3) // 4})[:k]
    bs = [0, w.batch - 1]
    return [(b, h) for b in bs for h in hs[: max(1, k // 2)]] + [(w.batch // 2, hs[-1])]


@pytest.mark.parametrize("name", ["mini_k3_mixer", "mamba3_siso", "long_7b"])
def test_full_size_sampled_pairs(name):
    """The bench's workloads at full size, default path; the oracle recomputes
    a few (row, head) pairs one by one."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    h = make_handle(w, "auto")
    dev = to_device(inp, w)
    out, fs, fc, _ = run_forward(h, w, dev, init_state_of(h, w, inp))
    pairs = _sampled_pairs(w)
    res = oracle.forward(w.dims(), inp, pairs=pairs)
    P = w.headdim
    for b, hh in pairs:
        sl = np.s_[b, :, hh * P:(hh + 1) * P]
        assert_close(out[sl], res["out"][sl], w.act_dtype, f"{name} ({b},{hh}) out")
        assert_close(fs[b, hh], res["final_ssm"][b, hh], w.act_dtype, f"{name} ({b},{hh}) state")
    if fc is not None:
        assert np.array_equal(fc, res["final_conv"])


def test_stage_conv_matches_oracle():
    w = _small("mini_k3_mixer", batch=2, seqlen=150, mean_doc_len=40)
    inp = make_inputs(w)
    rng = np.random.default_rng(2)
    inp["init_conv"] = np.asarray(np.round(rng.standard_normal((2, 3, w.conv_dim)) * 32) / 32,
                                  dtype=np.float32)
    want = oracle.conv_stage(w.dims(), inp)
    h = make_handle(w, "staged")
    dev = to_device(inp, w)
    init = state_from_numpy(h, w.batch, None, inp["init_conv"])
    u = h.stage_conv(dev["x"], dev["B"], dev["C"], dev["conv_w"], dev["conv_b"],
                     seq_idx=dev["seq_idx"], init_state=init)
    got = u.double().cpu().numpy()
    assert np.max(np.abs(got - want)) <= 2e-6 * max(1.0, np.max(np.abs(want)))


def test_stage_dt_matches_oracle():
    """dt and the segmented per-chunk cumsum: the sum of dt*a restarts at each
    chunk start and each document boundary (from the oracle's dt and a)."""
    w = _small("mamba3_siso", batch=2, seqlen=200)
    inp = make_inputs(w)
    inp["A"][0, 3:7, 5] = np.array([0.0, -1e-6, -1e-4, -2.0], dtype=np.float32)
    seq = np.stack([_docs_row(200, [1, 30, 64, 65, 100, 199]), _docs_row(200, [])])
    dt_ref, a_ref = oracle.dt_stage(w.dims(), inp)
    h = make_handle(w, "staged")
    dev = to_device(inp, w)
    dt, acs = h.stage_dt(dev["dt_raw"], dev["dt_bias"], dev["A"],
                         seq_idx=torch.from_numpy(seq).cuda())
    dt = dt.double().cpu().numpy()
    acs = acs.double().cpu().numpy()
    assert np.allclose(dt, dt_ref.transpose(0, 2, 1), rtol=2e-6, atol=1e-30)
    da = (dt_ref * a_ref).transpose(0, 2, 1)
    ref = np.empty_like(da)
    for b in range(2):
        for t in range(w.seqlen):
            start = t % 64 == 0 or seq[b, t] != seq[b, t - 1]
            ref[b, :, t] = da[b, :, t] if start else ref[b, :, t - 1] + da[b, :, t]
    scale = np.max(np.abs(ref))
    assert np.allclose(acs, ref, rtol=1e-5, atol=1e-6 * scale)


@pytest.mark.parametrize("path", PATHS)
def test_seq_idx_null_equals_all_zero_bitwise(path):
    w = _small("mini_k3_mixer", batch=2, seqlen=200, documents="none", init_state=True)
    inp = make_inputs(w)
    h = make_handle(w, path)
    dev = to_device(inp, w)
    a, sa, _, _ = run_forward(h, w, dev, init_state_of(h, w, inp))
    dev["seq_idx"] = torch.zeros(w.batch, w.seqlen, dtype=torch.int32, device="cuda")
    b, sb, _, _ = run_forward(h, w, dev, init_state_of(h, w, inp))
    assert np.array_equal(a, b) and np.array_equal(sa, sb)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("seed", [0, 1])
def test_documents_isolated_bitwise(path, seed):
    """Perturbing one packed document leaves every other document's outputs
    bit-identical (model card: exactly zero influence across documents)."""
    w = _small("mini_k3_mixer", batch=1, seqlen=260, documents="none", init_state=True,
               seed=30 + seed)
    inp = make_inputs(w)
    seq = _docs_row(w.seqlen, [1, 63, 64, 65, 128, 200, 259])[None]
    inp["seq_idx"] = seq
    h = make_handle(w, path)
    base, bs, bc, _ = run_forward(h, w, to_device(inp, w), init_state_of(h, w, inp))
    rng = np.random.default_rng(seed)
    ndoc = int(seq.max()) + 1
    for k in range(ndoc):
        sel = seq[0] == k
        pert = {kk: (None if v is None else np.array(v)) for kk, v in inp.items()}
        for key in ("x", "z", "B", "C"):
            pert[key][0, sel] = np.round(pert[key][0, sel] + rng.standard_normal(
                pert[key][0, sel].shape), 2).astype(np.float32)
        pert["dt_raw"][0, sel] += rng.standard_normal(pert["dt_raw"][0, sel].shape).astype(
            np.float32)
        out, s2, c2, _ = run_forward(h, w, to_device(pert, w), init_state_of(h, w, inp))
        assert np.array_equal(out[0, ~sel], base[0, ~sel]), k
        if k != ndoc - 1:
            assert np.array_equal(s2, bs) and np.array_equal(c2, bc), k


@pytest.mark.parametrize("path", PATHS)
def test_split_prefill_continues(path):
    w = _small("mini_k3_mixer", batch=2, seqlen=190, documents="none", init_state=True)
    inp = make_inputs(w)
    inp["seq_idx"] = np.stack([_docs_row(190, [100]), _docs_row(190, [])])
    res = oracle.forward(w.dims(), inp)
    h = make_handle(w, path)
    L1 = 70
    keys = ("x", "z", "B", "C", "dt_raw", "seq_idx")
    a = {k: (v[:, :L1] if k in keys and v is not None else v) for k, v in inp.items()}
    b = {k: (v[:, L1:] if k in keys and v is not None else v) for k, v in inp.items()}
    wa, wb = w.with_(seqlen=L1), w.with_(seqlen=190 - L1)
    o1, _, _, buf = run_forward(h, wa, to_device(a, wa), init_state_of(h, w, inp))
    o2, fs, fc, _ = run_forward(h, wb, to_device(b, wb), buf)
    out = np.concatenate([o1, o2], axis=1)
    assert_close(out, res["out"], w.act_dtype, "split prefill out")
    assert_close(fs, res["final_ssm"], w.act_dtype, "split prefill state")
    assert np.array_equal(fc, res["final_conv"])


@pytest.mark.parametrize("path", PATHS)
def test_in_place_state_carry(path):
    """init_state and final_state may be the same buffer."""
    w = _small("long_7b", batch=1, seqlen=150)
    inp = make_inputs(w)
    res = oracle.forward(w.dims(), inp)
    h = make_handle(w, path)
    buf = init_state_of(h, w, inp)
    dev = to_device(inp, w)
    out = h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"],
                    dev["C"], dev["D"], dev["conv_w"], dev["conv_b"], init_state=buf,
                    final_state=buf)
    torch.cuda.synchronize()
    fs, fc = state_to_numpy(h, buf, 1)
    assert_close(out.double().cpu().numpy(), res["out"], "bf16", "in-place out")
    assert_close(fs, res["final_ssm"], "bf16", "in-place state")
    assert np.array_equal(fc, res["final_conv"])


def _step_run(h, w, dev_params, step_inp, state):
    at = h.torch_dtype
    x = torch.from_numpy(step_inp["x"]).to(at).cuda()
    z = torch.from_numpy(step_inp["z"]).to(at).cuda()
    B = torch.from_numpy(step_inp["B"]).to(at).cuda()
    C = torch.from_numpy(step_inp["C"]).to(at).cuda()
    dtr = torch.from_numpy(step_inp["dt_raw"]).cuda()
    A = torch.from_numpy(step_inp["A"]).cuda() if "A" in step_inp else dev_params["A"]
    return h.step(x, z, dtr, dev_params["dt_bias"], A, B, C, dev_params["D"],
                  dev_params["conv_w"], dev_params["conv_b"], state=state)


@pytest.mark.parametrize("name", ["mini_k3_mixer", "mamba3_siso"])
def test_prefill_then_steps_small(name):
    w = _small(name, batch=3, seqlen=70, documents="none")
    inp = make_inputs(w)
    h = make_handle(w, "staged")
    dev = to_device(inp, w)
    _, _, _, state = run_forward(h, w, dev, None)
    r = oracle.forward(w.dims(), inp)
    ssm, conv = r["final_ssm"].astype(np.float32), (
        None if r["final_conv"] is None else r["final_conv"].astype(np.float32))
    for step in range(20):
        si = make_step_inputs(w, step)
        out = _step_run(h, w, dev, si, state)
        torch.cuda.synchronize()
        tok = {k: (v[:, None] if k in ("x", "z", "B", "C", "dt_raw", "A") else v)
               for k, v in si.items()}
        o_inp = dict(inp)
        o_inp.update(tok)
        if "A" not in si:
            o_inp["A"] = inp["A"]
        ro = oracle.step(w.dims(), o_inp, ssm, conv)
        assert_close(out.double().cpu().numpy(), ro["out"][:, 0], w.act_dtype, f"step {step}")
        ssm = ro["final_ssm"].astype(np.float32)
        conv = None if ro["final_conv"] is None else ro["final_conv"].astype(np.float32)
    fs, fc = state_to_numpy(h, state, w.batch)
    assert_close(fs, ssm, w.act_dtype, "state after steps")
    if fc is not None:
        assert np.array_equal(fc, conv)


def test_decode_full_size_sampled_rows():
    """batch 256 on the mini_k3 mixer shapes: a 2048-token prefill, then 512
    decode steps; the oracle follows 3 sampled rows through the same steps."""
    w = WORKLOADS["decode_b256"]
    inp = make_inputs(w)
    h = make_handle(w, "auto")
    dev = to_device(inp, w)
    _, _, _, state = run_forward(h, w, dev, None)
    rows = [0, 97, 255]
    sub = {k: (v[rows] if (v is not None and k in ("x", "z", "B", "C", "dt_raw", "seq_idx"))
               else v) for k, v in inp.items()}
    ws = w.with_(batch=len(rows))
    r = oracle.forward(ws.dims(), sub)
    ssm, conv = r["final_ssm"].astype(np.float32), r["final_conv"].astype(np.float32)
    fs, fc = state_to_numpy(h, state, w.batch)
    assert_close(fs[rows], r["final_ssm"], "bf16", "prefill state")
    assert np.array_equal(fc[rows], r["final_conv"])
    for step in range(w.decode_steps):
        si = make_step_inputs(w, step)
        out = _step_run(h, w, dev, si, state)
        if step % 64 == 0 or step == w.decode_steps - 1:
            torch.cuda.synchronize()
        tok = {k: v[rows][:, None] for k, v in si.items()}
        o_inp = dict(sub)
        o_inp.update(tok)
        ro = oracle.step(ws.dims(), o_inp, ssm, conv)
        if step % 64 == 0 or step == w.decode_steps - 1:
            got = out.double().cpu().numpy()[rows]
            assert_close(got, ro["out"][:, 0], "bf16", f"decode step {step}")
        ssm, conv = ro["final_ssm"].astype(np.float32), ro["final_conv"].astype(np.float32)
    fs, fc = state_to_numpy(h, state, w.batch)
    assert_close(fs[rows], ssm, "bf16", "state after 512 steps")
    assert np.array_equal(fc[rows].astype(np.float32), conv)


def test_empty_inputs():
    w = _small("mini_k3_mixer", batch=2, seqlen=64, documents="none", init_state=True)
    inp = make_inputs(w)
    h = make_handle(w, "staged")
    init = init_state_of(h, w, inp)
    fin = h.new_state(2)
    e = torch.empty(2, 0, w.nheads * w.headdim, dtype=torch.bfloat16, device="cuda")
    eb = torch.empty(2, 0, w.ngroups * w.dstate, dtype=torch.bfloat16, device="cuda")
    ef = torch.empty(2, 0, w.nheads, dtype=torch.float32, device="cuda")
    dev = to_device(inp, w)
    h.forward(e, e, ef, dev["dt_bias"], dev["A"], eb, eb, dev["D"], dev["conv_w"],
              dev["conv_b"], init_state=init, final_state=fin)
    torch.cuda.synchronize()
    assert torch.equal(fin, init)          # no token: the state passes through
    e0 = torch.empty(0, 5, w.nheads * w.headdim, dtype=torch.bfloat16, device="cuda")
    h.forward(e0, e0, ef[:0], dev["dt_bias"], dev["A"], eb[:0], eb[:0], dev["D"],
              dev["conv_w"], dev["conv_b"])
    torch.cuda.synchronize()


@pytest.mark.parametrize("dstate,dconv,a_per_token", [(128, 1, True), (64, 4, False), (128, 4, True)])
def test_bc_norm_on_the_fused_path(dstate, dconv, a_per_token):
    """B/C RMSNorm + per-head bias on the fused kernel: groups shared by several
    heads (so each head's bias must stay its own), norm weights other than one,
    packed documents, with and without the conv."""
    w = WORKLOADS["mamba3_siso"].with_(batch=2, seqlen=200, nheads=8, ngroups=2, dstate=dstate,
                                       dconv=dconv, a_per_token=a_per_token,
                                       documents="geometric", mean_doc_len=70, seed=21)
    inp = make_inputs(w)
    rng = np.random.Generator(np.random.PCG64(22))
    inp["B_norm_w"] = (1.0 + 0.3 * rng.standard_normal(dstate)).astype(np.float32)
    inp["C_norm_w"] = (1.0 + 0.3 * rng.standard_normal(dstate)).astype(np.float32)
    inp["B_bias"] = (0.1 * rng.standard_normal((w.nheads, dstate))).astype(np.float32)
    inp["C_bias"] = (0.1 * rng.standard_normal((w.nheads, dstate))).astype(np.float32)
    res = oracle.forward(w.dims(), inp)
    h = make_handle(w, "fused")
    assert h.path == "fused"
    dev = to_device(inp, w)
    out, fs, fc, _ = run_forward(h, w, dev, init_state_of(h, w, inp))
    _compare_all(w, inp, res, out, fs, fc, f"bc_norm N={dstate} conv={dconv}/fused")


def _ragged_case():
    w = _small("mini_k3_mixer", batch=4, seqlen=300, mean_doc_len=90).with_(init_state=True)
    inp = make_inputs(w)
    lengths = np.array([300, 128, 0, 65], dtype=np.int32)
    return w, inp, lengths


def _run_ragged(h, w, dev, init, lengths):
    fin = h.new_state(w.batch)
    lens = torch.from_numpy(lengths).cuda()
    out = h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"],
                    dev["C"], dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"],
                    init_state=init, final_state=fin, lengths=lens)
    torch.cuda.synchronize()
    h.check()
    return out, fin


@pytest.mark.parametrize("path", PATHS)
def test_ragged_batch_matches_oracle_with_zero_padding(path):
    """Ragged lengths (the full row, exactly two chunks, nothing, one chunk + 1):
    every element against the oracle, padding exactly +0.0, final state and conv
    history after each row's last real token."""
    w, inp, lengths = _ragged_case()
    res = oracle.forward(w.dims(), dict(inp, lengths=lengths))
    h = make_handle(w, path)
    dev = to_device(inp, w)
    out, fin = _run_ragged(h, w, dev, init_state_of(h, w, inp), lengths)
    bits = out.view(torch.int16)
    for b, L in enumerate(lengths):
        assert bool(torch.all(bits[b, L:] == 0)), f"row {b}: padding is not +0.0"
    s, c = state_to_numpy(h, fin, w.batch)
    _compare_all(w, inp, res, out.double().cpu().numpy(), s, c, f"ragged/{h.path}")


@pytest.mark.parametrize("path", PATHS)
def test_ragged_rows_equal_rows_run_alone(path):
    w, inp, lengths = _ragged_case()
    h = make_handle(w, path)
    dev = to_device(inp, w)
    out, fin = _run_ragged(h, w, dev, init_state_of(h, w, inp), lengths)
    s_all, c_all = state_to_numpy(h, fin, w.batch)
    o_all = out.double().cpu().numpy()
    for b, L in enumerate(lengths):
        if L == 0:
            continue
        wb = w.with_(batch=1, seqlen=int(L))
        one = {k: (None if v is None else
                   (np.ascontiguousarray(v[b:b + 1, :L]) if k in ("x", "z", "B", "C", "dt_raw", "seq_idx")
                    else (np.ascontiguousarray(v[b:b + 1]) if k in ("init_ssm", "init_conv") else v)))
               for k, v in inp.items()}
        h1 = make_handle(wb, path)
        o1, s1, c1, _ = run_forward(h1, wb, to_device(one, wb), init_state_of(h1, wb, one))
        rel = np.linalg.norm(o_all[b, :L] - o1[0]) / max(np.linalg.norm(o1[0]), 1e-30)
        assert rel <= 1e-6, f"row {b}: rel-L2 {rel:.2e} against the row run alone"
        assert np.allclose(s_all[b], s1[0], rtol=1e-6, atol=1e-6 * np.abs(s1[0]).max())
        if c1 is not None:
            assert np.array_equal(c_all[b], c1[0])


@pytest.mark.parametrize("path", PATHS)
def test_ragged_batch_without_conv_with_bc_norm(path):
    """The ragged variant of the no-conv, B/C-norm, d_state-128 kernels (per-token A)."""
    w = _small("mamba3_siso", batch=3, seqlen=200, nheads=8, ngroups=2)
    inp = make_inputs(w)
    lengths = np.array([200, 70, 0], dtype=np.int32)
    res = oracle.forward(w.dims(), dict(inp, lengths=lengths))
    h = make_handle(w, path)
    dev = to_device(inp, w)
    if w.bc_norm:
        h.set_bc_norm(dev["B_norm_w"], dev["C_norm_w"], dev["B_bias"], dev["C_bias"])
    out, fin = _run_ragged(h, w, dev, init_state_of(h, w, inp), lengths)
    bits = out.view(torch.int16)
    for b, L in enumerate(lengths):
        assert bool(torch.all(bits[b, L:] == 0)), f"row {b}: padding is not +0.0"
    s, c = state_to_numpy(h, fin, w.batch)
    _compare_all(w, inp, res, out.double().cpu().numpy(), s, c, f"ragged norm/{h.path}")


@pytest.mark.parametrize("path", PATHS)
def test_packed_documents_match_separate_calls(path):
    """Each document of a packed row against the same document run as its own
    call (model card, Checkpoint and training: packed and separately launched
    documents differ only by the reduction order of the fused prefix sums).
    Both runs see the same bf16 operands; the chunk grid falls differently on
    the document, so the results agree to the bf16 tolerance, not bit for bit.
    Documents of 1 token and boundaries on and beside the 64-token chunk edges
    are included."""
    w = _small("mini_k3_mixer", batch=1, seqlen=260, documents="none", init_state=False, seed=41)
    inp = make_inputs(w)
    seq = _docs_row(w.seqlen, [37, 64, 65, 150, 151, 230])[None]
    inp["seq_idx"] = seq
    h = make_handle(w, path)
    packed, _, _, _ = run_forward(h, w, to_device(inp, w), None, final=False)
    for k in range(int(seq.max()) + 1):
        idx = np.flatnonzero(seq[0] == k)
        lo, hi = int(idx[0]), int(idx[-1]) + 1
        wk = w.with_(seqlen=hi - lo)
        one = {key: (None if v is None else
                     (np.ascontiguousarray(v[:, lo:hi]) if key in ("x", "z", "B", "C", "dt_raw")
                      else v)) for key, v in inp.items()}
        one["seq_idx"] = None
        hk = make_handle(wk, path)
        alone, _, _, _ = run_forward(hk, wk, to_device(one, wk), None, final=False)
        assert_close(packed[:, lo:hi], alone, "bf16", f"document {k} packed vs alone ({h.path})")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", ["mini_k3_mixer", "mamba3_siso"])
def test_forward_of_one_token_equals_the_step(name, path):
    """Mamba3Block.step is the forward at L = 1 with the state carried: the
    decode kernel and a one-token forward from the same state give the same
    output and the same new state (to the bf16 tolerance: different kernels)."""
    w = _small(name, batch=3, seqlen=70, documents="none")
    inp = make_inputs(w)
    h = make_handle(w, path)
    dev = to_device(inp, w)
    _, _, _, state = run_forward(h, w, dev, None)
    carried = state.clone()
    si = make_step_inputs(w, 0)
    o_step = _step_run(h, w, dev, si, state)
    torch.cuda.synchronize()

    w1 = w.with_(seqlen=1)
    one = dict(inp)
    one.update({k: v[:, None] for k, v in si.items()})
    one["seq_idx"] = None
    o_fwd, s_fwd, c_fwd, _ = run_forward(h, w1, to_device(one, w1), carried)
    assert_close(o_step.double().cpu().numpy()[:, None], o_fwd, w.act_dtype, "step vs forward out")
    s_step, c_step = state_to_numpy(h, state, w.batch)
    assert_close(s_step, s_fwd, w.act_dtype, "step vs forward state")
    if c_step is not None:
        assert np.array_equal(c_step, c_fwd)
