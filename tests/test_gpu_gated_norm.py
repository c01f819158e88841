"""GPU parity of the gated RMSNorm after the scan (upstream Mamba-2's
norm(y * silu(z)), codestral_mamba.ts header: `mixer.norm.weight [d_inner]`)
against oracle.gated_norm applied to the oracle's forward output, at the bf16
tolerance (rel-L2 <= 5e-3, max-abs <= 2e-2 * max|ref|)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, init_state_of, make_handle, run_forward, to_device
from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs, make_step_inputs, round_bf16

pytestmark = pytest.mark.gpu


def _weight(n, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    return (1.0 + 0.3 * rng.standard_normal(n)).astype(np.float32)


@pytest.mark.parametrize("path", ["staged", "auto"])
@pytest.mark.parametrize("group", [0, 256])
def test_gated_norm_matches_oracle(path, group):
    """mini_k3_mixer shapes with packed documents: one norm per token (group 0 =
    d_inner) and upstream's grouped variant (d_inner / ngroups = 256)."""
    w = WORKLOADS["mini_k3_mixer"].with_(batch=2, seqlen=300, mean_doc_len=90)
    inp = make_inputs(w)
    d_inner = w.nheads * w.headdim
    wt = _weight(d_inner, 3)
    res = oracle.forward(w.dims(), inp)
    want = oracle.gated_norm(res["out"], wt, group or None, eps=1e-5)
    h = make_handle(w, path)
    h.set_gated_norm(torch.from_numpy(wt).cuda(), group_size=group, eps=1e-5)
    out, _, _, _ = run_forward(h, w, to_device(inp, w), None, final=False)
    assert_close(out, want, "bf16", f"gated norm group={group} ({h.path})")


def test_gated_norm_long_7b_rows_and_initial_state():
    w = WORKLOADS["long_7b"].with_(batch=1, seqlen=200, nheads=16)
    inp = make_inputs(w)
    d_inner = w.nheads * w.headdim
    wt = _weight(d_inner, 4)
    res = oracle.forward(w.dims(), inp)
    want = oracle.gated_norm(res["out"], wt, None, eps=1e-5)
    h = make_handle(w, "auto")
    h.set_gated_norm(torch.from_numpy(wt).cuda(), eps=1e-5)
    out, _, _, _ = run_forward(h, w, to_device(inp, w), init_state_of(h, w, inp), final=False)
    assert_close(out, want, "bf16", "gated norm long_7b")


def test_gated_norm_keeps_ragged_padding_zero():
    w = WORKLOADS["mini_k3_mixer"].with_(batch=3, seqlen=130, mean_doc_len=60)
    inp = make_inputs(w)
    lengths = np.array([130, 64, 0], dtype=np.int32)
    wt = -_weight(w.nheads * w.headdim, 5)          # negative weights: -0.0 would show
    res = oracle.forward(w.dims(), dict(inp, lengths=lengths))
    want = oracle.gated_norm(res["out"], wt, None, eps=1e-5)
    h = make_handle(w, "auto")
    h.set_gated_norm(torch.from_numpy(wt).cuda())
    dev = to_device(inp, w)
    out = h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"],
                    dev["C"], dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"],
                    lengths=torch.from_numpy(lengths).cuda())
    torch.cuda.synchronize()
    bits = out.view(torch.int16)
    for b, L in enumerate(lengths):
        assert bool(torch.all(bits[b, L:] == 0)), f"row {b}: padding is not +0.0"
    got = out.double().cpu().numpy()
    for b, L in enumerate(lengths):
        if L:
            assert_close(got[b, :L], want[b, :L], "bf16", f"ragged row {b}")


def test_gated_norm_on_the_decode_step():
    w = WORKLOADS["mini_k3_mixer"].with_(batch=3, seqlen=70, documents="none")
    inp = make_inputs(w)
    d_inner = w.nheads * w.headdim
    wt = _weight(d_inner, 6)
    h = make_handle(w, "auto")
    dev = to_device(inp, w)
    _, _, _, state = run_forward(h, w, dev, None)
    r = oracle.forward(w.dims(), inp)
    si = make_step_inputs(w, 0)
    h.set_gated_norm(torch.from_numpy(wt).cuda(), group_size=256)
    at = torch.bfloat16
    o = h.step(*(torch.from_numpy(si[k]).to(at).cuda() for k in ("x", "z")),
               torch.from_numpy(si["dt_raw"]).cuda(), dev["dt_bias"], dev["A"],
               torch.from_numpy(si["B"]).to(at).cuda(), torch.from_numpy(si["C"]).to(at).cuda(),
               dev["D"], dev["conv_w"], dev["conv_b"], state=state)
    torch.cuda.synchronize()
    tok = dict(inp)
    tok.update({k: v[:, None] for k, v in si.items()})
    ro = oracle.step(w.dims(), tok, r["final_ssm"].astype(np.float32),
                     r["final_conv"].astype(np.float32))
    want = oracle.gated_norm(ro["out"][:, 0], wt, 256, eps=1e-5)
    assert_close(o.double().cpu().numpy(), want, "bf16", "gated norm step")


def test_gated_norm_refuses_bad_groups():
    from selective_state_space_forward_b200 import ssd
    w = WORKLOADS["mini_k3_mixer"].with_(batch=1, seqlen=64)
    h = make_handle(w, "auto")
    for g in (3, 100, 4096):
        with pytest.raises(ssd.SSDError) as e:
            h.set_gated_norm(None, group_size=g)
        assert e.value.status == 1


def _packed(w, inp, pad):
    """A packed in_proj output (batch, seqlen, ld): [z | x | B | C | dt_raw | pad]
    in bf16, with dt_raw rounded to bf16 (the oracle gets the same values)."""
    HP, GN, H = w.nheads * w.headdim, w.ngroups * w.dstate, w.nheads
    dt = round_bf16(inp["dt_raw"])
    rng = np.random.Generator(np.random.PCG64(77))
    filler = round_bf16(rng.standard_normal((w.batch, w.seqlen, pad)))
    packed = np.concatenate([inp["z"], inp["x"], inp["B"], inp["C"], dt, filler], axis=2)
    assert packed.shape[2] == 2 * HP + 2 * GN + H + pad
    return torch.from_numpy(np.ascontiguousarray(packed, dtype=np.float32)).to(
        torch.bfloat16).cuda(), dict(inp, dt_raw=dt)


@pytest.mark.parametrize("path", ["staged", "auto"])
def test_packed_in_proj_input_with_gated_norm(path):
    """mini_k3_mixer shapes: the scan reads z, x, B, C and dt_raw in place from one
    packed in_proj row through row strides, then the gated norm (group 256) is
    applied; against oracle.gated_norm(oracle.forward(...)) on the same values."""
    w = WORKLOADS["mini_k3_mixer"].with_(batch=2, seqlen=300, mean_doc_len=90)
    inp = make_inputs(w)
    zxbcdt, ref_inp = _packed(w, inp, pad=8)         # 32 + 8 = a 16-byte multiple
    wt = _weight(w.nheads * w.headdim, 8)
    res = oracle.forward(w.dims(), ref_inp)
    want = oracle.gated_norm(res["out"], wt, 256, eps=1e-5)
    h = make_handle(w, path)
    dev = to_device(inp, w)
    h.set_gated_norm(torch.from_numpy(wt).cuda(), group_size=256)
    fin = h.new_state(w.batch)
    out = h.forward_packed(zxbcdt, dev["dt_bias"], dev["A"], dev["D"], dev["conv_w"],
                           dev["conv_b"], seq_idx=dev["seq_idx"], final_state=fin)
    torch.cuda.synchronize()
    h.check()
    assert_close(out.double().cpu().numpy(), want, "bf16", f"packed + gated norm ({h.path})")
    s, c = h.state_views(fin, w.batch)
    assert_close(s.double().cpu().numpy(), res["final_ssm"], "bf16", "packed final state")
    assert np.array_equal(c.double().cpu().numpy(), res["final_conv"])


@pytest.mark.parametrize("path", ["staged", "auto"])
def test_packed_equals_contiguous_forward_bitwise(path):
    """The same values through ssd_forward (contiguous tensors) and through
    ssd_forward_packed give the same bits: strides change addressing only."""
    w = WORKLOADS["long_7b"].with_(batch=2, seqlen=150, nheads=16)
    inp = make_inputs(w)
    inp["dt_raw"] = round_bf16(inp["dt_raw"])
    zxbcdt, _ = _packed(w, inp, pad=24)
    h = make_handle(w, path)
    dev = to_device(inp, w)
    init = init_state_of(h, w, inp)
    a, sa, _, _ = run_forward(h, w, dev, init)
    fin = h.new_state(w.batch)
    b = h.forward_packed(zxbcdt, dev["dt_bias"], dev["A"], dev["D"], dev["conv_w"],
                         dev["conv_b"], init_state=init, final_state=fin)
    torch.cuda.synchronize()
    assert np.array_equal(b.double().cpu().numpy(), a)
    assert np.array_equal(h.state_views(fin, w.batch)[0].double().cpu().numpy(), sa)
