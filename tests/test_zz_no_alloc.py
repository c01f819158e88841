"""ssd_forward_noalloc (the allocation-free forward) against ssd_forward.

Both entry points run the fused path's kernels; the no-alloc one takes its
workspace from a static device array of the library instead of a handle's
cudaMalloc'd block.  The checks: two calls in a row on one stream (different
shapes and inputs, so the second meets the first call's hand-off flags and
leftover scratch) each agree with ssd_forward; a repeated call is bit-identical
and moves no device memory; shapes beyond the static scratch and shapes the
fused path does not serve are refused before any launch.

This file is collected last on purpose: it must pass alone in a fresh process
(where its first call does the one-time set-up) and after every other test.
"""
import numpy as np
import pytest
import torch

from gpu_util import init_state_of, make_handle, to_device
from selective_state_space_forward_b200 import ssd
from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

# Same kernels on the same inputs: the results should agree to the last bit;
# the bound leaves room only for a different segment split of the scan.
REL_L2 = 1e-6
MAX_ABS = 1e-5

CASES = [
    # packed documents, ragged tail, dstate 64, no initial state
    WORKLOADS["mini_k3_mixer"].with_(batch=2, seqlen=1000, mean_doc_len=300),
    # dstate 128, one document per row, an initial state
    WORKLOADS["long_7b"].with_(batch=1, seqlen=3000),
]


def _noalloc(w, dev, init, fin, status, out=None, validate_finite=False):
    return ssd.forward_noalloc(
        dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"],
        dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"], init_state=init,
        out=out, final_state=fin, status=status, nheads=w.nheads, headdim=w.headdim,
        dstate=w.dstate, ngroups=w.ngroups, dconv=w.dconv, a_per_token=w.a_per_token,
        validate_finite=validate_finite)


def _handle_forward(h, w, dev, init):
    fin = h.new_state(w.batch)
    out = h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"],
                    dev["C"], dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"],
                    init_state=init, final_state=fin)
    torch.cuda.synchronize()
    h.check()
    return out, fin


def _close(got, want, what):
    g = got.double().cpu().numpy().ravel()
    r = want.double().cpu().numpy().ravel()
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    mx = np.abs(g - r).max() / max(np.abs(r).max(), 1e-30)
    assert rel <= REL_L2 and mx <= MAX_ABS, f"{what}: rel-L2 {rel:.3e}, max-abs {mx:.3e}"


def _status_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def test_noalloc_two_calls_in_a_row_match_forward():
    runs = []
    for w in CASES:
        inp = make_inputs(w)
        dev = to_device(inp, w)
        h = make_handle(w)
        assert h.path == "fused"
        init = init_state_of(h, w, inp)
        want_out, want_fin = _handle_forward(h, w, dev, init)
        runs.append((w, h, dev, init, want_out, want_fin))

    status = _status_word()
    got = []
    for w, h, dev, init, _, _ in runs:      # enqueued back to back, no sync between
        fin = h.new_state(w.batch)
        out = _noalloc(w, dev, init, fin, status)
        got.append((out, fin))
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
    for (w, h, _, _, want_out, want_fin), (out, fin) in zip(runs, got):
        _close(out, want_out, f"{w.name} out")
        s_got, c_got = h.state_views(fin, w.batch)
        s_want, c_want = h.state_views(want_fin, w.batch)
        _close(s_got, s_want, f"{w.name} final ssm")
        assert torch.equal(c_got, c_want), f"{w.name} final conv history"


def test_noalloc_repeat_is_identical_and_allocates_nothing():
    w = CASES[0]
    inp = make_inputs(w, seed=7)
    dev = to_device(inp, w)
    h = make_handle(w)
    status = _status_word()
    out1, fin1 = torch.empty_like(dev["x"]), h.new_state(w.batch)
    out2, fin2 = torch.empty_like(dev["x"]), h.new_state(w.batch)
    # the first call may do the per-device set-up and load the kernels' modules
    _noalloc(w, dev, None, fin1, status, out=out1)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    _noalloc(w, dev, None, fin2, status, out=out2)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert int(status.item()) == 0
    assert torch.equal(out1, out2)
    assert torch.equal(fin1, fin2)
    # a device allocation takes at least one 2 MiB page
    assert free_before - free_after < (2 << 20), (free_before, free_after)


def test_noalloc_refuses_shapes_beyond_the_static_scratch():
    status = _status_word()
    w = CASES[0]
    H, P, N, G = w.nheads, w.headdim, w.dstate, w.ngroups

    def call(batch, seqlen):
        x = torch.zeros(batch, seqlen, H * P, dtype=torch.bfloat16, device="cuda")
        bc = torch.zeros(batch, seqlen, G * N, dtype=torch.bfloat16, device="cuda")
        f = torch.zeros(batch, seqlen, H, dtype=torch.float32, device="cuda")
        hv = torch.zeros(H, dtype=torch.float32, device="cuda")
        cw = torch.zeros(H * P + 2 * G * N, 4, dtype=torch.bfloat16, device="cuda")
        cb = torch.zeros(H * P + 2 * G * N, dtype=torch.bfloat16, device="cuda")
        return ssd.forward_noalloc(x, x.clone(), f, hv, hv, bc, bc.clone(), hv, cw, cb,
                                   status=status, nheads=H, headdim=P, dstate=N, ngroups=G,
                                   dconv=4)

    # 30,000 tokens of this shape need about 69 MB of scratch (64 MiB held)
    with pytest.raises(ssd.SSDError) as e:
        call(1, 30000)
    assert e.value.status == 4 and "static scratch" in str(e.value)
    # 33 rows x 32 heads = 1056 (row, head) streams (1024 hand-off slots held)
    with pytest.raises(ssd.SSDError) as e:
        call(33, 1)
    assert e.value.status == 4
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_noalloc_refuses_what_the_fused_path_does_not_serve():
    w = CASES[0]
    dev = to_device(make_inputs(w.with_(batch=1, seqlen=64)), w.with_(batch=1, seqlen=64))
    status = _status_word()
    with pytest.raises(ssd.SSDError) as e:
        ssd.forward_noalloc(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"],
                            dev["B"], dev["C"], dev["D"], dev["conv_w"], dev["conv_b"],
                            status=status, nheads=w.nheads, headdim=w.headdim, dstate=w.dstate,
                            ngroups=w.ngroups, dconv=w.dconv, path="staged")
    assert e.value.status == 2
    with pytest.raises(ssd.SSDError) as e:
        ssd.forward_noalloc(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"],
                            dev["B"], dev["C"], dev["D"], dev["conv_w"], dev["conv_b"],
                            status=None, nheads=w.nheads, headdim=w.headdim, dstate=w.dstate,
                            ngroups=w.ngroups, dconv=w.dconv)
    assert e.value.status == 1


def test_noalloc_per_token_a_matches_forward():
    """Per-token A (floored at magnitude 1e-4), d_state 128, no conv: the no-alloc
    call against ssd_forward on a handle made with the same a_mode."""
    w = WORKLOADS["mamba3_siso"].with_(batch=2, seqlen=300, nheads=8, bc_norm=False, seed=13)
    inp = make_inputs(w)
    inp["A"][0, 5:9, 2] = np.array([0.0, -1e-6, -1e-4, -3.0], dtype=np.float32)
    dev = to_device(inp, w)
    h = make_handle(w)
    assert h.path == "fused"
    want_out, want_fin = _handle_forward(h, w, dev, None)
    status = _status_word()
    fin = h.new_state(w.batch)
    out = _noalloc(w, dev, None, fin, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _close(out, want_out, "per-token A out")
    _close(h.state_views(fin, w.batch)[0], h.state_views(want_fin, w.batch)[0],
           "per-token A final ssm")


def test_noalloc_validate_finite_reports_like_forward():
    """validate_finite: a clean call leaves the status word at 0; a NaN planted in
    one token of x reaches out and the final state, and the call ORs the
    non-finite bit (4) into the status word, as ssd_forward's check reports it."""
    w = CASES[0].with_(seqlen=200)
    inp = make_inputs(w, seed=5)
    dev = to_device(inp, w)
    status = _status_word()
    fin = ssd.Handle(w.nheads, w.headdim, w.dstate, w.ngroups, w.dconv, "bf16",
                     max_batch=w.batch, max_seqlen=w.seqlen).new_state(w.batch)
    _noalloc(w, dev, None, fin, status, validate_finite=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    dev["x"][0, 150, 3] = float("nan")
    _noalloc(w, dev, None, fin, status, validate_finite=True)
    torch.cuda.synchronize()
    assert int(status.item()) & 4, f"status {int(status.item()):#x}"
    h = ssd.Handle(w.nheads, w.headdim, w.dstate, w.ngroups, w.dconv, "bf16",
                   max_batch=w.batch, max_seqlen=w.seqlen, validate_finite=True)
    h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"],
              dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"],
              final_state=h.new_state(w.batch))
    with pytest.raises(ssd.SSDError) as e:
        h.check()
    assert e.value.status == 6 and "non-finite" in str(e.value)
