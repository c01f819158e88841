"""Argument validation through the C ABI with a real handle: every bad call is
refused by name before any launch (its output stays untouched), and a good
call writes nothing outside its output (guard bands)."""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import make_handle, to_device
from selective_state_space_forward_b200 import ssd
from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

SENTINEL = -12345.0


@pytest.fixture(scope="module")
def case():
    w = WORKLOADS["mini_k3_mixer"].with_(batch=2, seqlen=96, mean_doc_len=30)
    inp = make_inputs(w)
    h = make_handle(w, "staged", max_batch=2, max_seqlen=128)
    return w, h, to_device(inp, w)


def _raw_forward(h, w, dev, batch=None, seqlen=None, **over):
    args = dict(x=dev["x"], z=dev["z"], dt_raw=dev["dt_raw"], dt_bias=dev["dt_bias"], A=dev["A"],
                B=dev["B"], C=dev["C"], D=dev["D"], conv_w=dev["conv_w"], conv_b=dev["conv_b"],
                seq_idx=dev["seq_idx"], init=None, out=None, final=None)
    args.update(over)
    p = {k: (v if isinstance(v, int) or v is None else v.data_ptr()) for k, v in args.items()}
    return h.lib.ssd_forward(h._h, batch if batch is not None else w.batch,
                             seqlen if seqlen is not None else w.seqlen,
                             p["x"], p["z"], p["dt_raw"], p["dt_bias"], p["A"], p["B"], p["C"],
                             p["D"], p["conv_w"], p["conv_b"], p["seq_idx"], p["init"], p["out"],
                             p["final"], None)


def test_bad_arguments_are_refused_by_name(case):
    w, h, dev = case
    out = torch.full_like(dev["x"], SENTINEL)
    bad = [
        (dict(x=None, out=out), 1, "x"),
        (dict(dt_raw=None, out=out), 1, "dt_raw"),
        (dict(out=None), 1, "out"),
        (dict(conv_w=None, out=out), 1, "conv_w"),
        (dict(x=dev["x"].data_ptr() + 2, out=out), 3, "x"),
        (dict(B=dev["B"].data_ptr() + 8, out=out), 3, "B"),
        (dict(dt_raw=dev["dt_raw"].data_ptr() + 2, out=out), 3, "dt_raw"),
        (dict(out=dev["x"]), 1, "alias"),
    ]
    for over, status, word in bad:
        st = _raw_forward(h, w, dev, **over)
        assert st == status, (over.keys(), st)
        assert word in h.lib.ssd_last_error().decode()
    st = _raw_forward(h, w, dev, batch=3, out=out)
    assert st == 4 and "max_batch" in h.lib.ssd_last_error().decode()
    st = _raw_forward(h, w, dev, seqlen=129, out=out)
    assert st == 4 and "max_seqlen" in h.lib.ssd_last_error().decode()
    st = _raw_forward(h, w, dev, seqlen=-1, out=out)
    assert st == 1
    torch.cuda.synchronize()
    assert bool(torch.all(out == SENTINEL)), "a refused call wrote its output"


def test_conv_args_refused_without_conv():
    w = WORKLOADS["mamba3_siso"].with_(batch=1, seqlen=64)
    inp = make_inputs(w)
    h = make_handle(w, "staged")
    dev = to_device(inp, w)
    cw = torch.zeros(w.conv_dim, 4, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ssd.SSDError, match="conv_w"):
        h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"],
                  dev["D"], conv_w=cw, conv_b=cw[:, 0].contiguous())


@pytest.mark.parametrize("path", ["staged", "auto"])
def test_guard_bands_untouched(case, path):
    w, _, dev = case
    h = make_handle(w, path)
    n = dev["x"].numel()
    pad = 4096
    big = torch.full((n + 2 * pad,), SENTINEL, dtype=torch.bfloat16, device="cuda")
    out = big[pad:pad + n].view_as(dev["x"])
    sb = h.state_bytes(w.batch)
    sbig = torch.full((sb + 2 * 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    fin = sbig[4096:4096 + sb]
    h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"],
              dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"], out=out,
              final_state=fin)
    torch.cuda.synchronize()
    assert bool(torch.all(big[:pad] == SENTINEL)) and bool(torch.all(big[pad + n:] == SENTINEL))
    assert bool(torch.all(sbig[:4096] == 0xA5)) and bool(torch.all(sbig[4096 + sb:] == 0xA5))
    assert bool(torch.all(torch.isfinite(out.float())))


def test_check_reports_clean_status(case):
    w, h, dev = case
    h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"],
              dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"])
    h.check()


@pytest.mark.parametrize("path", ["staged", "auto"])
def test_validate_finite_reports_a_nan_in_the_results(path):
    """validate_finite: clean forward and step calls check clean; a NaN planted in
    z reaches out and ssd_check reports it; the check clears the word."""
    w = WORKLOADS["mini_k3_mixer"].with_(batch=1, seqlen=128, mean_doc_len=50)
    inp = make_inputs(w)
    dev = to_device(inp, w)
    h = ssd.Handle(w.nheads, w.headdim, w.dstate, w.ngroups, w.dconv, w.act_dtype,
                   max_batch=1, max_seqlen=128, path=path, validate_finite=True)
    fin = h.new_state(1)

    def fwd():
        return h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"],
                         dev["C"], dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"],
                         final_state=fin)

    fwd()
    h.check()
    dev["z"][0, 5, 3] = float("nan")
    fwd()
    with pytest.raises(ssd.SSDError, match="non-finite"):
        h.check()
    dev["z"][0, 5, 3] = 0.0
    fwd()
    h.check()
    # the decode step: a NaN in z reaches out
    x1, z1 = dev["x"][:, 0].contiguous(), dev["z"][:, 0].contiguous()
    z1[0, 7] = float("nan")
    h.step(x1, z1, dev["dt_raw"][:, 0].contiguous(), dev["dt_bias"], dev["A"],
           dev["B"][:, 0].contiguous(), dev["C"][:, 0].contiguous(), dev["D"], dev["conv_w"],
           dev["conv_b"], state=fin)
    with pytest.raises(ssd.SSDError, match="non-finite"):
        h.check()


@pytest.mark.parametrize("name", ["mini_k3_mixer", "mamba3_siso", "tiny_fp32"])
def test_state_bytes_without_a_handle_match_the_library(name):
    """The binding sizes ssd_forward_noalloc's state buffers itself; its count
    must be ssd_state_bytes'."""
    w = WORKLOADS[name]
    h = make_handle(w, max_batch=3, max_seqlen=64)
    for b in (0, 1, 3):
        assert ssd.state_bytes_for(w.nheads, w.headdim, w.dstate, w.ngroups, w.dconv,
                                   w.act_dtype, b) == h.state_bytes(b)
