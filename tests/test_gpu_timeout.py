"""The fused kernel's failure path, tested without a GPU fault.

Segments of a (row, head) stream hand their leaving state to the next segment
through a flag in device memory, and the waiting CTA spins on it with a bound.
A testing hook shortens the bound to 2 ms and withholds one stream's first
hand-off, so that wait runs out: the kernel must raise the timeout bit (read by
ssd_check as SSD_ERR_DEVICE), finish its own copies and tensor-core work, and
exit; the next call on the same handle must be correct against the oracle.

The decode kernel's blocks wait for bulk copies of their state; with the same
hook one block never requests its first state piece, so its wait runs out the
same way, and the next prefill and step on the handle are correct."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, make_handle, run_forward, to_device
from selective_state_space_forward_b200 import ssd
from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs, make_step_inputs

pytestmark = pytest.mark.gpu


def test_withheld_handoff_times_out_and_the_next_call_is_clean():
    # 160 (row, head) streams of 16 chunks on 148 SMs: the host splits every stream
    # into segments, so segment 1 of stream 0 waits for segment 0's hand-off
    w = WORKLOADS["mini_k3_mixer"].with_(batch=5, seqlen=1024, documents="none")
    inp = make_inputs(w)
    h = make_handle(w, "fused")
    assert h.path == "fused"
    dev = to_device(inp, w)
    h.set_wait_test(wait_limit_ns=2_000_000, withhold_stream=0)
    fin = h.new_state(w.batch)
    h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"],
              dev["D"], dev["conv_w"], dev["conv_b"], final_state=fin)
    torch.cuda.synchronize()
    with pytest.raises(ssd.SSDError) as e:
        h.check()
    assert e.value.status == 6 and "bounded wait timed out" in str(e.value)

    h.set_wait_test(0, -1)
    h.check()                                   # the status word was cleared
    out, fs, _, _ = run_forward(h, w, dev, None)
    res = oracle.forward(w.dims(), inp)
    assert_close(out, res["out"], "bf16", "forward after a timed-out call")
    assert_close(fs, res["final_ssm"], "bf16", "state after a timed-out call")


def test_withheld_decode_piece_times_out_and_the_next_step_is_clean():
    w = WORKLOADS["mini_k3_mixer"].with_(batch=4, seqlen=100, documents="none")
    inp = make_inputs(w)
    h = make_handle(w, "auto")
    dev = to_device(inp, w)
    si = make_step_inputs(w, 0)
    at = torch.bfloat16
    step_dev = [torch.from_numpy(si[k]).to(at).cuda() for k in ("x", "z")] + [
        torch.from_numpy(si["dt_raw"]).cuda(), dev["dt_bias"], dev["A"],
        torch.from_numpy(si["B"]).to(at).cuda(), torch.from_numpy(si["C"]).to(at).cuda(),
        dev["D"], dev["conv_w"], dev["conv_b"]]

    _, _, _, state = run_forward(h, w, dev, None)
    h.set_wait_test(wait_limit_ns=2_000_000, withhold_stream=w.ngroups + 1)   # row 1, group 1
    h.step(*step_dev, state=state)
    torch.cuda.synchronize()
    with pytest.raises(ssd.SSDError) as e:
        h.check()
    assert e.value.status == 6 and "bounded wait timed out" in str(e.value)

    # that call's state is invalid: prefill again, then a clean step against the oracle
    h.set_wait_test(0, -1)
    h.check()
    _, _, _, state = run_forward(h, w, dev, None)
    out = h.step(*step_dev, state=state)
    torch.cuda.synchronize()
    h.check()
    r = oracle.forward(w.dims(), inp)
    tok = dict(inp)
    tok.update({k: v[:, None] for k, v in si.items()})
    ro = oracle.step(w.dims(), tok, r["final_ssm"].astype(np.float32), r["final_conv"].astype(np.float32))
    assert_close(out.double().cpu().numpy(), ro["out"][:, 0], "bf16", "step after a timed-out step")


def test_wait_test_hook_validates_its_arguments():
    w = WORKLOADS["mini_k3_mixer"].with_(batch=1, seqlen=64)
    h = make_handle(w, "fused")
    for bad in (dict(wait_limit_ns=10, withhold_stream=-1), dict(wait_limit_ns=0, withhold_stream=-2)):
        with pytest.raises(ssd.SSDError) as e:
            h.set_wait_test(**bad)
        assert e.value.status == 1
