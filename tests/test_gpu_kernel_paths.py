"""GPU checks of kernel paths that the main parity tests reach only on some shapes.

- The decode step with more heads per B/C group than a block has threads (its
  per-head dt and decay loop), against the oracle's sequential recurrence; and
  on shapes whose state pieces (8 KB of a block's state each) end part-way:
  fewer rows than a piece holds, rows that fill only some of a block's warps,
  d_state 32 to 256.
- The staged path's chunk-output kernel on heads wider than one 64-column
  output block (headdim 128, and 72 with a part block) and a d_state that is
  not a power of two, element by element against the oracle.
- The S6 scan's two ways of bringing a chunk's raw inputs on chip: asynchronous
  copies into shared memory (16-byte aligned rows) and loads into registers (any
  other rows).  They compute the same values in the same order, so the outputs
  agree bit for bit; a bf16 d_inner that is not a multiple of 8 (the register
  path) is checked against the oracle too.
Tolerances as in the parity tests: bf16 rel-L2 <= 5e-3, max-abs <= 2e-2 max|ref|."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, make_handle, run_forward, state_to_numpy, to_device
from selective_state_space_forward_b200 import ssd
from selective_state_space_forward_b200.synthetic import (WORKLOADS, make_inputs, make_s6_inputs,
                                                           make_step_inputs)

pytestmark = pytest.mark.gpu


def test_decode_more_heads_per_group_than_threads():
    # 160 heads in one group: a decode block (128 threads) loops over its heads
    w = WORKLOADS["mini_k3_mixer"].with_(batch=2, seqlen=40, nheads=160, headdim=8, dstate=32,
                                         ngroups=1, documents="none")
    inp = make_inputs(w)
    h = make_handle(w, "auto")
    dev = to_device(inp, w)
    _, _, _, state = run_forward(h, w, dev, None)
    r = oracle.forward(w.dims(), inp)
    ssm, conv = r["final_ssm"].astype(np.float32), r["final_conv"].astype(np.float32)
    at = torch.bfloat16
    for step in range(3):
        si = make_step_inputs(w, step)
        out = h.step(*(torch.from_numpy(si[k]).to(at).cuda() for k in ("x", "z")),
                     torch.from_numpy(si["dt_raw"]).cuda(), dev["dt_bias"], dev["A"],
                     torch.from_numpy(si["B"]).to(at).cuda(), torch.from_numpy(si["C"]).to(at).cuda(),
                     dev["D"], dev["conv_w"], dev["conv_b"], state=state)
        torch.cuda.synchronize()
        tok = dict(inp)
        tok.update({k: v[:, None] for k, v in si.items()})
        ro = oracle.step(w.dims(), tok, ssm, conv)
        assert_close(out.double().cpu().numpy(), ro["out"][:, 0], "bf16", f"step {step}")
        ssm = ro["final_ssm"].astype(np.float32)
        conv = ro["final_conv"].astype(np.float32)
    fs, fc = state_to_numpy(h, state, w.batch)
    assert_close(fs, ssm, "bf16", "state after the steps")
    assert np.array_equal(fc, conv)


def _decode_steps(w, steps=3):
    inp = make_inputs(w)
    h = make_handle(w, "auto")
    dev = to_device(inp, w)
    _, _, _, state = run_forward(h, w, dev, None)
    r = oracle.forward(w.dims(), inp)
    ssm, conv = r["final_ssm"].astype(np.float32), r["final_conv"].astype(np.float32)
    at = torch.bfloat16
    for step in range(steps):
        si = make_step_inputs(w, step)
        out = h.step(*(torch.from_numpy(si[k]).to(at).cuda() for k in ("x", "z")),
                     torch.from_numpy(si["dt_raw"]).cuda(), dev["dt_bias"], dev["A"],
                     torch.from_numpy(si["B"]).to(at).cuda(), torch.from_numpy(si["C"]).to(at).cuda(),
                     dev["D"], dev["conv_w"], dev["conv_b"], state=state)
        torch.cuda.synchronize()
        h.check()
        tok = dict(inp)
        tok.update({k: v[:, None] for k, v in si.items()})
        ro = oracle.step(w.dims(), tok, ssm, conv)
        assert_close(out.double().cpu().numpy(), ro["out"][:, 0], "bf16", f"step {step}")
        ssm = ro["final_ssm"].astype(np.float32)
        conv = ro["final_conv"].astype(np.float32)
    fs, fc = state_to_numpy(h, state, w.batch)
    assert_close(fs, ssm, "bf16", "state after the steps")
    assert np.array_equal(fc, conv)


@pytest.mark.parametrize("nheads,headdim,dstate,ngroups", [
    (3, 8, 64, 1),      # 24 rows: one piece of 32 rows' room, the last 8 rows on two warps
    (2, 8, 256, 1),     # 8 rows per piece: two pieces, one warp each
    (6, 24, 128, 2),    # 72 rows per group: 16 rows per piece, a last piece of 8
    (5, 8, 32, 5),      # one head per group, 8 rows of 64 per piece
])
def test_decode_partial_state_pieces(nheads, headdim, dstate, ngroups):
    w = WORKLOADS["mini_k3_mixer"].with_(batch=3, seqlen=70, nheads=nheads, headdim=headdim,
                                         dstate=dstate, ngroups=ngroups, documents="none")
    _decode_steps(w)


@pytest.mark.parametrize("headdim,dstate", [(128, 128), (72, 200)])
def test_staged_wide_heads(headdim, dstate):
    w = WORKLOADS["mini_k3_mixer"].with_(batch=2, seqlen=150, nheads=2, headdim=headdim, dstate=dstate,
                                         ngroups=1, mean_doc_len=60)
    inp = make_inputs(w)
    res = oracle.forward(w.dims(), inp)
    h = make_handle(w, "staged")
    out, fs, fc, _ = run_forward(h, w, to_device(inp, w), None)
    assert_close(out, res["out"], "bf16", f"staged P={headdim} N={dstate} out")
    assert_close(fs, res["final_ssm"], "bf16", f"staged P={headdim} N={dstate} final state")
    assert np.array_equal(fc, res["final_conv"])


def _s6_dev(inp):
    return {k: (None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(
        torch.bfloat16 if k in ("u", "z", "B", "C") else torch.float32).cuda())
        for k, v in inp.items()}


def _s6_run(dev, u):
    Bb, L, DI = u.shape
    N = dev["A_log"].shape[1]
    fin = torch.empty(Bb, DI, N, dtype=torch.float32, device="cuda")
    out = ssd.s6_forward(u, dev["delta"], dev["delta_bias"], dev["A_log"], dev["B"], dev["C"],
                         dev["D"], z=dev["z"], init_state=dev["init"], final_state=fin)
    torch.cuda.synchronize()
    return out, fin


def test_s6_register_path_gives_the_async_paths_bits():
    inp = make_s6_inputs(2, 100, 96, 16, seed=21)
    dev = _s6_dev(inp)
    out_a, fin_a = _s6_run(dev, dev["u"])                  # 16-byte aligned rows: async copies
    flat = torch.empty(dev["u"].numel() + 1, dtype=torch.bfloat16, device="cuda")
    u_off = flat[1:].view(dev["u"].shape)                   # starts 2 bytes in: register loads
    u_off.copy_(dev["u"])
    assert u_off.data_ptr() % 16 != 0
    out_r, fin_r = _s6_run(dev, u_off)
    assert torch.equal(out_a.view(torch.int16), out_r.view(torch.int16))
    assert torch.equal(fin_a, fin_r)


def test_s6_bf16_d_inner_not_a_multiple_of_8():
    inp = make_s6_inputs(2, 90, 44, 16, seed=22)
    res = oracle.s6_forward(inp)
    dev = _s6_dev(inp)
    out, fin = _s6_run(dev, dev["u"])
    assert_close(out.double().cpu().numpy(), res["out"], "bf16", "S6 d_inner 44 out")
    assert_close(fin.double().cpu().numpy(), res["final"], "bf16", "S6 d_inner 44 final state")
