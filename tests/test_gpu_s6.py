"""GPU parity of the Mamba-1 selective scan (S6) through the C ABI against the
fp64 oracle.  Tolerances as for the SSD scan: bf16 activations rel-L2 <= 5e-3
and max-abs <= 2e-2 * max|ref|; fp32 rel-L2 <= 1e-5.  At the Falcon-Mamba-7B
mixer shape (d_inner 8192, d_state 16) the oracle checks slices of channels:
channels never mix, so a slice is its own scan."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close
from selective_state_space_forward_b200 import ssd
from selective_state_space_forward_b200.synthetic import make_s6_inputs

pytestmark = pytest.mark.gpu


def _inputs(B, L, DI, N, seed, bf16=True, gate=True, init=True):
    return make_s6_inputs(B, L, DI, N, seed, bf16=bf16, gate=gate, init=init)


def _gpu(inp, bf16=True):
    at = torch.bfloat16 if bf16 else torch.float32
    dev = {k: (None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(
        at if k in ("u", "z", "B", "C") else torch.float32).cuda()) for k, v in inp.items()}
    Bb, L, DI = inp["u"].shape
    N = inp["A_log"].shape[1]
    fin = torch.empty(Bb, DI, N, dtype=torch.float32, device="cuda")
    out = ssd.s6_forward(dev["u"], dev["delta"], dev["delta_bias"], dev["A_log"], dev["B"],
                         dev["C"], dev["D"], z=dev["z"], init_state=dev["init"], final_state=fin)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), fin.double().cpu().numpy()


@pytest.mark.parametrize("N", [8, 16, 32])
@pytest.mark.parametrize("gate,init", [(True, True), (False, False)])
def test_s6_small_bf16(N, gate, init):
    # 200 channels: a full block of 128 and a ragged one; 300 tokens: a ragged last chunk
    inp = _inputs(2, 300, 200, N, seed=N, gate=gate, init=init)
    res = oracle.s6_forward(inp)
    out, fin = _gpu(inp)
    assert_close(out, res["out"], "bf16", f"S6 N={N} out")
    assert_close(fin, res["final"], "bf16", f"S6 N={N} final state")


def test_s6_small_fp32():
    inp = _inputs(2, 150, 130, 16, seed=7, bf16=False)
    res = oracle.s6_forward(inp)
    out, fin = _gpu(inp, bf16=False)
    assert_close(out, res["out"], "f32", "S6 fp32 out")
    assert_close(fin, res["final"], "f32", "S6 fp32 final state")


def test_s6_falcon_mamba_7b_mixer_sampled_channels():
    B, L, DI, N = 2, 4096, 8192, 16
    inp = _inputs(B, L, DI, N, seed=9)
    out, fin = _gpu(inp)
    for lo, hi in ((0, 48), (4000, 4040), (DI - 40, DI)):
        sl = {k: (None if v is None else
                  (v[:, :, lo:hi] if k in ("u", "delta", "z") else
                   v[lo:hi] if k in ("A_log", "delta_bias", "D") else
                   v[:, lo:hi] if k == "init" else v)) for k, v in inp.items()}
        res = oracle.s6_forward(sl)
        assert_close(out[:, :, lo:hi], res["out"], "bf16", f"S6 7B channels {lo}:{hi} out")
        assert_close(fin[:, lo:hi], res["final"], "bf16", f"S6 7B channels {lo}:{hi} final")


def test_s6_refuses_bad_arguments_by_name():
    lib = ssd.load_library()
    u = torch.zeros(1, 8, 16, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(1, 8, 16, dtype=torch.float32, device="cuda")
    v = torch.zeros(16, dtype=torch.float32, device="cuda")
    a = torch.zeros(16, 24, dtype=torch.float32, device="cuda")
    bc = torch.zeros(1, 8, 24, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ssd.SSDError, match="dstate"):
        ssd.s6_forward(u, f, v, a, bc, bc, v)
    a16 = torch.zeros(16, 16, dtype=torch.float32, device="cuda")
    b16 = torch.zeros(1, 8, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ssd.SSDError, match="out may not alias"):
        ssd.s6_forward(u, f, v, a16, b16, b16, v, out=u)


def test_s6_split_sequence_continues_through_the_state():
    """Scanning tokens [0, 100) and then [100, 300) from the carried state gives
    the outputs and final state of one scan over [0, 300)."""
    inp = _inputs(2, 300, 200, 16, seed=11)
    out, fin = _gpu(inp)
    first = dict(inp, u=inp["u"][:, :100], delta=inp["delta"][:, :100], z=inp["z"][:, :100],
                 B=inp["B"][:, :100], C=inp["C"][:, :100])
    o1, f1 = _gpu(first)
    second = dict(inp, u=inp["u"][:, 100:], delta=inp["delta"][:, 100:], z=inp["z"][:, 100:],
                  B=inp["B"][:, 100:], C=inp["C"][:, 100:], init=f1.astype(np.float32))
    o2, f2 = _gpu(second)
    assert_close(np.concatenate([o1, o2], axis=1), out, "bf16", "S6 split outputs")
    assert_close(f2, fin, "bf16", "S6 split final state")


def test_s6_empty_inputs():
    """No token: the state passes through (zeros without an initial state); no row: nothing."""
    DI, N = 40, 8
    u = torch.empty(2, 0, DI, dtype=torch.bfloat16, device="cuda")
    f = torch.empty(2, 0, DI, dtype=torch.float32, device="cuda")
    bc = torch.empty(2, 0, N, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(DI, dtype=torch.float32, device="cuda")
    a = torch.zeros(DI, N, dtype=torch.float32, device="cuda")
    init = torch.randn(2, DI, N, device="cuda")
    fin = torch.full((2, DI, N), 7.0, device="cuda")
    ssd.s6_forward(u, f, v, a, bc, bc, v, init_state=init, final_state=fin)
    torch.cuda.synchronize()
    assert torch.equal(fin, init)
    ssd.s6_forward(u, f, v, a, bc, bc, v, final_state=fin)
    torch.cuda.synchronize()
    assert bool(torch.all(fin == 0.0))
    ssd.s6_forward(u[:0], f[:0], v, a, bc[:0], bc[:0], v)
    torch.cuda.synchronize()
