"""Helpers of the GPU parity tests: upload a workload, run it through the
C-ABI binding, and compare with the oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

from selective_state_space_forward_b200 import ssd
from selective_state_space_forward_b200.synthetic import Workload

# Tolerances on the gated output and the final state, against the fp64 oracle
# fed the same bf16-rounded inputs: relative L2 and max-abs as a fraction of
# the largest reference magnitude.
TOL = {"bf16": dict(rel_l2=5e-3, max_abs=2e-2), "f32": dict(rel_l2=1e-5, max_abs=1e-4)}

ACT_KEYS = ("x", "z", "B", "C", "conv_w", "conv_b")
F32_KEYS = ("dt_raw", "dt_bias", "A", "D", "B_norm_w", "C_norm_w", "B_bias", "C_bias")


def to_device(inp: dict, w: Workload) -> dict:
    at = torch.bfloat16 if w.act_dtype == "bf16" else torch.float32
    d = {}
    for k in ACT_KEYS:
        d[k] = None if inp.get(k) is None else torch.from_numpy(
            np.ascontiguousarray(inp[k])).to(at).cuda()
    for k in F32_KEYS:
        d[k] = None if inp.get(k) is None else torch.from_numpy(
            np.ascontiguousarray(inp[k], dtype=np.float32)).cuda()
    d["seq_idx"] = None if inp.get("seq_idx") is None else torch.from_numpy(
        np.ascontiguousarray(inp["seq_idx"], dtype=np.int32)).cuda()
    return d


def make_handle(w: Workload, path="auto", max_batch=None, max_seqlen=None) -> ssd.Handle:
    return ssd.Handle(w.nheads, w.headdim, w.dstate, w.ngroups, w.dconv, w.act_dtype,
                      a_per_token=w.a_per_token, bc_norm=w.bc_norm,
                      max_batch=max_batch or w.batch, max_seqlen=max_seqlen or w.seqlen,
                      path=path)


def state_from_numpy(h: ssd.Handle, batch: int, ssm=None, conv=None) -> torch.Tensor:
    buf = h.new_state(batch)
    s, c = h.state_views(buf, batch)
    if ssm is not None:
        s.copy_(torch.from_numpy(np.ascontiguousarray(ssm, dtype=np.float32)))
    if conv is not None and c is not None:
        c.copy_(torch.from_numpy(np.ascontiguousarray(conv, dtype=np.float32)).to(c.dtype))
    return buf


def state_to_numpy(h: ssd.Handle, buf: torch.Tensor, batch: int):
    s, c = h.state_views(buf, batch)
    return (s.double().cpu().numpy(), None if c is None else c.double().cpu().numpy())


def run_forward(h: ssd.Handle, w: Workload, dev: dict, init: torch.Tensor | None = None,
                final: bool = True, batch=None, seqlen=None):
    """Forward through the C ABI.  Returns (out f64, final ssm f64, final conv f64, final buf)."""
    if w.bc_norm:
        h.set_bc_norm(dev["B_norm_w"], dev["C_norm_w"], dev["B_bias"], dev["C_bias"])
    fin = h.new_state(w.batch) if final else None
    out = h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"],
                    dev["C"], dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"],
                    init_state=init, final_state=fin)
    torch.cuda.synchronize()
    h.check()
    o = out.double().cpu().numpy()
    if not final:
        return o, None, None, None
    s, c = state_to_numpy(h, fin, w.batch)
    return o, s, c, fin


def init_state_of(h: ssd.Handle, w: Workload, inp: dict):
    if inp.get("init_ssm") is None and inp.get("init_conv") is None:
        return None
    return state_from_numpy(h, w.batch, inp.get("init_ssm"), inp.get("init_conv"))


def errors(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    den = max(float(np.linalg.norm(want)), 1e-300)
    rel_l2 = float(np.linalg.norm(got - want)) / den
    max_abs = float(np.max(np.abs(got - want))) / max(float(np.max(np.abs(want))), 1e-300)
    return rel_l2, max_abs


def assert_close(got, want, act_dtype: str, what: str = ""):
    rel_l2, max_abs = errors(got, want)
    tol = TOL[act_dtype]
    assert rel_l2 <= tol["rel_l2"] and max_abs <= tol["max_abs"], (
        f"{what}: rel_l2={rel_l2:.3e} (tol {tol['rel_l2']:.0e}), "
        f"max_abs/max|ref|={max_abs:.3e} (tol {tol['max_abs']:.0e})")
    return rel_l2, max_abs
