"""GPU parity of ssd_backward (the vector-Jacobian product of a zero-state
prefill, mojolearn Mamba3Block method "backward") against the fp64 oracle.

Every gradient is compared element by element with oracle.backward on the
same bf16-rounded inputs and the same output gradient: relative L2 <= 5e-3 and
max-abs <= 2e-2 * max|ref| for bf16 activations, relative L2 <= 1e-5 for the
fp32 case (the backward computes in fp32 throughout).  The model card's gate
("Checkpoint and training"): a loss on one packed document gives exactly 0.0
gradient on every other document's tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, make_handle, to_device
from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs, make_output_grad

pytestmark = pytest.mark.gpu

TOKEN_GRADS = ("x", "z", "B", "C", "dt_raw")


def _docs_row(L, cuts):
    s = np.zeros(L, dtype=np.int32)
    for c in cuts:
        if 0 < c < L:
            s[c:] += 1
    return s


def _gout(w, seed):
    return make_output_grad(w, seed)


def _run(w, inp, gout, lengths=None):
    h = make_handle(w, "auto")
    dev = to_device(inp, w)
    if w.bc_norm:
        h.set_bc_norm(dev["B_norm_w"], dev["C_norm_w"], dev["B_bias"], dev["C_bias"])
    at = torch.bfloat16 if w.act_dtype == "bf16" else torch.float32
    g = h.backward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"],
                   dev["C"], dev["D"], dev["conv_w"], dev["conv_b"],
                   gout=torch.from_numpy(np.ascontiguousarray(gout)).to(at).cuda(),
                   seq_idx=dev["seq_idx"],
                   lengths=None if lengths is None else torch.from_numpy(lengths).cuda())
    torch.cuda.synchronize()
    h.check()
    return {k: v.double().cpu().numpy() for k, v in g.items()}, h


def _compare(got, want, dtype, what):
    tol = TOL[dtype]
    for k, ref in want.items():
        if ref is None:
            continue
        g = got[k]
        assert g.shape == ref.shape, (k, g.shape, ref.shape)
        assert np.all(np.isfinite(g)), f"{what}: non-finite values in d{k}"
        scale = max(float(np.max(np.abs(ref))), 1e-30)
        den = max(float(np.linalg.norm(ref)), 1e-30)
        rel = float(np.linalg.norm(g - ref)) / den
        mx = float(np.max(np.abs(g - ref))) / scale
        assert rel <= tol["rel_l2"] and mx <= tol["max_abs"], (
            f"{what} d{k}: rel_l2={rel:.3e}, max_abs/max|ref|={mx:.3e}")


SMALL = {
    # packed documents with boundaries on and beside chunk edges, conv, G < H
    "mini_k3_mixer": WORKLOADS["mini_k3_mixer"].with_(batch=2, seqlen=200, mean_doc_len=60),
    # per-token A (with floored values), B/C norm + per-head bias, no conv, N 128
    "mamba3_siso": WORKLOADS["mamba3_siso"].with_(batch=2, seqlen=150, nheads=8, ngroups=2),
    # N 128 with the conv, one document, a ragged last chunk
    "long_7b": WORKLOADS["long_7b"].with_(batch=1, seqlen=170, nheads=16, init_state=False),
    # fp32, no conv
    "tiny_fp32": WORKLOADS["tiny_fp32"],
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_backward_matches_oracle(name):
    w = SMALL[name]
    inp = make_inputs(w)
    if name == "mini_k3_mixer":
        inp["seq_idx"][0] = _docs_row(w.seqlen, [1, 63, 64, 65, 130, w.seqlen - 1])
    if name == "mamba3_siso":
        inp["A"][0, 3:7, 2] = np.array([0.0, -1e-6, -1e-4, -2.0], dtype=np.float32)
        rng = np.random.Generator(np.random.PCG64(17))
        inp["B_norm_w"] = (1.0 + 0.3 * rng.standard_normal(w.dstate)).astype(np.float32)
        inp["C_norm_w"] = (1.0 + 0.3 * rng.standard_normal(w.dstate)).astype(np.float32)
    gout = _gout(w, 100)
    want = oracle.backward(w.dims(), inp, gout)
    got, _ = _run(w, inp, gout)
    _compare(got, want, w.act_dtype, name)


def test_backward_ragged_rows():
    """Ragged lengths: padding tokens take exactly zero gradient, real ones match."""
    w = WORKLOADS["mini_k3_mixer"].with_(batch=3, seqlen=150, nheads=8, ngroups=2,
                                         mean_doc_len=50)
    inp = make_inputs(w)
    lengths = np.array([150, 64, 0], dtype=np.int32)
    gout = _gout(w, 101)
    want = oracle.backward(w.dims(), dict(inp, lengths=lengths), gout)
    got, _ = _run(w, inp, gout, lengths=lengths)
    _compare(got, want, "bf16", "ragged")
    for b, L in enumerate(lengths):
        for k in TOKEN_GRADS:
            assert np.all(got[k][b, L:] == 0.0), f"row {b}: d{k} on padding"


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_document_gate_exact_zero(seed):
    """A loss on one document only: every other document's token gradients are
    exactly 0.0 (model card, "Checkpoint and training")."""
    w = WORKLOADS["mini_k3_mixer"].with_(batch=1, seqlen=260, documents="none", seed=50 + seed)
    inp = make_inputs(w)
    seq = _docs_row(w.seqlen, [1, 63, 64, 65, 128, 200, 259])[None]
    inp["seq_idx"] = seq
    ndoc = int(seq.max()) + 1
    for k in range(ndoc):
        gout = _gout(w, 200 + k)
        gout[0, seq[0] != k] = 0.0
        got, _ = _run(w, inp, gout)
        other = seq[0] != k
        for key in TOKEN_GRADS:
            assert np.all(got[key][0, other] == 0.0), (k, key)
        assert np.any(got["x"][0, ~other] != 0.0), k


def test_backward_repeats_bit_for_bit():
    w = SMALL["mamba3_siso"]
    inp = make_inputs(w, seed=9)
    gout = _gout(w, 102)
    a, _ = _run(w, inp, gout)
    b, _ = _run(w, inp, gout)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_backward_mini_k3_mixer_shapes_long_rows():
    """The mini_k3_mixer layer (32 heads x 64, d_state 64, 8 groups, conv 4, packed
    documents) over 2 rows of 4096 tokens: every gradient against the oracle."""
    w = WORKLOADS["mini_k3_mixer"].with_(batch=2, seqlen=4096)
    inp = make_inputs(w)
    gout = _gout(w, 103)
    want = oracle.backward(w.dims(), inp, gout)
    got, _ = _run(w, inp, gout)
    _compare(got, want, "bf16", "mini_k3_mixer 2x4096")
