"""The forward on a caller's own stream and inside a captured CUDA graph.

The fused path forks its dt/cumsum kernel onto the handle's auxiliary stream
(an event from the caller's stream before it, an event back before the fused
kernel) and launches the fused kernel cooperatively; its segment hand-offs are
flags tagged with a per-call epoch.  The checks:

- on a side stream the forward gives the default stream's bits (fused and
  staged paths);
- captured once into a CUDA graph and replayed with new inputs copied into the
  captured buffers, every replay gives the bits of an eager call on the same
  inputs.  Alternating two input sets makes a replay that took the previous
  replay's hand-off flags for its own (the captured epoch is the same on every
  replay) read that replay's states and differ;
- the same with ragged rows (one full row, the rest a few tokens long), where
  CTAs reach a later segment of the full row while the segment before it is
  still running;
- ssd_forward_noalloc, captured and replayed the same way.
"""
import pytest
import torch

from gpu_util import init_state_of, make_handle, to_device
from selective_state_space_forward_b200 import ssd
from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

# More (row, head) streams than the persistent grid has CTAs (one per SM): the
# fused kernel then splits every stream into several segments to balance the
# last round of items, so the hand-off flags are in use.
CASES = {
    "mini_k3_mixer": WORKLOADS["mini_k3_mixer"].with_(batch=10, seqlen=700, mean_doc_len=300),
    "mamba3_siso": WORKLOADS["mamba3_siso"].with_(batch=4, seqlen=900),
    "long_7b": WORKLOADS["long_7b"].with_(batch=3, seqlen=1000),
}


def _same(a, b):
    """Bitwise equality (state buffers are bytes already)."""
    if a.dtype == torch.bfloat16:
        a, b = a.view(torch.int16), b.view(torch.int16)
    elif a.dtype == torch.float32:
        a, b = a.view(torch.int32), b.view(torch.int32)
    return torch.equal(a, b)


class _Call:
    """One forward's device buffers: inputs, init state, out and final state."""

    def __init__(self, h, w, seed, lengths=None):
        inp = make_inputs(w.with_(seed=seed))
        self.lengths = lengths
        self.dev = to_device(inp, w)
        self.init = init_state_of(h, w, inp)
        self.out = torch.empty_like(self.dev["x"])
        self.fin = h.new_state(w.batch)

    def copy_from(self, other):
        for k, v in self.dev.items():
            if v is not None:
                v.copy_(other.dev[k])
        if self.init is not None:
            self.init.copy_(other.init)

    def run(self, h):
        d = self.dev
        h.forward(d["x"], d["z"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                  d["conv_w"], d["conv_b"], seq_idx=d["seq_idx"], init_state=self.init,
                  out=self.out, final_state=self.fin, lengths=self.lengths)


def _handle(w, path):
    h = make_handle(w, path)
    if w.bc_norm:
        inp = make_inputs(w)
        dev = to_device(inp, w)
        h.set_bc_norm(dev["B_norm_w"], dev["C_norm_w"], dev["B_bias"], dev["C_bias"])
    return h


@pytest.mark.parametrize("path", ["fused", "staged"])
@pytest.mark.parametrize("name", ["mini_k3_mixer", "mamba3_siso"])
def test_side_stream_gives_the_default_streams_bits(name, path):
    w = CASES[name]
    h = _handle(w, path)
    ref = _Call(h, w, seed=11)
    ref.run(h)
    torch.cuda.synchronize()
    h.check()
    side = _Call(h, w, seed=11)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        side.run(h)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    h.check()
    assert _same(side.out, ref.out)
    assert _same(side.fin, ref.fin)


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):      # warm-up outside the graph
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


@pytest.mark.parametrize("path", ["fused", "staged"])
@pytest.mark.parametrize("name", ["mini_k3_mixer", "mamba3_siso", "long_7b"])
def test_graph_replays_match_eager_calls(name, path):
    w = CASES[name]
    h = _handle(w, path)
    eager = [_Call(h, w, seed=s) for s in (21, 22)]
    for c in eager:
        c.run(h)
    torch.cuda.synchronize()
    h.check()
    assert not _same(eager[0].out, eager[1].out)
    static = _Call(h, w, seed=21)
    g = _capture(lambda: static.run(h))
    for k in (1, 0, 1, 1, 0):
        static.copy_from(eager[k])
        g.replay()
        torch.cuda.synchronize()
        h.check()
        assert _same(static.out, eager[k].out), f"replay on input set {k}: out"
        assert _same(static.fin, eager[k].fin), f"replay on input set {k}: final state"
    del g


def test_graph_replays_with_ragged_rows():
    # Row 0 is full length, the others hold a few tokens: CTAs that finish the
    # short rows' items early start a later segment of row 0 while the segment
    # before it is still running, so each replay must wait for its own flags.
    w = CASES["mini_k3_mixer"]
    h = _handle(w, "fused")
    lens = torch.tensor([w.seqlen] + [5] * (w.batch - 1), dtype=torch.int32, device="cuda")
    eager = [_Call(h, w, seed=s, lengths=lens) for s in (41, 42)]
    for c in eager:
        c.run(h)
    torch.cuda.synchronize()
    h.check()
    static = _Call(h, w, seed=41, lengths=lens)
    g = _capture(lambda: static.run(h))
    for k in (1, 0, 1, 0):
        static.copy_from(eager[k])
        g.replay()
        torch.cuda.synchronize()
        h.check()
        assert _same(static.out[0], eager[k].out[0]), f"replay on input set {k}: row 0 out"
        assert _same(static.fin, eager[k].fin), f"replay on input set {k}: final state"
    del g


def _node_types(graph):
    """Types of a captured graph's nodes (cuda-python runtime bindings)."""
    from cuda.bindings import runtime as cr
    g = cr.cudaGraph_t(init_value=graph.raw_cuda_graph())
    err, _, n = cr.cudaGraphGetNodes(g)
    assert err == cr.cudaError_t.cudaSuccess
    err, nodes, n = cr.cudaGraphGetNodes(g, n)
    assert err == cr.cudaError_t.cudaSuccess
    types = []
    for node in nodes[:n]:
        err, t = cr.cudaGraphNodeGetType(node)
        assert err == cr.cudaError_t.cudaSuccess
        types.append(t)
    return cr, types


@pytest.mark.parametrize("path", ["fused", "staged"])
def test_captured_call_clears_the_handoff_flags(path):
    # Replays of one capture share its epoch, so a captured fused call must
    # clear its hand-off flags inside the graph: one memset node per fused
    # call, none on the staged path (which has no hand-offs).
    pytest.importorskip("cuda.bindings.runtime")
    w = CASES["mini_k3_mixer"]
    h = _handle(w, path)
    c = _Call(h, w, seed=51)
    c.run(h)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g):
        c.run(h)
    cr, types = _node_types(g)
    memsets = sum(t == cr.cudaGraphNodeType.cudaGraphNodeTypeMemset for t in types)
    kernels = sum(t == cr.cudaGraphNodeType.cudaGraphNodeTypeKernel for t in types)
    assert memsets == (1 if path == "fused" else 0), types
    assert kernels >= 3, types
    g.instantiate()
    g.replay()
    torch.cuda.synchronize()
    h.check()
    del g


def test_noalloc_graph_replays_match_eager_calls():
    w = CASES["mini_k3_mixer"]
    h = _handle(w, "fused")     # only for buffer sizes
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(c):
        d = c.dev
        ssd.forward_noalloc(d["x"], d["z"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"],
                            d["D"], d["conv_w"], d["conv_b"], seq_idx=d["seq_idx"],
                            init_state=c.init, out=c.out, final_state=c.fin, status=status,
                            nheads=w.nheads, headdim=w.headdim, dstate=w.dstate,
                            ngroups=w.ngroups, dconv=w.dconv, a_per_token=w.a_per_token)

    eager = [_Call(h, w, seed=s) for s in (31, 32)]
    for c in eager:
        run(c)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    static = _Call(h, w, seed=31)
    g = _capture(lambda: run(static))
    for k in (1, 0, 1):
        static.copy_from(eager[k])
        g.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert _same(static.out, eager[k].out), f"replay on input set {k}: out"
        assert _same(static.fin, eager[k].fin), f"replay on input set {k}: final state"
    del g
