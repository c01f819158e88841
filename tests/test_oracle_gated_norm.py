"""Pins of the oracle's gated RMSNorm, norm(y * silu(z)) * w (no GPU needed).

None of them re-derives the norm:
  * the RMSNorm identity: with unit weight, the mean square of each group's
    output is m / (m + eps), m the group's mean square in;
  * exact homogeneity at eps = 0: scaling the input by a power of two leaves
    the output unchanged bit for bit;
  * groups are independent: a group's output equals that group run alone as a
    one-group row with its slice of the weight, bit for bit;
  * the weight is per channel: a one-hot weight keeps one channel only.
"""
import numpy as np
import pytest

import oracle


def _gated(seed, rows=6, d=48):
    return np.random.default_rng(seed).standard_normal((rows, d)) * 3.0


def check_gated_norm(lib=None):
    """Names of the failing checks (used by the mutant battery too)."""
    bad = []
    g = _gated(1)
    for group in (48, 12):
        o = oracle.gated_norm(g, group=group, lib=lib)
        m = np.mean(g.reshape(6, -1, group) ** 2, axis=2)
        got = np.mean(o.reshape(6, -1, group) ** 2, axis=2)
        if not np.allclose(got, m / (m + 1e-5), rtol=1e-13, atol=0):
            bad.append("identity_group%d" % group)
    w = (1.0 + 0.5 * np.random.default_rng(2).standard_normal(48)).astype(np.float32)
    full = oracle.gated_norm(g, w, group=12, lib=lib)
    for j in range(4):
        alone = oracle.gated_norm(g[:, 12 * j:12 * (j + 1)], w[12 * j:12 * (j + 1)], lib=lib)
        if not np.array_equal(full[:, 12 * j:12 * (j + 1)], alone):
            bad.append("group_%d_alone" % j)
    a = oracle.gated_norm(g, w, group=12, eps=0.0, lib=lib)
    b = oracle.gated_norm(g * 2.0 ** 20, w, group=12, eps=0.0, lib=lib)
    if not np.array_equal(a, b):
        bad.append("homogeneity")
    onehot = np.zeros(48, np.float32)
    onehot[17] = 1.0
    o = oracle.gated_norm(g, onehot, lib=lib)
    keep = np.zeros(48, bool)
    keep[17] = True
    if not (np.all(o[:, ~keep] == 0.0) and np.all(o[:, 17] != 0.0)):
        bad.append("one_hot_weight")
    return bad


def test_gated_norm_pins(oracle_mod):
    assert check_gated_norm() == []


def test_gated_norm_of_the_forward_output(oracle_mod):
    """The step after the scan composes with forward: rows are tokens, the
    channel axis is d_inner = heads x headdim."""
    from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs
    w = WORKLOADS["tiny_fp32"].with_(seqlen=40)
    inp = make_inputs(w)
    out = oracle.forward(w.dims(), inp, final=False)["out"]
    o = oracle.gated_norm(out)
    m = np.mean(out ** 2, axis=-1)
    np.testing.assert_allclose(np.mean(o ** 2, axis=-1), m / (m + 1e-5), rtol=1e-13)


def test_gated_norm_refuses_bad_groups(oracle_mod):
    with pytest.raises(ValueError):
        oracle.gated_norm(_gated(3), group=7)
    with pytest.raises(ValueError):
        oracle.gated_norm(_gated(3), eps=-1.0)
