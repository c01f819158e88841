"""The binding's own checks, which need no GPU: before any call reaches the C
ABI (which sees bare pointers), every tensor must hold at least the elements
the call touches, and activation tensors must have the handle's channel
count.  A short tensor is refused by name instead of being read past its end
on the device."""
import pytest
import torch

from selective_state_space_forward_b200 import ssd

DIMS = dict(nheads=4, headdim=8, dstate=16, ngroups=2, dconv=4, a_per_token=False)


def _tensors(batch=2, seqlen=10, dims=DIMS, state_bytes=4096):
    H, P, N, G = dims["nheads"], dims["headdim"], dims["dstate"], dims["ngroups"]
    cd = H * P + 2 * G * N
    z = lambda *s, dt=torch.float32: torch.zeros(*s, dtype=dt)   # noqa: E731
    return dict(x=z(batch, seqlen, H * P), z=z(batch, seqlen, H * P), out=z(batch, seqlen, H * P),
                B=z(batch, seqlen, G * N), C=z(batch, seqlen, G * N), dt_raw=z(batch, seqlen, H),
                dt_bias=z(H), D=z(H),
                A=z(batch, seqlen, H) if dims.get("a_per_token") else z(H),
                conv_w=z(cd, 4), conv_b=z(cd), seq_idx=z(batch, seqlen, dt=torch.int32),
                lengths=z(batch, dt=torch.int32), init_state=z(state_bytes, dt=torch.uint8),
                final_state=z(state_bytes, dt=torch.uint8))


def test_exact_sizes_pass():
    ssd.check_forward_sizes(DIMS, 2, 10, 4096, **_tensors())
    ssd.check_forward_sizes(dict(DIMS, a_per_token=True), 2, 10, 4096,
                            **_tensors(dims=dict(DIMS, a_per_token=True)))
    # empty calls touch nothing
    ssd.check_forward_sizes(DIMS, 0, 10, 0, **_tensors(batch=0))
    ssd.check_forward_sizes(DIMS, 2, 0, 4096, **_tensors(seqlen=0))


@pytest.mark.parametrize("name", ["x", "z", "out", "B", "C", "dt_raw", "dt_bias", "D", "A",
                                  "conv_w", "conv_b", "seq_idx", "lengths", "init_state",
                                  "final_state"])
def test_a_short_tensor_is_refused_by_name(name):
    t = _tensors()
    t[name] = t[name].reshape(-1)[:-1]
    with pytest.raises(ValueError, match=name):
        ssd.check_forward_sizes(DIMS, 2, 10, 4096, **t)


def test_per_token_A_needs_a_value_per_token():
    t = _tensors()                       # per-head A: (H,)
    with pytest.raises(ValueError, match="A"):
        ssd.check_forward_sizes(dict(DIMS, a_per_token=True), 2, 10, 4096, **t)


def test_conv_tensors_are_not_sized_without_conv():
    t = _tensors()
    t["conv_w"] = t["conv_b"] = torch.zeros(1)
    ssd.check_forward_sizes(dict(DIMS, dconv=1), 2, 10, 4096, **t)


def test_activation_rank_and_channels():
    assert ssd._rows(torch.zeros(3, 5, 32), 32, "x") == (3, 5)
    assert ssd._rows(torch.zeros(0, 5, 32), 32, "x") == (0, 5)
    with pytest.raises(ValueError, match=r"x must be \(batch, seqlen, 32\)"):
        ssd._rows(torch.zeros(5, 32), 32, "x")
    with pytest.raises(ValueError, match="x must be"):
        ssd._rows(torch.zeros(3, 5, 33), 32, "x")


def test_state_bytes_layout():
    # fp32 SSM state, the conv history at the next 256-byte boundary, rounded to 256
    H, P, N, G = 4, 8, 16, 2
    ssm = 3 * H * P * N * 4                      # 6144, already a multiple of 256
    conv = 3 * 3 * (H * P + 2 * G * N) * 2       # 1728 bytes of bf16 history
    assert ssd.state_bytes_for(H, P, N, G, 4, "bf16", 3) == ((ssm + conv + 255) // 256) * 256
    assert ssd.state_bytes_for(H, P, N, G, 1, "bf16", 3) == ssm
    assert ssd.state_bytes_for(1, 8, 8, 1, 1, "f32", 1) == 256


def test_s6_sizes():
    kw = dict(delta=torch.zeros(2, 7, 5), delta_bias=torch.zeros(5), B=torch.zeros(2, 7, 8),
              C=torch.zeros(2, 7, 8), D=torch.zeros(5), z=torch.zeros(2, 7, 5),
              init_state=torch.zeros(2, 5, 8), out=torch.zeros(2, 7, 5),
              final_state=torch.zeros(2, 5, 8))
    ssd.check_s6_sizes(2, 7, 5, 8, **kw)
    for name in kw:
        bad = dict(kw)
        bad[name] = kw[name].reshape(-1)[:-1]
        with pytest.raises(ValueError, match=name):
            ssd.check_s6_sizes(2, 7, 5, 8, **bad)
