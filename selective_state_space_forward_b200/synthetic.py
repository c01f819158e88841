"""Seeded synthetic workloads for the SSD mixer scan.

This module only draws numbers: it holds none of the scan's arithmetic, and
both the CUDA path's tests/bench and the CPU oracle take their inputs from it.

Shapes follow the pages' models:
  * ``tiny_fp32``      a small fp32 parity case (1 x 256 tokens, 4 heads x 16,
                       d_state 16, 1 group, no conv).
  * ``mini_k3_mixer``  the Mamba-2 mixer of the 1024-wide Mini-K3-1H hybrid
                       (model card, Architecture: 32 heads x 64, d_state 64,
                       B/C groups 8, conv kernel 4; Checkpoint and training:
                       sequence 8192, local batch 5, packed documents).
  * ``mamba3_siso``    a Mamba-3 SISO scan sized like the 2.8B transplant
                       (d_inner 5120 = 80 heads x 64, d_state 128, 1 group; the
                       mojolearn Mamba3Block fixes head dim 64, d_state 128, one
                       group, B/C RMSNorm + per-head bias, A floor 1e-4).
  * ``long_7b``        a 7B-class Mamba-2 layer at 16K context (128 heads x 64,
                       d_state 128, 8 groups, conv 4) with a nonzero initial state.
  * ``decode_b256``    single-token decode, batch 256, on the mini_k3_mixer
                       shapes, continued from a 2048-token prefill.

Value recipe (every workload): x, z, B, C ~ N(0, 1); dt_raw ~ N(0, 1);
dt_bias = log(expm1(u)) with u log-uniform on [1e-3, 1e-1] (the inverse
softplus of the transplant article, so softplus(dt_bias) = u); per-head
A = -exp(A_log) with A_log = log(U[1, 16]); D ~ U[0, 1]; conv weight and bias
~ N(0, 0.5).  Activation tensors (x, z, B, C, conv weights) are drawn in fp64
and rounded to the activation dtype (bf16 round-to-nearest-even, via fp32);
dt_raw, dt_bias, A, D and states are fp32 ("Mamba control parameters: FP32",
model card).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    dconv: int            # 1 = no conv
    act_dtype: str        # "f32" | "bf16"
    a_per_token: bool = False
    bc_norm: bool = False
    documents: str = "none"   # "none" | "geometric"
    mean_doc_len: int = 1500
    init_state: bool = False
    seed: int = 0
    decode_steps: int = 0     # > 0: seqlen is the prefill, then this many single-token steps

    @property
    def conv_dim(self) -> int:
        return self.nheads * self.headdim + 2 * self.ngroups * self.dstate

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def dims(self) -> dict:
        """The shape/switch dict both the oracle and the binding accept."""
        return dict(batch=self.batch, seqlen=self.seqlen, nheads=self.nheads,
                    headdim=self.headdim, dstate=self.dstate, ngroups=self.ngroups,
                    dconv=self.dconv, a_per_token=int(self.a_per_token),
                    bc_norm=int(self.bc_norm))

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 256, 4, 16, 16, 1, 1, "f32", seed=0),
    "mini_k3_mixer": Workload("mini_k3_mixer", 5, 8192, 32, 64, 64, 8, 4, "bf16",
                              documents="geometric", mean_doc_len=1500, seed=1),
    "mamba3_siso": Workload("mamba3_siso", 4, 4096, 80, 64, 128, 1, 1, "bf16",
                            a_per_token=True, bc_norm=True, seed=2),
    "long_7b": Workload("long_7b", 2, 16384, 128, 64, 128, 8, 4, "bf16",
                        init_state=True, seed=3),
    "decode_b256": Workload("decode_b256", 256, 2048, 32, 64, 64, 8, 4, "bf16",
                            seed=4, decode_steps=512),
}


def round_bf16(a) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as float32."""
    a32 = np.asarray(a, dtype=np.float32)
    shape = a32.shape
    bits = np.ascontiguousarray(a32).reshape(-1).view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32).reshape(shape)


def _act(w: Workload, a) -> np.ndarray:
    return round_bf16(a) if w.act_dtype == "bf16" else np.asarray(a, dtype=np.float32)


def document_ids(rng: np.random.Generator, batch: int, seqlen: int, mean_len: int) -> np.ndarray:
    """Packed documents: geometric lengths (support >= 1, mean mean_len), packed
    left to right in each row, the last one truncated; the id is the ordinal
    of the document within its row."""
    seq = np.empty((batch, seqlen), dtype=np.int32)
    for b in range(batch):
        t, k = 0, 0
        while t < seqlen:
            n = int(rng.geometric(1.0 / mean_len))
            seq[b, t:t + n] = k
            t += n
            k += 1
    return seq


def softplus_inverse(u) -> np.ndarray:
    """log(exp(u) - 1): the dt_bias parameterisation of the transplant article."""
    u = np.asarray(u, dtype=np.float64)
    return np.log(np.expm1(u))


def make_inputs(w: Workload, seed: int | None = None) -> dict:
    """Draw every input of one forward call of workload w.

    Returns numpy arrays: x, z (batch, seqlen, H*P); B, C (batch, seqlen, G*N);
    dt_raw (batch, seqlen, H); dt_bias, D (H); A (H) or (batch, seqlen, H);
    conv_w (conv_dim, dconv), conv_b (conv_dim) or None; seq_idx (batch,
    seqlen) int32 or None; init_ssm (batch, H, P, N) or None; init_conv
    (batch, dconv-1, conv_dim) or None; B_norm_w, C_norm_w (N), B_bias,
    C_bias (H, N) or None.  Float arrays are float32 holding exactly the
    values the device receives.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    Bb, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    out = {}
    out["x"] = _act(w, rng.standard_normal((Bb, L, H * P)))
    out["z"] = _act(w, rng.standard_normal((Bb, L, H * P)))
    out["B"] = _act(w, rng.standard_normal((Bb, L, G * N)))
    out["C"] = _act(w, rng.standard_normal((Bb, L, G * N)))
    out["dt_raw"] = rng.standard_normal((Bb, L, H)).astype(np.float32)
    u = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), H))
    out["dt_bias"] = softplus_inverse(u).astype(np.float32)
    if w.a_per_token:
        v = rng.standard_normal((Bb, L, H))
        sp = np.logaddexp(0.0, v)
        out["A"] = (-np.maximum(sp, 1e-4)).astype(np.float32)
    else:
        out["A"] = (-np.exp(np.log(rng.uniform(1.0, 16.0, H)))).astype(np.float32)
    out["D"] = rng.uniform(0.0, 1.0, H).astype(np.float32)
    if w.dconv > 1:
        out["conv_w"] = _act(w, 0.5 * rng.standard_normal((w.conv_dim, w.dconv)))
        out["conv_b"] = _act(w, 0.5 * rng.standard_normal(w.conv_dim))
    else:
        out["conv_w"] = out["conv_b"] = None
    out["seq_idx"] = (document_ids(rng, Bb, L, w.mean_doc_len)
                      if w.documents == "geometric" else None)
    out["init_ssm"] = (0.1 * rng.standard_normal((Bb, H, P, N))).astype(np.float32) \
        if w.init_state else None
    out["init_conv"] = None
    if w.bc_norm:
        out["B_norm_w"] = np.ones(N, dtype=np.float32)
        out["C_norm_w"] = np.ones(N, dtype=np.float32)
        out["B_bias"] = (0.02 * rng.standard_normal((H, N))).astype(np.float32)
        out["C_bias"] = (0.02 * rng.standard_normal((H, N))).astype(np.float32)
    else:
        out["B_norm_w"] = out["C_norm_w"] = out["B_bias"] = out["C_bias"] = None
    return out


def make_output_grad(w: Workload, seed: int) -> np.ndarray:
    """A seeded gradient of the loss with respect to `out` for the backward:
    N(0, 1) of shape (batch, seqlen, H*P), rounded to the activation dtype."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return _act(w, rng.standard_normal((w.batch, w.seqlen, w.nheads * w.headdim)))


def make_s6_inputs(batch: int, seqlen: int, d_inner: int, dstate: int, seed: int,
                   bf16: bool = True, gate: bool = True, init: bool = True) -> dict:
    """Seeded inputs of the Mamba-1 selective scan (S6): u, z, B, C ~ N(0, 1) in the
    activation dtype; delta ~ N(-2, 1); A_log = log U[1, dstate] per (channel,
    state); delta_bias ~ U[-2, 0]; D ~ U[0, 1]; initial state ~ N(0, 0.1).  z and
    the initial state are None when not asked for."""
    rng = np.random.Generator(np.random.PCG64(seed))
    act = round_bf16 if bf16 else (lambda a: np.asarray(a, dtype=np.float32))
    f = np.float32
    B, L, DI, N = batch, seqlen, d_inner, dstate
    return dict(u=act(rng.standard_normal((B, L, DI))),
                delta=(rng.standard_normal((B, L, DI)) - 2.0).astype(f),
                z=act(rng.standard_normal((B, L, DI))) if gate else None,
                B=act(rng.standard_normal((B, L, N))), C=act(rng.standard_normal((B, L, N))),
                A_log=np.log(rng.uniform(1.0, N, (DI, N))).astype(f),
                delta_bias=rng.uniform(-2.0, 0.0, DI).astype(f),
                D=rng.uniform(0.0, 1.0, DI).astype(f),
                init=(0.1 * rng.standard_normal((B, DI, N))).astype(f) if init else None)


def make_step_inputs(w: Workload, step: int, seed: int | None = None) -> dict:
    """Fresh draws for decode step `step` (same distributions, one token per row):
    x, z (batch, H*P); B, C (batch, G*N); dt_raw (batch, H); A (batch, H) when
    per token.  Parameters (dt_bias, A per head, D, conv weights) are those of
    make_inputs."""
    base = w.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64([base, 7919, step]))
    Bb, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    out = {
        "x": _act(w, rng.standard_normal((Bb, H * P))),
        "z": _act(w, rng.standard_normal((Bb, H * P))),
        "B": _act(w, rng.standard_normal((Bb, G * N))),
        "C": _act(w, rng.standard_normal((Bb, G * N))),
        "dt_raw": rng.standard_normal((Bb, H)).astype(np.float32),
    }
    if w.a_per_token:
        v = rng.standard_normal((Bb, H))
        out["A"] = (-np.maximum(np.logaddexp(0.0, v), 1e-4)).astype(np.float32)
    return out
