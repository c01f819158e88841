"""CPU fp64 oracle of the SSD mixer scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it, and it
never loads the CUDA library: the two share no code.

The arithmetic lives in ``ssd_oracle.c`` (plain sequential recurrence in
double precision, one (batch, head) pair per thread); this module only builds
that file with gcc and passes numpy arrays to it through ctypes.  What the C
code computes, and which page passage each step follows, is written at the
top of ``ssd_oracle.c``.

A decode step is ``forward`` at ``seqlen == 1`` with the carried state as the
initial state ("the same computation as forward at L = 1", mojolearn
Mamba3Block.step).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libssd_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile ssd_oracle.c (or another copy of it) into a shared library."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
             "-ffp-contract=off", src, "-o", tmp, "-lm"])
        os.replace(tmp, out)
    return out


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "dconv",
        "a_per_token", "bc_norm")]


_FP = ctypes.POINTER(ctypes.c_float)


class _Inputs(ctypes.Structure):
    _fields_ = [(n, _FP) for n in (
        "x", "z", "Bm", "Cm", "dt_raw", "dt_bias", "A", "D", "conv_w", "conv_b")] + [
        ("seq_idx", ctypes.POINTER(ctypes.c_int32))] + [
        (n, _FP) for n in ("init_ssm", "init_conv", "bn_w", "cn_w", "bn_bias", "cn_bias")] + [
        ("lengths", ctypes.POINTER(ctypes.c_int32))]


class _S6Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("batch", "seqlen", "d_inner", "dstate")]


class _S6Inputs(ctypes.Structure):
    _fields_ = [(n, _FP) for n in ("u", "delta", "delta_bias", "A_log", "Bm", "Cm", "D", "z",
                                   "init")]


class _Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.POINTER(ctypes.c_double)) for n in (
        "x", "z", "Bm", "Cm", "dt_raw", "dt_bias", "A", "D", "conv_w", "conv_b",
        "bn_w", "cn_w", "bn_bias", "cn_bias")]


def _bind(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_forward.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Inputs),
                                   ctypes.POINTER(ctypes.c_int32), ctypes.c_int,
                                   ctypes.c_int, dp, dp, dp]
    lib.oracle_forward.restype = ctypes.c_int
    lib.oracle_conv.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Inputs), dp]
    lib.oracle_conv.restype = ctypes.c_int
    lib.oracle_dt.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Inputs), dp, dp]
    lib.oracle_dt.restype = ctypes.c_int
    lib.oracle_bcnorm.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Inputs), dp, dp]
    lib.oracle_bcnorm.restype = ctypes.c_int
    lib.oracle_default_threads.restype = ctypes.c_int
    lib.oracle_s6_forward.argtypes = [ctypes.POINTER(_S6Dims), ctypes.POINTER(_S6Inputs),
                                      ctypes.c_int, dp, dp]
    lib.oracle_s6_forward.restype = ctypes.c_int
    lib.oracle_backward.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Inputs), _FP,
                                    ctypes.c_int, ctypes.POINTER(_Grads)]
    lib.oracle_backward.restype = ctypes.c_int
    lib.oracle_gated_norm.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                      dp, _FP, dp]
    lib.oracle_gated_norm.restype = ctypes.c_int
    return lib


def _load(lib=None):
    """The default oracle library, or `lib` when a test passes a variant build."""
    global _lib
    if lib is not None:
        return lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def load_variant(path: str):
    """Bind another build of ssd_oracle.c (used by tests that plant mistakes)."""
    return _bind(path)


def default_threads() -> int:
    return int(_load().oracle_default_threads())


def _f32(a, keep):
    if a is None:
        return None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    keep.append(a)
    return a.ctypes.data_as(_FP)


def _marshal(dims: dict, inp: dict):
    d = _Dims(batch=dims["batch"], seqlen=dims["seqlen"], nheads=dims["nheads"],
              headdim=dims["headdim"], dstate=dims["dstate"], ngroups=dims["ngroups"],
              dconv=dims.get("dconv", 1), a_per_token=int(dims.get("a_per_token", 0)),
              bc_norm=int(dims.get("bc_norm", 0)))
    keep = []
    seq = inp.get("seq_idx")
    if seq is not None:
        seq = np.ascontiguousarray(np.asarray(seq, dtype=np.int32))
        keep.append(seq)
    lens = inp.get("lengths")
    if lens is not None:
        lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32))
        keep.append(lens)
    i = _Inputs(
        x=_f32(inp["x"], keep), z=_f32(inp["z"], keep), Bm=_f32(inp["B"], keep),
        Cm=_f32(inp["C"], keep), dt_raw=_f32(inp["dt_raw"], keep),
        dt_bias=_f32(inp["dt_bias"], keep), A=_f32(inp["A"], keep), D=_f32(inp["D"], keep),
        conv_w=_f32(inp.get("conv_w"), keep), conv_b=_f32(inp.get("conv_b"), keep),
        seq_idx=seq.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) if seq is not None else None,
        init_ssm=_f32(inp.get("init_ssm"), keep), init_conv=_f32(inp.get("init_conv"), keep),
        bn_w=_f32(inp.get("B_norm_w"), keep), cn_w=_f32(inp.get("C_norm_w"), keep),
        bn_bias=_f32(inp.get("B_bias"), keep), cn_bias=_f32(inp.get("C_bias"), keep),
        lengths=lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) if lens is not None else None)
    return d, i, keep


def _dptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if a is not None else None


def forward(dims: dict, inp: dict, pairs=None, threads: int = 0, final: bool = True,
            lib=None) -> dict:
    """Run the sequential fp64 recurrence.

    dims: batch, seqlen, nheads, headdim, dstate, ngroups, dconv (1 = no conv),
    a_per_token, bc_norm.  inp: numpy arrays named x, z, B, C, dt_raw, dt_bias,
    A, D, conv_w, conv_b, seq_idx, init_ssm, init_conv, B_norm_w, C_norm_w,
    B_bias, C_bias (missing optional ones = None).  pairs: iterable of (b, h) to
    compute (others stay NaN), or None for all.

    Returns {"out": (batch, seqlen, H*P) f64, "final_ssm": (batch, H, P, N) f64,
    "final_conv": (batch, dconv-1, conv_dim) f64 or None, "threads": int}.
    """
    lib = _load(lib)
    d, i, keep = _marshal(dims, inp)
    Bb, L, H, P, N, G, K = (dims["batch"], dims["seqlen"], dims["nheads"], dims["headdim"],
                            dims["dstate"], dims["ngroups"], dims.get("dconv", 1))
    out = np.full((Bb, L, H * P), np.nan)
    fin = np.full((Bb, H, P, N), np.nan) if final else None
    fconv = np.zeros((Bb, K - 1, H * P + 2 * G * N)) if (final and K > 1) else None
    parr, npairs = None, 0
    if pairs is not None:
        pl = np.ascontiguousarray(np.asarray(list(pairs), dtype=np.int32).reshape(-1, 2))
        keep.append(pl)
        parr, npairs = pl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), pl.shape[0]
    nt = lib.oracle_forward(ctypes.byref(d), ctypes.byref(i), parr, npairs, int(threads),
                            _dptr(out), _dptr(fin), _dptr(fconv))
    if nt < 0:
        raise ValueError("oracle_forward rejected its arguments")
    return {"out": out, "final_ssm": fin, "final_conv": fconv, "threads": nt}


def conv_stage(dims: dict, inp: dict, lib=None) -> np.ndarray:
    """conv+SiLU output of every x|B|C channel, (batch, seqlen, conv_dim) f64."""
    lib = _load(lib)
    d, i, keep = _marshal(dims, inp)
    cd = dims["nheads"] * dims["headdim"] + 2 * dims["ngroups"] * dims["dstate"]
    u = np.empty((dims["batch"], dims["seqlen"], cd))
    if lib.oracle_conv(ctypes.byref(d), ctypes.byref(i), _dptr(u)) != 0:
        raise ValueError("oracle_conv rejected its arguments")
    return u


def dt_stage(dims: dict, inp: dict, lib=None):
    """(dt, a): softplus(dt_raw + dt_bias) and the (floored) decay rate, (batch, seqlen, H) f64."""
    lib = _load(lib)
    d, i, keep = _marshal(dims, inp)
    shape = (dims["batch"], dims["seqlen"], dims["nheads"])
    dt, a = np.empty(shape), np.empty(shape)
    if lib.oracle_dt(ctypes.byref(d), ctypes.byref(i), _dptr(dt), _dptr(a)) != 0:
        raise ValueError("oracle_dt rejected its arguments")
    return dt, a


def bcnorm_stage(dims: dict, inp: dict, lib=None):
    """(B_hat, C_hat): per-head RMSNorm(B)*w + bias, (batch, seqlen, H, N) f64 each."""
    lib = _load(lib)
    d, i, keep = _marshal(dims, inp)
    shape = (dims["batch"], dims["seqlen"], dims["nheads"], dims["dstate"])
    bh, ch = np.empty(shape), np.empty(shape)
    if lib.oracle_bcnorm(ctypes.byref(d), ctypes.byref(i), _dptr(bh), _dptr(ch)) != 0:
        raise ValueError("oracle_bcnorm rejected its arguments")
    return bh, ch


def step(dims: dict, inp: dict, state_ssm, state_conv, threads: int = 0, lib=None) -> dict:
    """One decode token per row: forward at seqlen 1 from the carried state.

    inp holds (batch, 1, ...) arrays; returns out (batch, 1, H*P) and the new
    state (final_ssm, final_conv).
    """
    d = dict(dims)
    d["seqlen"] = 1
    i = dict(inp)
    i["seq_idx"] = None
    i["init_ssm"] = state_ssm
    i["init_conv"] = state_conv
    return forward(d, i, threads=threads, lib=lib)


def s6_forward(inp: dict, threads: int = 0, lib=None) -> dict:
    """The Mamba-1 selective scan (S6), sequential fp64.

    inp: numpy arrays u, delta, z (batch, seqlen, d_inner; z may be None), B, C
    (batch, seqlen, dstate), A_log (d_inner, dstate), delta_bias, D (d_inner),
    init (batch, d_inner, dstate) or None.  Returns {"out": (batch, seqlen,
    d_inner) f64, "final": (batch, d_inner, dstate) f64}.
    """
    lib = _load(lib)
    Bb, L, DI = inp["u"].shape
    N = inp["B"].shape[2]
    keep = []
    d = _S6Dims(batch=Bb, seqlen=L, d_inner=DI, dstate=N)
    i = _S6Inputs(u=_f32(inp["u"], keep), delta=_f32(inp["delta"], keep),
                  delta_bias=_f32(inp["delta_bias"], keep), A_log=_f32(inp["A_log"], keep),
                  Bm=_f32(inp["B"], keep), Cm=_f32(inp["C"], keep), D=_f32(inp["D"], keep),
                  z=_f32(inp.get("z"), keep), init=_f32(inp.get("init"), keep))
    out = np.full((Bb, L, DI), np.nan)
    fin = np.full((Bb, DI, N), np.nan)
    if lib.oracle_s6_forward(ctypes.byref(d), ctypes.byref(i), int(threads), _dptr(out), _dptr(fin)) < 0:
        raise ValueError("oracle_s6_forward rejected its arguments")
    return {"out": out, "final": fin}


def backward(dims: dict, inp: dict, gout, threads: int = 0, lib=None) -> dict:
    """Gradients of a zero-state prefill (the vector-Jacobian product of forward).

    dims / inp as for ``forward`` (init_ssm and init_conv must be None); gout is
    the gradient of the loss with respect to ``out``, (batch, seqlen, H*P).
    Returns float64 gradients under the input names: x, z, B, C, dt_raw,
    dt_bias, A, D, and conv_w, conv_b (with a conv) and B_norm_w, C_norm_w,
    B_bias, C_bias (with the B/C norm); the others are None.
    """
    lib = _load(lib)
    if inp.get("init_ssm") is not None or inp.get("init_conv") is not None:
        raise ValueError("backward is defined for a zero-state prefill only")
    d, i, keep = _marshal(dims, inp)
    Bb, L, H, P, N, G, K = (dims["batch"], dims["seqlen"], dims["nheads"], dims["headdim"],
                            dims["dstate"], dims["ngroups"], dims.get("dconv", 1))
    cd = H * P + 2 * G * N
    norm = bool(dims.get("bc_norm"))
    g = {
        "x": np.zeros((Bb, L, H * P)), "z": np.zeros((Bb, L, H * P)),
        "B": np.zeros((Bb, L, G * N)), "C": np.zeros((Bb, L, G * N)),
        "dt_raw": np.zeros((Bb, L, H)), "dt_bias": np.zeros(H),
        "A": np.zeros((Bb, L, H) if dims.get("a_per_token") else H), "D": np.zeros(H),
        "conv_w": np.zeros((cd, K)) if K > 1 else None, "conv_b": np.zeros(cd) if K > 1 else None,
        "B_norm_w": np.zeros(N) if norm else None, "C_norm_w": np.zeros(N) if norm else None,
        "B_bias": np.zeros((H, N)) if norm else None, "C_bias": np.zeros((H, N)) if norm else None,
    }
    gr = _Grads(x=_dptr(g["x"]), z=_dptr(g["z"]), Bm=_dptr(g["B"]), Cm=_dptr(g["C"]),
                dt_raw=_dptr(g["dt_raw"]), dt_bias=_dptr(g["dt_bias"]), A=_dptr(g["A"]),
                D=_dptr(g["D"]), conv_w=_dptr(g["conv_w"]), conv_b=_dptr(g["conv_b"]),
                bn_w=_dptr(g["B_norm_w"]), cn_w=_dptr(g["C_norm_w"]),
                bn_bias=_dptr(g["B_bias"]), cn_bias=_dptr(g["C_bias"]))
    go = _f32(gout, keep)
    if lib.oracle_backward(ctypes.byref(d), ctypes.byref(i), go, int(threads), ctypes.byref(gr)) < 0:
        raise ValueError("oracle_backward rejected its arguments")
    return g


def gated_norm(gated, weight=None, group: int | None = None, eps: float = 1e-5, lib=None):
    """RMSNorm of the gated scan output (``forward``'s out = y * silu(z)) times
    the per-channel weight: upstream Mamba-2's norm(y * silu(z)).

    gated: (..., d_inner) float64; weight: (d_inner) or None (ones); group:
    channels per norm group (default d_inner, one norm per token).
    """
    lib = _load(lib)
    g = np.ascontiguousarray(np.asarray(gated, dtype=np.float64))
    d_inner = g.shape[-1]
    rows = g.size // d_inner if d_inner else 0
    keep = []
    out = np.empty_like(g)
    rc = lib.oracle_gated_norm(int(rows), int(d_inner), int(group or d_inner), float(eps),
                               _dptr(g), _f32(weight, keep), _dptr(out))
    if rc != 0:
        raise ValueError("oracle_gated_norm rejected its arguments")
    return out
