"""ctypes binding of libssd.so (include/ssd.h): argument marshalling only.

Every step of the scan runs in the library's CUDA kernels; this module turns
torch tensors into device pointers and ssd_* status codes into exceptions.
It never computes on the host and has no fallback: if libssd.so is missing it
raises.

    h = Handle(nheads=32, headdim=64, dstate=64, ngroups=8, dconv=4,
               act_dtype="bf16", max_batch=5, max_seqlen=8192)
    out = h.forward(x, z, dt_raw, dt_bias, A, B, C, D, conv_w, conv_b, seq_idx=seq)
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd.so")

SSD_OK = 0
STATUS_NAMES = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED",
                3: "SSD_ERR_ALIGNMENT", 4: "SSD_ERR_SHAPE_EXCEEDS_MAX", 5: "SSD_ERR_CUDA",
                6: "SSD_ERR_DEVICE"}
PATHS = {"auto": 0, "fused": 1, "staged": 2}
PATH_NAMES = {1: "fused", 2: "staged"}
DTYPES = {"f32": (0, torch.float32), "bf16": (1, torch.bfloat16)}

# Every symbol include/ssd.h declares.
EXPORTS = ("ssd_create", "ssd_destroy", "ssd_get_path", "ssd_set_bc_norm", "ssd_state_bytes",
           "ssd_state_conv_offset", "ssd_forward", "ssd_step", "ssd_stage_conv", "ssd_stage_dt",
           "ssd_set_timing_events", "ssd_launch_count", "ssd_check", "ssd_last_error",
           "ssd_status_string", "ssd_forward_noalloc", "ssd_forward_ragged", "ssd_s6_forward",
           "ssd_backward_workspace_bytes", "ssd_backward", "ssd_set_gated_norm",
           "ssd_forward_packed", "ssd_ex2_throughput", "ssd_set_wait_test")


class SSDError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class Desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "nheads", "headdim", "dstate", "ngroups", "dconv", "chunk", "act_dtype", "a_mode",
        "bc_norm", "max_batch", "max_seqlen", "path", "validate_finite")]


class Grads(ctypes.Structure):
    """ssd_grads: device pointers of the backward's fp32 gradient outputs."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "x", "z", "B", "C", "dt_raw", "dt_bias", "A", "D", "conv_w", "conv_b", "B_norm_w",
        "C_norm_w", "B_bias", "C_bias")]


_lib = None


def load_library(path: str = LIB_PATH):
    """Open libssd.so and declare its signatures (raises when it was not built)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m selective_state_space_forward_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.ssd_create.argtypes = [ctypes.POINTER(Desc), ctypes.POINTER(vp)]
    lib.ssd_destroy.argtypes = [vp]
    lib.ssd_destroy.restype = None
    lib.ssd_get_path.argtypes = [vp]
    lib.ssd_get_path.restype = i32
    lib.ssd_set_bc_norm.argtypes = [vp, vp, vp, vp, vp]
    lib.ssd_state_bytes.argtypes = [vp, i32]
    lib.ssd_state_bytes.restype = sz
    lib.ssd_state_conv_offset.argtypes = [vp, i32]
    lib.ssd_state_conv_offset.restype = sz
    lib.ssd_forward.argtypes = [vp, i32, i32] + [vp] * 14 + [vp]
    lib.ssd_forward_ragged.argtypes = [vp, i32, i32] + [vp] * 15 + [vp]
    lib.ssd_s6_forward.argtypes = [i32, i32, i32, i32, i32] + [vp] * 11 + [vp]
    lib.ssd_step.argtypes = [vp, i32] + [vp] * 13
    lib.ssd_stage_conv.argtypes = [vp, i32, i32] + [vp] * 9
    lib.ssd_stage_dt.argtypes = [vp, i32, i32] + [vp] * 7
    lib.ssd_set_timing_events.argtypes = [vp, vp, vp]
    lib.ssd_launch_count.argtypes = [vp]
    lib.ssd_launch_count.restype = ctypes.c_uint64
    lib.ssd_check.argtypes = [vp, vp]
    lib.ssd_last_error.argtypes = []
    lib.ssd_last_error.restype = ctypes.c_char_p
    lib.ssd_status_string.argtypes = [ctypes.c_int]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_forward_noalloc.argtypes = [ctypes.POINTER(Desc), i32, i32] + [vp] * 15 + [vp]
    lib.ssd_set_gated_norm.argtypes = [vp, i32, vp, i32, ctypes.c_float]
    lib.ssd_ex2_throughput.argtypes = [ctypes.POINTER(ctypes.c_double), vp]
    lib.ssd_set_wait_test.argtypes = [vp, ctypes.c_uint64, i32]
    lib.ssd_forward_packed.argtypes = [vp, i32, i32, vp, ctypes.c_int64] + [vp] * 9 + [vp]
    lib.ssd_backward_workspace_bytes.argtypes = [vp, i32, i32]
    lib.ssd_backward_workspace_bytes.restype = sz
    lib.ssd_backward.argtypes = [vp, i32, i32] + [vp] * 13 + [ctypes.POINTER(Grads), vp, sz, vp]
    for f in ("ssd_create", "ssd_set_bc_norm", "ssd_forward", "ssd_step", "ssd_stage_conv",
              "ssd_stage_dt", "ssd_set_timing_events", "ssd_check", "ssd_forward_noalloc",
              "ssd_forward_ragged", "ssd_s6_forward", "ssd_backward", "ssd_set_gated_norm",
              "ssd_forward_packed", "ssd_ex2_throughput", "ssd_set_wait_test"):
        getattr(lib, f).restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


def _raise(lib, st: int):
    if st != SSD_OK:
        raise SSDError(st, lib.ssd_last_error().decode())


def _ptr(t, dtype=None, name="tensor"):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() and not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise TypeError(f"{name} must be contiguous")
    return t.data_ptr() or None


def _need(t, count: int, name: str):
    """Refuse a tensor that holds fewer elements than the call reads or writes
    through its pointer (the C ABI sees only the pointer)."""
    if isinstance(t, torch.Tensor) and t.numel() < count:
        raise ValueError(f"{name} holds {t.numel()} elements; the call touches {count}")


def _align256(v: int) -> int:
    return (v + 255) & ~255


def state_bytes_for(nheads, headdim, dstate, ngroups, dconv, act_dtype, batch) -> int:
    """ssd_state_bytes without a handle: the fp32 SSM state (batch, H, P, N), then
    at the next 256-byte boundary the conv history (batch, 3, conv_dim) in the
    activation dtype (none when dconv is 1), the whole rounded up to 256 bytes."""
    n = _align256(batch * nheads * headdim * dstate * 4)
    if dconv == 4:
        es = 2 if act_dtype == "bf16" else 4
        n += batch * 3 * (nheads * headdim + 2 * ngroups * dstate) * es
    return _align256(n)


def check_forward_sizes(dims: dict, batch: int, seqlen: int, state_bytes: int, *, x, z, dt_raw,
                        dt_bias, A, B, C, D, conv_w=None, conv_b=None, seq_idx=None,
                        init_state=None, out=None, final_state=None, lengths=None):
    """Element counts of a forward's (or, at seqlen 1, a step's) tensors against
    the shape the call reads: every pointer the library dereferences must
    cover what it touches.  dims: nheads, headdim, dstate, ngroups, dconv,
    a_per_token."""
    H, P, N, G = dims["nheads"], dims["headdim"], dims["dstate"], dims["ngroups"]
    tok = batch * seqlen
    for t, n in (("x", x), ("z", z), ("out", out)):
        _need(n, tok * H * P, t)
    _need(B, tok * G * N, "B")
    _need(C, tok * G * N, "C")
    _need(dt_raw, tok * H, "dt_raw")
    _need(dt_bias, H, "dt_bias")
    _need(D, H, "D")
    _need(A, tok * H if dims.get("a_per_token") else H, "A")
    if dims.get("dconv", 1) == 4:
        cd = H * P + 2 * G * N
        _need(conv_w, cd * 4, "conv_w")
        _need(conv_b, cd, "conv_b")
    _need(seq_idx, tok, "seq_idx")
    _need(lengths, batch, "lengths")
    _need(init_state, state_bytes, "init_state")
    _need(final_state, state_bytes, "final_state")


def _rows(x, per_token: int, name: str, rank: int = 3):
    """(batch, seqlen) of a (batch, seqlen, per_token) activation tensor."""
    if not isinstance(x, torch.Tensor) or x.dim() != rank or x.shape[-1] != per_token:
        want = "(batch, seqlen, %d)" % per_token if rank == 3 else "(batch, %d)" % per_token
        got = tuple(x.shape) if isinstance(x, torch.Tensor) else type(x).__name__
        raise ValueError(f"{name} must be {want}, got {got}")
    return (x.shape[0], x.shape[1]) if rank == 3 else (x.shape[0], 1)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Handle:
    """One layer shape: an ssd_handle plus its (library-owned) workspace."""

    def __init__(self, nheads, headdim, dstate, ngroups=1, dconv=4, act_dtype="bf16",
                 a_per_token=False, bc_norm=False, max_batch=1, max_seqlen=1, path="auto",
                 validate_finite=False, lib=None):
        self.lib = lib or load_library()
        self.nheads, self.headdim, self.dstate, self.ngroups = nheads, headdim, dstate, ngroups
        self.dconv, self.act_dtype = dconv, act_dtype
        self.a_per_token, self.bc_norm = bool(a_per_token), bool(bc_norm)
        self.torch_dtype = DTYPES[act_dtype][1]
        d = Desc(nheads=nheads, headdim=headdim, dstate=dstate, ngroups=ngroups, dconv=dconv,
                 chunk=64, act_dtype=DTYPES[act_dtype][0], a_mode=int(bool(a_per_token)),
                 bc_norm=int(bool(bc_norm)), max_batch=max_batch, max_seqlen=max_seqlen,
                 path=PATHS[path], validate_finite=int(bool(validate_finite)))
        h = ctypes.c_void_p()
        _raise(self.lib, self.lib.ssd_create(ctypes.byref(d), ctypes.byref(h)))
        self._h = h
        self._keep = ()
        self.path = PATH_NAMES.get(self.lib.ssd_get_path(h), "?")

    @property
    def dims(self) -> dict:
        return dict(nheads=self.nheads, headdim=self.headdim, dstate=self.dstate,
                    ngroups=self.ngroups, dconv=self.dconv, a_per_token=self.a_per_token)

    @property
    def conv_dim(self):
        return self.nheads * self.headdim + 2 * self.ngroups * self.dstate

    def close(self):
        if getattr(self, "_h", None):
            self.lib.ssd_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- state buffers -------------------------------------------------------------
    def state_bytes(self, batch: int) -> int:
        return int(self.lib.ssd_state_bytes(self._h, batch))

    def conv_offset(self, batch: int) -> int:
        return int(self.lib.ssd_state_conv_offset(self._h, batch))

    def new_state(self, batch: int, device="cuda") -> torch.Tensor:
        """A zero (fresh) state buffer for `batch` rows, as raw bytes."""
        return torch.zeros(self.state_bytes(batch), dtype=torch.uint8, device=device)

    def state_views(self, buf: torch.Tensor, batch: int):
        """(ssm (batch, H, P, N) fp32, conv history (batch, 3, conv_dim) or None) views of buf."""
        n = batch * self.nheads * self.headdim * self.dstate
        ssm = buf[:n * 4].view(torch.float32).view(batch, self.nheads, self.headdim, self.dstate)
        conv = None
        if self.dconv == 4:
            off = self.conv_offset(batch)
            es = 2 if self.act_dtype == "bf16" else 4
            conv = buf[off:off + batch * 3 * self.conv_dim * es].view(self.torch_dtype).view(
                batch, 3, self.conv_dim)
        return ssm, conv

    # ---- calls -----------------------------------------------------------------------
    def set_bc_norm(self, B_norm_w=None, C_norm_w=None, B_bias=None, C_bias=None):
        f = torch.float32
        self._keep = (B_norm_w, C_norm_w, B_bias, C_bias)
        _raise(self.lib, self.lib.ssd_set_bc_norm(
            self._h, _ptr(B_norm_w, f, "B_norm_w"), _ptr(C_norm_w, f, "C_norm_w"),
            _ptr(B_bias, f, "B_bias"), _ptr(C_bias, f, "C_bias")))

    def forward(self, x, z, dt_raw, dt_bias, A, B, C, D, conv_w=None, conv_b=None, seq_idx=None,
                init_state=None, out=None, final_state=None, stream=None, lengths=None):
        """ssd_forward, or ssd_forward_ragged when `lengths` (an int32 CUDA tensor of
        per-row real-token counts) is given; returns `out` (allocated like x when not given)."""
        at, f = self.torch_dtype, torch.float32
        batch, seqlen = _rows(x, self.nheads * self.headdim, "x")
        if out is None:
            out = torch.empty_like(x)
        check_forward_sizes(self.dims, batch, seqlen, self.state_bytes(batch), x=x, z=z,
                            dt_raw=dt_raw, dt_bias=dt_bias, A=A, B=B, C=C, D=D, conv_w=conv_w,
                            conv_b=conv_b, seq_idx=seq_idx, init_state=init_state, out=out,
                            final_state=final_state, lengths=lengths)
        if lengths is not None:
            _raise(self.lib, self.lib.ssd_forward_ragged(
                self._h, batch, seqlen, _ptr(lengths, torch.int32, "lengths"), _ptr(x, at, "x"),
                _ptr(z, at, "z"), _ptr(dt_raw, f, "dt_raw"), _ptr(dt_bias, f, "dt_bias"),
                _ptr(A, f, "A"), _ptr(B, at, "B"), _ptr(C, at, "C"), _ptr(D, f, "D"),
                _ptr(conv_w, at, "conv_w"), _ptr(conv_b, at, "conv_b"),
                _ptr(seq_idx, torch.int32, "seq_idx"), _ptr(init_state, torch.uint8, "init_state"),
                _ptr(out, at, "out"), _ptr(final_state, torch.uint8, "final_state"),
                _stream(stream)))
            return out
        _raise(self.lib, self.lib.ssd_forward(
            self._h, batch, seqlen, _ptr(x, at, "x"), _ptr(z, at, "z"),
            _ptr(dt_raw, f, "dt_raw"), _ptr(dt_bias, f, "dt_bias"), _ptr(A, f, "A"),
            _ptr(B, at, "B"), _ptr(C, at, "C"), _ptr(D, f, "D"), _ptr(conv_w, at, "conv_w"),
            _ptr(conv_b, at, "conv_b"), _ptr(seq_idx, torch.int32, "seq_idx"),
            _ptr(init_state, torch.uint8, "init_state"), _ptr(out, at, "out"),
            _ptr(final_state, torch.uint8, "final_state"), _stream(stream)))
        return out

    def packed_width(self) -> int:
        """Columns of a packed in_proj row: z, x, B, C, dt_raw."""
        return 2 * self.nheads * self.headdim + 2 * self.ngroups * self.dstate + self.nheads

    def forward_packed(self, zxbcdt, dt_bias, A, D, conv_w=None, conv_b=None, seq_idx=None,
                       init_state=None, out=None, final_state=None, stream=None):
        """ssd_forward_packed: zxbcdt is a (batch, seqlen, ld) activation tensor whose rows
        hold [z | x | B | C | dt_raw] from column 0 (a view of a wider buffer is fine as
        long as its last dimension is contiguous); returns `out`."""
        at, f = self.torch_dtype, torch.float32
        if not isinstance(zxbcdt, torch.Tensor) or zxbcdt.dim() != 3:
            raise ValueError("zxbcdt must be (batch, seqlen, ld)")
        batch, seqlen, width = zxbcdt.shape
        if width < self.packed_width():
            raise ValueError(f"zxbcdt rows hold {width} columns; {self.packed_width()} needed")
        if zxbcdt.dtype != at or (zxbcdt.numel() and not zxbcdt.is_cuda):
            raise TypeError(f"zxbcdt must be a CUDA {at} tensor")
        if zxbcdt.stride(2) != 1 or zxbcdt.stride(0) != seqlen * zxbcdt.stride(1):
            raise TypeError("zxbcdt must have contiguous rows of equal stride")
        ld = zxbcdt.stride(1)
        if out is None:
            out = torch.empty(batch, seqlen, self.nheads * self.headdim, dtype=at,
                              device=zxbcdt.device)
        HP = self.nheads * self.headdim
        _need(out, batch * seqlen * HP, "out")
        _need(dt_bias, self.nheads, "dt_bias")
        _need(D, self.nheads, "D")
        _need(A, batch * seqlen * self.nheads if self.a_per_token else self.nheads, "A")
        if self.dconv == 4:
            _need(conv_w, self.conv_dim * 4, "conv_w")
            _need(conv_b, self.conv_dim, "conv_b")
        _need(seq_idx, batch * seqlen, "seq_idx")
        _need(init_state, self.state_bytes(batch), "init_state")
        _need(final_state, self.state_bytes(batch), "final_state")
        _raise(self.lib, self.lib.ssd_forward_packed(
            self._h, batch, seqlen, zxbcdt.data_ptr() or None, ld, _ptr(dt_bias, f, "dt_bias"),
            _ptr(A, f, "A"), _ptr(D, f, "D"), _ptr(conv_w, at, "conv_w"),
            _ptr(conv_b, at, "conv_b"), _ptr(seq_idx, torch.int32, "seq_idx"),
            _ptr(init_state, torch.uint8, "init_state"), _ptr(out, at, "out"),
            _ptr(final_state, torch.uint8, "final_state"), _stream(stream)))
        return out

    def step(self, x, z, dt_raw, dt_bias, A, B, C, D, conv_w=None, conv_b=None, state=None,
             out=None, stream=None):
        """ssd_step: one token per row, `state` updated in place; returns `out`."""
        at, f = self.torch_dtype, torch.float32
        batch = x.shape[0] if isinstance(x, torch.Tensor) and x.dim() >= 1 else 0
        if not isinstance(x, torch.Tensor) or x.numel() != batch * self.nheads * self.headdim:
            raise ValueError(f"x must hold one token of {self.nheads * self.headdim} channels per row")
        if out is None:
            out = torch.empty_like(x)
        check_forward_sizes(self.dims, batch, 1, self.state_bytes(batch), x=x, z=z, dt_raw=dt_raw,
                            dt_bias=dt_bias, A=A, B=B, C=C, D=D, conv_w=conv_w, conv_b=conv_b,
                            init_state=state, out=out)
        _raise(self.lib, self.lib.ssd_step(
            self._h, batch, _ptr(x, at, "x"), _ptr(z, at, "z"), _ptr(dt_raw, f, "dt_raw"),
            _ptr(dt_bias, f, "dt_bias"), _ptr(A, f, "A"), _ptr(B, at, "B"), _ptr(C, at, "C"),
            _ptr(D, f, "D"), _ptr(conv_w, at, "conv_w"), _ptr(conv_b, at, "conv_b"),
            _ptr(state, torch.uint8, "state"), _ptr(out, at, "out"), _stream(stream)))
        return out

    def stage_conv(self, x, B, C, conv_w, conv_b, seq_idx=None, init_state=None, u=None,
                   stream=None):
        at = self.torch_dtype
        batch, seqlen = _rows(x, self.nheads * self.headdim, "x")
        if u is None:
            u = torch.empty(batch, seqlen, self.conv_dim, dtype=torch.float32, device=x.device)
        gn = self.ngroups * self.dstate
        _need(B, batch * seqlen * gn, "B")
        _need(C, batch * seqlen * gn, "C")
        _need(conv_w, self.conv_dim * 4, "conv_w")
        _need(conv_b, self.conv_dim, "conv_b")
        _need(seq_idx, batch * seqlen, "seq_idx")
        _need(init_state, self.state_bytes(batch), "init_state")
        _need(u, batch * seqlen * self.conv_dim, "u")
        _raise(self.lib, self.lib.ssd_stage_conv(
            self._h, batch, seqlen, _ptr(x, at, "x"), _ptr(B, at, "B"), _ptr(C, at, "C"),
            _ptr(conv_w, at, "conv_w"), _ptr(conv_b, at, "conv_b"),
            _ptr(seq_idx, torch.int32, "seq_idx"), _ptr(init_state, torch.uint8, "init_state"),
            _ptr(u, torch.float32, "u"), _stream(stream)))
        return u

    def stage_dt(self, dt_raw, dt_bias, A, seq_idx=None, stream=None):
        f = torch.float32
        batch, seqlen = _rows(dt_raw, self.nheads, "dt_raw")
        _need(dt_bias, self.nheads, "dt_bias")
        _need(A, batch * seqlen * self.nheads if self.a_per_token else self.nheads, "A")
        _need(seq_idx, batch * seqlen, "seq_idx")
        dt = torch.empty(batch, self.nheads, seqlen, dtype=f, device=dt_raw.device)
        acs = torch.empty_like(dt)
        _raise(self.lib, self.lib.ssd_stage_dt(
            self._h, batch, seqlen, _ptr(dt_raw, f, "dt_raw"), _ptr(dt_bias, f, "dt_bias"),
            _ptr(A, f, "A"), _ptr(seq_idx, torch.int32, "seq_idx"), _ptr(dt, f, "dt"),
            _ptr(acs, f, "acs"), _stream(stream)))
        return dt, acs

    def set_gated_norm(self, weight=None, group_size: int = 0, eps: float = 1e-5,
                       enable: bool = True):
        """ssd_set_gated_norm: later forwards and steps write norm(y * silu(z)) * weight."""
        self._gn_keep = weight
        _raise(self.lib, self.lib.ssd_set_gated_norm(
            self._h, int(bool(enable)), _ptr(weight, torch.float32, "weight"), int(group_size),
            float(eps)))

    def backward_workspace_bytes(self, batch: int, seqlen: int) -> int:
        return int(self.lib.ssd_backward_workspace_bytes(self._h, batch, seqlen))

    def backward(self, x, z, dt_raw, dt_bias, A, B, C, D, conv_w=None, conv_b=None, gout=None,
                 seq_idx=None, lengths=None, workspace=None, grads=None, stream=None):
        """ssd_backward of a zero-state prefill: returns a dict of fp32 gradients named like
        the inputs (x, z, B, C, dt_raw, dt_bias, A, D, and conv_w, conv_b with the conv,
        B_norm_w, C_norm_w, B_bias, C_bias with the B/C norm).  `grads` may hold
        preallocated outputs; `workspace` a uint8 CUDA tensor of at least
        backward_workspace_bytes(batch, seqlen) bytes."""
        at, f = self.torch_dtype, torch.float32
        batch, seqlen = _rows(x, self.nheads * self.headdim, "x")
        check_forward_sizes(self.dims, batch, seqlen, self.state_bytes(batch), x=x, z=z,
                            dt_raw=dt_raw, dt_bias=dt_bias, A=A, B=B, C=C, D=D, conv_w=conv_w,
                            conv_b=conv_b, seq_idx=seq_idx, out=gout, lengths=lengths)
        H, N, dev = self.nheads, self.dstate, x.device
        need = {"x": (batch, seqlen, H * self.headdim), "z": (batch, seqlen, H * self.headdim),
                "B": (batch, seqlen, self.ngroups * N), "C": (batch, seqlen, self.ngroups * N),
                "dt_raw": (batch, seqlen, H), "dt_bias": (H,), "D": (H,),
                "A": (batch, seqlen, H) if self.a_per_token else (H,)}
        if self.dconv == 4:
            need.update(conv_w=(self.conv_dim, 4), conv_b=(self.conv_dim,))
        if self.bc_norm:
            need.update(B_norm_w=(N,), C_norm_w=(N,), B_bias=(H, N), C_bias=(H, N))
        g = dict(grads or {})
        for k, shape in need.items():
            if g.get(k) is None:
                g[k] = torch.empty(shape, dtype=f, device=dev)
            else:
                _need(g[k], int(torch.Size(shape).numel()), "grads." + k)
        ws_bytes = self.backward_workspace_bytes(batch, seqlen)
        if workspace is None:
            workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
        _need(workspace, ws_bytes, "workspace")
        gr = Grads(**{k: _ptr(v, f, "grads." + k) for k, v in g.items()})
        _raise(self.lib, self.lib.ssd_backward(
            self._h, batch, seqlen, _ptr(lengths, torch.int32, "lengths"), _ptr(x, at, "x"),
            _ptr(z, at, "z"), _ptr(dt_raw, f, "dt_raw"), _ptr(dt_bias, f, "dt_bias"),
            _ptr(A, f, "A"), _ptr(B, at, "B"), _ptr(C, at, "C"), _ptr(D, f, "D"),
            _ptr(conv_w, at, "conv_w"), _ptr(conv_b, at, "conv_b"),
            _ptr(seq_idx, torch.int32, "seq_idx"), _ptr(gout, at, "gout"), ctypes.byref(gr),
            _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)))
        return g

    def set_timing_events(self, start=None, stop=None):
        """Bracket the main kernel of later calls with these torch.cuda.Events."""
        _raise(self.lib, self.lib.ssd_set_timing_events(
            self._h, start.cuda_event if start is not None else None,
            stop.cuda_event if stop is not None else None))

    def set_wait_test(self, wait_limit_ns: int = 0, withhold_stream: int = -1):
        """ssd_set_wait_test: bound the fused kernel's waits and withhold one hand-off."""
        _raise(self.lib, self.lib.ssd_set_wait_test(self._h, int(wait_limit_ns),
                                                    int(withhold_stream)))

    def launch_count(self) -> int:
        return int(self.lib.ssd_launch_count(self._h))

    def check(self, stream=None):
        _raise(self.lib, self.lib.ssd_check(self._h, _stream(stream)))


def forward_noalloc(x, z, dt_raw, dt_bias, A, B, C, D, conv_w=None, conv_b=None, seq_idx=None,
                    init_state=None, out=None, final_state=None, *, status, nheads, headdim,
                    dstate, ngroups=1, dconv=4, a_per_token=False, validate_finite=False,
                    max_batch=None, max_seqlen=None, path="auto", stream=None, lib=None):
    """ssd_forward_noalloc: the fused forward with no handle and no device allocation by the
    library (its scratch is a static device array).  `status` is a one-element int32 CUDA
    tensor the kernels OR error bits into; `out` and the state buffers are laid out as for
    Handle.forward.  a_per_token: A is (batch, seqlen, H), floored at magnitude 1e-4;
    validate_finite: the call also scans out and the final state for NaN or infinity and
    ORs bit 4 into `status`.  Returns `out` (allocated like x when not given)."""
    lib = lib or load_library()
    at, f = torch.bfloat16, torch.float32
    batch, seqlen = _rows(x, nheads * headdim, "x")
    d = Desc(nheads=nheads, headdim=headdim, dstate=dstate, ngroups=ngroups, dconv=dconv,
             chunk=64, act_dtype=DTYPES["bf16"][0], a_mode=int(bool(a_per_token)), bc_norm=0,
             max_batch=max_batch or max(batch, 1), max_seqlen=max_seqlen or max(seqlen, 1),
             path=PATHS[path], validate_finite=int(bool(validate_finite)))
    if out is None:
        out = torch.empty_like(x)
    dims = dict(nheads=nheads, headdim=headdim, dstate=dstate, ngroups=ngroups, dconv=dconv,
                a_per_token=bool(a_per_token))
    check_forward_sizes(dims, batch, seqlen,
                        state_bytes_for(nheads, headdim, dstate, ngroups, dconv, "bf16", batch),
                        x=x, z=z, dt_raw=dt_raw, dt_bias=dt_bias, A=A, B=B, C=C, D=D,
                        conv_w=conv_w, conv_b=conv_b, seq_idx=seq_idx, init_state=init_state,
                        out=out, final_state=final_state)
    _need(status, 1, "status")
    _raise(lib, lib.ssd_forward_noalloc(
        ctypes.byref(d), batch, seqlen, _ptr(x, at, "x"), _ptr(z, at, "z"),
        _ptr(dt_raw, f, "dt_raw"), _ptr(dt_bias, f, "dt_bias"), _ptr(A, f, "A"),
        _ptr(B, at, "B"), _ptr(C, at, "C"), _ptr(D, f, "D"), _ptr(conv_w, at, "conv_w"),
        _ptr(conv_b, at, "conv_b"), _ptr(seq_idx, torch.int32, "seq_idx"),
        _ptr(init_state, torch.uint8, "init_state"), _ptr(out, at, "out"),
        _ptr(final_state, torch.uint8, "final_state"), _ptr(status, torch.int32, "status"),
        _stream(stream)))
    return out


def ex2_throughput(stream=None, lib=None) -> float:
    """ssd_ex2_throughput: measured hardware exp2 results per second on this device."""
    lib = lib or load_library()
    v = ctypes.c_double(0.0)
    _raise(lib, lib.ssd_ex2_throughput(ctypes.byref(v), _stream(stream)))
    return v.value


def s6_forward(u, delta, delta_bias, A_log, B, C, D, z=None, init_state=None, out=None,
               final_state=None, stream=None, lib=None):
    """ssd_s6_forward (the Mamba-1 selective scan); returns `out` (allocated like u when
    not given).  u, z, B, C: bf16 or fp32 CUDA tensors; the rest fp32."""
    lib = lib or load_library()
    f = torch.float32
    if u.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("u must be bf16 or fp32")
    at = u.dtype
    if u.dim() != 3:
        raise ValueError(f"u must be (batch, seqlen, d_inner), got {tuple(u.shape)}")
    batch, seqlen, d_inner = u.shape
    if not isinstance(A_log, torch.Tensor) or A_log.dim() != 2 or A_log.shape[0] != d_inner:
        raise ValueError(f"A_log must be (d_inner, dstate) = ({d_inner}, dstate)")
    dstate = A_log.shape[1]
    if out is None:
        out = torch.empty_like(u)
    check_s6_sizes(batch, seqlen, d_inner, dstate, delta=delta, delta_bias=delta_bias, B=B, C=C,
                   D=D, z=z, init_state=init_state, out=out, final_state=final_state)
    _raise(lib, lib.ssd_s6_forward(
        batch, seqlen, d_inner, dstate, 1 if at == torch.bfloat16 else 0, _ptr(u, at, "u"),
        _ptr(delta, f, "delta"), _ptr(delta_bias, f, "delta_bias"), _ptr(A_log, f, "A_log"),
        _ptr(B, at, "B"), _ptr(C, at, "C"), _ptr(D, f, "D"), _ptr(z, at, "z"),
        _ptr(init_state, f, "init_state"), _ptr(out, at, "out"), _ptr(final_state, f, "final_state"),
        _stream(stream)))
    return out


def check_s6_sizes(batch, seqlen, d_inner, dstate, *, delta, delta_bias, B, C, D, z=None,
                   init_state=None, out=None, final_state=None):
    """Element counts of ssd_s6_forward's tensors against the shape it reads."""
    tok = batch * seqlen
    _need(delta, tok * d_inner, "delta")
    _need(z, tok * d_inner, "z")
    _need(out, tok * d_inner, "out")
    _need(B, tok * dstate, "B")
    _need(C, tok * dstate, "C")
    _need(delta_bias, d_inner, "delta_bias")
    _need(D, d_inner, "D")
    _need(init_state, batch * d_inner * dstate, "init_state")
    _need(final_state, batch * d_inner * dstate, "final_state")
