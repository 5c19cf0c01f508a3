"""Thin ctypes binding over libreplayssm.so (include/replayssm.h).

Argument marshalling only: every function checks dtypes/devices, turns torch
tensors into raw pointers and strides, and calls the C entry point of the same
name.  All compute runs in the library's CUDA kernels; there is no CPU path.
If the library is missing, every entry point raises.

PyTorch is used for device memory and streams: `ReplayState` allocates the
caller-owned buffers the C ABI expects (sizes from replayssm_state_bytes).

A Mamba-2 layer decoded step by step (shapes of one layer, bf16 inputs):

    layer = Layer("m2", batch, nheads, headdim, dstate, ngroups=G, window=16,
                  in_dtype=torch.bfloat16)
    state = ReplayState(layer)
    replayssm_init(layer, state, S0)               # fp32 [B][H][P][N] on the GPU
    for t in range(T):                             # x [B][H][P], dt [B][H], Bm/Cm [B][G][N]
        replayssm_decode_step(layer, state, dict(x=x[t], dt=dt[t], Bm=Bm[t], Cm=Cm[t],
                                                 A=A, D=D), y[t])
    replayssm_materialize(layer, state, S_out, A)  # the full state, out of place

Speculative rounds use replayssm_verify_commit (drafts with a draft axis after
the batch axis, the previous round's accepted counts) and replayssm_commit.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libreplayssm.so")

# enums (replayssm.h)
RSSM_OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "unsupported dtype",
                4: "pointer not 16-byte aligned", 5: "buffer capacity exceeded",
                6: "CUDA launch error", 7: "device wait timed out",
                8: "unsupported by this build", 9: "buffer state out of range"}
KIND = {"m2": 0, "gdn": 1, "kda": 2}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}
FMT = {"none": 0, "fp8": 1, "nvfp4": 2}
BYTES = {"h0": 0, "buf0": 1, "buf1": 2, "buf2": 3, "buf3": 4, "buf4": 5, "buf5": 6, "len": 7,
         "rc": 8, "rc_scale": 9, "rc_gscale": 10, "status": 11, "full_state": 12, "y": 13}


class Desc(C.Structure):
    _fields_ = [("kind", C.c_int32), ("batch", C.c_int32), ("nheads", C.c_int32),
                ("headdim", C.c_int32), ("dstate", C.c_int32), ("ngroups", C.c_int32),
                ("window", C.c_int32), ("draft_max", C.c_int32), ("in_dtype", C.c_int32),
                ("read_fmt", C.c_int32), ("ckpt_fmt", C.c_int32), ("scale", C.c_float)]


class State(C.Structure):
    _fields_ = [("h0", C.c_void_p), ("buf", C.c_void_p * 6), ("len", C.c_void_p),
                ("rc", C.c_void_p), ("rc_scale", C.c_void_p), ("rc_gscale", C.c_void_p),
                ("status", C.c_void_p)]


class StepIn(C.Structure):
    _fields_ = [("in_", C.c_void_p * 5), ("A", C.c_void_p), ("D", C.c_void_p),
                ("batch_stride", C.c_int64 * 5), ("y_batch_stride", C.c_int64)]


ENTRY_POINTS = {
    "replayssm_validate": (C.c_int, [C.POINTER(Desc)]),
    "replayssm_capacity": (C.c_int32, [C.POINTER(Desc)]),
    "replayssm_state_bytes": (C.c_size_t, [C.POINTER(Desc), C.c_int32]),
    "replayssm_status_string": (C.c_char_p, [C.c_int]),
    "replayssm_last_cuda_error": (C.c_char_p, []),
    "replayssm_init": (C.c_int, [C.POINTER(Desc), C.POINTER(State), C.c_void_p, C.c_void_p]),
    "replayssm_decode_step": (C.c_int, [C.POINTER(Desc), C.POINTER(State), C.POINTER(StepIn),
                                        C.c_void_p, C.c_void_p]),
    "replayssm_flush": (C.c_int, [C.POINTER(Desc), C.POINTER(State), C.c_void_p, C.c_int32,
                                  C.c_void_p]),
    "replayssm_decode_step_inplace": (C.c_int, [C.POINTER(Desc), C.POINTER(State), C.c_void_p,
                                                C.c_void_p, C.c_void_p, C.c_void_p]),
    "replayssm_verify_commit": (C.c_int, [C.POINTER(Desc), C.POINTER(State), C.c_void_p,
                                          C.POINTER(StepIn), C.c_int32, C.c_void_p, C.c_void_p]),
    "replayssm_commit": (C.c_int, [C.POINTER(Desc), C.POINTER(State), C.c_void_p, C.c_void_p,
                                   C.c_void_p]),
    "replayssm_full_decode_step": (C.c_int, [C.POINTER(Desc), C.c_void_p, C.POINTER(StepIn),
                                             C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p]),
    "replayssm_materialize": (C.c_int, [C.POINTER(Desc), C.POINTER(State), C.c_void_p,
                                        C.c_void_p, C.c_void_p]),
    "replayssm_quantize": (C.c_int, [C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_void_p,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "replayssm_set_test_hooks": (C.c_int, [C.c_int64, C.c_int32]),
}

_lib = None


def lib():
    """Load libreplayssm.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m ssm_state_storage_b200.build` (no CPU fallback exists)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in ENTRY_POINTS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class ReplayError(RuntimeError):
    pass


def _ok(rc: int, what: str):
    if rc != RSSM_OK:
        extra = ""
        if rc == 6:
            extra = f": {lib().replayssm_last_cuda_error().decode()}"
        raise ReplayError(f"{what}: {STATUS_NAMES.get(rc, rc)} (status {rc}){extra}")


# ------------------------------------------------------------------- layer spec

@dataclass
class Layer:
    """One SSM layer's decode-state description (rssm_desc)."""
    kind: str            # "m2" | "gdn" | "kda"
    batch: int
    nheads: int
    headdim: int         # M2 P; GDN d_v
    dstate: int          # M2 N; GDN d_k
    ngroups: int = 0     # M2 G
    window: int = 16
    draft_max: int = 0
    in_dtype: torch.dtype = torch.bfloat16
    read_fmt: str = "none"
    ckpt_fmt: str = "none"
    scale: float = 1.0

    def desc(self) -> Desc:
        return Desc(KIND[self.kind], self.batch, self.nheads, self.headdim, self.dstate,
                    self.ngroups, self.window, self.draft_max, DTYPE[self.in_dtype],
                    FMT[self.read_fmt], FMT[self.ckpt_fmt], float(self.scale))

    @property
    def G(self):
        return self.ngroups if self.kind == "m2" else self.nheads

    def capacity(self) -> int:
        d = self.desc()
        return int(lib().replayssm_capacity(C.byref(d)))

    def nbytes(self, which: str) -> int:
        d = self.desc()
        return int(lib().replayssm_state_bytes(C.byref(d), BYTES[which]))


class ReplayState:
    """Caller-owned device buffers of a replay state, allocated with torch."""

    def __init__(self, layer: Layer, device="cuda"):
        d = layer.desc()
        _ok(lib().replayssm_validate(C.byref(d)), "replayssm_validate")
        self.layer = layer
        B, H, P, N, G = layer.batch, layer.nheads, layer.headdim, layer.dstate, layer.G
        cap = layer.capacity()
        self.cap = cap
        dt_in = layer.in_dtype
        f32 = torch.float32
        if layer.kind == "m2":
            self.h0 = torch.zeros(B, H, P, N, dtype=f32, device=device)
            self.buf = [torch.zeros(B, H, cap, P, dtype=dt_in, device=device),
                        torch.zeros(B, H, cap, dtype=f32, device=device),
                        torch.zeros(B, G, cap, N, dtype=dt_in, device=device),
                        torch.zeros(B, G, cap, N, dtype=dt_in, device=device)]
        else:
            self.h0 = torch.zeros(B, H, N, P, dtype=f32, device=device)
            alpha_shape = (B, H, cap, N) if layer.kind == "kda" else (B, H, cap)
            self.buf = [torch.zeros(B, H, cap, N, dtype=dt_in, device=device),
                        torch.zeros(B, H, cap, N, dtype=dt_in, device=device),
                        torch.zeros(B, H, cap, P, dtype=dt_in, device=device),
                        torch.zeros(*alpha_shape, dtype=f32, device=device),
                        torch.zeros(B, H, cap, dtype=f32, device=device),
                        torch.zeros(B, H, cap, P, dtype=f32, device=device)]
        for i, t in enumerate(self.buf):
            assert t.numel() * t.element_size() == layer.nbytes(f"buf{i}")
        assert self.h0.numel() * 4 == layer.nbytes("h0")
        self.len = torch.zeros(B, H, dtype=torch.int32, device=device)
        self.status_word = torch.zeros(1, dtype=torch.int32, device=device)
        u8 = torch.uint8
        self.rc = self.rc_scale = self.rc_gscale = None
        if layer.read_fmt == "fp8":
            self.rc = torch.zeros(B, H, P, N, dtype=u8, device=device)
        elif layer.read_fmt == "nvfp4":
            self.rc = torch.zeros(B, H, P, N // 2, dtype=u8, device=device)
            self.rc_scale = torch.zeros(B, H, P, N // 16, dtype=u8, device=device)
            self.rc_gscale = torch.zeros(B, H, dtype=f32, device=device)

    def cstate(self) -> State:
        s = State()
        s.h0 = self.h0.data_ptr()
        for i in range(6):
            s.buf[i] = self.buf[i].data_ptr() if i < len(self.buf) else None
        s.len = self.len.data_ptr()
        s.rc = self.rc.data_ptr() if self.rc is not None else None
        s.rc_scale = self.rc_scale.data_ptr() if self.rc_scale is not None else None
        s.rc_gscale = self.rc_gscale.data_ptr() if self.rc_gscale is not None else None
        s.status = self.status_word.data_ptr()
        return s

    def status(self) -> int:
        """Device status word (synchronises the current stream)."""
        return int(self.status_word.item())

    def clear_status(self):
        self.status_word.zero_()


# -------------------------------------------------------------- marshalling

def _stream(stream):
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


def _dev(t: torch.Tensor, dtype, what):
    if not t.is_cuda:
        raise ReplayError(f"{what}: tensor must live on a CUDA device (no CPU path)")
    if t.dtype != dtype:
        raise ReplayError(f"{what}: dtype {t.dtype}, expected {dtype}")
    return t


def _batched(t: torch.Tensor, dtype, what):
    """Pointer + batch stride of a [B, ...] tensor whose per-sequence part is dense."""
    _dev(t, dtype, what)
    if t.dim() == 0 or t.shape[0] == 0:
        return t.data_ptr(), 0
    if not t[0].is_contiguous():
        raise ReplayError(f"{what}: per-sequence slice must be contiguous")
    return t.data_ptr(), t.stride(0)


def _dense(t, dtype, what):
    _dev(t, dtype, what)
    if not t.is_contiguous():
        raise ReplayError(f"{what}: must be contiguous")
    return t.data_ptr()


def _step_in(layer: Layer, inp: dict, y: torch.Tensor | None = None) -> StepIn:
    s = StepIn()
    f32, dti = torch.float32, layer.in_dtype
    if layer.kind == "m2":
        names = [("x", dti), ("dt", dti), ("Bm", dti), ("Cm", dti)]
    else:
        names = [("q", dti), ("k", dti), ("v", dti), ("alpha", f32), ("beta", f32)]
    for i, (nm, dt) in enumerate(names):
        ptr, bs = _batched(inp[nm], dt, nm)
        s.in_[i] = ptr
        s.batch_stride[i] = bs
    if layer.kind == "m2":
        s.A = _dense(inp["A"], f32, "A")
        s.D = _dense(inp["D"], f32, "D")
    if y is not None:
        _, s.y_batch_stride = _batched(y, f32, "y")
    return s


# ------------------------------------------------------------- entry points

def replayssm_init(layer: Layer, state: ReplayState, S0: torch.Tensor, stream=None):
    d, cs = layer.desc(), state.cstate()
    _ok(lib().replayssm_init(C.byref(d), C.byref(cs), _dense(S0, torch.float32, "S0"),
                             _stream(stream)), "replayssm_init")


def replayssm_decode_step(layer: Layer, state: ReplayState, inp: dict, y: torch.Tensor,
                          stream=None):
    d, cs = layer.desc(), state.cstate()
    si = _step_in(layer, inp, y)
    _ok(lib().replayssm_decode_step(C.byref(d), C.byref(cs), C.byref(si), y.data_ptr(),
                                    _stream(stream)), "replayssm_decode_step")


def replayssm_decode_step_inplace(layer: Layer, state: ReplayState, y: torch.Tensor,
                                  A: torch.Tensor | None = None, D: torch.Tensor | None = None,
                                  stream=None):
    """A decode step whose record the caller already wrote into slot len of
    the record buffers (state.buf[i][..., len, ...])."""
    d, cs = layer.desc(), state.cstate()
    a = _dense(A, torch.float32, "A") if A is not None else None
    dd = _dense(D, torch.float32, "D") if D is not None else None
    _ok(lib().replayssm_decode_step_inplace(C.byref(d), C.byref(cs), a, dd,
                                            _dense(y, torch.float32, "y"), _stream(stream)),
        "replayssm_decode_step_inplace")


def replayssm_flush(layer: Layer, state: ReplayState, A: torch.Tensor | None = None,
                    force: bool = False, stream=None):
    d, cs = layer.desc(), state.cstate()
    a = _dense(A, torch.float32, "A") if A is not None else None
    _ok(lib().replayssm_flush(C.byref(d), C.byref(cs), a, int(bool(force)), _stream(stream)),
        "replayssm_flush")


def replayssm_verify_commit(layer: Layer, state: ReplayState, accepted_prev, drafts: dict,
                            y: torch.Tensor, stream=None):
    """Mamba-2 drafts: x [B,n,H,P], dt [B,n,H], Bm/Cm [B,n,G,N], A, D; y [B,n,H,P].
    Gated DeltaNet drafts: q, k [B,n,H,DK], v [B,n,H,DV], alpha, beta [B,n,H];
    y [B,n,H,DV]."""
    d, cs = layer.desc(), state.cstate()
    n = drafts["x" if layer.kind == "m2" else "q"].shape[1]
    si = _step_in(layer, drafts, y)
    acc = _dense(accepted_prev, torch.int32, "accepted_prev") if accepted_prev is not None else None
    _ok(lib().replayssm_verify_commit(C.byref(d), C.byref(cs), acc, C.byref(si), int(n),
                                      y.data_ptr(), _stream(stream)), "replayssm_verify_commit")


def replayssm_commit(layer: Layer, state: ReplayState, accepted: torch.Tensor,
                     A: torch.Tensor | None = None, stream=None):
    """Close a speculative round (A: Mamba-2 decay rates; None for GDN)."""
    d, cs = layer.desc(), state.cstate()
    a = _dense(A, torch.float32, "A") if A is not None else None
    _ok(lib().replayssm_commit(C.byref(d), C.byref(cs), _dense(accepted, torch.int32, "accepted"),
                               a, _stream(stream)), "replayssm_commit")


def replayssm_full_decode_step(layer: Layer, S: torch.Tensor, inp: dict, y: torch.Tensor,
                               limit: torch.Tensor | None = None, step_index: int = 0,
                               stream=None):
    d = layer.desc()
    si = _step_in(layer, inp, y)
    lim = _dense(limit, torch.int32, "limit") if limit is not None else None
    _ok(lib().replayssm_full_decode_step(C.byref(d), _dense(S, torch.float32, "S"), C.byref(si),
                                         y.data_ptr(), lim, int(step_index), _stream(stream)),
        "replayssm_full_decode_step")


def replayssm_materialize(layer: Layer, state: ReplayState, S_out: torch.Tensor,
                          A: torch.Tensor | None = None, stream=None):
    d, cs = layer.desc(), state.cstate()
    a = _dense(A, torch.float32, "A") if A is not None else None
    _ok(lib().replayssm_materialize(C.byref(d), C.byref(cs), a,
                                    _dense(S_out, torch.float32, "S_out"), _stream(stream)),
        "replayssm_materialize")


def replayssm_quantize(fmt: str, src: torch.Tensor, codes: torch.Tensor,
                       scales: torch.Tensor | None = None, gscale: torch.Tensor | None = None,
                       stream=None):
    """src [..., rows, cols] fp32: every [rows, cols] slice is one tile."""
    rows, cols = src.shape[-2:]
    ntile = src.numel() // (rows * cols) if src.numel() else 0
    _ok(lib().replayssm_quantize(FMT[fmt], ntile, rows, cols, _dense(src, torch.float32, "src"),
                                 _dense(codes, torch.uint8, "codes"),
                                 _dense(scales, torch.uint8, "scales") if scales is not None else None,
                                 _dense(gscale, torch.float32, "gscale") if gscale is not None else None,
                                 _stream(stream)), "replayssm_quantize")


def replayssm_status_string(code: int) -> str:
    return lib().replayssm_status_string(int(code)).decode()


def replayssm_validate(layer: Layer) -> int:
    d = layer.desc()
    return int(lib().replayssm_validate(C.byref(d)))


def replayssm_set_test_hooks(consumer_wait_ns: int = 0, withhold_item: int = -1):
    """Test hook of the bounded device waits (see include/replayssm.h):
    shorten the compute warps' wait limit and make the staging warp skip one
    work item.  Call with no arguments to restore the defaults."""
    _ok(lib().replayssm_set_test_hooks(int(consumer_wait_ns), int(withhold_item)),
        "replayssm_set_test_hooks")
