"""ctypes wrapper over the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY.  Imported by tests/, by __graft_entry__.smoke() and by
the cpu_baseline / --impl reference legs of bench.py; never by the product
package.  It shares no code with the CUDA path: inputs come from the seeded
workload generators (which hold none of the method's arithmetic) and are
converted here to float64.

Array conventions follow oracle.h.  Every function takes and returns numpy
arrays; state-carrying calls work on an explicit record-buffer object so that
runs can be composed (decode steps, then a forced flush, then more steps ...).
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

FMT = {"none": 0, "fp8": 1, "nvfp4": 2}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        dp = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        ip = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        lp = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
        fp = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        up = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
        i = C.c_int
        L.oracle_m2_conventional.argtypes = [i, i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp, dp, lp, lp]
        L.oracle_m2_replay.argtypes = [i, i, i, i, i, i, i, i, i, i, dp, dp, dp, dp, dp, ip,
                                       dp, dp, dp, dp, dp, dp, dp, ip, ip, lp, lp]
        L.oracle_m2_flush.argtypes = [i, i, i, i, i, i, i, i, dp, dp, dp, dp, ip, dp]
        L.oracle_m2_materialize.argtypes = [i, i, i, i, i, dp, dp, dp, dp, ip, dp, dp]
        L.oracle_m2_verify_replay.argtypes = [i, i, i, i, i, i, i, i, i, dp, dp, dp, dp, dp, ip,
                                              dp, dp, dp, dp, dp, dp, ip, dp, ip]
        L.oracle_m2_verify_snapshot.argtypes = [i, i, i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp,
                                                ip, dp, lp]
        L.oracle_gdn_conventional.argtypes = [i, i, i, i, i, C.c_double, dp, dp, dp, dp, dp, dp,
                                              dp, lp, lp]
        L.oracle_gdn_replay.argtypes = [i, i, i, i, i, i, i, C.c_double, dp, dp, dp, dp, dp, dp,
                                        ip, dp, dp, dp, dp, dp, dp, ip, ip, lp, lp]
        L.oracle_gdn_flush.argtypes = [i, i, i, i, i, i, i, dp, dp, dp, dp, dp, ip]
        L.oracle_gdn_verify_replay.argtypes = [i, i, i, i, i, i, i, i, C.c_double, dp, dp, dp,
                                               dp, dp, dp, ip, dp, dp, dp, dp, dp, ip, dp, ip]
        L.oracle_gdn_verify_snapshot.argtypes = [i, i, i, i, i, i, C.c_double, dp, dp, dp, dp,
                                                 dp, dp, ip, dp, lp]
        L.oracle_gdn_materialize.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, ip, dp]
        L.oracle_kda_conventional.argtypes = [i, i, i, i, i, C.c_double, dp, dp, dp, dp, dp, dp,
                                              dp, lp, lp]
        L.oracle_kda_replay.argtypes = [i, i, i, i, i, i, i, C.c_double, dp, dp, dp, dp, dp, dp,
                                        ip, dp, dp, dp, dp, dp, dp, ip, ip, lp, lp]
        L.oracle_kda_flush.argtypes = [i, i, i, i, i, i, i, dp, dp, dp, dp, dp, ip]
        L.oracle_kda_materialize.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, ip, dp]
        L.oracle_e4m3_encode.argtypes = [C.c_float]
        L.oracle_e4m3_encode.restype = C.c_uint8
        L.oracle_e4m3_decode.argtypes = [C.c_uint8]
        L.oracle_e4m3_decode.restype = C.c_double
        L.oracle_e2m1_encode.argtypes = [C.c_float]
        L.oracle_e2m1_encode.restype = C.c_uint8
        L.oracle_e2m1_decode.argtypes = [C.c_uint8]
        L.oracle_e2m1_decode.restype = C.c_double
        L.oracle_fp8_quant.argtypes = [C.c_longlong, fp, up]
        L.oracle_fp8_dequant.argtypes = [C.c_longlong, up, fp]
        L.oracle_nvfp4_quant.argtypes = [i, i, i, fp, up, up, fp]
        L.oracle_nvfp4_dequant.argtypes = [i, i, i, up, up, fp, fp]
        L.oracle_quantize_ckpt.argtypes = [i, i, i, i, dp]
        _lib = L
    return _lib


def _f64(a):
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: bad argument or buffer state (rc={rc})")


# --------------------------------------------------------------------- Mamba-2

def m2_conventional(S0, x, dt, Bm, Cm, A, D):
    """Token-by-token Mamba-2 decode.  Returns (y[T,B,H,P], S_final, reads, writes)."""
    S = _f64(S0).copy()
    x, dt, Bm, Cm, A, D = map(_f64, (x, dt, Bm, Cm, A, D))
    T, B, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    y = np.zeros((T, B, H, P))
    rd = np.zeros((B, H), np.int64)
    wr = np.zeros((B, H), np.int64)
    _check(lib().oracle_m2_conventional(T, B, H, P, N, G, S, x, dt, Bm, Cm, A, D, y, rd, wr),
           "m2_conventional")
    return y, S, rd, wr


class M2Replay:
    """Checkpoint + record buffer for every (sequence, head) of a Mamba-2 layer."""

    def __init__(self, h0, G, L=16, cap=None, read_fmt="none", ckpt_fmt="none"):
        self.h0 = _f64(h0).copy()
        B, H, P, N = self.h0.shape
        self.B, self.H, self.P, self.N, self.G = B, H, P, N, G
        self.L = L
        self.cap = cap if cap is not None else L
        self.read_fmt, self.ckpt_fmt = FMT[read_fmt], FMT[ckpt_fmt]
        cap = self.cap
        self.rec_x = np.zeros((B, H, cap, P))
        self.rec_dt = np.zeros((B, H, cap))
        self.rec_B = np.zeros((B, H, cap, N))
        self.rec_C = np.zeros((B, H, cap, N))
        self.len = np.zeros((B, H), np.int32)
        self.reads = np.zeros((B, H), np.int64)
        self.writes = np.zeros((B, H), np.int64)
        if self.ckpt_fmt:
            quantize_ckpt(ckpt_fmt, self.h0)

    def decode(self, x, dt, Bm, Cm, A, D):
        """Run T decode steps.  Returns (y[T,B,H,P], len_trace[T,B,H], flush_trace[T,B,H])."""
        x, dt, Bm, Cm, A, D = map(_f64, (x, dt, Bm, Cm, A, D))
        T = x.shape[0]
        y = np.zeros((T, self.B, self.H, self.P))
        lt = np.zeros((T, self.B, self.H), np.int32)
        ft = np.zeros((T, self.B, self.H), np.int32)
        _check(lib().oracle_m2_replay(T, self.B, self.H, self.P, self.N, self.G, self.L, self.cap,
                                      self.read_fmt, self.ckpt_fmt, self.h0, self.rec_x,
                                      self.rec_dt, self.rec_B, self.rec_C, self.len,
                                      x, dt, Bm, Cm, A, D, y, lt, ft, self.reads, self.writes),
               "m2_replay")
        return y, lt, ft

    def flush(self, A, force=False):
        _check(lib().oracle_m2_flush(self.B, self.H, self.P, self.N, self.L, self.cap, int(force),
                                     self.ckpt_fmt, self.h0, self.rec_x, self.rec_dt, self.rec_B,
                                     self.len, _f64(A)), "m2_flush")

    def materialize(self, A):
        S = np.zeros_like(self.h0)
        _check(lib().oracle_m2_materialize(self.B, self.H, self.P, self.N, self.cap, self.h0,
                                           self.rec_x, self.rec_dt, self.rec_B, self.len,
                                           _f64(A), S), "m2_materialize")
        return S

    def verify(self, x, dt, Bm, Cm, A, D, acc):
        """R speculative rounds: append Dn drafts, evaluate them output-only,
        commit acc[r, b] of them.  x is [R,B,Dn,H,P].  Returns (y, len_trace[R,B,H])."""
        x, dt, Bm, Cm, A, D = map(_f64, (x, dt, Bm, Cm, A, D))
        acc = _i32(acc)
        R, B, Dn, H, P = x.shape
        y = np.zeros((R, B, Dn, H, P))
        lt = np.zeros((R, B, H), np.int32)
        _check(lib().oracle_m2_verify_replay(R, B, H, P, self.N, self.G, self.L, self.cap, Dn,
                                             self.h0, self.rec_x, self.rec_dt, self.rec_B,
                                             self.rec_C, self.len, x, dt, Bm, Cm, A, D, acc, y, lt),
               "m2_verify_replay")
        return y, lt


def m2_verify_snapshot(S0, x, dt, Bm, Cm, A, D, acc):
    """Snapshot-and-restore speculative decoding on the full state.
    Returns (y[R,B,Dn,H,P], S_final, state_copies[B,H])."""
    S = _f64(S0).copy()
    x, dt, Bm, Cm, A, D = map(_f64, (x, dt, Bm, Cm, A, D))
    acc = _i32(acc)
    R, B, Dn, H, P = x.shape
    G, N = Bm.shape[3], Bm.shape[4]
    y = np.zeros((R, B, Dn, H, P))
    cp = np.zeros((B, H), np.int64)
    _check(lib().oracle_m2_verify_snapshot(R, B, H, P, N, G, Dn, S, x, dt, Bm, Cm, A, D, acc, y,
                                           cp), "m2_verify_snapshot")
    return y, S, cp


# --------------------------------------------------------------- Gated DeltaNet

def gdn_conventional(S0, q, k, v, alpha, beta, scale=1.0):
    """Token-by-token gated delta rule.  Returns (o[T,B,H,DV], S_final, reads, writes)."""
    S = _f64(S0).copy()
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    T, B, H, DK = q.shape
    DV = v.shape[3]
    o = np.zeros((T, B, H, DV))
    rd = np.zeros((B, H), np.int64)
    wr = np.zeros((B, H), np.int64)
    _check(lib().oracle_gdn_conventional(T, B, H, DK, DV, float(scale), S, q, k, v, alpha, beta,
                                         o, rd, wr), "gdn_conventional")
    return o, S, rd, wr


def gdn_verify_snapshot(S0, q, k, v, alpha, beta, acc, scale=1.0):
    """Snapshot-and-restore speculative decoding of the full GDN state.
    Returns (o[R,B,Dn,H,DV], S_final, state_copies[B,H])."""
    S = _f64(S0).copy()
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    acc = _i32(acc)
    R, B, Dn, H, DK = q.shape
    DV = v.shape[-1]
    o = np.zeros((R, B, Dn, H, DV))
    copies = np.zeros((B, H), np.int64)
    _check(lib().oracle_gdn_verify_snapshot(R, B, H, DK, DV, Dn, float(scale), S, q, k, v,
                                            alpha, beta, acc, o, copies), "gdn_verify_snapshot")
    return o, S, copies


class GDNReplay:
    def __init__(self, h0, L=16, cap=None, scale=1.0):
        self.h0 = _f64(h0).copy()
        B, H, DK, DV = self.h0.shape
        self.B, self.H, self.DK, self.DV = B, H, DK, DV
        self.L, self.cap, self.scale = L, (cap if cap is not None else L), float(scale)
        cap = self.cap
        self.rec_q = np.zeros((B, H, cap, DK))
        self.rec_k = np.zeros((B, H, cap, DK))
        self.rec_v = np.zeros((B, H, cap, DV))
        self.rec_alpha = np.zeros((B, H, cap))
        self.rec_beta = np.zeros((B, H, cap))
        self.len = np.zeros((B, H), np.int32)
        self.reads = np.zeros((B, H), np.int64)
        self.writes = np.zeros((B, H), np.int64)

    def decode(self, q, k, v, alpha, beta):
        q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
        T = q.shape[0]
        o = np.zeros((T, self.B, self.H, self.DV))
        lt = np.zeros((T, self.B, self.H), np.int32)
        ft = np.zeros((T, self.B, self.H), np.int32)
        _check(lib().oracle_gdn_replay(T, self.B, self.H, self.DK, self.DV, self.L, self.cap,
                                       self.scale, self.h0, self.rec_q, self.rec_k, self.rec_v,
                                       self.rec_alpha, self.rec_beta, self.len, q, k, v, alpha,
                                       beta, o, lt, ft, self.reads, self.writes), "gdn_replay")
        return o, lt, ft

    def flush(self, force=False):
        _check(lib().oracle_gdn_flush(self.B, self.H, self.DK, self.DV, self.L, self.cap,
                                      int(force), self.h0, self.rec_k, self.rec_v,
                                      self.rec_alpha, self.rec_beta, self.len), "gdn_flush")

    def verify(self, q, k, v, alpha, beta, acc):
        """R speculative rounds: append Dn drafts, evaluate them output-only,
        commit acc[r, b] of them.  q is [R,B,Dn,H,DK].  Returns (o, len_trace[R,B,H])."""
        q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
        acc = _i32(acc)
        R, B, Dn, H, _ = q.shape
        o = np.zeros((R, B, Dn, H, self.DV))
        lt = np.zeros((R, B, H), np.int32)
        _check(lib().oracle_gdn_verify_replay(R, B, H, self.DK, self.DV, self.L, self.cap, Dn,
                                              self.scale, self.h0, self.rec_q, self.rec_k,
                                              self.rec_v, self.rec_alpha, self.rec_beta,
                                              self.len, q, k, v, alpha, beta, acc, o, lt),
               "gdn_verify_replay")
        return o, lt

    def materialize(self):
        S = np.zeros_like(self.h0)
        _check(lib().oracle_gdn_materialize(self.B, self.H, self.DK, self.DV, self.cap, self.h0,
                                            self.rec_k, self.rec_v, self.rec_alpha,
                                            self.rec_beta, self.len, S), "gdn_materialize")
        return S


# ---------------------------------------------------------- Kimi Delta Attention

def kda_conventional(S0, q, k, v, alpha, beta, scale=1.0):
    """Token-by-token gated delta rule with per-channel decay alpha [T,B,H,DK].
    Returns (o[T,B,H,DV], S_final, reads, writes)."""
    S = _f64(S0).copy()
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    T, B, H, DK = q.shape
    DV = v.shape[3]
    o = np.zeros((T, B, H, DV))
    rd = np.zeros((B, H), np.int64)
    wr = np.zeros((B, H), np.int64)
    _check(lib().oracle_kda_conventional(T, B, H, DK, DV, float(scale), S, q, k, v, alpha, beta,
                                         o, rd, wr), "kda_conventional")
    return o, S, rd, wr


class KDAReplay:
    """Checkpoint + record buffer (q, k, v, per-channel alpha, beta) for every
    (sequence, head) of a Kimi Delta Attention layer."""

    def __init__(self, h0, L=16, cap=None, scale=1.0):
        self.h0 = _f64(h0).copy()
        B, H, DK, DV = self.h0.shape
        self.B, self.H, self.DK, self.DV = B, H, DK, DV
        self.L, self.cap, self.scale = L, (cap if cap is not None else L), float(scale)
        cap = self.cap
        self.rec_q = np.zeros((B, H, cap, DK))
        self.rec_k = np.zeros((B, H, cap, DK))
        self.rec_v = np.zeros((B, H, cap, DV))
        self.rec_alpha = np.zeros((B, H, cap, DK))
        self.rec_beta = np.zeros((B, H, cap))
        self.len = np.zeros((B, H), np.int32)
        self.reads = np.zeros((B, H), np.int64)
        self.writes = np.zeros((B, H), np.int64)

    def decode(self, q, k, v, alpha, beta):
        q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
        T = q.shape[0]
        o = np.zeros((T, self.B, self.H, self.DV))
        lt = np.zeros((T, self.B, self.H), np.int32)
        ft = np.zeros((T, self.B, self.H), np.int32)
        _check(lib().oracle_kda_replay(T, self.B, self.H, self.DK, self.DV, self.L, self.cap,
                                       self.scale, self.h0, self.rec_q, self.rec_k, self.rec_v,
                                       self.rec_alpha, self.rec_beta, self.len, q, k, v, alpha,
                                       beta, o, lt, ft, self.reads, self.writes), "kda_replay")
        return o, lt, ft

    def flush(self, force=False):
        _check(lib().oracle_kda_flush(self.B, self.H, self.DK, self.DV, self.L, self.cap,
                                      int(force), self.h0, self.rec_k, self.rec_v,
                                      self.rec_alpha, self.rec_beta, self.len), "kda_flush")

    def materialize(self):
        S = np.zeros_like(self.h0)
        _check(lib().oracle_kda_materialize(self.B, self.H, self.DK, self.DV, self.cap, self.h0,
                                            self.rec_k, self.rec_v, self.rec_alpha,
                                            self.rec_beta, self.len, S), "kda_materialize")
        return S


# ----------------------------------------------------------------------- codecs

def e4m3_encode(v: float) -> int:
    return int(lib().oracle_e4m3_encode(float(v)))


def e4m3_decode(c: int) -> float:
    return float(lib().oracle_e4m3_decode(int(c)))


def e2m1_encode(v: float) -> int:
    return int(lib().oracle_e2m1_encode(float(v)))


def e2m1_decode(c: int) -> float:
    return float(lib().oracle_e2m1_decode(int(c)))


def fp8_quant(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    c = np.zeros(x.shape, np.uint8)
    _check(lib().oracle_fp8_quant(x.size, x.reshape(-1), c.reshape(-1)), "fp8_quant")
    return c


def fp8_dequant(c):
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.zeros(c.shape, np.float32)
    _check(lib().oracle_fp8_dequant(c.size, c.reshape(-1), out.reshape(-1)), "fp8_dequant")
    return out


def nvfp4_quant(x):
    """x: [..., rows, cols] fp32; every [rows, cols] slice is one tile."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape[-2:]
    lead = x.shape[:-2]
    nt = int(np.prod(lead)) if lead else 1
    codes = np.zeros(lead + (rows, cols // 2), np.uint8)
    scales = np.zeros(lead + (rows, cols // 16), np.uint8)
    gs = np.zeros(lead if lead else (1,), np.float32)
    _check(lib().oracle_nvfp4_quant(nt, rows, cols, x.reshape(-1), codes.reshape(-1),
                                    scales.reshape(-1), gs.reshape(-1)), "nvfp4_quant")
    return codes, scales, gs


def nvfp4_dequant(codes, scales, gs):
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    gs = np.ascontiguousarray(gs, np.float32)
    rows, half = codes.shape[-2:]
    cols = half * 2
    lead = codes.shape[:-2]
    nt = int(np.prod(lead)) if lead else 1
    out = np.zeros(lead + (rows, cols), np.float32)
    _check(lib().oracle_nvfp4_dequant(nt, rows, cols, codes.reshape(-1), scales.reshape(-1),
                                      gs.reshape(-1), out.reshape(-1)), "nvfp4_dequant")
    return out


def quantize_ckpt(fmt, h):
    """In place: h <- deq(Q(fp32(h))) per [rows, cols] tile (last two axes)."""
    rows, cols = h.shape[-2:]
    nt = int(np.prod(h.shape[:-2])) if h.ndim > 2 else 1
    assert h.dtype == np.float64 and h.flags.c_contiguous
    _check(lib().oracle_quantize_ckpt(FMT[fmt], nt, rows, cols, h.reshape(-1)), "quantize_ckpt")
    return h
