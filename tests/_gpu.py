"""Helpers that drive the CUDA path through the Python binding of the C ABI
for the parity tests.  Inputs come from the seeded workload generators; the
expected values come from the CPU oracle only."""
import numpy as np
import torch

from ssm_state_storage_b200 import replayssm as rs
from ssm_state_storage_b200 import workloads as wl


def layer_for(w: wl.Workload, **kw) -> rs.Layer:
    if w.kind == "m2":
        return rs.Layer("m2", w.B, w.H, w.P, w.N, ngroups=w.G, window=w.L,
                        draft_max=kw.pop("draft_max", w.n_draft), in_dtype=w.in_dtype, **kw)
    return rs.Layer(w.kind, w.B, w.H, w.P, w.N, window=w.L,
                    draft_max=kw.pop("draft_max", w.n_draft), in_dtype=w.in_dtype, **kw)


def to_dev(d: dict, dev="cuda"):
    return {k: v.to(dev) for k, v in d.items()}


def m2_replay_run(w, A, D, S0, steps, T=None, layer=None, check_h0_untouched=False):
    """Run T replay decode steps.  Returns dict(y[T,B,H,P], len[T,B,H], state)."""
    layer = layer or layer_for(w)
    st = rs.ReplayState(layer)
    rs.replayssm_init(layer, st, S0.cuda())
    T = steps["x"].shape[0] if T is None else T
    dev = to_dev(steps)
    Ad, Dd = A.cuda(), D.cuda()
    y = torch.empty(T, w.B, w.H, w.P, device="cuda")
    lens = torch.empty(T, w.B, w.H, dtype=torch.int32, device="cuda")
    untouched = True
    for t in range(T):
        prev = st.h0.clone() if check_h0_untouched else None
        inp = dict(x=dev["x"][t], dt=dev["dt"][t], Bm=dev["Bm"][t], Cm=dev["Cm"][t], A=Ad, D=Dd)
        rs.replayssm_decode_step(layer, st, inp, y[t])
        lens[t] = st.len
        if check_h0_untouched and (t + 1) % w.L != 0:
            untouched = untouched and bool(torch.equal(prev, st.h0))
    torch.cuda.synchronize()
    return dict(y=y.cpu().numpy(), len=lens.cpu().numpy(), state=st, layer=layer,
                untouched=untouched)


def m2_full_run(w, A, D, S0, steps, layer=None):
    layer = layer or layer_for(w)
    S = S0.clone().cuda()
    dev = to_dev(steps)
    T = steps["x"].shape[0]
    y = torch.empty(T, w.B, w.H, w.P, device="cuda")
    Ad, Dd = A.cuda(), D.cuda()
    for t in range(T):
        inp = dict(x=dev["x"][t], dt=dev["dt"][t], Bm=dev["Bm"][t], Cm=dev["Cm"][t], A=Ad, D=Dd)
        rs.replayssm_full_decode_step(layer, S, inp, y[t])
    torch.cuda.synchronize()
    return y.cpu().numpy(), S.cpu().double().numpy()


def gdn_replay_run(w, S0, steps, layer=None, check_h0_untouched=False):
    layer = layer or layer_for(w)
    st = rs.ReplayState(layer)
    rs.replayssm_init(layer, st, S0.cuda())
    dev = to_dev(steps)
    T = steps["q"].shape[0]
    o = torch.empty(T, w.B, w.H, w.P, device="cuda")
    lens = torch.empty(T, w.B, w.H, dtype=torch.int32, device="cuda")
    untouched = True
    for t in range(T):
        prev = st.h0.clone() if check_h0_untouched else None
        inp = {k: dev[k][t] for k in ("q", "k", "v", "alpha", "beta")}
        rs.replayssm_decode_step(layer, st, inp, o[t])
        lens[t] = st.len
        if check_h0_untouched and (t + 1) % w.L != 0:
            untouched = untouched and bool(torch.equal(prev, st.h0))
    torch.cuda.synchronize()
    return dict(y=o.cpu().numpy(), len=lens.cpu().numpy(), state=st, layer=layer,
                untouched=untouched)


def gdn_full_run(w, S0, steps, layer=None):
    layer = layer or layer_for(w)
    S = S0.clone().cuda()
    dev = to_dev(steps)
    T = steps["q"].shape[0]
    o = torch.empty(T, w.B, w.H, w.P, device="cuda")
    for t in range(T):
        inp = {k: dev[k][t] for k in ("q", "k", "v", "alpha", "beta")}
        rs.replayssm_full_decode_step(layer, S, inp, o[t])
    torch.cuda.synchronize()
    return o.cpu().numpy(), S.cpu().double().numpy()


def f64(t):
    return t.detach().cpu().double().numpy()


def m2_buffer_matches(state, orc, G_heads):
    """Slots below len: GPU records (rounded storage) equal the oracle's records
    exactly.  G_heads: number of heads per group."""
    ln = state.len.cpu().numpy()
    assert np.array_equal(ln, orc.len)
    xb, dtb, Bb, Cb = (f64(t) for t in state.buf[:4])
    n = int(ln.max()) if ln.size else 0
    for b in range(ln.shape[0]):
        for h in range(ln.shape[1]):
            k = int(ln[b, h])
            g = h // G_heads
            if not (np.array_equal(xb[b, h, :k], orc.rec_x[b, h, :k])
                    and np.array_equal(dtb[b, h, :k], orc.rec_dt[b, h, :k])
                    and np.array_equal(Bb[b, g, :k], orc.rec_B[b, h, :k])
                    and np.array_equal(Cb[b, g, :k], orc.rec_C[b, h, :k])):
                return False
    return True
