"""Small fixed runs of one kernel each, for ncu captures (one kernel, a few
launches, a checkpoint larger than the 126 MB L2, a few GB on the device):

    python -m ssm_state_storage_b200.profile_cases verify [batch]
        8 speculative verify rounds of m2_verify (default batch 64: a 256 MiB
        checkpoint), the previous round's acceptance committed each round
    python -m ssm_state_storage_b200.profile_cases gdn [batch]
        20 decode steps of gdn_serving (default batch 64: a 512 MiB checkpoint)
    python -m ssm_state_storage_b200.profile_cases m2 [batch]
        32 decode steps of m2_serving (default batch 64: a 256 MiB checkpoint;
        launches 16 and 32 are flush steps)
    python -m ssm_state_storage_b200.profile_cases gdn_verify [batch]
        8 speculative verify rounds of gdn_verify (default batch 64)
    python -m ssm_state_storage_b200.profile_cases kda [batch]
        20 decode steps of kda_serving (default batch 64)

Each run checks the device status word and exits non-zero if it is set.
"""
import sys

import torch

from . import replayssm as rs
from . import workloads as wl


def verify(batch=64, rounds=8):
    w = wl.make("m2_verify", B=batch)
    g = wl.Generator(w)
    A, D = (t.cuda() for t in g.params())
    S0 = g.initial_state()
    rd = {k: v.cuda() for k, v in g.rounds(rounds).items()}
    layer = rs.Layer("m2", w.B, w.H, w.P, w.N, ngroups=w.G, window=w.L, draft_max=w.n_draft,
                     in_dtype=w.in_dtype)
    y = torch.empty(w.B, w.n_draft, w.H, w.P, device="cuda")
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    for r in range(rounds):
        drafts = dict(x=rd["x"][r], dt=rd["dt"][r], Bm=rd["Bm"][r], Cm=rd["Cm"][r], A=A, D=D)
        rs.replayssm_verify_commit(layer, state, rd["acc"][r - 1] if r else None, drafts, y)
    torch.cuda.synchronize()
    return state.status()


def gdn(batch=64, steps=20):
    w = wl.make("gdn_serving", B=batch)
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = {k: v.cuda() for k, v in g.steps(steps).items()}
    layer = rs.Layer("gdn", w.B, w.H, w.P, w.N, window=w.L, in_dtype=w.in_dtype)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    y = torch.empty(w.B, w.H, w.P, device="cuda")
    for t in range(steps):
        rs.replayssm_decode_step(layer, state, {k: st[k][t] for k in st}, y)
    torch.cuda.synchronize()
    return state.status()


def m2(batch=64, steps=32):
    w = wl.make("m2_serving", B=batch)
    g = wl.Generator(w)
    A, D = (t.cuda() for t in g.params())
    S0 = g.initial_state()
    st = {k: v.cuda() for k, v in g.steps(steps).items()}
    layer = rs.Layer("m2", w.B, w.H, w.P, w.N, ngroups=w.G, window=w.L, in_dtype=w.in_dtype)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    y = torch.empty(w.B, w.H, w.P, device="cuda")
    for t in range(steps):
        inp = dict(x=st["x"][t], dt=st["dt"][t], Bm=st["Bm"][t], Cm=st["Cm"][t], A=A, D=D)
        rs.replayssm_decode_step(layer, state, inp, y)
    torch.cuda.synchronize()
    return state.status()


def gdn_verify(batch=64, rounds=8):
    w = wl.make("gdn_verify", B=batch)
    g = wl.Generator(w)
    S0 = g.initial_state()
    rd = {k: v.cuda() for k, v in g.rounds(rounds).items()}
    layer = rs.Layer("gdn", w.B, w.H, w.P, w.N, window=w.L, draft_max=w.n_draft,
                     in_dtype=w.in_dtype)
    y = torch.empty(w.B, w.n_draft, w.H, w.P, device="cuda")
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    for r in range(rounds):
        drafts = {k: rd[k][r] for k in ("q", "k", "v", "alpha", "beta")}
        rs.replayssm_verify_commit(layer, state, rd["acc"][r - 1] if r else None, drafts, y)
    torch.cuda.synchronize()
    return state.status()


def kda(batch=64, steps=20):
    w = wl.make("kda_serving", B=batch)
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = {k: v.cuda() for k, v in g.steps(steps).items()}
    layer = rs.Layer("kda", w.B, w.H, w.P, w.N, window=w.L, in_dtype=w.in_dtype)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    y = torch.empty(w.B, w.H, w.P, device="cuda")
    for t in range(steps):
        rs.replayssm_decode_step(layer, state, {k: st[k][t] for k in st}, y)
    torch.cuda.synchronize()
    return state.status()


def main(argv):
    cases = {"verify": verify, "gdn": gdn, "m2": m2, "gdn_verify": gdn_verify, "kda": kda}
    if len(argv) < 1 or argv[0] not in cases:
        print(__doc__)
        return 2
    status = cases[argv[0]](*(int(a) for a in argv[1:2]))
    print(argv[0], "status", status)
    return 0 if status == 0 else 1


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
