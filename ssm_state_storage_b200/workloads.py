"""Seeded synthetic inputs for the SSM-layer decode workloads.

This module only draws random numbers in the distributions the workloads name
and rounds them once to their storage dtypes; it contains none of the decode
arithmetic.  It is the single source of inputs for both the CUDA path and the
CPU oracle.

Every sequence b owns a torch CPU generator seeded from (workload seed, b), so
the inputs of a sequence do not depend on the batch size or on how many steps
are drawn: a subset of sequences, or a prefix of the steps, is bit-identical to
the corresponding slice of the full draw.  Draw order per sequence: initial
state, then per step the step's tensors in the order listed below.  Per-head
parameters (A, D) come from a generator seeded by the workload seed alone.
All draws are float64 and are rounded once to the storage dtype.

Workloads (sizes of the SSM layer decode step):
  m2_tiny      Mamba-2, batch 4, 8 heads, headdim 64, d_state 64, 1 group,
               fp32 inputs, 64 steps, window 16 (4 flushes).
  m2_serving   Mamba-2, batch 256, 128 heads, headdim 64, d_state 128,
               16 groups (8 heads share B/C), bf16 inputs, fp32 checkpoint,
               512 steps, window 16.
  gdn_serving  Gated DeltaNet, batch 256, 32 heads, d_k = d_v = 128, bf16
               q/k/v, fp32 alpha/beta, fp32 checkpoint, 512 steps, window 16.
  m2_readcopy  m2_serving shapes at batch 64 over 8192 steps.
  m2_verify    m2_serving heads at batch 512, 4 drafts per round, 256 rounds.
  gdn_verify   gdn_serving heads at batch 256, 4 drafts per round, 256 rounds.
  kda_serving  Kimi Delta Attention on the gdn_serving shapes (batch 256, 32
               heads, d_k = d_v = 128), one decay per key channel.

Distributions: x, B, C ~ N(0,1); dt = softplus(N(0,1) - 2);
A_h = -exp(U(0, ln 16)); D_h ~ N(0,1); initial state 0.1 * N(0,1) (standard
deviation 0.1); GDN q, k ~ N(0,1) then L2-normalised; v ~ N(0,1);
alpha = exp(-softplus(N(0,1))) (KDA: drawn per key channel); beta =
sigmoid(N(0,1)); verify acceptance length ~ Uniform{0..n_draft}.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

F32, BF16 = torch.float32, torch.bfloat16


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "m2" or "gdn"
    B: int
    H: int
    P: int               # M2 headdim; GDN d_v
    N: int               # M2 d_state; GDN d_k
    G: int               # M2 groups; GDN: == H
    T: int               # decode steps (or verify rounds for m2_verify)
    L: int = 16          # window (buffer length)
    in_dtype: torch.dtype = BF16
    seed: int = 1000
    n_draft: int = 0

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "m2_tiny": Workload("m2_tiny", "m2", B=4, H=8, P=64, N=64, G=1, T=64, in_dtype=F32, seed=1000),
    "m2_serving": Workload("m2_serving", "m2", B=256, H=128, P=64, N=128, G=16, T=512, seed=1001),
    "gdn_serving": Workload("gdn_serving", "gdn", B=256, H=32, P=128, N=128, G=32, T=512, seed=1002),
    "m2_readcopy": Workload("m2_readcopy", "m2", B=64, H=128, P=64, N=128, G=16, T=8192, seed=1003),
    "m2_verify": Workload("m2_verify", "m2", B=512, H=128, P=64, N=128, G=16, T=256, seed=1004,
                          n_draft=4),
    "gdn_verify": Workload("gdn_verify", "gdn", B=256, H=32, P=128, N=128, G=32, T=256,
                           seed=1005, n_draft=4),
    "kda_serving": Workload("kda_serving", "kda", B=256, H=32, P=128, N=128, G=32, T=512,
                            seed=1006),
}


def _seq_seed(w: Workload, b: int) -> int:
    return (w.seed * 1_000_003 + 7919 * (b + 1)) % (2**63 - 1)


def _softplus(z):
    return torch.nn.functional.softplus(z)


class _Seq:
    """Per-sequence generator with a step cursor (steps must be drawn in order)."""

    def __init__(self, w: Workload, b: int):
        self.w, self.b = w, b
        self.g = torch.Generator("cpu")
        self.g.manual_seed(_seq_seed(w, b))
        self.state_drawn = False
        self.cursor = 0

    def n(self, *shape):
        return torch.randn(*shape, generator=self.g, dtype=torch.float64)

    def state(self):
        assert not self.state_drawn
        self.state_drawn = True
        w = self.w
        return 0.1 * self.n(w.H, w.P, w.N) if w.kind == "m2" else 0.1 * self.n(w.H, w.N, w.P)

    def m2_step(self):
        w = self.w
        x = self.n(w.H, w.P)
        dt = _softplus(self.n(w.H) - 2.0)
        Bm = self.n(w.G, w.N)
        Cm = self.n(w.G, w.N)
        return x, dt, Bm, Cm

    def gdn_step(self):
        w = self.w
        q = self.n(w.H, w.N)
        k = self.n(w.H, w.N)
        v = self.n(w.H, w.P)
        a = torch.exp(-_softplus(self.n(w.H, w.N) if w.kind == "kda" else self.n(w.H)))
        be = torch.sigmoid(self.n(w.H))
        q = q / q.norm(dim=-1, keepdim=True)
        k = k / k.norm(dim=-1, keepdim=True)
        return q, k, v, a, be

    def accept(self):
        return int(torch.randint(0, self.w.n_draft + 1, (1,), generator=self.g).item())


class Generator:
    """Draws the inputs of workload `w` for sequences `seqs` (default: all)."""

    def __init__(self, w: Workload, seqs=None):
        self.w = w
        self.seqs = list(range(w.B)) if seqs is None else [int(s) for s in seqs]
        self._s = [_Seq(w, b) for b in self.seqs]

    # per-head parameters (Mamba-2) -- independent of the sequence subset
    def params(self):
        w = self.w
        g = torch.Generator("cpu")
        g.manual_seed(w.seed)
        A = -torch.exp(torch.rand(w.H, generator=g, dtype=torch.float64) * math.log(16.0))
        D = torch.randn(w.H, generator=g, dtype=torch.float64)
        return A.to(F32), D.to(F32)

    def initial_state(self) -> torch.Tensor:
        """fp32 [B][H][P][N] (M2) or [B][H][DK][DV] (GDN)."""
        return torch.stack([s.state() for s in self._s]).to(F32)

    def steps(self, T: int):
        """Next T decode steps, stacked [T][B]...  M2: dict(x, dt, Bm, Cm);
        GDN: dict(q, k, v, alpha, beta).  Storage dtypes: x/B/C/dt, q/k/v in
        the workload's input dtype; alpha/beta fp32."""
        w = self.w
        dt_ = w.in_dtype
        if w.kind == "m2":
            xs, dts, Bs, Cs = [], [], [], []
            for _ in range(T):
                row = [s.m2_step() for s in self._s]
                xs.append(torch.stack([r[0] for r in row]).to(dt_))
                dts.append(torch.stack([r[1] for r in row]).to(dt_))
                Bs.append(torch.stack([r[2] for r in row]).to(dt_))
                Cs.append(torch.stack([r[3] for r in row]).to(dt_))
            for s in self._s:
                s.cursor += T
            return dict(x=torch.stack(xs), dt=torch.stack(dts), Bm=torch.stack(Bs),
                        Cm=torch.stack(Cs))
        qs, ks, vs, als, bes = [], [], [], [], []
        for _ in range(T):
            row = [s.gdn_step() for s in self._s]
            qs.append(torch.stack([r[0] for r in row]).to(dt_))
            ks.append(torch.stack([r[1] for r in row]).to(dt_))
            vs.append(torch.stack([r[2] for r in row]).to(dt_))
            als.append(torch.stack([r[3] for r in row]).to(F32))
            bes.append(torch.stack([r[4] for r in row]).to(F32))
        for s in self._s:
            s.cursor += T
        return dict(q=torch.stack(qs), k=torch.stack(ks), v=torch.stack(vs),
                    alpha=torch.stack(als), beta=torch.stack(bes))

    def rounds(self, R: int):
        """Next R speculative rounds: drafts stacked [R][B][Dn]... plus
        acceptance lengths acc[R][B] (int32).  Mamba-2: x, dt, Bm, Cm in the
        input dtype; GDN: q, k, v in the input dtype, alpha, beta fp32."""
        w = self.w
        assert w.n_draft > 0
        dt_ = w.in_dtype
        if w.kind == "m2":
            names, draw = ("x", "dt", "Bm", "Cm"), _Seq.m2_step
            dts = {k: dt_ for k in names}
        else:
            names, draw = ("q", "k", "v", "alpha", "beta"), _Seq.gdn_step
            dts = {"q": dt_, "k": dt_, "v": dt_, "alpha": F32, "beta": F32}
        out = {k: [] for k in names}
        accs = []
        for _ in range(R):
            per = {k: [] for k in out}
            acc_r = []
            for s in self._s:
                ds = [draw(s) for _ in range(w.n_draft)]
                for i, k in enumerate(names):
                    per[k].append(torch.stack([d[i] for d in ds]))
                acc_r.append(s.accept())
            for k in out:
                out[k].append(torch.stack(per[k]).to(dts[k]))
            accs.append(torch.tensor(acc_r, dtype=torch.int32))
        res = {k: torch.stack(v) for k, v in out.items()}
        res["acc"] = torch.stack(accs)
        return res


def make(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.with_(**overrides) if overrides else w
