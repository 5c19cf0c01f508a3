"""Long-horizon decoding on the GPU: the fp32 replay path against the fp64
oracle over many flushes, and the error ordering of the low-precision
variants (read copy over an fp32 checkpoint vs a quantised checkpoint)."""
import numpy as np
import pytest
import torch

import oracle
from ssm_state_storage_b200 import replayssm as rs
from ssm_state_storage_b200 import workloads as wl
from tests import _gpu
from tests._util import norm_err, rel_err

pytestmark = pytest.mark.gpu
T = 1024


def _decode(w, A, D, S0, st, **kw):
    layer = _gpu.layer_for(w, **kw)
    return _gpu.m2_replay_run(w, A, D, S0, st, layer=layer)


@pytest.fixture(scope="module")
def runs():
    w = wl.make("m2_readcopy", B=2, H=16, G=2)
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    st = g.steps(T)
    out = {"fp32": _decode(w, A, D, S0, st)}
    for kind in ("read_fmt", "ckpt_fmt"):
        for fmt in ("fp8", "nvfp4"):
            out[f"{kind}:{fmt}"] = _decode(w, A, D, S0, st, **{kind: fmt})
    yc, _, _, _ = oracle.m2_conventional(S0, st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    return w, out, yc


def test_fp32_replay_matches_oracle_over_64_flushes(runs):
    """1024 steps = 64 windows: per-step error against the fp64 conventional
    recurrence stays within the fp32 tolerance (no accumulation over folds)."""
    w, out, yc = runs
    got = out["fp32"]
    errs = [rel_err(a, b) for a, b in zip(got["y"], yc)]
    assert max(errs) < 1e-4, max(errs)
    assert got["state"].status() == 0


def _curve(out, key):
    ref = out["fp32"]["y"]
    return np.array([norm_err(a, b) for a, b in zip(out[key]["y"], ref)])


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_read_copy_error_stays_bounded_quantised_checkpoint_drifts(runs, fmt):
    """[sitech §Bounding quantisation error]: the read copy's error enters the
    output only, so it does not grow with the horizon; quantising the
    checkpoint itself feeds the error back into the recurrence."""
    w, out, _ = runs
    rc = _curve(out, f"read_fmt:{fmt}")
    ck = _curve(out, f"ckpt_fmt:{fmt}")
    early, late = slice(16, 144), slice(T - 128, T)
    print(fmt, "read copy early/late", rc[early].mean(), rc[late].mean(),
          "checkpoint early/late", ck[early].mean(), ck[late].mean())
    assert rc[late].mean() < 3.0 * rc[early].mean()
    assert ck[late].mean() > rc[late].mean()
