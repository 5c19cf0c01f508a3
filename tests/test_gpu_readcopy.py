"""Low-precision read copy on the GPU: codes bit-exact against the oracle's
codec on the same fp32 input, the fp32 recurrence untouched by the copy, and
output error within the per-format bounds."""
import numpy as np
import pytest
import torch

import oracle
from ssm_state_storage_b200 import replayssm as rs
from ssm_state_storage_b200 import workloads as wl
from tests import _gpu
from tests._util import norm_err, per_step_rel_err

pytestmark = pytest.mark.gpu

# Normwise output error of GPU read-copy decoding against the oracle running
# the same read format, per step.  The copy is built from each side's own fp32
# checkpoint, so a code can land one step apart where the two checkpoints
# straddle a rounding boundary; the bounds allow for that.
BOUND = {"fp8": 1e-3, "nvfp4": 1e-2}


def _special_values(n, rng):
    x = rng.standard_normal(n).astype(np.float32) * np.exp(rng.uniform(-12, 7, n)).astype(np.float32)
    x[:64] = 0.0
    x[64:128] = -0.0
    x[128:192] = np.float32(1e-30)
    x[192:256] = np.float32(600.0)
    x[256:320] = -np.float32(5000.0)
    return x


@pytest.mark.parametrize("rows,cols", [(64, 128), (64, 64), (128, 128)])
def test_quantize_codes_bit_exact(rows, cols):
    rng = np.random.default_rng(rows * 7 + cols)
    ntile = 24
    x = _special_values(ntile * rows * cols, rng).reshape(ntile, rows, cols)
    x[3] = 0.0                     # an all-zero tile
    x[5] *= np.float32(1e-6)       # a tiny tile: block scales near E4M3 subnormals
    xd = torch.from_numpy(x).cuda()
    c8 = torch.empty(ntile, rows, cols, dtype=torch.uint8, device="cuda")
    rs.replayssm_quantize("fp8", xd, c8)
    assert np.array_equal(c8.cpu().numpy(), oracle.fp8_quant(x))
    c4 = torch.empty(ntile, rows, cols // 2, dtype=torch.uint8, device="cuda")
    sc = torch.empty(ntile, rows, cols // 16, dtype=torch.uint8, device="cuda")
    gs = torch.empty(ntile, device="cuda")
    rs.replayssm_quantize("nvfp4", xd, c4, sc, gs)
    oc, osc, ogs = oracle.nvfp4_quant(x)
    assert np.array_equal(gs.cpu().numpy(), ogs)
    assert np.array_equal(sc.cpu().numpy(), osc)
    assert np.array_equal(c4.cpu().numpy(), oc)


def _run(fmt_kind, fmt, T=48, B=2, H=16, G=2):
    w = wl.make("m2_readcopy", B=B, H=H, G=G)
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    st = g.steps(T)
    kw = {fmt_kind: fmt} if fmt != "none" else {}
    layer = _gpu.layer_for(w, **kw)
    got = _gpu.m2_replay_run(w, A, D, S0, st, layer=layer)
    return w, A, D, S0, st, got


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_read_copy_keeps_fp32_checkpoint(fmt):
    """[sitech §Bounding quantisation error]: the read copy never feeds the
    recurrence, so the fp32 checkpoints are bit-identical with it on or off;
    the fused fold epilogue writes the same codes the standalone quantiser
    produces from the stored checkpoint."""
    w, A, D, S0, st, ref = _run("read_fmt", "none")
    _, _, _, _, _, got = _run("read_fmt", fmt)
    assert torch.equal(got["state"].h0, ref["state"].h0)
    s = got["state"]
    if fmt == "fp8":
        c = torch.empty_like(s.rc)
        rs.replayssm_quantize("fp8", s.h0, c)
        assert torch.equal(c, s.rc)
    else:
        c, sc, gs = torch.empty_like(s.rc), torch.empty_like(s.rc_scale), torch.empty_like(s.rc_gscale)
        rs.replayssm_quantize("nvfp4", s.h0, c, sc, gs)
        assert torch.equal(c, s.rc) and torch.equal(sc, s.rc_scale) and torch.equal(gs, s.rc_gscale)
    assert 0 < norm_err(got["y"], ref["y"]) < 0.2


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
@pytest.mark.parametrize("kind", ["read_fmt", "ckpt_fmt"])
def test_low_precision_outputs_match_oracle(kind, fmt):
    w, A, D, S0, st, got = _run(kind, fmt)
    orc = oracle.M2Replay(S0, G=w.G, L=w.L, **{kind: fmt})
    y, lt, _ = orc.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    assert np.array_equal(got["len"], lt)
    errs = [norm_err(a, b) for a, b in zip(got["y"], y)]
    assert max(errs) < BOUND[fmt], (kind, fmt, max(errs))
    if kind == "ckpt_fmt" and fmt == "fp8":
        # the stored checkpoint holds only FP8-representable values
        h = got["state"].h0
        c = torch.empty(h.shape, dtype=torch.uint8, device="cuda")
        rs.replayssm_quantize("fp8", h, c)
        np.testing.assert_array_equal(oracle.fp8_dequant(c.cpu().numpy()), h.cpu().numpy())


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_read_copy_full_batch_sampled(fmt):
    """m2_readcopy at its batch of 64 (many work items per CTA, the read-copy
    ring layout) over 20 steps including a flush; 2 sequences checked."""
    w = wl.make("m2_readcopy")
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    st = g.steps(20)
    got = _gpu.m2_replay_run(w, A, D, S0, st, layer=_gpu.layer_for(w, read_fmt=fmt))
    assert got["state"].status() == 0
    seqs = [0, 63]
    sub = {k: v[:, seqs] for k, v in st.items()}
    orc = oracle.M2Replay(S0[seqs], G=w.G, L=w.L, read_fmt=fmt)
    y, lt, _ = orc.decode(sub["x"], sub["dt"], sub["Bm"], sub["Cm"], A, D)
    assert np.array_equal(got["len"][:, seqs], lt)
    errs = [norm_err(a, b) for a, b in zip(got["y"][:, seqs], y)]
    assert max(errs) < BOUND[fmt], max(errs)
