"""Pins for the low-precision read-copy formats and the read-copy semantics of
the CPU oracle (no GPU)."""
import numpy as np
import pytest

from ssm_state_storage_b200 import workloads as wl
from tests._util import norm_err, read_formats

E4M3_FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_format_tables_match_spec(oracle_mod):
    for fmt, code, val in read_formats():
        dec = oracle_mod.e4m3_decode if fmt == "e4m3" else oracle_mod.e2m1_decode
        assert dec(code) == val, (fmt, hex(code))
    assert np.isnan(oracle_mod.e4m3_decode(0x7F)) and np.isnan(oracle_mod.e4m3_decode(0xFF))


def test_encode_decode_round_trip(oracle_mod):
    for c in E4M3_FINITE:
        v = oracle_mod.e4m3_decode(c)
        assert oracle_mod.e4m3_encode(v) == c, hex(c)
    for c in range(16):
        assert oracle_mod.e2m1_encode(oracle_mod.e2m1_decode(c)) == c


def _argmin_encode(v, values, codes):
    """Independent reference: nearest representable value, ties to the even
    code, magnitudes beyond the largest finite value saturate."""
    a = abs(v)
    mag_codes = [(val, c) for val, c in zip(values, codes) if val >= 0]
    best = min(mag_codes, key=lambda vc: (abs(vc[0] - a), vc[1] % 2))
    c = best[1]
    if a >= max(vc[0] for vc in mag_codes):
        c = max(mag_codes)[1]
    return c


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_encode_is_nearest_even(oracle_mod, fmt):
    if fmt == "e4m3":
        codes = list(range(0x7F))
        dec, enc, sbit = oracle_mod.e4m3_decode, oracle_mod.e4m3_encode, 0x80
    else:
        codes = list(range(8))
        dec, enc, sbit = oracle_mod.e2m1_decode, oracle_mod.e2m1_encode, 0x8
    values = [dec(c) for c in codes]
    rng = np.random.default_rng(0)
    top = max(values)
    samples = list(np.float32(rng.uniform(0, top * 1.2, 3000)))
    samples += list(np.float32(np.exp(rng.uniform(np.log(1e-4), np.log(top), 2000))))
    # exact midpoints and their fp32 neighbours
    for lo, hi in zip(values[:-1], values[1:]):
        m = np.float32((lo + hi) / 2)
        samples += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9))]
    samples += [np.float32(top * 4), np.float32(1e30)]
    for s in samples:
        s = float(s)
        want = _argmin_encode(s, values, codes)
        assert enc(s) == want, (fmt, s)
        assert enc(-s) == (want | sbit), (fmt, -s)


def test_fp8_relative_error_bound(oracle_mod):
    rng = np.random.default_rng(1)
    x = np.float32(rng.standard_normal(20000) * np.exp(rng.uniform(-4, 5, 20000)))
    x = x[np.abs(x) < 448]
    xr = oracle_mod.fp8_dequant(oracle_mod.fp8_quant(x))
    normal = np.abs(x) >= 2.0 ** -6
    # 3 mantissa bits: half an ulp is 2^-4 relative in the normal range
    assert np.all(np.abs(xr - x)[normal] <= 2.0 ** -4 * np.abs(x[normal]))
    # subnormal spacing 2^-9: error at most 2^-10
    assert np.all(np.abs(xr - x)[~normal] <= 2.0 ** -10)


def test_nvfp4_tile_structure_and_bound(oracle_mod):
    rng = np.random.default_rng(2)
    x = np.float32(0.3 * rng.standard_normal((3, 8, 64)))
    x[1, 2, 16:32] = 0.0  # an all-zero block
    codes, scales, gs = oracle_mod.nvfp4_quant(x)
    assert codes.shape == (3, 8, 32) and scales.shape == (3, 8, 4) and gs.shape == (3,)
    np.testing.assert_allclose(gs, np.abs(x).reshape(3, -1).max(1) / 2688.0, rtol=1e-7)
    xr = oracle_mod.nvfp4_dequant(codes, scales, gs)
    assert np.all(xr[1, 2, 16:32] == 0) and scales[1, 2, 1] == 0
    # per-block step d = s_b * s_g; E2M1 spacing is at most 2 (between 4 and 6),
    # and the largest magnitude in a block lands within [5.6, 6.4] * d, so the
    # error never exceeds one d
    sb = np.vectorize(oracle_mod.e4m3_decode)(scales).astype(np.float32)
    d = np.repeat(sb * gs[:, None, None], 16, axis=-1)
    assert np.all(np.abs(xr - x) <= d * (1 + 1e-6))
    # codes: even element in the low nibble
    lo = codes & 0xF
    v0 = np.vectorize(oracle_mod.e2m1_decode)(lo) * d[..., 0::2]
    np.testing.assert_allclose(v0, xr[..., 0::2], rtol=1e-6, atol=0)


def _drift_run(oracle_mod, T, read_fmt="none", ckpt_fmt="none"):
    w = wl.make("m2_readcopy", B=1, H=16, G=2)
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    st = g.steps(T)
    rp = oracle_mod.M2Replay(S0, G=w.G, L=w.L, read_fmt=read_fmt, ckpt_fmt=ckpt_fmt)
    y, _, _ = rp.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    return rp, y


def test_read_copy_leaves_recurrence_untouched(oracle_mod):
    """[sitech §Bounding quantisation error]: the low-precision copy serves reads
    only, so the high-precision checkpoints are the same with it on or off."""
    ref, y_ref = _drift_run(oracle_mod, 48)
    for fmt in ("fp8", "nvfp4"):
        rp, y = _drift_run(oracle_mod, 48, read_fmt=fmt)
        np.testing.assert_array_equal(rp.h0, ref.h0)
        np.testing.assert_array_equal(rp.rec_x, ref.rec_x)
        assert 0 < norm_err(y, y_ref) < 0.1


def test_quantised_checkpoint_is_representable(oracle_mod):
    rp, _ = _drift_run(oracle_mod, 32, ckpt_fmt="fp8")
    f = rp.h0.astype(np.float32)
    np.testing.assert_array_equal(oracle_mod.fp8_dequant(oracle_mod.fp8_quant(f)), f)


@pytest.mark.slow
def test_read_copy_error_does_not_accumulate(oracle_mod):
    """Qualitative ordering only (magnitudes are not pinned by the pages): over
    a long run the output error of read-copy decoding stays below that of
    storing the checkpoint itself in the same format."""
    T = 256
    _, y_ref = _drift_run(oracle_mod, T)
    for fmt in ("fp8", "nvfp4"):
        _, y_rc = _drift_run(oracle_mod, T, read_fmt=fmt)
        _, y_q = _drift_run(oracle_mod, T, ckpt_fmt=fmt)
        tail = slice(T - 64, T)
        e_rc = norm_err(y_rc[tail], y_ref[tail])
        e_q = norm_err(y_q[tail], y_ref[tail])
        assert e_rc < e_q, (fmt, e_rc, e_q)
