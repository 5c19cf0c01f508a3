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


def _e4m3_value(c):
    """E4M3 decoded from the format definition (OCP MX v1.0 §5.3: 1 sign bit,
    4 exponent bits with bias 7, 3 mantissa bits, subnormals at exponent 0),
    independent of the oracle's decoder; checked against the golden table."""
    s = -1.0 if c & 0x80 else 1.0
    e, m = (c >> 3) & 0xF, c & 7
    return s * (m / 8.0 * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))


def _block_ratios(x, scales, gs):
    """Per 16-element block: its largest magnitude over the block's step s_b * s_g."""
    sb = np.vectorize(_e4m3_value)(scales)
    bmax = np.abs(x).reshape(*x.shape[:-1], -1, 16).max(-1)
    return bmax, bmax / (sb * gs[:, None, None])


def test_nvfp4_block_scale_maps_block_max_to_top_code(oracle_mod):
    """The block scale is fixed by the format, not by the oracle's formula: the
    largest magnitude of every block must land on E2M1's top value 6 within
    the E4M3 rounding of the scale (3 mantissa bits: a relative step of at most
    2^-4 either way), i.e. bmax / (s_b s_g) in [6/(1+2^-4), 6/(1-2^-4)] =
    [5.65, 6.4] whenever the scale bmax / (6 s_g) is an E4M3 normal number.
    A block scale twice too large (bmax -> ~3) or half too small (bmax ->
    ~12, saturating) fails this.  The block holding the tile maximum gets the
    largest finite E4M3 scale, 448, which pins the per-tile scale."""
    for fmt, code, val in read_formats():
        if fmt == "e4m3":
            assert _e4m3_value(code) == val, hex(code)
    rng = np.random.default_rng(3)
    # blocks whose magnitudes span ~5 decades inside one tile, plus zeros
    scale = np.exp(rng.uniform(-6, 3, (6, 16, 8, 1))).repeat(16, -1).reshape(6, 16, 128)
    x = rng.standard_normal((6, 16, 128)) * scale
    x = np.float32(x)
    x[2, 5, 32:48] = 0.0
    codes, scales, gs = oracle_mod.nvfp4_quant(x)
    bmax, ratio = _block_ratios(x, scales, gs)
    lo, hi = 6.0 / (1.0 + 2.0 ** -4), 6.0 / (1.0 - 2.0 ** -4)
    normal = bmax / (6.0 * gs[:, None, None]) >= 2.0 ** -6
    assert normal.sum() > 0.9 * normal.size  # the pin covers nearly every block
    assert np.all((ratio[normal] >= lo) & (ratio[normal] <= hi)), (ratio[normal].min(), ratio[normal].max())
    assert np.all(scales[bmax == 0] == 0)
    for t in range(x.shape[0]):
        r, b = np.unravel_index(np.argmax(bmax[t]), bmax[t].shape)
        assert _e4m3_value(scales[t, r, b]) == 448.0
    # the pin rejects a mis-scaled block scale in either direction
    for wrong in (2.0, 0.5):
        bad = bmax / (np.vectorize(_e4m3_value)(scales) * wrong * gs[:, None, None])
        assert not np.all((bad[normal] >= lo) & (bad[normal] <= hi)), wrong
