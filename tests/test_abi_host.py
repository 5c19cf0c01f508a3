"""The C-ABI library loads and exports every entry point the header declares;
host-side validation answers without touching a GPU (no compute calls here)."""
import ctypes as C
import os
import re

import pytest
import torch

from ssm_state_storage_b200 import replayssm as rs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


def _declared():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if fn.endswith(".h"):
            txt = open(os.path.join(HEADER_DIR, fn)).read()
            names |= set(re.findall(r"^[A-Za-z_][\w \*]*?\b(replayssm_\w+)\s*\(", txt, re.M))
    return names


@pytest.fixture(scope="module")
def lib():
    from ssm_state_storage_b200 import build
    build.build()
    return rs.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 12
    for n in sorted(names):
        assert hasattr(lib, n), n
    assert names <= set(rs.ENTRY_POINTS), names - set(rs.ENTRY_POINTS)


def _m2(**kw):
    base = dict(kind="m2", batch=256, nheads=128, headdim=64, dstate=128, ngroups=16)
    base.update(kw)
    return rs.Layer(**base)


def test_validation_and_sizes(lib):
    L = _m2()
    assert rs.replayssm_validate(L) == 0
    assert L.capacity() == 16
    assert _m2(draft_max=4).capacity() == 19
    assert L.nbytes("h0") == 256 * 128 * 64 * 128 * 4
    assert L.nbytes("buf0") == 256 * 128 * 16 * 64 * 2
    assert L.nbytes("buf2") == 256 * 16 * 16 * 128 * 2
    assert L.nbytes("len") == 256 * 128 * 4
    assert _m2(read_fmt="nvfp4").nbytes("rc") == 256 * 128 * 64 * 64
    assert _m2(read_fmt="nvfp4").nbytes("rc_scale") == 256 * 128 * 64 * 8
    assert rs.replayssm_validate(_m2(headdim=96)) == 2          # shape
    assert rs.replayssm_validate(_m2(ngroups=3)) == 2            # H % G
    assert rs.replayssm_validate(_m2(window=17)) == 5            # capacity
    assert rs.replayssm_validate(_m2(draft_max=5)) == 5
    assert rs.replayssm_validate(_m2(read_fmt="fp8", ckpt_fmt="fp8")) == 1
    g = rs.Layer("gdn", 8, 32, 128, 128)
    assert rs.replayssm_validate(g) == 0 and g.capacity() == 16
    assert rs.replayssm_validate(rs.Layer("gdn", 8, 32, 64, 128)) == 2
    assert rs.replayssm_validate(rs.Layer("gdn", 8, 32, 128, 128, draft_max=2)) == 0
    assert rs.Layer("gdn", 8, 32, 128, 128, draft_max=4).capacity() == 19
    assert rs.replayssm_validate(rs.Layer("gdn", 8, 32, 128, 128, read_fmt="fp8")) == 8
    assert rs.replayssm_status_string(9) == "buffer state out of range"


def test_null_arguments_rejected_before_launch(lib):
    L = _m2(batch=2)
    d = L.desc()
    st = rs.State()
    si = rs.StepIn()
    # no CUDA call is made: every check fails first
    assert lib.replayssm_decode_step(C.byref(d), C.byref(st), C.byref(si), None, None) == 1
    assert lib.replayssm_decode_step(None, C.byref(st), C.byref(si), None, None) == 1
    assert lib.replayssm_flush(C.byref(d), None, None, 0, None) == 1
    assert lib.replayssm_verify_commit(C.byref(d), C.byref(st), None, C.byref(si), 1, None,
                                       None) in (1, 5)
    assert lib.replayssm_quantize(7, 1, 1, 16, None, None, None, None, None) == 1


def test_cpu_tensors_are_refused():
    """The binding refuses host tensors for device arguments: there is no CPU path."""
    L = _m2(batch=1, nheads=8, ngroups=1)
    x = torch.zeros(1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(rs.ReplayError):
        rs._step_in(L, dict(x=x, dt=x[..., 0], Bm=x, Cm=x, A=torch.zeros(8), D=torch.zeros(8)))


def test_empty_batch_returns_ok_without_reading_pointers(lib):
    """batch = 0: every stateful call answers RSSM_OK on the host, with null
    state and input pointers, and launches nothing; argument kinds the call
    cannot serve are still refused."""
    st, si = rs.State(), rs.StepIn()
    for kind in ("m2", "gdn"):
        L = _m2(batch=0) if kind == "m2" else rs.Layer("gdn", 0, 32, 128, 128)
        d = L.desc()
        assert lib.replayssm_init(C.byref(d), C.byref(st), None, None) == 0
        assert lib.replayssm_decode_step(C.byref(d), C.byref(st), C.byref(si), None, None) == 0
        assert lib.replayssm_flush(C.byref(d), C.byref(st), None, 1, None) == 0
        assert lib.replayssm_full_decode_step(C.byref(d), None, C.byref(si), None, None, 0,
                                              None) == 0
        assert lib.replayssm_materialize(C.byref(d), C.byref(st), None, None, None) == 0
    d = _m2(batch=0, draft_max=4).desc()
    assert lib.replayssm_verify_commit(C.byref(d), C.byref(st), None, C.byref(si), 4, None,
                                       None) == 0
    assert lib.replayssm_commit(C.byref(d), C.byref(st), None, None, None) == 0
    g = rs.Layer("gdn", 0, 32, 128, 128, draft_max=4).desc()
    assert lib.replayssm_verify_commit(C.byref(g), C.byref(st), None, C.byref(si), 4, None,
                                       None) == 0
    assert lib.replayssm_commit(C.byref(g), C.byref(st), None, None, None) == 0
    g = rs.Layer("gdn", 0, 32, 128, 128, read_fmt="fp8").desc()
    assert lib.replayssm_verify_commit(C.byref(g), C.byref(st), None, C.byref(si), 1, None,
                                       None) == 8          # no GDN read copy


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses never-dereferenced fake device addresses: host-only check")
def test_host_checks_on_fake_addresses(lib):
    """Alignment, draft-count and draft-row checks answer before any launch.
    The addresses are fake (never dereferenced); every call returns at a host
    check, so the test runs only where no GPU is present."""
    L = _m2(batch=2, nheads=16, ngroups=2, draft_max=4)
    d = L.desc()
    st = rs.State()
    ok = 0x10000
    st.h0, st.len, st.status = C.c_void_p(ok), C.c_void_p(ok), C.c_void_p(ok)
    for i in range(4):
        st.buf[i] = ok
    si = rs.StepIn()
    for i in range(4):
        si.in_[i] = ok
    si.A = si.D = C.c_void_p(ok)
    st.h0 = C.c_void_p(ok + 4)                               # misaligned checkpoint
    assert lib.replayssm_decode_step(C.byref(d), C.byref(st), C.byref(si), C.c_void_p(ok),
                                     None) == 4
    st.h0 = C.c_void_p(ok)
    assert lib.replayssm_verify_commit(C.byref(d), C.byref(st), None, C.byref(si), 5,
                                       C.c_void_p(ok), None) == 5   # n_draft > draft_max
    assert lib.replayssm_verify_commit(C.byref(d), C.byref(st), None, C.byref(si), 0,
                                       C.c_void_p(ok), None) == 5   # n_draft < 1
    si.in_[0] = ok + 2                                       # misaligned draft x rows
    assert lib.replayssm_verify_commit(C.byref(d), C.byref(st), None, C.byref(si), 4,
                                       C.c_void_p(ok), None) == 4
    si.in_[0] = ok
    si.batch_stride[2] = 2 * 16 * 128 + 1                    # B batch stride not 16-byte
    assert lib.replayssm_verify_commit(C.byref(d), C.byref(st), None, C.byref(si), 4,
                                       C.c_void_p(ok), None) == 4
    big = _m2(batch=2, nheads=32, ngroups=2, draft_max=4).desc()   # 16 heads per group
    assert lib.replayssm_verify_commit(C.byref(big), C.byref(st), None, C.byref(si), 4,
                                       C.c_void_p(ok), None) == 8


def test_test_hooks_entry_point_validates_and_resets():
    from ssm_state_storage_b200 import replayssm as rs
    with pytest.raises(rs.ReplayError, match="invalid"):
        rs.replayssm_set_test_hooks(1000, -2)
    rs.replayssm_set_test_hooks(1000, 3)
    rs.replayssm_set_test_hooks()  # back to the defaults


def test_kda_descriptor_and_sizes():
    from ssm_state_storage_b200 import replayssm as rs
    L = rs.Layer("kda", 4, 8, 128, 128)
    assert rs.replayssm_validate(L) == 0
    assert L.nbytes("buf3") == 4 * 8 * 16 * 128 * 4     # one decay per key channel
    assert L.nbytes("buf4") == 4 * 8 * 16 * 4
    assert L.nbytes("buf5") == 4 * 8 * 16 * 128 * 4
    assert rs.replayssm_validate(rs.Layer("kda", 4, 8, 128, 128, draft_max=2)) == 8
    assert rs.replayssm_validate(rs.Layer("kda", 4, 8, 64, 128)) == 2
