"""The algorithmic byte model (the roofline numerators) against sizes written
out from the storage layout: fp32 state tiles, bf16 inputs, fp32 buffered dt,
the read-copy formats (FP8: one byte per element; NVFP4: half a byte per
element, one E4M3 scale per 16 elements, one fp32 scale per tile)."""
from ssm_state_storage_b200 import bytes_model as bm

P, N, HPG, IN = 64, 128, 8, 2
STATE = P * N * 4                    # 32768
X, DT, Y = P * IN, IN, P * 4         # 128, 2, 256
BC = 2 * N * IN / HPG                # B and C of the group, per head: 64
B_SHARE = N * IN / HPG               # B of a buffered record, per head: 32
REC = X + 4 + B_SHARE                # buffered x, fp32 dt, B: 164


def test_replay_step_bytes_from_the_layout():
    cur = X + DT + BC                   # this step's inputs: 194
    app = X + 4 + BC                    # its record appended: 196
    assert bm.m2_replay_bytes(1, 16, P, N, HPG, IN) == STATE + cur + app + Y
    assert bm.m2_replay_bytes(9, 16, P, N, HPG, IN) == STATE + 8 * REC + cur + app + Y
    # the flush step appends nothing and writes the checkpoint once
    assert bm.m2_replay_bytes(16, 16, P, N, HPG, IN) == 2 * STATE + 15 * REC + cur + Y
    assert bm.m2_conventional_bytes(P, N, HPG, IN) == 2 * STATE + cur + Y


def test_read_copy_bytes_from_the_formats():
    assert bm.rc_tile_bytes(P, N, "fp8") == 8192
    assert bm.rc_tile_bytes(P, N, "nvfp4") == 4096 + 512 + 4
    for fmt in ("fp8", "nvfp4"):
        rc = bm.rc_tile_bytes(P, N, fmt)
        for k in (1, 7, 15):  # non-flush: the copy replaces the fp32 read
            assert bm.m2_replay_bytes_rc(k, 16, P, N, HPG, IN, fmt) == \
                bm.m2_replay_bytes(k, 16, P, N, HPG, IN) - STATE + rc
        # flush: copy read for the output, fp32 read + write for the fold, new copy written
        assert bm.m2_replay_bytes_rc(16, 16, P, N, HPG, IN, fmt) == \
            bm.m2_replay_bytes(16, 16, P, N, HPG, IN) + 2 * rc


def test_window_ratio_is_about_half():
    """[sitech §Reducing state traffic]: the dominant traffic is roughly halved."""
    r = bm.m2_replay_window_bytes(16, P, N, HPG, IN) / (16 * bm.m2_conventional_bytes(P, N, HPG, IN))
    assert 0.5 < r < 0.6
