"""Algorithmic HBM bytes of the decode paths (the roofline numerators).

Counts the bytes a step must move at minimum given the storage layout, not
what the hardware happens to move:
  conventional (full-state) step, per head-token:
      read + write the fp32 state, read the step inputs (x, dt, the group's
      B and C shared by its heads), write y.
  replay step with k records after the append (k = 1..window), per head-token:
      read h0, read the k-1 buffered records (x, dt and the group's B; C of
      past records is never needed), read the step inputs, append the record
      (not on the flush step, whose buffer empties), write y, and on the flush
      step write h0 once.
[sitech.ge, "NVIDIA ו-Dao AI Lab הציגו ReplaySSM…", §Reducing state traffic and
simplifying rollback]: a 16-token window costs 16 state reads and 16 writes
conventionally, against one checkpoint write for ReplaySSM.
"""
from __future__ import annotations


def m2_sizes(P, N, hpg, in_bytes):
    state = P * N * 4
    x = P * in_bytes
    dt_in = in_bytes
    bc_share = 2 * N * in_bytes / hpg      # B and C of the group, per head
    b_share = N * in_bytes / hpg
    y = P * 4
    return state, x, dt_in, bc_share, b_share, y


def m2_conventional_bytes(P, N, hpg, in_bytes):
    state, x, dt_in, bc, _, y = m2_sizes(P, N, hpg, in_bytes)
    return 2 * state + x + dt_in + bc + y


def m2_replay_bytes(k, L, P, N, hpg, in_bytes):
    """Bytes of one replay step for one head whose buffer holds k records
    after the append (the buffered dt is stored as fp32)."""
    state, x, dt_in, bc, b_share, y = m2_sizes(P, N, hpg, in_bytes)
    rec_read = x + 4 + b_share
    flush = k == L
    append = 0 if flush else (x + 4 + bc)
    return state + (k - 1) * rec_read + (x + dt_in + bc) + append + y + (state if flush else 0)


def m2_replay_window_bytes(L, P, N, hpg, in_bytes):
    return sum(m2_replay_bytes(k, L, P, N, hpg, in_bytes) for k in range(1, L + 1))


def rc_tile_bytes(P, N, fmt):
    """Bytes of one head's low-precision read copy: FP8 E4M3 codes, or NVFP4
    E2M1 codes (two per byte) + one E4M3 scale per 16 elements + the fp32
    per-tile scale."""
    if fmt == "fp8":
        return P * N
    if fmt == "nvfp4":
        return P * N // 2 + P * N // 16 + 4
    raise ValueError(fmt)


def m2_replay_bytes_rc(k, L, P, N, hpg, in_bytes, fmt):
    """Replay step whose outputs read the low-precision copy instead of the
    fp32 checkpoint: the copy replaces the fp32 read; on the flush step the fold
    still reads and writes the fp32 checkpoint and writes the new copy."""
    state = P * N * 4
    rc = rc_tile_bytes(P, N, fmt)
    flush = k == L
    return m2_replay_bytes(k, L, P, N, hpg, in_bytes) - state + rc + ((state + rc) if flush else 0)


def m2_replay_window_bytes_rc(L, P, N, hpg, in_bytes, fmt):
    return sum(m2_replay_bytes_rc(k, L, P, N, hpg, in_bytes, fmt) for k in range(1, L + 1))


def gdn_conventional_bytes(DK, DV, in_bytes):
    state = DK * DV * 4
    return 2 * state + (2 * DK + DV) * in_bytes + 8 + DV * 4


def gdn_replay_bytes(k, L, DK, DV, in_bytes):
    """Gated DeltaNet replay step as the kernel runs it: every past record
    contributes its key, its cached u (fp32) and its alpha; this step reads
    q, k, v, alpha, beta, appends them with its u (not on the flush step),
    writes the output, and on the flush step writes the checkpoint."""
    state = DK * DV * 4
    rec_read = DK * in_bytes + DV * 4 + 4
    cur = (2 * DK + DV) * in_bytes + 8
    flush = k == L
    append = 0 if flush else cur + DV * 4
    return state + (k - 1) * rec_read + cur + append + DV * 4 + (state if flush else 0)


def gdn_replay_window_bytes(L, DK, DV, in_bytes):
    return sum(gdn_replay_bytes(k, L, DK, DV, in_bytes) for k in range(1, L + 1))


def gdn_replay_bytes_records(k, L, DK, DV, in_bytes):
    """The same step counted with the plain record of the layer inputs only
    (q, k, v in the input dtype, alpha, beta fp32) and no cached corrections:
    a past record contributes the fields a replay needs (k, v, alpha, beta),
    the current record is read and appended, the output written, and the
    checkpoint written on the flush step."""
    state = DK * DV * 4
    rec_read = (DK + DV) * in_bytes + 8
    cur = (2 * DK + DV) * in_bytes + 8
    flush = k == L
    append = 0 if flush else cur
    return state + (k - 1) * rec_read + cur + append + DV * 4 + (state if flush else 0)


def gdn_replay_window_bytes_records(L, DK, DV, in_bytes):
    return sum(gdn_replay_bytes_records(k, L, DK, DV, in_bytes) for k in range(1, L + 1))


def gdn_verify_round_bytes(n1, fold, nd, DK, DV, in_bytes):
    """One Gated DeltaNet speculative round for one head: read h0, the n1
    committed records (key, cached correction, alpha), the nd drafts (q, k, v,
    alpha, beta); append the drafts with their corrections; write nd outputs;
    write h0 once when the commit folds."""
    state = DK * DV * 4
    rec = DK * in_bytes + DV * 4 + 4
    draft = (2 * DK + DV) * in_bytes + 8
    return (state + n1 * rec + nd * draft + nd * (draft + DV * 4) + nd * DV * 4
            + (state if fold else 0))


def kda_conventional_bytes(DK, DV, in_bytes):
    """Kimi Delta Attention full-state step: read + write the state, read q,
    k, v, the per-channel decay (fp32) and beta, write the output."""
    state = DK * DV * 4
    return 2 * state + (2 * DK + DV) * in_bytes + DK * 4 + 4 + DV * 4


def kda_replay_bytes(k, L, DK, DV, in_bytes):
    """Kimi Delta Attention replay step as the kernel runs it: every past
    record contributes its key, its per-channel decay and its cached
    correction; this step reads q, k, v, alpha, beta, appends them with the
    correction (not on the flush step), writes the output, and on the flush
    step writes the checkpoint."""
    state = DK * DV * 4
    rec_read = DK * in_bytes + DK * 4 + DV * 4
    cur = (2 * DK + DV) * in_bytes + DK * 4 + 4
    flush = k == L
    append = 0 if flush else cur + DV * 4
    return state + (k - 1) * rec_read + cur + append + DV * 4 + (state if flush else 0)


def kda_replay_window_bytes(L, DK, DV, in_bytes):
    return sum(kda_replay_bytes(k, L, DK, DV, in_bytes) for k in range(1, L + 1))
