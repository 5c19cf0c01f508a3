"""Shared test helpers (comparison metrics and fixture readers)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rel_err(got, ref, axis_rms=None):
    """Max element error relative to max(|ref|, 1e-2 * rms(ref)).

    Element-wise relative error is undefined where the reference crosses zero,
    so each element's error is scaled by its own magnitude but never by less
    than one hundredth of the RMS of the whole output tensor.
    """
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    den = np.maximum(np.abs(ref), 1e-2 * rms)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(got - ref) / den)) if ref.size else 0.0


def norm_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (d if d else 1.0))


def per_step_rel_err(got, ref):
    """rel_err evaluated separately for every leading-axis slice; returns the max."""
    return max(rel_err(g, r) for g, r in zip(got, ref))


class Worst(float):
    """A float (the error) that also describes where the worst element is."""

    def __new__(cls, value, where):
        obj = super().__new__(cls, value)
        obj.where = where
        return obj

    def __repr__(self):
        return f"{float(self):.3e} ({self.where})"


def worst_step_err(got, ref):
    """per_step_rel_err plus the step, index and values of the worst element."""
    best = Worst(0.0, "")
    for t, (g, r) in enumerate(zip(got, ref)):
        g = np.asarray(g, np.float64)
        r = np.asarray(r, np.float64)
        rms = np.sqrt(np.mean(r * r)) if r.size else 0.0
        den = np.maximum(np.abs(r), 1e-2 * rms)
        den = np.where(den == 0, 1.0, den)
        e = np.abs(g - r) / den
        i = int(np.argmax(e))
        if e.flat[i] > best:
            idx = np.unravel_index(i, r.shape)
            best = Worst(float(e.flat[i]), f"step {t} index {tuple(int(v) for v in idx)} got "
                         f"{g.flat[i]:.9g} ref {r.flat[i]:.9g} rms {rms:.4g}")
    return best


def read_kv(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()
            out[k] = int(v)
    return out


def read_formats(name="ocp_formats.txt"):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fmt, code, val = line.split()
            rows.append((fmt, int(code, 16), float(val)))
    return rows
