"""Shared helpers of the GPU parity tests (uploading seeded inputs, comparing
selections with the exemptions the method allows, error metrics)."""
from __future__ import annotations

import numpy as np

import oracle
from synth.device import DeviceStep, MappedHostBuffer, bits_of, to_dev  # noqa: F401

# output tolerance for bf16 inputs with fp32 accumulation (max abs / mean abs)
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# a selection may differ from the oracle's only where a cumulative mass lies this
# close to the threshold, or where two blocks' masses tie to this relative precision
MASS_EXEMPT = 1e-5


def selection_lists(idx: np.ndarray, cnt: np.ndarray):
    H, n = cnt.shape
    return [[idx[h, i, :cnt[h, i]].astype(np.int64) for i in range(n)] for h in range(H)]


EXEMPT_LOG = []  # (what, head, row, kind, margin) of every exempt row, for the test log


def check_selection(gpu, ref, probs, tau, what=""):
    """Compare per-row kept block lists.  A differing row is accepted only if
    (a) a cumulative ranked mass lies within MASS_EXEMPT of tau at the cut, or
    (b) the lists have equal length and differ only by blocks whose masses tie
        within MASS_EXEMPT relative.
    Each exempt row is printed and appended to EXEMPT_LOG with its margin (the
    distance of the cumulative mass from tau, or the relative mass gap of the tie).
    Returns (#rows, #exempt rows)."""
    rows = exempt = 0
    for h in range(len(ref)):
        for i in range(len(ref[h])):
            rows += 1
            g = np.asarray(gpu[h][i])
            o = np.asarray(ref[h][i])
            if g.shape == o.shape and np.array_equal(g, o):
                continue
            p = probs[h, i]
            assert len(g) >= 1 and np.all(np.diff(g) > 0) and g.min() >= 0 and g.max() < len(p), (what, h, i, g)
            order = sorted(range(len(p)), key=lambda j: (-p[j], j))
            cum = np.cumsum(p[order])
            lo, hi = min(len(g), len(o)), max(len(g), len(o))
            gaps = [abs(cum[k - 1] - tau[h]) for k in range(max(lo, 1), hi + 1)]
            near = min(gaps) <= MASS_EXEMPT
            tie, gap = False, float("inf")
            if len(g) == len(o):
                pin = p[g].min()
                pout = np.delete(p, g).max() if len(g) < len(p) else -1.0
                gap = (pout - pin) / max(p.max(), 1e-30)
                tie = pin >= pout - MASS_EXEMPT * max(p.max(), 1e-30)
            assert near or tie, (what, h, i, g.tolist(), o.tolist(), float(cum[lo - 1]), float(tau[h]))
            kind, margin = ("threshold", float(min(gaps))) if near else ("tie", float(gap))
            EXEMPT_LOG.append((what, h, i, kind, margin))
            print(f"exempt row {what} h={h} i={i}: {kind} margin {margin:.3e} (gpu {g.tolist()} oracle {o.tolist()})")
            exempt += 1
    return rows, exempt


def check_selection_both(gpu_inter, gpu_intra, Q, Kc, Kq, tau, what="", max_frac=0.01):
    """GPU selections against the oracle twice: with the block means and scores that
    decide the lists rounded to fp32 (the kernels' precision), and in fp64 throughout.
    The same exemptions apply to both; exempt rows stay rare (<= max_frac)."""
    out = {}
    for dt in (np.float32, np.float64):
        ref = oracle.block_select(Q, Kc, Kq, tau, dtype=dt)
        n1, e1 = check_selection(gpu_inter, ref.inter, ref.p_inter, tau, f"{what} inter {dt.__name__}")
        n2, e2 = check_selection(gpu_intra, ref.intra, ref.p_intra, tau, f"{what} intra {dt.__name__}")
        assert e1 + e2 <= max(2, int((n1 + n2) * max_frac)), (what, dt, e1, e2, n1, n2)
        out[dt.__name__] = (n1 + n2, e1 + e2)
    return out


def check_pages(gpu_sel, ref_sel, scores, Kp):
    """Page selections equal, unless the Kp-th and (Kp+1)-th scores tie within 1e-5 relative."""
    if np.array_equal(np.sort(gpu_sel), np.sort(ref_sel)):
        return False
    s = np.sort(scores[np.isfinite(scores)])[::-1]
    assert len(s) > Kp and abs(s[Kp - 1] - s[Kp]) <= 1e-5 * np.abs(s).max(), (gpu_sel, ref_sel)
    return True


def errors(got, ref):
    d = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))
    return float(d.max()), float(d.mean())


def assert_close(got, ref, what="", max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    assert np.all(np.isfinite(got)), what
    mx, mn = errors(got, ref)
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max abs {mx:.3e} (<= {max_abs}), mean abs {mn:.3e} (<= {mean_abs})"
    return mx, mn


def sample_rows(Lq: int, n: int, seed: int = 0) -> np.ndarray:
    """Rows spanning the chunk: first/last of every few blocks plus the ragged tail."""
    rng = np.random.default_rng(seed)
    fixed = {0, 63, 64, 127, 128, Lq - 1, Lq - 2, (Lq // 64) * 64, max(0, (Lq // 128) * 128 - 1)}
    fixed = {r for r in fixed if 0 <= r < Lq}
    rest = rng.choice(Lq, size=min(Lq, max(0, n - len(fixed))), replace=False)
    return np.array(sorted(fixed | set(rest.tolist())), dtype=np.int64)
