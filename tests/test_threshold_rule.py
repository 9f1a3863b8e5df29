"""The quantizer decides codes without a division per weight: for each
group it derives, per nearest-code test, the smallest |x| whose quotient
fl32(|x|/s) passes the test, from the exact rounding boundary next to the
test's midpoint (fp64 product, rounded up to fp32).  This checks that rule
against the plain definition (IEEE fp32 division, then the midpoint compare
with ties to the even index) on inputs placed on and around every boundary.
Host arithmetic only (numpy); no GPU."""
import numpy as np
import pytest

MAGS = {0: [0, .5, 1, 1.5, 2, 2.5, 3, 3.5], 1: [0, .5, 1, 1.5, 2, 3, 4, 6], 2: [0, .25, .5, 1, 2, 4, 8, 16]}


def boundaries(fmt):
    mags = np.array(MAGS[fmt], np.float32)
    mid = (np.float32(0.5) * (mags[:-1] + mags[1:])).astype(np.float32)
    hb, tie = [], []
    for i, m in enumerate(mid):
        if i % 2 == 0:
            lo, hi = m, np.nextafter(m, np.float32(np.inf))
        else:
            lo, hi = np.nextafter(m, np.float32(0)), m
        hb.append(0.5 * (float(lo) + float(hi)))
        tie.append((int(np.array(hi, np.float32).view(np.uint32)) & 1) == 0)
    return mid, hb, tie


def idx_division(ax, s, mid):
    q = np.float32(ax) / np.float32(s)  # IEEE binary32, round to nearest even
    return sum(1 for i, m in enumerate(mid) if q > m or (q == m and i % 2 == 1))


def threshold(hb, tie, s):
    H = hb * float(s)  # exact in fp64
    T = np.float32(H)
    if float(T) < H:
        T = np.nextafter(T, np.float32(np.inf))  # round up to fp32
    if float(T) == H and not tie:
        T = np.nextafter(T, np.float32(np.inf))
    return T


def idx_threshold(ax, s, hb, tie):
    return sum(1 for h, t in zip(hb, tie) if np.float32(ax) >= threshold(h, t, s))


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_threshold_rule_matches_division(fmt):
    mid, hb, tie = boundaries(fmt)
    rng = np.random.default_rng(100 + fmt)
    scales = list(rng.uniform(1e-3, 1.0, 150).astype(np.float32))
    scales += [np.float32(np.float16(v)) for v in rng.uniform(1e-4, 0.1, 100)]  # fp16-representable
    scales += [np.float32(2.0 ** e) for e in range(-10, 4)]
    scales += [np.float32(1e-39), np.float32(3e-42)]  # subnormal scales
    checked = 0
    for s in scales:
        for h in hb:
            base = np.float32(h * float(s))
            cands = [base]
            for _ in range(3):
                cands.append(np.nextafter(cands[-1], np.float32(np.inf)))
            c = base
            for _ in range(3):
                c = np.nextafter(c, np.float32(0))
                cands.append(c)
            for ax in cands:
                assert idx_threshold(ax, s, hb, tie) == idx_division(ax, s, mid), (fmt, float(s), float(ax))
                checked += 1
        for ax in rng.uniform(0, 8 * float(s), 40).astype(np.float32):
            assert idx_threshold(ax, s, hb, tie) == idx_division(ax, s, mid)
    assert checked > 1000
