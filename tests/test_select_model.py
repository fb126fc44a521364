"""The selection kernel's algorithm, replayed on the CPU against the oracle's selection.

The GPU select kernels do not sort. They map fp32 scores to order-preserving unsigned keys
and take the best candidates in one of three ways: repeated argmax (largest key, then
lowest tile index) when a few are needed, or a bitwise binary search for a threshold key
(with an early exit when the count is exact), or (the fixed and budget modes' radix
kernel) a search that narrows a key range from the candidates' [min, max] through at most
256 buckets of 2^shift keys per pass, ending early on a bucket that holds exactly the keys
still needed; each is followed by taking tied keys in index order. The
cumulative-mass mode searches the fp32 bits of positive pooled probabilities and counts mass
instead of keys. This module replays those steps in NumPy, with the kernel's fp32
arithmetic, and checks on many random rows with heavy ties that they select exactly what a
plain sort (the oracle's top_outside) selects. It pins the algorithm the kernel implements,
not the kernel itself; the GPU parity tests pin the kernel.
"""
import numpy as np
import pytest

from oracle import bsa_oracle as O


def order_key(f: np.ndarray) -> np.ndarray:
    f = np.where(f == 0.0, np.float32(0.0), f.astype(np.float32))
    u = f.view(np.uint32)
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def select_by_count(keys: np.ndarray, cand: np.ndarray, extra: int) -> np.ndarray:
    """Candidates (bool mask) the kernel selects for `extra` extra tiles."""
    kr = np.where(cand, keys, 0).astype(np.uint64)
    ncand = int(cand.sum())
    extra = max(0, min(extra, ncand))
    idx = np.arange(kr.size, dtype=np.uint64)
    if extra == 0:
        thr, need_eq = 0xFFFFFFFF, 0
    elif extra == ncand:
        thr, need_eq = 1, 0
    elif extra <= 32:
        kr = kr.copy()
        for _ in range(extra):
            v = (kr << np.uint64(32)) | (np.uint64(0xFFFFFFFF) - idx)
            ok = (kr > 1) & (kr != 0xFFFFFFFF)
            best = int(np.where(ok, v, 0).max())
            jbest = 0xFFFFFFFF - (best & 0xFFFFFFFF)
            kr[jbest] = 0xFFFFFFFF
        thr, need_eq = 0xFFFFFFFE, 0
    else:
        t, exact = 0, False
        for bit in range(31, -1, -1):
            if exact:
                break
            cand_t = t | (1 << bit)
            c = int((kr >= cand_t).sum())
            if c >= extra:
                t = cand_t
            exact = c == extra
        if exact:
            thr, need_eq = t - 1, 0
        else:
            thr, need_eq = t, extra - int((kr > t).sum())
    eq = cand & (kr == thr)
    rank = np.cumsum(eq) - eq
    return cand & ((kr > thr) | (eq & (rank < need_eq)))


def select_by_range(keys: np.ndarray, cand: np.ndarray, extra: int, bucket_bits: int = 8) -> np.ndarray:
    """The radix kernel's selection: keys >= t_ge, plus the first need_eq keys equal to thr
    in index order. bucket_bits = 8 is the kernel (at most 2^8 buckets per pass)."""
    kr = np.where(cand, keys, 0).astype(np.uint64)
    ncand = int(cand.sum())
    extra = max(0, min(extra, ncand))
    thr, need_eq = 0, 0
    if extra == 0:
        t_ge = 0xFFFFFFFF + 1                      # nothing
    elif extra == ncand:
        t_ge = 1
    else:
        lo, hi = int(kr[cand].min()), int(kr[cand].max())
        remaining, done = extra, False
        while not done:
            span = hi - lo
            shift = 0 if span < (1 << bucket_bits) else span.bit_length() - bucket_bits
            inr = cand & (kr >= lo) & (kr <= hi)
            bucket = (kr[inr].astype(np.int64) - lo) >> shift
            cnt = np.bincount(bucket, minlength=1 << bucket_bits)
            suf = np.cumsum(cnt[::-1])[::-1]
            d = int(np.nonzero(suf >= remaining)[0].max())
            above = int(suf[d + 1]) if d + 1 < cnt.size else 0
            at = int(cnt[d])
            remaining -= above
            blo = lo + (d << shift)
            bhi = min(hi, blo + (1 << shift) - 1)
            if at == remaining:
                t_ge, done = blo, True
            elif shift == 0:
                thr, t_ge, need_eq, done = blo, blo + 1, remaining, True
            lo, hi = blo, bhi
    eq = cand & (kr == thr) & (need_eq > 0)
    rank = np.cumsum(eq) - eq
    return cand & ((kr >= t_ge) | (eq & (rank < need_eq)))


def select_by_mass(e: np.ndarray, cand: np.ndarray, need: np.float32) -> np.ndarray:
    """Cumulative-mass mode: e are the unnormalised fp32 pooled probabilities."""
    kr = np.where(cand, np.maximum(e.astype(np.float32).view(np.uint32), 1), 0).astype(np.uint64)
    val = kr.astype(np.uint32).view(np.float32)
    if not need > 0:
        return np.zeros_like(cand)
    total = np.float32(val[cand].sum(dtype=np.float32))
    if total < need:
        return cand.copy()
    t = 0
    for bit in range(30, -1, -1):
        cand_t = t | (1 << bit)
        if np.float32(val[kr >= cand_t].sum(dtype=np.float32)) >= need:
            t = cand_t
    above = np.float32(val[kr > t].sum(dtype=np.float32))
    eqc = int((kr == t).sum())
    pt = np.array([t], np.uint32).view(np.float32)[0]
    need_eq = max(1, min(int(np.ceil(np.float32(need - above) / pt)), eqc))
    eq = kr == t
    rank = np.cumsum(eq) - eq
    return cand & ((kr > t) | (eq & (rank < need_eq)))


def _rows(rng, n_rows, n):
    for _ in range(n_rows):
        levels = int(rng.integers(2, 40))
        s = rng.integers(-levels, levels, size=n).astype(np.float32) * np.float32(rng.uniform(0.01, 3.0))
        if rng.random() < 0.3:
            s[rng.random(n) < 0.2] = 0.0
            s[rng.random(n) < 0.1] = -0.0
        cand = rng.random(n) < rng.uniform(0.3, 1.0)
        yield s, cand


@pytest.mark.parametrize("n", [60, 624, 2160])
def test_count_selection_matches_sort(n):
    rng = np.random.default_rng(n)
    for s, cand in _rows(rng, 200 if n < 1000 else 60, n):
        for extra in (0, 1, 3, 17, 32, 33, 80, int(cand.sum()), int(cand.sum()) + 5):
            got = select_by_count(order_key(s), cand, extra)
            want = np.zeros(n, bool)
            want[O.top_outside(s.astype(np.float64), ~cand, min(extra, int(cand.sum())))] = True
            assert np.array_equal(got, want), (n, extra)


@pytest.mark.parametrize("n", [60, 624, 2160])
def test_range_selection_matches_sort(n):
    rng = np.random.default_rng(7 + n)
    for s, cand in _rows(rng, 200 if n < 1000 else 60, n):
        for extra in (0, 1, 3, 17, 32, 33, 80, int(cand.sum()), int(cand.sum()) + 5):
            got = select_by_range(order_key(s), cand, extra)
            want = np.zeros(n, bool)
            want[O.top_outside(s.astype(np.float64), ~cand, min(extra, int(cand.sum())))] = True
            assert np.array_equal(got, want), (n, extra)


def test_range_selection_spread_and_outliers():
    """Scores spread over many binades and rows with a few huge outliers (the range is
    then dominated by them, so the first pass puts nearly every key in one bucket)."""
    rng = np.random.default_rng(11)
    for _ in range(200):
        n = int(rng.integers(40, 700))
        s = (rng.standard_normal(n) * np.exp(rng.uniform(-8, 8, n))).astype(np.float32)
        if rng.random() < 0.5:
            s[rng.integers(0, n, 3)] = np.float32(1e30)
        cand = rng.random(n) < 0.8
        for extra in (1, 5, 40, int(cand.sum()) - 1):
            got = select_by_range(order_key(s), cand, extra)
            want = np.zeros(n, bool)
            want[O.top_outside(s.astype(np.float64), ~cand, max(0, min(extra, int(cand.sum()))))] = True
            assert np.array_equal(got, want)


def test_planted_range_bucket_off_by_one_is_caught():
    """Taking the bucket below the right one (the boundary one bucket too low) must
    disagree with the sort somewhere."""
    rng = np.random.default_rng(13)

    def wrong(keys, cand, extra):
        kr = np.where(cand, keys, 0).astype(np.uint64)
        lo, hi = int(kr[cand].min()), int(kr[cand].max())
        shift = max(0, (hi - lo).bit_length() - 8)
        cnt = np.bincount((kr[cand].astype(np.int64) - lo) >> shift, minlength=256)
        suf = np.cumsum(cnt[::-1])[::-1]
        d = max(0, int(np.nonzero(suf >= extra)[0].max()) - 1)
        return cand & (kr >= lo + (d << shift))

    bad = 0
    for s, cand in _rows(rng, 60, 624):
        extra = 30
        if int(cand.sum()) <= extra:
            continue
        want = np.zeros(s.size, bool)
        want[O.top_outside(s.astype(np.float64), ~cand, extra)] = True
        bad += int(not np.array_equal(wrong(order_key(s), cand, extra), want))
    assert bad > 0


@pytest.mark.parametrize("n", [60, 624])
def test_mass_selection_matches_sorted_prefix(n):
    """On scores spread apart (no fp32 near-ties), the mass search takes exactly the
    shortest prefix of the (score desc, index asc) order whose fp32 mass reaches the need."""
    rng = np.random.default_rng(100 + n)
    for _ in range(150):
        s = (rng.permutation(n).astype(np.float32) * np.float32(0.05)).astype(np.float32)
        cand = rng.random(n) < 0.7
        e = np.exp2((s - s.max()) * np.float32(1.3)).astype(np.float32)
        total = np.float32(e[cand].sum(dtype=np.float32))
        need = np.float32(total * np.float32(rng.uniform(0.05, 1.05)))
        got = select_by_mass(e, cand, need)
        order = np.lexsort((np.arange(n), -s.astype(np.float64)))
        want = np.zeros(n, bool)
        acc = 0.0
        for j in order:
            if not cand[j]:
                continue
            if acc >= need:
                break
            want[j] = True
            acc += float(e[j])
        # the fp32 sums of the search and the float64 running sum may differ only where the
        # running mass passes within float32 rounding of the need
        if not np.array_equal(got, want):
            cum = np.cumsum([float(e[j]) for j in order if cand[j]])
            assert np.min(np.abs(cum - float(need))) < 1e-5 * float(total)


def test_mass_ties_taken_in_index_order():
    """Equal probabilities: the ceil rule takes the lowest-indexed tied tiles."""
    e = np.full(40, np.float32(0.25))
    cand = np.ones(40, bool)
    cand[[3, 7]] = False
    got = select_by_mass(e, cand, np.float32(1.6))                      # needs 7 tiles (1.75)
    want = np.zeros(40, bool)
    want[[j for j in range(40) if cand[j]][:7]] = True
    assert np.array_equal(got, want)


def test_planted_tie_order_is_caught():
    """Taking tied keys from the highest index down must disagree with the sort somewhere."""
    rng = np.random.default_rng(5)
    mismatches = 0
    for s, cand in _rows(rng, 100, 624):
        keys = order_key(s)
        for extra in (40, 90):
            kr = np.where(cand, keys, 0).astype(np.uint64)
            good = select_by_count(keys, cand, extra)
            n_sel = int(good.sum())
            # planted: the same count, ties broken toward the higher index
            order = np.lexsort((-np.arange(s.size), -kr.astype(np.float64)))
            bad = np.zeros(s.size, bool)
            bad[[j for j in order if cand[j]][:n_sel]] = True
            mismatches += not np.array_equal(bad, good)
    assert mismatches > 0
