"""The order-statistic identity behind the 4:8 selection of the prefill kernel
(csrc/ssa_fwd.cu, nm8_n4): with the two halves of an 8-group sorted
descending (a, c), the k-th largest of the group is the largest, over
i + j = k, of min(i-th largest of a, j-th largest of c), the 0-th being
+inf.  The kernel takes k = 4 (its keep threshold t) and k = 5 (nx, for the
tie test).  Checked here against a plain sort on random groups, groups with
repeated values, and groups with -inf (masked) keys, in float32 as the
kernel computes.  The kernel's own selections are compared with the oracle's
keep masks bit for bit by the GPU parity tests."""
import numpy as np
import pytest


def _kth_by_merge(a, c, k):
    """k-th largest (1-based) of the union of two descending lists of four."""
    big = np.float32(np.inf)
    A = [big] + list(a)
    C = [big] + list(c)
    best = np.float32(-np.inf)
    for i in range(0, 5):
        j = k - i
        if 0 <= j <= 4:
            best = max(best, min(A[i], C[j]))
    return best


def _kernel_t_nx(v):
    """t and nx exactly as the kernel forms them from the sorted halves."""
    a = np.sort(v[:4])[::-1]
    c = np.sort(v[4:])[::-1]
    t = max(max(c[3], min(a[0], c[2]), min(a[1], c[1])), max(min(a[2], c[0]), a[3]))
    nx = max(max(min(a[0], c[3]), min(a[1], c[2]), min(a[2], c[1])), min(a[3], c[0]))
    return np.float32(t), np.float32(nx)


@pytest.mark.parametrize("kind", ["normal", "ties", "masked"])
def test_fourth_and_fifth_largest_from_sorted_halves(kind):
    rng = np.random.default_rng({"normal": 1, "ties": 2, "masked": 3}[kind])
    for _ in range(20000):
        if kind == "normal":
            v = rng.standard_normal(8).astype(np.float32)
        elif kind == "ties":
            v = rng.choice(np.array([-1.0, 0.0, 0.5, 2.0], np.float32), size=8)
        else:
            v = rng.standard_normal(8).astype(np.float32)
            v[rng.random(8) < 0.4] = -np.inf
        srt = np.sort(v)[::-1]
        t, nx = _kernel_t_nx(v)
        assert t == srt[3] or (np.isneginf(t) and np.isneginf(srt[3])), (v, t)
        assert nx == srt[4] or (np.isneginf(nx) and np.isneginf(srt[4])), (v, nx)
        a = np.sort(v[:4])[::-1]
        c = np.sort(v[4:])[::-1]
        for k in range(1, 9):
            got = _kth_by_merge(a, c, k)
            assert got == srt[k - 1] or (np.isneginf(got) and np.isneginf(srt[k - 1]))


def test_a_wrong_merge_index_is_caught():
    """Planted mistake: pairing the halves' i-th with the (k - i + 1)-th
    instead of the (k - i)-th must fail on random groups."""
    rng = np.random.default_rng(4)
    bad = 0
    for _ in range(2000):
        v = rng.standard_normal(8).astype(np.float32)
        a = np.sort(v[:4])[::-1]
        c = np.sort(v[4:])[::-1]
        A = [np.inf] + list(a)
        C = [np.inf] + list(c)
        wrong = max(min(A[i], C[min(4, 4 - i + 1)]) for i in range(0, 5))
        bad += wrong != np.sort(v)[::-1][3]
    assert bad > 0
