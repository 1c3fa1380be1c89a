"""The tree sampler's top-k launch filters the values it offers to the
per-thread candidate lists by a warp threshold; this checks, on the CPU,
that the filter cannot change the slab's top_k.

The model follows the launch's steps for one slab: 128 threads in warps of
32, rounds of four 16-byte vectors per thread (eight bf16 logits each), a
sorted list of KM entries per thread (larger value first, ties to the
smaller index; -inf and NaN never enter), and, per round, the warp
threshold: the top_k-th largest of the lanes' round maxima, found by top_k
rounds that each take the warp maximum and retire it from the lowest lane
holding it; the threshold only grows. Values below it are not offered. The
slab's result -- top_k block-wide argmax rounds over the list heads -- must
equal the plain top_k of the slab in (value desc, index asc) order, with or
without the filter, on rows with many exact ties (values on a coarse grid,
as bf16 logits are) and with -inf entries.
"""
import numpy as np
import pytest

THREADS, WARP, ROUND_VECS, VEC = 128, 32, 4, 8


def _better(a, ia, b, ib):
    return a > b or (a == b and ia < ib)


class _List:
    def __init__(self, km):
        self.v = [-np.inf] * km
        self.i = [np.iinfo(np.int64).max] * km

    def offer(self, x, idx):
        if not (x > -np.inf) or not _better(x, idx, self.v[-1], self.i[-1]):
            return
        self.v[-1], self.i[-1] = x, idx
        for e in range(len(self.v) - 1, 0, -1):
            if _better(self.v[e], self.i[e], self.v[e - 1], self.i[e - 1]):
                self.v[e], self.v[e - 1] = self.v[e - 1], self.v[e]
                self.i[e], self.i[e - 1] = self.i[e - 1], self.i[e]

    def pop(self):
        self.v = self.v[1:] + [-np.inf]
        self.i = self.i[1:] + [np.iinfo(np.int64).max]


def _kth_of_lanes(xs, k):
    xs = list(xs)
    kth = -np.inf
    for _ in range(k):
        m = max(xs)
        kth = m
        if not (m > -np.inf):
            break
        xs[xs.index(m)] = -np.inf  # the lowest lane holding it
    return kth


def _slab_topk(vals, top_k, km, use_threshold):
    n = vals.size
    nvec = n // VEC
    lists = [_List(km) for _ in range(THREADS)]
    thr = [-np.inf] * (THREADS // WARP)
    step = THREADS * ROUND_VECS
    for r0 in range(0, nvec, step):
        rmax = [-np.inf] * THREADS
        for t in range(THREADS):
            for k in range(ROUND_VECS):
                vi = r0 + t + k * THREADS
                if vi < nvec:
                    seg = vals[vi * VEC:(vi + 1) * VEC]
                    finite = seg[~np.isnan(seg)]
                    if finite.size:
                        rmax[t] = max(rmax[t], float(finite.max()))
        for w in range(THREADS // WARP):
            if use_threshold:
                thr[w] = max(thr[w], _kth_of_lanes(rmax[w * WARP:(w + 1) * WARP], top_k))
        for t in range(THREADS):
            for k in range(ROUND_VECS):
                vi = r0 + t + k * THREADS
                if vi < nvec:
                    for e in range(VEC):
                        x = float(vals[vi * VEC + e])
                        if x >= thr[t // WARP]:
                            lists[t].offer(x, vi * VEC + e)
    out = []
    for _ in range(top_k):
        best = max(range(THREADS), key=lambda t: (lists[t].v[0], -lists[t].i[0]))
        v, i = lists[best].v[0], lists[best].i[0]
        if not (v > -np.inf):
            out.append((-np.inf, -1))
            continue
        out.append((v, i))
        lists[best].pop()
    return out


def _plain_topk(vals, top_k):
    order = sorted((i for i in range(vals.size) if vals[i] > -np.inf),
                   key=lambda i: (-vals[i], i))
    got = [(float(vals[i]), i) for i in order[:top_k]]
    return got + [(-np.inf, -1)] * (top_k - len(got))


@pytest.mark.parametrize("n,top_k,km,levels,seed", [
    (4096, 4, 4, 16, 1),      # one round, heavy ties
    (4096, 4, 4, 1000, 2),    # one round, few ties
    (12288, 8, 8, 24, 3),     # three rounds: the threshold carries over
    (12288, 2, 4, 6, 4),      # lists longer than top_k, very heavy ties
    (2048, 16, 16, 40, 5),    # top_k 16 (the launch offers every value there)
])
def test_threshold_keeps_the_slab_topk(n, top_k, km, levels, seed):
    rng = np.random.default_rng(seed)
    vals = np.round(rng.normal(0.0, 2.0, n) * levels / 8.0) / (levels / 8.0)
    vals[rng.choice(n, size=n // 50, replace=False)] = -np.inf
    want = _plain_topk(vals, top_k)
    assert _slab_topk(vals, top_k, km, use_threshold=True) == want
    assert _slab_topk(vals, top_k, km, use_threshold=False) == want


def test_threshold_with_few_finite_values():
    vals = np.full(4096, -np.inf)
    vals[[5, 900, 4000]] = [1.0, 1.0, 0.5]
    assert _slab_topk(vals, 4, 4, use_threshold=True) == \
        [(1.0, 5), (1.0, 900), (0.5, 4000), (-np.inf, -1)]


def test_threshold_when_the_top_values_sit_in_one_warp():
    # the four largest values in the first vectors of threads 0..3 (one warp,
    # four lanes): the threshold is the fourth of them, and the fourth must
    # still be offered
    rng = np.random.default_rng(7)
    vals = rng.normal(0.0, 1.0, 4096)
    for t, v in enumerate((9.0, 8.0, 7.0, 6.0)):
        vals[t * VEC + 3] = v
    want = [(9.0, 3), (8.0, 11), (7.0, 19), (6.0, 27)]
    assert _plain_topk(vals, 4) == want
    assert _slab_topk(vals, 4, 4, use_threshold=True) == want
