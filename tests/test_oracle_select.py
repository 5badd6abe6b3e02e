"""Pins for the oracle's top-K selector with question protection (MarkTechPost page,
sections "Comment TokenGate a-t-il appris le fonctionnement de la réduction des
tokens ?" — a top-K selector keeps the best-scoring tokens; only the document may
be dropped, the question never — and "Comment déployer TokenGate ?" — {state}
marks the droppable document, max_kept_prefill_tokens is the budget).

Reading: per sequence keep min(k_doc, |doc|) document tokens by score (ties to the
lower position, -0 == +0, NaN below -inf) plus every token outside the document,
in ascending position order."""
import itertools
import json
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f(v):
    return float(v) if not isinstance(v, str) else float(v.replace("inf", "inf"))


def _run(orc, scores, doc, k):
    s = np.array([_f(v) for v in scores], np.float32)
    idx, cu = orc.select_topk(s, [0, len(s)], [doc[0]], [doc[1]], [k])
    return idx.tolist(), cu


def test_golden_cases(orc):
    cases = json.load(open(os.path.join(GOLDEN, "select_cases.json")))["cases"]
    for c in cases:
        kept, cu = _run(orc, c["scores"], c["doc"], c["k_doc"])
        assert kept == c["kept"], c
        assert cu.tolist() == [0, len(c["kept"])]


def _rank_key(f):
    """Brute-force side: map a float32 to a sortable tuple, NaN lowest, -0 == +0."""
    if math.isnan(f):
        return (0, 0.0)
    return (1, 0.0 if f == 0 else float(f))


def _brute_force(scores, db, de, k):
    """Enumerate every k-subset of the document; exactly one satisfies 'every kept
    token beats every dropped one (higher score, or equal score and lower
    position)'. Returns it with the protected tokens, ascending."""
    doc = list(range(db, de))
    k = min(max(k, 0), len(doc))
    valid = []
    for sub in itertools.combinations(doc, k):
        s = set(sub)
        ok = True
        for a in sub:
            for b in doc:
                if b in s:
                    continue
                ka, kb = _rank_key(scores[a]), _rank_key(scores[b])
                if not (ka > kb or (ka == kb and a < b)):
                    ok = False
                    break
            if not ok:
                break
        if ok:
            valid.append(s)
    assert len(valid) == 1, "the tie rule must single out one subset"
    keep = valid[0] | (set(range(len(scores))) - set(doc))
    return sorted(keep)


def test_exhaustive_tiny_against_brute_force(orc):
    # every score pattern over a small alphabet with ties, signed zeros and specials
    alphabet = np.array([np.nan, -np.inf, -1.0, -0.0, 0.0, 1.0, np.inf], np.float32)
    rng = np.random.default_rng(11)
    n_checked = 0
    for n in range(1, 8):
        for trial in range(60 if n > 3 else 200):
            s = alphabet[rng.integers(0, len(alphabet), n)]
            db = int(rng.integers(0, n + 1))
            de = int(rng.integers(db, n + 1))
            for k in range(0, de - db + 2):
                got, _ = _run(orc, s.tolist(), (db, de), k)
                assert got == _brute_force(s, db, de, k), (s, db, de, k)
                n_checked += 1
    assert n_checked > 1000


def _check_invariants(scores, cu, db, de, kd, idx, cuk):
    B = len(db)
    for b in range(B):
        base, n = cu[b], cu[b + 1] - cu[b]
        got = idx[cuk[b]:cuk[b + 1]] - base
        assert np.all(np.diff(got) > 0), "ascending, no duplicates"
        assert np.all((got >= 0) & (got < n))
        nd = de[b] - db[b]
        doc_kept = got[(got >= db[b]) & (got < de[b])]
        assert len(doc_kept) == min(kd[b], nd), "exactly K document tokens"
        prot = np.r_[0:db[b], de[b]:n]
        assert np.isin(prot, got).all(), "question never dropped"
        s = scores[base:base + n]
        dropped = np.setdiff1d(np.arange(db[b], de[b]), doc_kept)
        if len(doc_kept) and len(dropped):
            assert s[doc_kept].min() >= s[dropped].max(), "threshold separation"
            thr = s[doc_kept].min()
            tie_kept = doc_kept[s[doc_kept] == thr]
            tie_drop = dropped[s[dropped] == thr]
            if len(tie_drop):
                assert tie_kept.max() < tie_drop.min(), "ties to the lower position"


def test_invariants_batch_with_ties(orc):
    rng = np.random.default_rng(3)
    lens = [4096, 1, 700, 3000, 64]
    cu = np.r_[0, np.cumsum(lens)].astype(np.int32)
    # coarse values -> many exact ties
    scores = (rng.integers(-50, 50, cu[-1]) / 8.0).astype(np.float32)
    db = [0, 0, 100, 0, 10]
    de = [4096 - 256, 1, 650, 3000, 10]
    kd = [409, 5, 20, 0, 3]
    idx, cuk = orc.select_topk(scores, cu, db, de, kd)
    _check_invariants(scores, cu, db, de, kd, idx, cuk)
    assert cuk[-1] == len(idx)


def test_against_numpy_lexsort_witness(orc):
    # finite scores: the kept document set is the first k of a lexsort by
    # (-score, position) -- a library sort, independent of the oracle's comparator
    rng = np.random.default_rng(5)
    n, q, k = 5000, 300, 777
    s = rng.standard_normal(n).astype(np.float32)
    s[rng.integers(0, n - q, 400)] = s[123]          # exact ties straddling nothing in particular
    order = np.lexsort((np.arange(n - q), -s[: n - q].astype(np.float64)))
    want = np.sort(np.r_[order[:k], np.arange(n - q, n)])
    idx, _ = orc.select_topk(s, [0, n], [0], [n - q], [k])
    np.testing.assert_array_equal(idx, want)


def test_bad_span_rejected(orc):
    with pytest.raises(ValueError):
        orc.select_topk(np.zeros(4, np.float32), [0, 4], [3], [2], [1])
    with pytest.raises(ValueError):
        orc.select_topk(np.zeros(4, np.float32), [0, 4], [0], [5], [1])
