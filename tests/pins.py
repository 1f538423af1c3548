"""Checks that pin the CPU oracle to things other than itself.

Each ``check_*`` function raises AssertionError when the oracle (``oracle``
package, whichever library is loaded) disagrees with an independent fact:
an independent implementation (numpy's Philox), a library routine (python's
sort, numpy.take, scipy's vq and softmax, torch's bf16 cast), a closed form,
an invariant, or a hand-derived golden case.  ``test_oracle_pins.py`` runs
them on the oracle; ``test_oracle_mutants.py`` runs them on deliberately
broken copies of the oracle and expects each copy to be caught.
"""
from __future__ import annotations

import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
U64 = (1 << 64) - 1


def numpy_philox_block(ctr, key):
    """Philox4x64-10 block(ctr) from numpy, which pre-increments its counter."""
    v = sum(int(c) << (64 * i) for i, c in enumerate(ctr))
    v = (v - 1) % (1 << 256)
    cm = np.array([(v >> (64 * i)) & U64 for i in range(4)], dtype=np.uint64)
    g = np.random.Philox(key=np.array([int(k) for k in key], dtype=np.uint64), counter=cm)
    return [int(x) for x in g.random_raw(4)]


def check_philox():
    rng = np.random.default_rng(7)
    cases = [([0, 0, 0, 0], [0, 0]), ([U64, U64, U64, U64], [U64, U64]), ([1, 0, 0, 0], [1, 2])]
    for _ in range(40):
        cases.append(([int(x) for x in rng.integers(0, 2**63, 4, dtype=np.int64)],
                      [int(x) for x in rng.integers(0, 2**63, 2, dtype=np.int64)]))
    for ctr, key in cases:
        got = [int(x) for x in oracle.philox4x64_10(ctr, key)]
        assert got == numpy_philox_block(ctr, key), (ctr, key)


def check_random_score():
    rng = np.random.default_rng(11)
    for _ in range(60):
        seed, rnd = int(rng.integers(0, 2**40)), int(rng.integers(0, 1000))
        r, l, h, pos = (int(x) for x in rng.integers(0, 5000, 4))
        for shared in (False, True):
            want = numpy_philox_block([pos, U64 if shared else h, l, r], [seed, rnd])[0] >> 32
            assert oracle.random_score(seed, rnd, r, l, h, pos, shared) == want


def check_retention():
    with open(os.path.join(GOLDEN, "retention_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        got = oracle.retention(c["L"], c["P"], c["K"])
        assert (got.M, got.R, got.noop, got.over_budget) == (c["M"], c["R"], c["noop"], c["over_budget"]), c
    # invariant: retained = min(K, L) whenever K >= P
    for L in range(0, 40, 3):
        for P in range(0, L + 1, 5):
            for K in range(P, 50, 7):
                assert oracle.retention(L, P, K).R == min(K, L)


def check_select():
    rng = np.random.default_rng(3)
    for trial in range(200):
        N = int(rng.integers(1, 60))
        M = int(rng.integers(0, N + 1))
        score = rng.integers(0, 4, N).astype(np.float64)  # many ties
        pos = np.sort(rng.choice(10_000, N, replace=False)).astype(np.int64)
        slot = np.arange(5, 5 + N, dtype=np.int64)
        got = oracle.select_topk(score, pos, slot, M)
        order = sorted(range(N), key=lambda j: (-score[j], pos[j]))
        want = np.sort(slot[order[:M]])
        assert np.array_equal(got, want), (trial, got, want)
        kept = set(got.tolist())
        for j in range(N):  # dominance: every kept beats every evicted
            for e in range(N):
                if slot[j] in kept and slot[e] not in kept:
                    assert score[j] > score[e] or (score[j] == score[e] and pos[j] < pos[e])


def check_compact():
    rng = np.random.default_rng(5)
    for _ in range(30):
        L = int(rng.integers(1, 70))
        P = int(rng.integers(0, L + 1))
        rows = rng.integers(0, 255, (L, 24), dtype=np.uint8)
        kept = np.sort(rng.choice(np.arange(P, L), int(rng.integers(0, L - P + 1)), replace=False))
        got = oracle.compact_rows(rows, P, kept)
        want = np.take(rows, np.concatenate([np.arange(P), kept]).astype(np.int64), axis=0)
        assert np.array_equal(got, want)


def check_random_round_invariants():
    seed, rnd = 9, 3
    P, K, L = 16, 64, 256
    pos_in = np.arange(L, dtype=np.int32) * 3 + 7  # increasing, not equal to slots
    for shared in (False, True):
        kept_by_head = []
        for h in range(4):
            kept, pos_out = oracle.random_round_segment(seed, rnd, 2, 1, h, shared, P, K, pos_in)
            assert len(kept) == K
            assert np.array_equal(kept[:P], np.arange(P))
            assert np.all(np.diff(kept) > 0)
            assert np.array_equal(pos_out, pos_in[kept])
            # recompute the scores independently and check dominance
            sc = np.array([numpy_philox_block([int(p), U64 if shared else h, 1, 2], [seed, rnd])[0] >> 32
                           for p in pos_in[P:]], dtype=np.float64)
            keep = np.zeros(L - P, bool)
            keep[kept[P:] - P] = True
            assert sc[keep].min() >= sc[~keep].max()
            kept_by_head.append(kept)
        same = all(np.array_equal(kept_by_head[0], k) for k in kept_by_head[1:])
        assert same == shared


def _steady_state(S, P, M, E, rounds, seed):
    """S segments at steady state; returns survivors of the first E arrivals per round."""
    stride = P + M + E
    pos = np.tile(np.arange(P + M, dtype=np.int32), (S, 1))
    next_pos = P + M
    rlh = np.stack([np.arange(S) // 64, (np.arange(S) // 8) % 8, np.arange(S) % 8], 1)
    lpk = np.tile([P + M + E, P, P + M], (S, 1))
    tracked = None
    surv = []
    for rd in range(rounds):
        new = np.arange(next_pos, next_pos + E, dtype=np.int32)
        next_pos += E
        full = np.concatenate([pos, np.tile(new, (S, 1))], 1)
        if rd == 0:
            tracked = new
        out, R = oracle.random_round_batch(seed, rd, False, rlh, lpk, full)
        assert np.all(R == P + M)
        pos = np.ascontiguousarray(out[:, :P + M])
        surv.append(int(np.isin(pos, tracked).sum()))
    return surv


def check_survival():
    S, P, M, E, rounds = 4000, 16, 48, 16, 8
    p = M / (M + E)
    surv = _steady_state(S, P, M, E, rounds, seed=21)
    n0 = S * E
    for n, got in enumerate(surv, start=1):
        q = p ** n
        sd = np.sqrt(n0 * q * (1 - q))
        assert abs(got - n0 * q) < 5 * sd + 1, (n, got, n0 * q)
    # one round, uniform survivors over candidate positions (chi^2)
    from scipy.stats import chisquare
    P2, K2, L2 = 16, 64, 256
    counts = np.zeros(L2 - P2)
    pos_in = np.arange(L2, dtype=np.int32)
    S2 = 3000
    rlh = np.stack([np.arange(S2), np.zeros(S2, int), np.zeros(S2, int)], 1)
    lpk = np.tile([L2, P2, K2], (S2, 1))
    out, R = oracle.random_round_batch(5, 0, False, rlh, lpk, np.tile(pos_in, (S2, 1)))
    for s in range(S2):
        counts[out[s, P2:R[s]] - P2] += 1
    assert abs(counts.sum() / (S2 * (L2 - P2)) - (K2 - P2) / (L2 - P2)) < 1e-12
    assert chisquare(counts).pvalue > 1e-4


def check_head_independence():
    P, K, L = 16, 64, 256
    M, N = K - P, L - P
    pos_in = np.arange(L, dtype=np.int32)
    ov = []
    for r in range(300):
        a, _ = oracle.random_round_segment(4, 0, r, 0, 0, False, P, K, pos_in)
        b, _ = oracle.random_round_segment(4, 0, r, 0, 1, False, P, K, pos_in)
        ov.append(len(set(a[P:].tolist()) & set(b[P:].tolist())))
    # independent uniform M-subsets of N overlap by M^2/N on average
    assert abs(np.mean(ov) - M * M / N) < 5 * np.std(ov) / np.sqrt(len(ov)) + 0.05


def check_bf16():
    import torch
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(3000), rng.standard_normal(500) * 1e-3,
                        rng.standard_normal(500) * 1e4]).astype(np.float32)
    # exact ties: halfway between two bf16 values
    x = np.concatenate([x, np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, -(1.0 + 2**-8)], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def check_beacon_update():
    from scipy.cluster.vq import vq
    rng = np.random.default_rng(8)
    n, B, d = 96, 8, 16
    pts = rng.standard_normal((n, d))
    c0 = pts[(np.arange(B) * n) // B]
    c1, cnt1, a1 = oracle.beacon_update(pts, np.zeros((B, d)), np.zeros(B), init=True)
    code, _ = vq(pts, c0)
    assert np.array_equal(a1, code)
    hist = [[] for _ in range(B)]
    for p, i in enumerate(a1):
        hist[i].append(pts[p])
    for i in range(B):
        if hist[i]:
            assert np.allclose(c1[i], np.mean(hist[i], 0), rtol=1e-12, atol=1e-12)
            assert cnt1[i] == len(hist[i])
        else:
            assert np.array_equal(c1[i], c0[i]) and cnt1[i] == 0
    # later updates: still the mean of every point ever assigned
    c, cnt = c1, cnt1
    for step in range(4):
        new = rng.standard_normal((64, d)) + step
        code, _ = vq(new, c)
        c, cnt, a = oracle.beacon_update(new, c, cnt, init=False)
        assert np.array_equal(a, code)
        for p, i in enumerate(a):
            hist[i].append(new[p])
        for i in range(B):
            if hist[i]:
                assert np.allclose(c[i], np.mean(hist[i], 0), rtol=1e-10, atol=1e-12)
                assert cnt[i] == len(hist[i])
    try:
        oracle.beacon_update(pts[:B - 1], np.zeros((B, d)), np.zeros(B), init=True)
    except ValueError:
        pass
    else:
        raise AssertionError("n_pts < B on the first update must fail")


def check_beacon_score():
    from scipy.special import softmax
    rng = np.random.default_rng(4)
    for (L, P, B, d) in [(50, 5, 3, 8), (33, 0, 1, 16), (64, 16, 4, 64)]:
        keys = rng.standard_normal((L, d))
        bea = rng.standard_normal((B, d))
        sc, lse = oracle.beacon_score(keys, bea, P)
        Z = bea @ keys.T / np.sqrt(d)
        want = softmax(Z, axis=1).max(0)[P:]
        assert np.allclose(sc, want, rtol=1e-12, atol=0)
        assert np.allclose(lse, np.log(np.exp(Z).sum(1)), rtol=1e-12)
    # identical keys: every key gets 1/L, whatever the beacons
    keys = np.tile(rng.standard_normal(8), (40, 1))
    sc, _ = oracle.beacon_score(keys, rng.standard_normal((3, 8)), 4)
    assert np.allclose(sc, 1 / 40, rtol=1e-12)
    # B = 1: ranking == ranking of the dot product c.k_j
    keys = rng.standard_normal((30, 8))
    c = rng.standard_normal((1, 8))
    sc, _ = oracle.beacon_score(keys, c, 0)
    assert np.array_equal(np.argsort(-sc, kind="stable"), np.argsort(-(keys @ c[0]), kind="stable"))
    # one-hot keys e_0..e_{L-1} and beacon alpha*e_m: closed form
    d, L, m, alpha = 16, 10, 3, 5.0
    keys = np.eye(d)[:L]
    c = np.zeros((1, d))
    c[0, m] = alpha
    sc, _ = oracle.beacon_score(keys, c, 0)
    e = np.exp(alpha / np.sqrt(d))
    want = np.full(L, 1 / (e + L - 1))
    want[m] = e / (e + L - 1)
    assert np.allclose(sc, want, rtol=1e-13)


def check_block_score():
    rng = np.random.default_rng(13)
    for _ in range(40):
        seed, rnd = int(rng.integers(0, 2**40)), int(rng.integers(0, 100))
        r, l, h, pos = (int(x) for x in rng.integers(0, 5000, 4))
        block = int(rng.choice([1, 2, 16, 64, 256]))
        for shared in (False, True):
            want = numpy_philox_block([pos // block, U64 if shared else h, l, r], [seed, rnd])[0] >> 32
            assert oracle.random_score_block(seed, rnd, r, l, h, pos, shared, block) == want


def check_hole_fill():
    rng = np.random.default_rng(17)
    for _ in range(200):
        L = int(rng.integers(1, 80))
        R = int(rng.integers(0, L + 1))
        kept = np.sort(rng.choice(L, R, replace=False)).astype(np.int64)
        src = oracle.hole_fill(R, kept)
        assert sorted(src.tolist()) == kept.tolist()            # same rows survive
        for s in kept[kept < R]:
            assert src[s] == s                                   # survivors below R stay
        holes = [s for s in range(R) if s not in set(kept.tolist())]
        movers = kept[kept >= R].tolist()
        assert [int(src[s]) for s in holes] == movers            # holes in order take movers in order


def check_random_round_ex():
    rng = np.random.default_rng(19)
    P, K, L = 16, 64, 256
    pos_in = (np.arange(L) * 2 + 5).astype(np.int32)
    for trial in range(30):
        seed, rnd, h = int(rng.integers(0, 2**32)), int(rng.integers(0, 50)), int(rng.integers(0, 8))
        # block 1, ordered: the pinned per-token round
        want = oracle.random_round_segment(seed, rnd, 3, 2, h, False, P, K, pos_in)[1]
        assert np.array_equal(oracle.random_round_segment_ex(seed, rnd, 3, 2, h, False, 1, False, P, K, pos_in), want)
        # hole filling keeps the same positions; those already below R stay put
        hf = oracle.random_round_segment_ex(seed, rnd, 3, 2, h, False, 1, True, P, K, pos_in)
        assert sorted(hf.tolist()) == sorted(want.tolist())
        for s in range(K):
            if pos_in[s] in set(want.tolist()):
                assert hf[s] == pos_in[s]
        # block-granular draws split at most one block of candidates
        for block in (4, 16, 64):
            out = oracle.random_round_segment_ex(seed, rnd, 3, 2, h, False, block, False, P, K, pos_in)
            kept = set(out.tolist())
            blocks = {}
            for pos in pos_in[P:]:
                blocks.setdefault(int(pos) // block, []).append(int(pos) in kept)
            split = sum(1 for v in blocks.values() if any(v) and not all(v))
            assert split <= 1, (block, split)
            assert len(out) == K and np.array_equal(out[:P], pos_in[:P])


def check_beacon_trigger_score():
    from scipy.special import softmax
    rng = np.random.default_rng(31)
    for (L, P, B, d) in [(40, 4, 3, 8), (64, 0, 5, 16), (33, 10, 1, 32)]:
        keys = rng.standard_normal((L, d))
        bea = rng.standard_normal((B, d))
        trig = rng.integers(0, 20, B).astype(np.float64)
        trig[0] += 1
        sc = oracle.beacon_trigger_score(keys, bea, trig, P)
        A = softmax(bea @ keys.T / np.sqrt(d), axis=1)  # [B, L]
        want = (trig / trig.sum()) @ A
        assert np.allclose(sc, want[P:], rtol=1e-12, atol=1e-15)
        # scaling the counts changes nothing
        assert np.allclose(oracle.beacon_trigger_score(keys, bea, 7 * trig, P), sc, rtol=1e-13, atol=0)
        # one-hot trigger: that beacon's attention row
        b = int(rng.integers(B))
        oh = np.zeros(B)
        oh[b] = 3
        assert np.allclose(oracle.beacon_trigger_score(keys, bea, oh, P), A[b, P:], rtol=1e-12, atol=1e-15)
    # mass conservation over all keys (P = 0)
    keys = rng.standard_normal((50, 8))
    sc = oracle.beacon_trigger_score(keys, rng.standard_normal((4, 8)), np.array([1.0, 0, 5, 2]), 0)
    assert abs(sc.sum() - 1.0) <= 1e-12
    # identical keys: 1/L whatever the beacons and triggers
    keys = np.tile(rng.standard_normal(8), (25, 1))
    sc = oracle.beacon_trigger_score(keys, rng.standard_normal((3, 8)), np.array([2.0, 1, 0]), 5)
    assert np.allclose(sc, 1 / 25, rtol=1e-12)
    # no trigger at all: zeros
    sc = oracle.beacon_trigger_score(keys, rng.standard_normal((3, 8)), np.zeros(3), 5)
    assert np.array_equal(sc, np.zeros(20))


def check_decode_attention():
    from scipy.special import logsumexp, softmax
    rng = np.random.default_rng(23)
    for (L, d, scale) in [(1, 8, None), (37, 16, None), (200, 64, 0.3), (5, 128, 2.0)]:
        q = rng.standard_normal(d)
        k = rng.standard_normal((L, d))
        v = rng.standard_normal((L, d))
        sc = 1 / np.sqrt(d) if scale is None else scale
        out, lse = oracle.decode_attention(q, k, v, scale)
        s = sc * (k @ q)
        assert np.allclose(out, softmax(s) @ v, rtol=1e-12, atol=1e-14)
        assert abs(lse - logsumexp(s)) <= 1e-12 * max(1.0, abs(lse))
        # joint permutation of the rows changes nothing
        perm = rng.permutation(L)
        out2, lse2 = oracle.decode_attention(q, k[perm], v[perm], scale)
        assert np.allclose(out2, out, rtol=1e-12, atol=1e-14) and abs(lse2 - lse) <= 1e-12 * max(1.0, abs(lse))
    # one row: the value row itself, lse = the score
    q, k, v = rng.standard_normal(8), rng.standard_normal((1, 8)), rng.standard_normal((1, 8))
    out, lse = oracle.decode_attention(q, k, v)
    assert np.array_equal(out, v[0]) and abs(lse - (k[0] @ q) / np.sqrt(8)) <= 1e-15
    # zero query: the mean of the values, lse = log L
    v = rng.standard_normal((50, 16))
    out, lse = oracle.decode_attention(np.zeros(16), rng.standard_normal((50, 16)), v)
    assert np.allclose(out, v.mean(0), rtol=1e-12, atol=1e-15) and abs(lse - np.log(50)) <= 1e-13
    # large scale: all weight on the best key (no overflow)
    k = rng.standard_normal((20, 16))
    q = rng.standard_normal(16)
    v = rng.standard_normal((20, 16))
    out, lse = oracle.decode_attention(q, k, v, scale=1e4)
    j = int(np.argmax(k @ q))
    assert np.allclose(out, v[j], rtol=1e-9, atol=1e-12) and np.isfinite(lse)
    # empty: zeros and -inf
    out, lse = oracle.decode_attention(np.ones(4), np.zeros((0, 4)), np.zeros((0, 4)))
    assert np.array_equal(out, np.zeros(4)) and lse == -np.inf


def check_decode_attention_gqa():
    rng = np.random.default_rng(29)
    Hq, Hkv, L, d = 8, 2, 30, 16
    q = rng.standard_normal((Hq, d))
    k = rng.standard_normal((Hkv, L, d))
    v = np.stack([np.full((L, d), 3.0), np.full((L, d), 7.0)])  # marker value per KV head
    out, lse = oracle.decode_attention_gqa(q, k, v)
    G = Hq // Hkv
    for hq in range(Hq):
        assert np.allclose(out[hq], 3.0 if hq // G == 0 else 7.0, rtol=1e-13)
        s = k[hq // G] @ q[hq] / np.sqrt(d)
        assert abs(lse[hq] - np.log(np.exp(s).sum())) <= 1e-12 * abs(lse[hq]) + 1e-13


ALL = [check_philox, check_random_score, check_retention, check_select, check_compact,
       check_random_round_invariants, check_survival, check_head_independence, check_bf16,
       check_beacon_update, check_beacon_score, check_block_score, check_hole_fill, check_random_round_ex,
       check_decode_attention, check_decode_attention_gqa, check_beacon_trigger_score]
