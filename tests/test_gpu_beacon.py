"""BeaconKV update and scoring on the GPU against the oracle.

Staged parity: the oracle's beacon update is compared assignment by
assignment (exact, or a counted near-tie), then recomputed from the GPU's
assignments (fp32 vs double running means); the oracle's scores are computed
from the GPU's scoring copy of the beacons and the pre-round keys, then
compared within |g - o| <= 1e-5 + 1e-3|o| and within the strict relative
gate |g - o| <= 1e-9 + 1e-4|o|; the kept set must match the oracle's except
within 1e-4*tau of the threshold tau, with equal counts.

The "sharp" cases scale the decode queries to norm sqrt(d): beacons are then
long enough that the softmax over the keys is far from uniform, and scores
spread over several orders of magnitude instead of sitting near 1/L."""
import math

import numpy as np
import pytest
import torch

import oracle
from decode_kv_cache_paged_b200 import workloads as wl
from gpu_helpers import band_check, check_scores, dense_layer, make_context

pytestmark = pytest.mark.gpu


def _fill_recording(ctx, w, gen, interleave=False):
    """Fill like workloads.fill, keeping the queries of the last W steps per request.  With interleave, the
    requests take turns appending 16 tokens (one page) at a time, so no request holds consecutive page ids."""
    R = w.num_requests
    W = w.query_window
    plans = []
    for r in range(R):
        P, L = int(w.prompt[r]), int(w.length[r])
        q_from = L - min(W, L - P)
        steps, done = [], 0  # (tokens, protect, with queries)
        while done < P:
            T = min(16 if interleave else 256, P - done)
            steps.append((T, True, False))
            done += T
        while done < L:
            T = min(256 if done < q_from and not interleave else 16, (q_from if done < q_from else L) - done)
            steps.append((T, False, done >= q_from))
            done += T
        plans.append(steps)
    if interleave:
        order = [(r, plans[r][i]) for i in range(max(len(pl) for pl in plans)) for r in range(R) if i < len(plans[r])]
    else:
        order = [(r, st) for r in range(R) for st in plans[r]]
    qs = {r: [] for r in range(R)}
    for r, (T, protect, with_q) in order:
        ids = np.array([r], np.int32)
        k, v = gen.kv(1, T)
        if protect:
            ctx.append(ids, k, v, None, protect=True)
            continue
        q = gen.queries(1, T) if with_q else None
        ctx.append(ids, k, v, q)
        if q is not None:
            qs[r].append(q[0].float().cpu().numpy().astype(np.float64))  # [Ly, T, Hq, d]
    return {r: np.concatenate(qs[r], axis=1)[:, -W:] for r in range(R)}  # [Ly, steps, Hq, d]


def run_beacon(w, sample=None, score_impl=None, sinks=None, compaction="ordered", selector="beacon", k_hook=None,
               interleave=False):
    ctx = make_context(w)
    if score_impl is not None:
        ctx.set_option(0, score_impl)
    gen = wl.Generator(w, "cuda")
    qwin = _fill_recording(ctx, w, gen, interleave)
    R, Ly, H, d, B, G = w.num_requests, w.num_layers, w.num_kv_heads, w.head_dim, w.num_beacons, w.G
    W = w.query_window
    assign = torch.full((R, Ly, H, W * G), -1, dtype=torch.int32, device="cuda")
    ctx.update_beacons(assign_out=assign)
    ctx.sync()
    st = ctx.state_tensors()
    g_beacons = st["beacons"].cpu().numpy().astype(np.float64)
    g_scoring = st["beacons_scoring"].float().cpu().numpy().astype(np.float64)
    g_counts = st["beacon_counts"].cpu().numpy()
    g_trig = st["beacon_triggers"].cpu().numpy()
    g_assign = assign.cpu().numpy()
    # the scoring copy is the fp32 beacon rounded to the cache dtype (torch's RNE cast)
    assert torch.equal(st["beacons_scoring"], st["beacons"].to(ctx.dtype))
    segs = [(r, l, h) for r in range(R) for l in range(Ly) for h in range(H)]
    if isinstance(sample, list):
        segs = list(sample)  # explicit (request, layer, head) segments
    elif sample is not None:
        segs = [segs[i] for i in np.random.default_rng(0).choice(len(segs), sample, replace=False)]
    near_ties = 0
    for (r, l, h) in segs:
        pts = oracle.segment_points(qwin[r][l], h, G)
        n = len(pts)
        ga = g_assign[r, l, h, :n]
        c_o, cnt_o, a_o = oracle.beacon_update(pts, np.zeros((B, d)), np.zeros(B), init=True)
        if not np.array_equal(a_o, ga):
            # differing assignments must be near-ties of the squared distance
            c0 = pts[(np.arange(B) * n) // B]
            for p in np.nonzero(a_o != ga)[0]:
                d_o = np.sum((pts[p] - c0[a_o[p]]) ** 2)
                d_g = np.sum((pts[p] - c0[ga[p]]) ** 2)
                assert abs(d_o - d_g) <= 1e-5 * max(d_o, 1e-30), (r, l, h, p, d_o, d_g)
                near_ties += 1
        c_s, cnt_s, _ = oracle.beacon_update(pts, np.zeros((B, d)), np.zeros(B), init=True, assign_override=ga)
        assert np.array_equal(cnt_s, g_counts[r, l, h])
        # trigger shares: this update's points per beacon / points (one fp32 division)
        share = (np.bincount(ga, minlength=B).astype(np.float32) / np.float32(n)).astype(np.float32)
        assert np.array_equal(g_trig[r, l, h], share), (r, l, h)
        assert np.allclose(g_beacons[r, l, h], c_s, rtol=1e-5, atol=1e-6), (r, l, h)
    # the round
    if k_hook is not None:
        k_hook(ctx)  # edits the cached keys before the pre-round snapshot
    lengths, prompts = ctx.lengths()
    cap = int(lengths.max())
    need_l = sorted({l for (_, l, _) in segs})
    pre = {l: dense_layer(ctx, l, range(R), cap, lengths, with_kv=True) if sample is None else None
           for l in need_l}
    if sample is not None:
        # only the sampled (request, layer) pairs, to bound device memory
        for l in need_l:
            rs = sorted({r for (r, ll, _) in segs if ll == l})
            pos, k, v = dense_layer(ctx, l, rs, cap, lengths, with_kv=True)
            full_pos = np.full((R,) + pos.shape[1:], -1, np.int64)
            full_k = torch.zeros((R,) + tuple(k.shape[1:]), dtype=k.dtype, device=k.device)
            full_v = torch.zeros_like(full_k)
            idx = torch.as_tensor(rs, device=k.device)
            full_pos[rs] = pos
            full_k[idx] = k
            full_v[idx] = v
            pre[l] = (full_pos, full_k, full_v)
    scores = torch.zeros((R, Ly, H, ctx.spec.max_seq_len), dtype=torch.float32, device="cuda")
    budgets = w.budget.astype(np.int32)
    stats = ctx.compress(selector, budgets, w.philox_seed, debug_scores=scores, stats=True,
                         sink_tokens=sinks, compaction=compaction)
    ctx.sync()
    new_len, _ = ctx.lengths()
    g_scores = scores.cpu().numpy()
    max_rel = 0.0
    differ = in_abs = in_rel = 0
    for (r, l, h) in segs:
        L, P, K = int(lengths[r]), int(prompts[r]), int(budgets[r])
        if sinks is not None:
            P = min(P, sinks)
        keys = pre[l][1][r, h, :L].float().cpu().numpy().astype(np.float64)
        if selector == "beacon_trigger":
            o_sc = oracle.beacon_trigger_score(keys, g_scoring[r, l, h], g_trig[r, l, h].astype(np.float64), P)
        else:
            o_sc, _ = oracle.beacon_score(keys, g_scoring[r, l, h], P)
        if L <= K:
            continue
        N, M = L - P, max(0, K - P)
        assert new_len[r] == P + M
        if M == 0:
            continue
        max_rel = max(max_rel, check_scores(g_scores[r, l, h, :N], o_sc))
        post_pos, post_k, post_v = dense_layer(ctx, l, [r], int(new_len[r]), new_len, with_kv=True)
        gpu_kept = np.searchsorted(pre[l][0][r, h, :L], post_pos[0, h])
        assert np.array_equal(pre[l][0][r, h, gpu_kept], post_pos[0, h])
        assert np.array_equal(gpu_kept[:P], np.arange(P))
        if compaction == "hole_fill":
            # same kept set as order-preserving compaction, laid out by hole filling
            assert np.array_equal(gpu_kept, oracle.hole_fill(P + M, np.sort(gpu_kept)))
        dd, ia, ir = band_check(np.sort(gpu_kept)[P:], o_sc, P, M, N)
        differ += dd
        in_abs += ia
        in_rel += ir
        # compacted bytes follow the GPU's own selection exactly
        ks = torch.as_tensor(gpu_kept, device="cuda")
        assert torch.equal(post_k[0, h], pre[l][1][r, h, ks])
        assert torch.equal(post_v[0, h], pre[l][2][r, h, ks])
    ctx.close()
    return {"near_tie_assignments": near_ties, "max_rel_score_err": max_rel, "index_differ": differ,
            "in_band_abs": in_abs, "in_band_rel": in_rel, "stats": stats}


def test_tiny_beacon():
    out = run_beacon(wl.tiny())
    assert out["index_differ"] == 0


def test_beacon_serving_small():
    out = run_beacon(wl.beacon_serving(R=3, layers=2))
    print(out)


def test_beacon_serving_full_size_sampled():
    out = run_beacon(wl.beacon_serving(), sample=24)
    print(out)


@pytest.mark.parametrize("c", [2, 4, 8, 16])
def test_ragged_beacon_sampled(c):
    """Ragged lengths 4096..32768 (the ragged sweep's first 4 requests, 2 layers) at 2x, 4x, 8x and 16x
    compression, including prompts close to and over the budget: sampled segments."""
    w = wl.scaled(wl.ragged(c), num_requests=4, num_layers=2)
    out = run_beacon(w, sample=12)
    print(c, out)


@pytest.mark.parametrize("c", [4, 8])
def test_ragged_cluster_trigger_sampled(c):
    """The cluster-trigger selector on a ragged slice (first 4 requests, 2 layers) at 4x and 8x."""
    w = wl.scaled(wl.ragged(c), num_requests=4, num_layers=2)
    out = run_beacon(w, sample=12, selector="beacon_trigger")
    print(c, out)


def test_long_trace_sampled():
    w = wl.scaled(wl.long_trace(), num_requests=2, num_layers=4)
    out = run_beacon(w, sample=3)
    print(out)


def test_long_trace_every_request():
    """All 8 requests of the long trace (two layers of 32768 keys each, 256 beacons): one sampled segment of
    every request, on alternating layers and heads."""
    w = wl.scaled(wl.long_trace(), num_layers=2)
    segs = [(r, r % 2, (3 * r) % 8) for r in range(8)]
    out = run_beacon(w, sample=segs)
    print(out)


def test_large_survivor_count():
    """Beacon selection on segments of 32768 and 9000 keys keeping most of them: the rank map is too large for the
    persistent select form's shared memory budget, so the round takes the one-CTA-per-segment kernel."""
    P = np.array([0, 100])
    L = np.array([32768, 9000])
    K = np.array([30000, 8000])
    w = wl.Workload("large_m_beacon", 2, 1, 2, 128, P, L, K, selectors=("beacon",), num_q_heads=8,
                    num_beacons=64, query_window=64, n_components=64, data_seed=47, philox_seed=53)
    out = run_beacon(w)
    print(out)


def _sharp(w):
    return wl.scaled(w, query_norm=math.sqrt(w.head_dim))


@pytest.mark.parametrize("selector", ["beacon", "beacon_trigger"])
@pytest.mark.parametrize("impl", [1, 2], ids=["simt", "tcgen05"])
def test_sharp_beacon_serving(impl, selector):
    """Queries of norm sqrt(d) at the beacon-serving shape (3 requests, 2 layers, every segment), both score
    kernels and both beacon selectors, under the strict gate."""
    out = run_beacon(_sharp(wl.beacon_serving(R=3, layers=2)), score_impl=impl, selector=selector)
    print(impl, selector, out)
    assert out["max_rel_score_err"] < 1e-4


@pytest.mark.parametrize("selector", ["beacon", "beacon_trigger"])
@pytest.mark.parametrize("impl", [1, 2], ids=["simt", "tcgen05"])
def test_sharp_long_trace(impl, selector):
    """Queries of norm sqrt(d) at the long-trace shape (32768 keys, 256 beacons; 2 requests, 2 layers,
    4 sampled segments), both score kernels and both beacon selectors, under the strict gate."""
    w = _sharp(wl.scaled(wl.long_trace(), num_requests=2, num_layers=2))
    out = run_beacon(w, sample=[(0, 0, 1), (0, 1, 6), (1, 0, 4), (1, 1, 3)], score_impl=impl, selector=selector)
    print(impl, selector, out)
    assert out["max_rel_score_err"] < 1e-4


@pytest.mark.parametrize("sinks,compaction", [(4, "ordered"), (None, "hole_fill"), (0, "hole_fill")])
def test_beacon_round_options(sinks, compaction):
    """Sink-only protection and hole-filling compaction under the beacon selector."""
    out = run_beacon(wl.beacon_serving(R=3, layers=2), sinks=sinks, compaction=compaction)
    print(sinks, compaction, out)


@pytest.mark.parametrize("impl", [1, 2], ids=["simt", "tcgen05"])
def test_cluster_trigger_selector(impl):
    """The cluster-trigger score (trigger-share-weighted beacon attention) on both kernels."""
    out = run_beacon(wl.beacon_serving(R=3, layers=2), score_impl=impl, selector="beacon_trigger")
    print(impl, out)


def test_cluster_trigger_256_beacons():
    w = wl.scaled(wl.long_trace(), num_requests=1, num_layers=2)
    w.length = np.array([4133])
    w.budget = np.array([1000])
    w.prompt = np.array([77])
    out = run_beacon(w, score_impl=2, selector="beacon_trigger", compaction="hole_fill")
    print(out)


@pytest.mark.parametrize("impl", [1, 2], ids=["simt", "tcgen05"])
def test_score_kernels_small(impl):
    """Both beacon-score kernels (SIMT fp32 and tcgen05) against the oracle."""
    out = run_beacon(wl.beacon_serving(R=2, layers=2), score_impl=impl)
    print(impl, out)


@pytest.mark.parametrize("B", [128, 192])
def test_tcgen05_non_duplicated_beacon_tiles(B):
    """128 beacons (one beacon copy per tile, four 128-column accumulator buffers) and 192 (two 128-row
    halves, two 256-column buffers)."""
    w = wl.beacon_serving(R=2, layers=2)
    w.num_beacons = B
    out = run_beacon(w, score_impl=2)
    print(B, out)


def test_tcgen05_256_beacons():
    """The 256-beacon path of the tensor-core kernel (two M=128 halves in pass 1)."""
    w = wl.scaled(wl.long_trace(), num_requests=1, num_layers=2)
    w.length = np.array([4133])
    w.budget = np.array([1000])
    w.prompt = np.array([77])
    out = run_beacon(w, score_impl=2)
    print(out)


def test_tcgen05_scattered_pages():
    """Two requests filled one page at a time in turn: no 8-page key tile has consecutive page ids, so every
    tile comes in as per-page boxes (with consecutive ids a tile is two 8-page boxes)."""
    w = wl.beacon_serving(R=2, layers=2)
    out = run_beacon(w, score_impl=2, interleave=True)
    print(out)


def _plant_dominant_keys(slots, z):
    """Overwrites the keys at `slots` of every segment with a multiple of the segment's scoring beacon 0,
    scaled so that z_0j = c_0.k_j / sqrt(d) is about z: a logit far above every earlier one."""
    def hook(ctx):
        st = ctx.state_tensors()
        bt = st["block_table"].cpu().numpy()
        c0 = st["beacons_scoring"][:, :, :, 0, :].float()  # [R, Ly, H, d]
        R, Ly, H, d = c0.shape
        for r in range(R):
            for l in range(Ly):
                for h in range(H):
                    lam = z * d ** 0.5 / float((c0[r, l, h] ** 2).sum())
                    for j in slots:
                        ctx.k_pool[l, int(bt[r, j // 16]), h, j % 16] = (lam * c0[r, l, h]).to(ctx.dtype)
        ctx.sync()
    return hook


@pytest.mark.parametrize("B", [64, 256])
def test_tcgen05_logit_far_above_running_max(B):
    """Keys whose logit sits ~200 above every earlier key of the segment: the pass-1 chunk sum against the
    running reference would overflow, so that chunk must take the exact rescaling path.  Slot 1000 lies in
    a full 64-key chunk of a full tile, slot 3100 in a later one."""
    w = wl.scaled(wl.long_trace(), num_requests=1, num_layers=2)
    w.num_beacons = B
    w.length = np.array([4133])
    w.budget = np.array([1000])
    w.prompt = np.array([77])
    out = run_beacon(w, score_impl=2, k_hook=_plant_dominant_keys([1000, 3100], 200.0))
    print(B, out)


@pytest.mark.parametrize("impl,B,W,Hq", [(1, 64, 64, 32), (2, 64, 64, 32), (2, 32, 64, 32), (2, 96, 64, 32),
                                         (2, 128, 64, 32), (2, 256, 64, 32), (2, 64, 40, 32), (2, 64, 50, 16),
                                         (2, 192, 64, 32), (2, 160, 100, 16), (2, 256, 256, 32),
                                         (2, 64, 64, 24), (2, 256, 96, 24)],
                         ids=["simt-64", "tc-64", "tc-32", "tc-96", "tc-128", "tc-256", "tc-64-160pts",
                              "tc-64-G2-100pts", "tc-192", "tc-160-G2-200pts", "tc-256-1024pts",
                              "tc-64-G3", "tc-256-G3"])
def test_second_update_against_oracle(impl, B, W, Hq):
    """A later (non-initial) update: fp32 beacons with counts, new points.
    The oracle recomputes it from the GPU's beacons and counts before the
    update; assignments may differ only on near-ties within the kernels'
    error bound (fp32 rounding, plus 2^-18 sum|x_k c_k| per dot product for
    the tensor-core kernel's two-term bf16 split of the beacons).  Two cases
    leave the last 128-point tile partly filled (160 points; G = 2 with 100
    points, a single partial tile).  More than 128 beacons split over a CTA
    pair: 192 and 160 (second halves of 64 and 32 beacons, the latter with a
    partial last tile) and 256 over the long trace's 1024-point window.  G = 3 (24 query heads) does not
    divide a 128-point tile into whole ring slots: those updates take the one-CTA-per-segment kernel."""
    w = wl.beacon_serving(R=2, layers=2)
    w.num_beacons = B
    w.num_q_heads = Hq
    w.query_window = max(W, B // (Hq // 8))  # the first update needs at least B points
    ctx = make_context(w, headroom=256)
    ctx.set_option(1, impl)
    gen = wl.Generator(w, "cuda")
    _fill_recording(ctx, w, gen)
    ctx.update_beacons()
    ctx.sync()
    st = ctx.state_tensors()
    c_before = st["beacons"].double().cpu().numpy()
    n_before = st["beacon_counts"].cpu().numpy().astype(np.int64)
    R, Ly, H, d, G = 2, 2, 8, 128, Hq // 8
    W = w.query_window
    q = gen.queries(R, W)
    k, v = gen.kv(R, W)
    ctx.append(np.arange(R, dtype=np.int32), k, v, q)
    assign = torch.full((R, Ly, H, w.query_window * G), -1, dtype=torch.int32, device="cuda")
    ctx.update_beacons(assign_out=assign)
    ctx.sync()
    g_beacons = st["beacons"].double().cpu().numpy()
    g_counts = st["beacon_counts"].cpu().numpy()
    g_assign = assign.cpu().numpy()
    qn = q.float().cpu().numpy().astype(np.float64)  # [R, Ly, W, Hq, d]
    ties = 0
    for r in range(R):
        for l in range(Ly):
            for h in range(H):
                pts = oracle.segment_points(qn[r, l], h, G)
                c0 = c_before[r, l, h]
                _, _, a_o = oracle.beacon_update(pts, c0, n_before[r, l, h], init=False)
                ga = g_assign[r, l, h, :len(pts)]
                for p in np.nonzero(a_o != ga)[0]:
                    d_o = np.sum((pts[p] - c0[a_o[p]]) ** 2)
                    d_g = np.sum((pts[p] - c0[ga[p]]) ** 2)
                    bound = 4 * 2.0 ** -18 * max(np.abs(pts[p] * c0[a_o[p]]).sum(),
                                                 np.abs(pts[p] * c0[ga[p]]).sum()) + 1e-5 * d_o
                    assert d_g - d_o <= bound, (r, l, h, p, d_o, d_g, bound)
                    ties += 1
                c_s, cnt_s, _ = oracle.beacon_update(pts, c0, n_before[r, l, h], init=False, assign_override=ga)
                assert np.array_equal(cnt_s, g_counts[r, l, h])
                assert np.allclose(g_beacons[r, l, h], c_s, rtol=1e-5, atol=1e-6)
    ctx.close()
    print("near-tie assignments:", ties)
