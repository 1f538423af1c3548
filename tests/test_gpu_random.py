"""Random-Attention rounds on the GPU against the oracle: position maps, K/V
bytes and the 32-bit Philox scores, bit-exact, over several steady-state
rounds, ragged lengths and the degenerate cases of the retention rule."""
import numpy as np
import pytest
import torch

import oracle
from decode_kv_cache_paged_b200 import workloads as wl
from gpu_helpers import check_random_layer, dense_layer, make_context, oracle_random_round

pytestmark = pytest.mark.gpu


def _edge_workload(d=128, dtype="bf16", layers=2, H=4):
    # request: (P, L, K) covering the regimes of the retention rule
    cases = [
        (1024, 2112, 2048),  # serving shape: evict 64 of 1088
        (16, 256, 64),       # tiny shape
        (0, 300, 100),       # no prompt
        (300, 600, 200),     # prompt over budget: keep only the prompt
        (64, 100, 64),       # prompt fills the budget exactly
        (100, 150, 200),     # no-op: L <= K
        (10, 1200, 11),      # keep one generated position
        (5, 1300, 1303),     # no-op by 3
        (7, 4133, 1000),     # several tiles, ragged tail
        (0, 0, 10),          # empty request
        (33, 9000, 8900),    # large N, few evictions
    ]
    P = np.array([c[0] for c in cases])
    L = np.array([c[1] for c in cases])
    K = np.array([c[2] for c in cases])
    return wl.Workload("edge", len(cases), layers, H, d, P, L, K, dtype=dtype,
                       selectors=("random", "random_shared"), trigger=40, data_seed=77, philox_seed=5)


def run_rounds(w, selector, rounds, seed, kv_layers=None, req_sample=None, check_scores_n=200):
    torch.manual_seed(0)
    headroom = max(0, int(max(w.budget.max(), w.prompt.max()) + w.trigger - w.length.max()))
    ctx = make_context(w, headroom=headroom)
    gen = wl.Generator(w, "cuda")
    wl.fill(ctx, w, gen, with_queries=False)
    R, Ly, H = w.num_requests, w.num_layers, w.num_kv_heads
    reqs = list(range(R)) if req_sample is None else list(req_sample)
    kv_layers = list(range(Ly)) if kv_layers is None else list(kv_layers)
    budgets = w.budget.astype(np.int32)
    shared = selector == "random_shared"
    for rd in range(rounds):
        lengths, prompts = ctx.lengths()
        cap = int(max(lengths.max(), 16))
        pre = {}
        for l in range(Ly):
            pre[l] = dense_layer(ctx, l, reqs, cap, lengths, with_kv=l in kv_layers)
        dbg = torch.zeros((R, Ly, H, ctx.spec.max_seq_len), dtype=torch.int32, device="cuda")
        stats = ctx.compress(selector, budgets, seed, debug_scores=dbg, stats=True)
        ctx.sync()
        assert stats["round"] == rd
        new_len, _ = ctx.lengths()
        exp = oracle_random_round({l: pre[l][0] for l in pre}, lengths, prompts, budgets, seed, rd, shared,
                                  range(Ly), H, reqs)
        moved_total = 0
        for l in range(Ly):
            post = dense_layer(ctx, l, reqs, cap, new_len, with_kv=l in kv_layers)
            pre_kv = (pre[l][1], pre[l][2]) if l in kv_layers else None
            post_kv = (post[1], post[2]) if l in kv_layers else None
            check_random_layer(ctx, reqs, lengths, pre[l][0], post[0], exp[l][0], exp[l][1], new_len,
                               pre_kv, post_kv, tag=f"round {rd} layer {l}")
            # moved rows: survivors after the first evicted slot
            for i, r in enumerate(reqs):
                for h in range(H):
                    L, P, Rn = int(lengths[r]), int(prompts[r]), int(exp[l][1][i, h])
                    if Rn < L and Rn > P:
                        same = pre[l][0][i, h, :Rn] == exp[l][0][i, h, :Rn]
                        first = int(np.argmin(same)) if not same.all() else Rn
                        moved_total += Rn - first
        if req_sample is None:
            assert stats["moved_rows"] == moved_total
            assert stats["head_positions"] == int(lengths.sum()) * Ly * H
        # debug scores: the 32-bit Philox draws of a sample of candidates
        dbg_np = dbg.cpu().numpy().view(np.uint32)
        rng = np.random.default_rng(rd)
        checked = 0
        for _ in range(check_scores_n):
            i = int(rng.integers(len(reqs)))
            r = reqs[i]
            L, P, K = int(lengths[r]), int(prompts[r]), int(budgets[r])
            if L <= K or L - P == 0 or K - P <= 0:
                continue
            l, h = int(rng.integers(Ly)), int(rng.integers(H))
            j = int(rng.integers(L - P))
            pos = int(pre[l][0][i, h, P + j])
            want = oracle.random_score(seed, rd, r, l, h, pos, shared)
            assert int(dbg_np[r, l, h, j]) == want, (r, l, h, j)
            checked += 1
        # steady state: the trigger window of new tokens
        k, v = gen.kv(R, w.trigger)
        ctx.append(np.arange(R, dtype=np.int32), k, v)
    ctx.sync()
    ctx.close()


def test_tiny_random():
    w = wl.tiny()
    w.num_beacons = 0
    run_rounds(w, "random", rounds=3, seed=w.philox_seed)


def test_tiny_random_shared():
    w = wl.tiny()
    w.num_beacons = 0
    run_rounds(w, "random_shared", rounds=2, seed=w.philox_seed)


@pytest.mark.parametrize("selector", ["random", "random_shared"])
def test_edge_cases_bf16(selector):
    run_rounds(_edge_workload(), selector, rounds=3, seed=123)


def test_edge_cases_d64_and_f32():
    run_rounds(_edge_workload(d=64, layers=1, H=2), "random", rounds=2, seed=9)
    run_rounds(_edge_workload(d=128, dtype="f32", layers=1, H=2), "random", rounds=2, seed=10)


def test_shared_variant_identical_across_heads():
    w = _edge_workload(layers=1, H=4)
    ctx = make_context(w)
    gen = wl.Generator(w, "cuda")
    wl.fill(ctx, w, gen, with_queries=False)
    ctx.compress("random_shared", w.budget.astype(np.int32), 3)
    ctx.sync()
    ln, _ = ctx.lengths()
    pos, _, _ = dense_layer(ctx, 0, range(w.num_requests), int(ln.max()), ln, with_kv=False)
    for h in range(1, 4):
        assert np.array_equal(pos[:, h], pos[:, 0])
    ctx.close()


def test_serving_shape_small():
    """The random serving round's shapes on 8 requests x 4 layers, 4 rounds."""
    w = wl.random_serving(R=8, layers=4)
    run_rounds(w, "random", rounds=4, seed=w.philox_seed, kv_layers=[0, 3])


def test_serving_full_size():
    """128 requests x 36 layers x 8 KV heads (the benchmarked round): every
    segment's position map and 32-bit scores; K/V bytes of two layers."""
    w = wl.random_serving()
    run_rounds(w, "random", rounds=2, seed=w.philox_seed, kv_layers=[0, 35], check_scores_n=2000)


@pytest.mark.parametrize("c,sel", [(2, "random"), (4, "random"), (4, "random_shared"), (8, "random"),
                                   (8, "random_shared"), (16, "random_shared")])
def test_ragged_sweep_slice(c, sel):
    """Ragged lengths 4096..32768 with prompts 128..1536 at 2x, 4x, 8x and 16x compression (12-layer slice; at
    4x and 8x some prompts come close to or over the budget), random and shared selectors: every position map,
    the K/V bytes of one layer and a sample of the 32-bit draws."""
    w = wl.scaled(wl.ragged(c), num_layers=12, num_beacons=0, query_window=0, num_q_heads=8)
    run_rounds(w, sel, rounds=1, seed=w.philox_seed, kv_layers=[5], check_scores_n=500)


@pytest.mark.parametrize("selector", ["random", "random_shared"])
def test_large_survivor_counts(selector):
    """Segments of up to 32768 candidates that keep most of them: the rank map is too large for the persistent
    form's shared memory budget, so the round takes the one-CTA-per-segment kernel (two rounds)."""
    cases = [(0, 32768, 30000), (100, 20000, 19000), (50, 5000, 4000), (7, 4133, 1000)]
    P = np.array([c[0] for c in cases])
    L = np.array([c[1] for c in cases])
    K = np.array([c[2] for c in cases])
    w = wl.Workload("large_m", len(cases), 1, 2, 128, P, L, K, selectors=(selector,), trigger=40,
                    data_seed=41, philox_seed=43)
    run_rounds(w, selector, rounds=2, seed=w.philox_seed, check_scores_n=400)
