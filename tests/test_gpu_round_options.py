"""Round options on the GPU against the oracle: sink-only protection,
block-granular Philox draws and hole-filling compaction (kvc_compress_ex).

Every segment's position map must equal the oracle's exactly, K/V rows must
be the bytes of the slot the oracle names, the 32-bit draws of a sample of
candidates must equal the oracle's block draw, and the moved-row count must
equal the number of slots whose content changed.  Several rounds run back to
back, so rounds after a hole-filling round (slots out of position order,
ties split by position) are covered too."""
import numpy as np
import pytest
import torch

import oracle
from decode_kv_cache_paged_b200 import KvcError, workloads as wl
from gpu_helpers import as_bytes, dense_layer, make_context

pytestmark = pytest.mark.gpu


def _workload(layers=2, H=4, d=128):
    # (P, L, K): serving shape, prompt over budget, prompt-heavy, no-op,
    # ragged multi-tile, empty, large N
    cases = [
        (1024, 2112, 2048),
        (300, 600, 200),
        (900, 1000, 960),
        (100, 150, 200),
        (7, 4133, 1000),
        (0, 0, 10),
        (33, 9000, 8900),
        (64, 1500, 700),
    ]
    P = np.array([c[0] for c in cases])
    L = np.array([c[1] for c in cases])
    K = np.array([c[2] for c in cases])
    return wl.Workload("options", len(cases), layers, H, d, P, L, K, dtype="bf16",
                       selectors=("random", "random_shared"), trigger=40, data_seed=31, philox_seed=17)


def _pre_slot_of(pre_pos_seg: np.ndarray, post_pos_seg: np.ndarray) -> np.ndarray:
    """Pre-round slot of every post-round position (positions are unique)."""
    order = np.argsort(pre_pos_seg, kind="stable")
    idx = order[np.searchsorted(pre_pos_seg[order], post_pos_seg)]
    assert np.array_equal(pre_pos_seg[idx], post_pos_seg)
    return idx


def run_option_rounds(w, selector, plan, seed, kv_layers=(0,), check_scores_n=300, extra_pages=0):
    """plan: list of per-round dicts with keys sinks (None or S), block, compaction."""
    headroom = max(0, int(max(w.budget.max(), w.prompt.max()) + w.trigger - w.length.max()))
    ctx = make_context(w, headroom=headroom, extra_pages=extra_pages)
    gen = wl.Generator(w, "cuda")
    wl.fill(ctx, w, gen, with_queries=False)
    R, Ly, H = w.num_requests, w.num_layers, w.num_kv_heads
    reqs = list(range(R))
    budgets = w.budget.astype(np.int32)
    shared = selector == "random_shared"
    for rd, opt in enumerate(plan):
        sinks, block, comp = opt.get("sinks"), opt.get("block", 1), opt.get("compaction", "ordered")
        hole = comp == "hole_fill"
        lengths, prompts = ctx.lengths()
        cap = int(max(lengths.max(), 16))
        pre = {l: dense_layer(ctx, l, reqs, cap, lengths, with_kv=l in kv_layers) for l in range(Ly)}
        dbg = torch.zeros((R, Ly, H, ctx.spec.max_seq_len), dtype=torch.int32, device="cuda")
        stats = ctx.compress(selector, budgets, seed, debug_scores=dbg, stats=True, sink_tokens=sinks,
                             block=block, compaction=comp)
        ctx.sync()
        new_len, new_prompt = ctx.lengths()
        p_eff = np.array([int(prompts[r]) if sinks is None else min(int(prompts[r]), sinks) for r in reqs])
        for r in reqs:
            evicts = lengths[r] > budgets[r]
            assert new_prompt[r] == (p_eff[r] if evicts else prompts[r]), (rd, r)
        moved = 0
        for l in range(Ly):
            pre_pos = pre[l][0]
            n = len(reqs)
            rlh = np.array([[r, l, h] for r in reqs for h in range(H)], np.int64)
            lpk = np.array([[lengths[r], p_eff[r], budgets[r]] for r in reqs for h in range(H)], np.int64)
            pos_in = np.ascontiguousarray(pre_pos.reshape(n * H, cap), dtype=np.int32)
            exp_pos, exp_R = oracle.random_round_batch_ex(seed, rd, shared, block, hole, rlh, lpk, pos_in)
            exp_pos = exp_pos.reshape(n, H, cap).astype(np.int64)
            exp_R = exp_R.reshape(n, H)
            post = dense_layer(ctx, l, reqs, cap, new_len, with_kv=l in kv_layers)
            for i, r in enumerate(reqs):
                for h in range(H):
                    Rn = int(exp_R[i, h])
                    assert new_len[r] == Rn, (rd, l, r, h)
                    assert np.array_equal(post[0][i, h, :Rn], exp_pos[i, h, :Rn]), (rd, l, r, h)
                    moved += int(np.sum(pre_pos[i, h, :Rn] != exp_pos[i, h, :Rn]))
                    if l in kv_layers and Rn > 0:
                        L = int(lengths[r])
                        src = torch.as_tensor(_pre_slot_of(pre_pos[i, h, :L], exp_pos[i, h, :Rn]), device="cuda")
                        for a, b in ((post[1], pre[l][1]), (post[2], pre[l][2])):
                            assert np.array_equal(as_bytes(a[i, h, :Rn]), as_bytes(b[i, h, src])), (rd, l, r, h)
        assert stats["moved_rows"] == moved, (rd, stats["moved_rows"], moved)
        dbg_np = dbg.cpu().numpy().view(np.uint32)
        rng = np.random.default_rng(100 + rd)
        for _ in range(check_scores_n):
            r = int(rng.integers(R))
            L, P, K = int(lengths[r]), int(p_eff[r]), int(budgets[r])
            if L <= K or L - P == 0 or K - P <= 0:
                continue
            l, h = int(rng.integers(Ly)), int(rng.integers(H))
            j = int(rng.integers(L - P))
            pos = int(pre[l][0][r, h, P + j])
            assert int(dbg_np[r, l, h, j]) == oracle.random_score_block(seed, rd, r, l, h, pos, shared, block)
        k, v = gen.kv(R, w.trigger)
        ctx.append(np.arange(R, dtype=np.int32), k, v)
    ctx.sync()
    ctx.close()


@pytest.mark.parametrize("sinks", [0, 4, 128])
def test_sink_protection(sinks):
    plan = [{"sinks": sinks}, {"sinks": sinks}, {}]
    run_option_rounds(_workload(), "random", plan, seed=5)


@pytest.mark.parametrize("block", [16, 64, 256])
@pytest.mark.parametrize("selector", ["random", "random_shared"])
def test_block_draws(block, selector):
    run_option_rounds(_workload(), selector, [{"block": block}, {"block": block}], seed=11)


@pytest.mark.parametrize("selector", ["random", "random_shared"])
def test_block_draws_as_long_as_the_segment(selector):
    """One draw for a whole segment (block 32768: every candidate ties and the lowest slots stay, so no row
    moves) and two draws for the 4133-slot request (block 4096: a few dozen rows move): the persistent select
    form's rounds whose copy is empty or a single chunk."""
    run_option_rounds(_workload(), selector, [{"block": 32768}, {"block": 4096}, {}], seed=13)


def test_block_one_equals_default():
    w = _workload(layers=1, H=2)
    run_option_rounds(w, "random", [{"block": 1}, {}], seed=3)


def test_hole_fill_then_ordered():
    """Hole filling, hole filling again on the scrambled slots, then an
    order-preserving round that must split ties by position."""
    plan = [{"compaction": "hole_fill"}, {"compaction": "hole_fill"}, {}, {"block": 16}]
    run_option_rounds(_workload(), "random", plan, seed=23, kv_layers=(0, 1))


def test_hole_fill_blocks_and_sinks():
    plan = [{"compaction": "hole_fill", "block": 64, "sinks": 4},
            {"compaction": "hole_fill", "block": 16},
            {"block": 64, "sinks": 4}]
    run_option_rounds(_workload(), "random_shared", plan, seed=29)


def test_serving_shape_hole_fill():
    w = wl.random_serving(R=8, layers=4)
    run_option_rounds(w, "random", [{"compaction": "hole_fill"}] * 3 + [{}], seed=w.philox_seed,
                      kv_layers=(0, 3))


def test_invalid_options():
    w = _workload(layers=1, H=2)
    ctx = make_context(w)
    b = w.budget.astype(np.int32)
    for kw in ({"block": 0}, {"block": 40000}, {"compaction": 7}):
        with pytest.raises(KvcError):
            ctx.compress("random", b, 1, **kw)
    with pytest.raises(KvcError):
        ctx.compress("beacon", b, 1, block=16)
    ctx.close()
