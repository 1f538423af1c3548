"""Decode attention over the paged cache (kvc_decode_attention) against the
oracle.

Tolerance, derived from the kernel's fp32 arithmetic (u = 2^-24) with the
probabilistic rounding-error model of Higham and Mary (SIAM J. Sci. Comput.
2019: a sum of n rounded terms errs by at most lambda*sqrt(n)*u times the sum
of magnitudes, with probability 1 - 2 exp(-lambda^2 (1-u)^2 / 2); lambda = 8
here).  Products of bf16 values are exact in fp32.  For one query row:
  score error (natural-log units): ds <= lambda*sqrt(d + 6)*u*A + u*|s - m| + 3u,
    A = max_j scale*sum_i |q_i k_ji|, the scale*log2(e) rounding of q and the
    exp2f error (<= 2 ulp) included;
  out error per dimension c: <= max_j |v_jc| * (2*ds + 2*lambda*sqrt(L + 64)*u);
  lse error: <= ds + lambda*sqrt(L + 64)*u.
A separate test with a zero query and small-integer values is exact up to
the final division: every row must be counted exactly once."""
import numpy as np
import pytest
import torch

import oracle
from decode_kv_cache_paged_b200 import KvcError, workloads as wl
from gpu_helpers import dense_layer, make_context

pytestmark = pytest.mark.gpu

U = 2.0 ** -24
LAM = 8.0


def _workload(d=128, dtype="bf16", layers=2, H=2, Hq=8):
    cases = [  # (P, L, K)
        (1024, 2112, 2048),
        (0, 1, 10),
        (0, 0, 10),
        (16, 17, 64),
        (7, 4133, 1000),
        (33, 9000, 8900),
        (5, 63, 100),
    ]
    P = np.array([c[0] for c in cases])
    L = np.array([c[1] for c in cases])
    K = np.array([c[2] for c in cases])
    w = wl.Workload("attention", len(cases), layers, H, d, P, L, K, dtype=dtype,
                    selectors=("random",), trigger=40, data_seed=41, philox_seed=7)
    w.num_q_heads = Hq
    w.num_beacons = 0
    w.query_window = 0
    return w


def _check(ctx, w, q, out, lse, layers, scale=None, tag=""):
    """Every (layer, request, query head) row against the oracle."""
    lengths, _ = ctx.lengths()
    R, H, Hq, d = w.num_requests, w.num_kv_heads, ctx.spec.num_q_heads, w.head_dim
    G = Hq // H
    cap = int(max(lengths.max(), 16))
    out_np = out.cpu().numpy().astype(np.float64)
    lse_np = lse.cpu().numpy().astype(np.float64)
    q64 = q.float().cpu().numpy().astype(np.float64)
    sc = 1 / np.sqrt(d) if scale is None else scale
    worst = 0.0
    for li, l in enumerate(layers):
        _, k, v = dense_layer(ctx, l, range(R), cap, lengths, with_kv=True)
        k64 = k.float().cpu().numpy().astype(np.float64)
        v64 = v.float().cpu().numpy().astype(np.float64)
        for r in range(R):
            L = int(lengths[r])
            o_o, o_lse = oracle.decode_attention_gqa(q64[li, r], k64[r, :, :L], v64[r, :, :L], sc)
            if L == 0:
                assert np.all(out_np[li, r] == 0.0) and np.all(np.isneginf(lse_np[li, r])), (tag, l, r)
                continue
            for hq in range(Hq):
                h = hq // G
                s = sc * (k64[r, h, :L] @ q64[li, r, hq])
                A = np.max(sc * (np.abs(k64[r, h, :L]) @ np.abs(q64[li, r, hq])))
                ds = LAM * np.sqrt(d + 6) * U * A + U * np.max(s.max() - s) + 3 * U
                acc = LAM * np.sqrt(L + 64) * U
                tol = np.max(np.abs(v64[r, h, :L]), axis=0) * (2 * ds + 2 * acc) + 1e-30
                err = np.abs(out_np[li, r, hq] - o_o[hq])
                assert np.all(err <= tol), (tag, l, r, hq, float(err.max()), float(tol.min()))
                assert abs(lse_np[li, r, hq] - o_lse[hq]) <= ds + acc + 4 * U * abs(o_lse[hq]), (tag, l, r, hq)
                worst = max(worst, float((err / tol).max()))
    return worst


def _run(w, layer_begin=0, layer_count=None, rounds=(), scale=None, seed=0):
    headroom = max(0, int(max(w.budget.max(), w.prompt.max()) + w.trigger - w.length.max()))
    ctx = make_context(w, headroom=headroom)
    gen = wl.Generator(w, "cuda")
    wl.fill(ctx, w, gen, with_queries=False)
    for opts in rounds:
        ctx.compress("random", w.budget.astype(np.int32), 99, **opts)
    lc = w.num_layers - layer_begin if layer_count is None else layer_count
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((lc, w.num_requests, ctx.spec.num_q_heads, w.head_dim), generator=g, device="cuda")
    q = q.to(ctx.dtype)
    out, lse = ctx.decode_attention(q, layer_begin=layer_begin, scale=0.0 if scale is None else scale)
    ctx.sync()
    worst = _check(ctx, w, q, out, lse, list(range(layer_begin, layer_begin + lc)), scale)
    ctx.close()
    return worst


@pytest.mark.parametrize("Hq", [2, 8, 16], ids=["G1", "G4", "G8"])
def test_gqa_groups(Hq):
    print(_run(_workload(Hq=Hq)))


def test_after_ordered_round():
    print(_run(_workload(), rounds=[{}]))


def test_after_hole_filling_rounds():
    """Slots out of position order: attention must not depend on it."""
    print(_run(_workload(), rounds=[{"compaction": "hole_fill"}, {"compaction": "hole_fill", "block": 16}]))


@pytest.mark.parametrize("dtype,d", [("f32", 128), ("bf16", 64), ("f32", 64)])
def test_dtypes_and_head_dims(dtype, d):
    print(_run(_workload(d=d, dtype=dtype)))


def test_layer_subset_and_scale():
    w = _workload(layers=4)
    print(_run(w, layer_begin=1, layer_count=2, scale=0.05))


def test_many_layers_single_split():
    """Enough (layer, request, head) units that no split is needed."""
    w = wl.random_serving(R=16, layers=8)
    w.num_q_heads = 32
    print(_run(w))


def test_serving_full_size_sampled():
    """The benchmarked step: 128 requests x 36 layers x 8 KV heads, 32 query heads, 2048 rows after a
    round; 24 sampled (layer, request) pairs, every query head, against the oracle."""
    w = wl.random_serving()
    w.num_q_heads = 32
    ctx = make_context(w)
    gen = wl.Generator(w, "cuda")
    wl.fill(ctx, w, gen, with_queries=False)
    ctx.compress("random", w.budget.astype(np.int32), w.philox_seed)
    g = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn((w.num_layers, w.num_requests, 32, w.head_dim), generator=g, device="cuda").to(ctx.dtype)
    out, lse = ctx.decode_attention(q)
    ctx.sync()
    lengths, _ = ctx.lengths()
    rng = np.random.default_rng(3)
    sc = 1 / np.sqrt(w.head_dim)
    G = 32 // w.num_kv_heads
    worst = 0.0
    for _ in range(24):
        l, r = int(rng.integers(w.num_layers)), int(rng.integers(w.num_requests))
        L = int(lengths[r])
        _, k, v = dense_layer(ctx, l, [r], L, lengths, with_kv=True)
        k64 = k[0].float().cpu().numpy().astype(np.float64)
        v64 = v[0].float().cpu().numpy().astype(np.float64)
        q64 = q[l, r].float().cpu().numpy().astype(np.float64)
        o_o, o_lse = oracle.decode_attention_gqa(q64, k64, v64, sc)
        got = out[l, r].cpu().numpy().astype(np.float64)
        got_lse = lse[l, r].cpu().numpy().astype(np.float64)
        for hq in range(32):
            h = hq // G
            s = sc * (k64[h] @ q64[hq])
            A = np.max(sc * (np.abs(k64[h]) @ np.abs(q64[hq])))
            ds = LAM * np.sqrt(w.head_dim + 6) * U * A + U * np.max(s.max() - s) + 3 * U
            acc = LAM * np.sqrt(L + 64) * U
            tol = np.max(np.abs(v64[h]), axis=0) * (2 * ds + 2 * acc)
            err = np.abs(got[hq] - o_o[hq])
            assert np.all(err <= tol), (l, r, hq, float(err.max()))
            assert abs(got_lse[hq] - o_lse[hq]) <= ds + acc + 4 * U * abs(o_lse[hq]), (l, r, hq)
            worst = max(worst, float((err / tol).max()))
    print("worst error / bound:", worst)
    ctx.close()


def test_every_row_counted_exactly():
    """Zero query, integer values: out = exact mean of the rows (one rounding)."""
    w = _workload()
    ctx = make_context(w)
    gen = wl.Generator(w, "cuda")
    wl.fill(ctx, w, gen, with_queries=False)
    st = ctx.state_tensors()
    gi = torch.Generator(device="cuda").manual_seed(5)
    ctx.v_pool.copy_(torch.randint(-8, 9, ctx.v_pool.shape, generator=gi, device="cuda").to(ctx.dtype))
    q = torch.zeros((w.num_layers, w.num_requests, ctx.spec.num_q_heads, w.head_dim), dtype=ctx.dtype,
                    device="cuda")
    out, lse = ctx.decode_attention(q)
    ctx.sync()
    lengths, _ = ctx.lengths()
    G = ctx.spec.num_q_heads // w.num_kv_heads
    for l in range(w.num_layers):
        _, _, v = dense_layer(ctx, l, range(w.num_requests), int(lengths.max()), lengths)
        v64 = v.float().cpu().numpy().astype(np.float64)
        for r in range(w.num_requests):
            L = int(lengths[r])
            if L == 0:
                continue
            want = v64[r, :, :L].sum(1) / L  # [H, d], sums exact
            got = out[l, r].cpu().numpy().astype(np.float64)
            for hq in range(ctx.spec.num_q_heads):
                assert np.all(np.abs(got[hq] - want[hq // G]) <= 2 * U * np.abs(want[hq // G]) + 1e-30), (l, r, hq)
                assert abs(float(lse[l, r, hq]) - np.log(L)) <= 8 * U * max(1.0, np.log(L)), (l, r, hq)
    del st
    ctx.close()


def test_invalid_arguments():
    w = _workload(layers=2)
    ctx = make_context(w)
    q = torch.zeros((2, w.num_requests, ctx.spec.num_q_heads, w.head_dim), dtype=ctx.dtype, device="cuda")
    with pytest.raises(KvcError):
        ctx.decode_attention(q, layer_begin=1)  # layers 1..2 of 2
    with pytest.raises(KvcError):
        ctx.decode_attention(q, scale=-1.0)
    ctx.close()
