"""Helpers shared by the GPU parity tests.

The device state is read back with plain torch indexing of the pools and of
the workspace views (independent of the library's own gather kernel), and
compared with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from decode_kv_cache_paged_b200 import Context, ContextSpec, workloads as wl

# Beacon-score tolerances, two gates, both asserted.
# Stated gate: |gpu - oracle| <= ABS + REL*|oracle| for scores; selected
# indices may differ only within BAND (absolute) of the M-th oracle score.
# At the serving shapes scores sit near 1/L (~5e-4), so the stated gate alone
# would admit a 2 % score error and almost every candidate into the band.
SCORE_ABS, SCORE_REL, BAND = 1e-5, 1e-3, 1e-4
# Strict gate: relative score error <= STRICT_REL (floor STRICT_ABS for
# scores that underflow), and indices may differ only within STRICT_BAND*tau
# of the threshold tau.  The kernels' fp32 arithmetic (bf16 x bf16 products
# exact, fp32 sums over <= 32768 keys, exp2 with ~2^-22 relative error) puts
# the relative score error near 1e-5; two scores each off by at most that can
# only swap places when they lie within ~2e-5*tau of each other.
STRICT_ABS, STRICT_REL, STRICT_BAND = 1e-9, 1e-4, 1e-4


def make_context(w: wl.Workload, headroom: int = 0, device="cuda", extra_pages: int = 0) -> Context:
    spec = ContextSpec(num_requests=w.num_requests, num_layers=w.num_layers, num_kv_heads=w.num_kv_heads,
                       head_dim=w.head_dim, max_seq_len=w.max_seq_len(headroom),
                       num_pages=w.pages_needed(headroom) + w.num_requests + extra_pages,
                       num_q_heads=w.num_q_heads or w.num_kv_heads, num_beacons=w.num_beacons,
                       query_window=w.query_window)
    return Context(spec, dtype=wl.torch_dtype(w.dtype), device=device)


def seg_rows(ctx: Context, layer: int, reqs, cap: int):
    """Global row index [n, Hkv, cap] of slot s of each (request, head) segment (-1 past the table)."""
    st = ctx.state_tensors()
    bt = st["block_table"][torch.as_tensor(np.asarray(reqs), device=ctx.device).long()]  # [n, maxp]
    H = ctx.spec.num_kv_heads
    slots = torch.arange(cap, device=ctx.device)
    page = bt[:, slots // 16].long()  # [n, cap]
    h = torch.arange(H, device=ctx.device).view(1, H, 1)
    rows = ((layer * ctx.spec.num_pages + page.unsqueeze(1)) * H + h) * 16 + (slots % 16).view(1, 1, cap)
    return rows, page.unsqueeze(1).expand_as(rows) >= 0


def dense_layer(ctx: Context, layer: int, reqs, cap: int, lengths, with_kv: bool = True):
    """(pos [n,H,cap] int64 numpy, k, v [n,H,cap,d] torch on device or None) of the
    requests' segments in one layer; slots at or past the request's length read as
    -1 (pos) / 0 (k, v)."""
    rows, ok = seg_rows(ctx, layer, reqs, cap)
    ln = torch.as_tensor(np.asarray([lengths[r] for r in reqs]), device=ctx.device).view(-1, 1, 1)
    ok = ok & (torch.arange(cap, device=ctx.device).view(1, 1, cap) < ln)
    st = ctx.state_tensors()
    pos_flat = st["pos_map"].reshape(-1)
    safe = torch.where(ok, rows, torch.zeros_like(rows))
    pos = torch.where(ok, pos_flat[safe], torch.full_like(safe, -1, dtype=torch.int32))
    k = v = None
    if with_kv:
        d = ctx.spec.head_dim
        kf = ctx.k_pool.reshape(-1, d)
        vf = ctx.v_pool.reshape(-1, d)
        m = ok.unsqueeze(-1)
        k = torch.where(m, kf[safe.reshape(-1)].reshape(*rows.shape, d), torch.zeros((), dtype=kf.dtype, device=kf.device))
        v = torch.where(m, vf[safe.reshape(-1)].reshape(*rows.shape, d), torch.zeros((), dtype=vf.dtype, device=vf.device))
    return pos.cpu().numpy().astype(np.int64), k, v


def as_bytes(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a tensor's last dim (bit-exact comparisons)."""
    t = t.contiguous()
    return t.view(torch.uint8).cpu().numpy() if t.dtype != torch.uint8 else t.cpu().numpy()


def oracle_random_round(pre_pos: dict, lengths, prompts, budgets, seed: int, rnd: int, shared: bool,
                        layers, H: int, reqs):
    """Expected post-round position maps from the oracle for every segment.

    pre_pos[l] is [n, H, cap] for requests `reqs`.  Returns dict l -> (pos [n,H,cap], R [n])."""
    out = {}
    for l in layers:
        P = pre_pos[l]
        n, _, cap = P.shape
        rlh = np.array([[r, l, h] for r in reqs for h in range(H)], np.int64)
        lpk = np.array([[lengths[r], prompts[r], budgets[r]] for r in reqs for h in range(H)], np.int64)
        pos_in = np.ascontiguousarray(P.reshape(n * H, cap), dtype=np.int32)
        # slots past L must not be read by the oracle: it only looks at [0, L)
        pos_out, R = oracle.random_round_batch(seed, rnd, shared, rlh, lpk, pos_in)
        out[l] = (pos_out.reshape(n, H, cap).astype(np.int64), R.reshape(n, H))
    return out


def kept_slots(pre_pos_seg: np.ndarray, post_pos_seg: np.ndarray) -> np.ndarray:
    """Slots (pre-round) of the positions present after the round (positions are unique and increasing)."""
    idx = np.searchsorted(pre_pos_seg, post_pos_seg)
    assert np.array_equal(pre_pos_seg[idx], post_pos_seg)
    return idx


def check_random_layer(ctx, reqs, lengths_pre, pre_pos, post_pos, exp_pos, exp_R, new_len, pre_kv=None,
                       post_kv=None, tag=""):
    """Position maps exact for every segment of one layer; K/V bytes exact where given."""
    H = ctx.spec.num_kv_heads
    for i, r in enumerate(reqs):
        for h in range(H):
            Rn = int(exp_R[i, h])
            assert new_len[r] == Rn, (tag, r, new_len[r], Rn)
            assert np.array_equal(post_pos[i, h, :Rn], exp_pos[i, h, :Rn]), (tag, r, h)
            if pre_kv is not None:
                L = int(lengths_pre[r])
                ks = torch.as_tensor(kept_slots(pre_pos[i, h, :L], exp_pos[i, h, :Rn]), device=ctx.device)
                for pre_t, post_t in zip(pre_kv, post_kv):
                    assert np.array_equal(as_bytes(post_t[i, h, :Rn]), as_bytes(pre_t[i, h, ks])), (tag, r, h)


def band_check(gpu_kept: np.ndarray, oracle_scores: np.ndarray, P: int, M: int, N: int):
    """Kept set equal to the oracle's except for positions whose oracle score lies
    within STRICT_BAND*tau of the threshold tau (which also puts them within the
    absolute BAND); returns (n_differ, n_in_band_abs, n_in_band_rel)."""
    s32 = oracle_scores.astype(np.float32).astype(np.float64)
    order = sorted(range(N), key=lambda j: (-s32[j], j))
    o_kept = np.zeros(N, bool)
    o_kept[order[:M]] = True
    g = np.zeros(N, bool)
    g[gpu_kept - P] = True
    assert g.sum() == M
    tau = s32[order[M - 1]] if M > 0 else np.inf
    differ = np.nonzero(g != o_kept)[0]
    for j in differ:
        assert abs(oracle_scores[j] - tau) <= BAND, (j, oracle_scores[j], tau)
        assert abs(oracle_scores[j] - tau) <= STRICT_BAND * abs(tau), ("strict band", j, oracle_scores[j], tau)
    in_abs = int(np.sum(np.abs(oracle_scores - tau) <= BAND))
    in_rel = int(np.sum(np.abs(oracle_scores - tau) <= BAND * abs(tau)))
    return len(differ), in_abs, in_rel


def check_scores(gpu: np.ndarray, ora: np.ndarray):
    """Both score gates, element by element; returns the largest relative error."""
    err = np.abs(gpu.astype(np.float64) - ora)
    bad = err > SCORE_ABS + SCORE_REL * np.abs(ora)
    assert not bad.any(), (np.nonzero(bad)[0][:8], gpu[bad][:8], ora[bad][:8])
    bad = err > STRICT_ABS + STRICT_REL * np.abs(ora)
    assert not bad.any(), ("strict", np.nonzero(bad)[0][:8], gpu[bad][:8], ora[bad][:8])
    return float((err / np.maximum(np.abs(ora), 1e-30)).max())
