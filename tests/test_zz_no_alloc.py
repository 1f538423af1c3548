"""kvc_beacon_select_noalloc, the entry point for callers that cannot allocate
device memory (graph-capturing code, plug-ins confined to another engine's
memory arena, hosts without a device allocator).

It must agree with kvc_compress(KVC_SEL_BEACON) on the same keys and beacons,
and with the oracle's beacon score and selection under both score gates
(the stated one and the strict relative one), on two calls in a row of
different shapes, while keeping its scratch in the library's own fixed device
array.  Also covered: fp32 keys, the no-eviction and prompt-only rounds
(scores_out left untouched), a call at exactly the scratch limit, and a NaN
key (its segment's candidates rank last).  Collected last so that a failure
here stops a -x run only after every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import decode_kv_cache_paged_b200 as kvc
import oracle
from decode_kv_cache_paged_b200 import Context, ContextSpec
from gpu_helpers import band_check, check_scores

pytestmark = pytest.mark.gpu

SENTINEL = -7.25


def _vp(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _call(keys, beacons, S, L, P, K, B, d, dtype, kept, scores):
    stream = torch.cuda.current_stream()
    dt = kvc.KVC_BF16 if dtype == torch.bfloat16 else kvc.KVC_F32
    st = kvc.kvc_beacon_select_noalloc(_vp(keys), _vp(beacons), S, L, P, K, B, d, dt, _vp(kept), _vp(scores),
                                       ctypes.c_void_p(stream.cuda_stream))
    assert st == kvc.KVC_OK, kvc.kvc_last_error(None)
    torch.cuda.synchronize()


def _against_oracle(keys, beacons, P, M, got_scores, got_kept, segs):
    """Scores of the listed segments within both gates of the oracle's; kept sets equal outside the
    strict threshold band."""
    kd = keys.float().cpu().numpy().astype(np.float64)
    cd = beacons.float().cpu().numpy().astype(np.float64)
    L = kd.shape[1]
    N = L - P
    for h in segs:
        o_sc, _ = oracle.beacon_score(kd[h], cd[h], P)
        check_scores(got_scores[h], o_sc)
        assert np.array_equal(got_kept[h, :P], np.arange(P))
        band_check(got_kept[h, P:], o_sc, P, M, N)


def _one_case(seed, H, L, P, K, B, d, dtype=torch.bfloat16, W=16):
    """Context path vs allocation-free path on H dense segments (1 request, 1 layer), and both vs the oracle."""
    G = 2
    spec = ContextSpec(num_requests=1, num_layers=1, num_kv_heads=H, head_dim=d, max_seq_len=(L + 15) // 16 * 16,
                       num_pages=(L + 15) // 16 + 2, num_q_heads=H * G, num_beacons=B, query_window=W)
    ctx = Context(spec, dtype=dtype)
    g = torch.Generator(device="cuda").manual_seed(seed)
    k = torch.randn((1, 1, L, H, d), generator=g, device="cuda").to(dtype)
    v = torch.randn((1, 1, L, H, d), generator=g, device="cuda").to(dtype)
    q = torch.randn((1, 1, W, H * G, d), generator=g, device="cuda").to(dtype)
    ctx.append([0], k[:, :, :P].contiguous(), v[:, :, :P].contiguous(), protect=True)
    ctx.append([0], k[:, :, P:L - W].contiguous(), v[:, :, P:L - W].contiguous())
    ctx.append([0], k[:, :, L - W:].contiguous(), v[:, :, L - W:].contiguous(), q)
    ctx.update_beacons()
    keys = k[0, 0].permute(1, 0, 2).contiguous()                        # [H, L, d]
    beacons = ctx.state_tensors()["beacons_scoring"][0, 0].contiguous()  # [H, B, d]
    N, M = L - P, (max(0, K - P) if L > K else L - P)
    R = P + M
    dbg = torch.zeros((1, 1, H, spec.max_seq_len), dtype=torch.float32, device="cuda")
    ctx.compress("beacon", np.array([K], np.int32), 0, debug_scores=dbg)
    ctx.sync()
    _, _, pos = ctx.gather_dense(0, cap=R)
    want_kept = pos[0].cpu().numpy()          # positions == slots in the first round
    want_scores = dbg[0, 0, :, :N].cpu().numpy().astype(np.float64)

    kept = torch.full((H, R), -1, dtype=torch.int32, device="cuda")
    scores = torch.full((H, max(N, 1)), SENTINEL, dtype=torch.float32, device="cuda")
    _call(keys, beacons, H, L, P, K, B, d, dtype, kept, scores)
    got_scores = scores.cpu().numpy().astype(np.float64)
    got_kept = kept.cpu().numpy()
    evicts_some = L > K and 0 < M < N
    if not evicts_some:
        # nothing to rank: the prompt (and every candidate when L <= K) stays, scores_out untouched
        assert np.array_equal(got_kept, np.tile(np.arange(R), (H, 1)))
        assert np.all(got_scores == SENTINEL)
        assert np.array_equal(got_kept, want_kept)
        ctx.close()
        return
    # the context path: same scores (same arithmetic in the same order), same kept sets up to the band
    check_scores(got_scores, want_scores)
    for h in range(H):
        assert np.array_equal(got_kept[h, :P], np.arange(P))
        assert np.all(np.diff(got_kept[h]) > 0)
        band_check(want_kept[h, P:], got_scores[h], P, M, N)
    # the oracle
    _against_oracle(keys, beacons, P, M, got_scores, got_kept, range(H))
    ctx.close()


def test_noalloc_matches_compress_two_calls_in_a_row():
    _one_case(seed=1, H=4, L=700, P=60, K=300, B=16, d=128)
    _one_case(seed=2, H=8, L=450, P=32, K=128, B=8, d=64)


def test_noalloc_f32_keys():
    _one_case(seed=3, H=2, L=530, P=17, K=200, B=12, d=128, dtype=torch.float32)


@pytest.mark.parametrize("L,P,K", [(300, 40, 300), (300, 40, 512), (400, 120, 100), (400, 120, 120)],
                         ids=["L=K", "L<K", "K<P", "K=P"])
def test_noalloc_nothing_to_rank(L, P, K):
    """No eviction (L <= K) and prompt-only rounds (K <= P < L): kept slots only, scores_out untouched."""
    _one_case(seed=4, H=2, L=L, P=P, K=K, B=8, d=64)


def test_noalloc_at_the_scratch_limit():
    """S*(L-P) exactly 2^20 scores: accepted, and sampled segments match the oracle."""
    S, L, P, K, B, d = 32, 32768, 0, 8192, 8, 64
    g = torch.Generator(device="cuda").manual_seed(5)
    keys = torch.randn((S, L, d), generator=g, device="cuda").bfloat16()
    beacons = (torch.randn((S, B, d), generator=g, device="cuda") * 0.3).bfloat16()
    kept = torch.full((S, K), -1, dtype=torch.int32, device="cuda")
    scores = torch.zeros((S, L - P), dtype=torch.float32, device="cuda")
    _call(keys, beacons, S, L, P, K, B, d, torch.bfloat16, kept, scores)
    _against_oracle(keys, beacons, P, K - P, scores.cpu().numpy().astype(np.float64), kept.cpu().numpy(),
                    [0, 13, 31])


def test_noalloc_nan_key_ranks_last():
    """A NaN key makes its segment's scores NaN; they rank below every score, so the segment keeps its lowest
    candidates.  The other segment is unaffected."""
    S, L, P, K, B, d = 2, 600, 50, 250, 8, 128
    g = torch.Generator(device="cuda").manual_seed(6)
    keys = torch.randn((S, L, d), generator=g, device="cuda").bfloat16()
    beacons = (torch.randn((S, B, d), generator=g, device="cuda") * 0.3).bfloat16()
    keys[1, 321, 7] = float("nan")
    kept = torch.full((S, K), -1, dtype=torch.int32, device="cuda")
    scores = torch.zeros((S, L - P), dtype=torch.float32, device="cuda")
    _call(keys, beacons, S, L, P, K, B, d, torch.bfloat16, kept, scores)
    sc, kp = scores.cpu().numpy().astype(np.float64), kept.cpu().numpy()
    assert np.all(np.isnan(sc[1]))
    assert np.array_equal(kp[1], np.arange(K))
    _against_oracle(keys, beacons, P, K - P, sc, kp, [0])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    t = torch.zeros(16, dtype=torch.int32, device="cuda")
    st = kvc.kvc_beacon_select_noalloc(_vp(t), _vp(t), 64, 32768, 0, 100, 4, 128, kvc.KVC_BF16, _vp(t), None, None)
    assert st == kvc.KVC_ERR_INVALID_ARG
    assert b"scratch limit" in kvc.kvc_last_error(None)
    # 64 scores over the limit (64 x 16385); the size check comes before any launch
    st = kvc.kvc_beacon_select_noalloc(_vp(t), _vp(t), 64, 16385, 0, 100, 4, 128, kvc.KVC_BF16, _vp(t), None,
                                       None)
    assert st == kvc.KVC_ERR_INVALID_ARG
    assert b"scratch limit" in kvc.kvc_last_error(None)
