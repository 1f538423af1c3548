"""kvc_beacon_select_noalloc, the entry point for callers that cannot allocate
device memory (graph-capturing code, plug-ins confined to another engine's
memory arena, hosts without a device allocator): it must agree with
kvc_compress(KVC_SEL_BEACON) on the same keys and beacons, on two calls in a
row of different shapes, while keeping its scratch in the library's own
fixed device array.  Collected last so that a failure here stops a -x run only
after every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import decode_kv_cache_paged_b200 as kvc
from decode_kv_cache_paged_b200 import Context, ContextSpec
from gpu_helpers import BAND, SCORE_ABS, SCORE_REL

pytestmark = pytest.mark.gpu


def _vp(t):
    return ctypes.c_void_p(t.data_ptr())


def _one_case(seed, H, L, P, K, B, d, W=16):
    """Context path vs allocation-free path on H dense segments (1 request, 1 layer)."""
    G = 2
    spec = ContextSpec(num_requests=1, num_layers=1, num_kv_heads=H, head_dim=d, max_seq_len=(L + 15) // 16 * 16,
                       num_pages=(L + 15) // 16 + 2, num_q_heads=H * G, num_beacons=B, query_window=W)
    ctx = Context(spec, dtype=torch.bfloat16)
    g = torch.Generator(device="cuda").manual_seed(seed)
    k = torch.randn((1, 1, L, H, d), generator=g, device="cuda").bfloat16()
    v = torch.randn((1, 1, L, H, d), generator=g, device="cuda").bfloat16()
    q = torch.randn((1, 1, W, H * G, d), generator=g, device="cuda").bfloat16()
    ctx.append([0], k[:, :, :P].contiguous(), v[:, :, :P].contiguous(), protect=True)
    ctx.append([0], k[:, :, P:L - W].contiguous(), v[:, :, P:L - W].contiguous())
    ctx.append([0], k[:, :, L - W:].contiguous(), v[:, :, L - W:].contiguous(), q)
    ctx.update_beacons()
    keys = k[0, 0].permute(1, 0, 2).contiguous()                        # [H, L, d]
    beacons = ctx.state_tensors()["beacons_scoring"][0, 0].contiguous()  # [H, B, d]
    N, M = L - P, (K - P if L > K else L - P)
    R = P + M
    dbg = torch.zeros((1, 1, H, spec.max_seq_len), dtype=torch.float32, device="cuda")
    ctx.compress("beacon", np.array([K], np.int32), 0, debug_scores=dbg)
    ctx.sync()
    _, _, pos = ctx.gather_dense(0, cap=R)
    want_kept = pos[0].cpu().numpy()          # positions == slots in the first round
    want_scores = dbg[0, 0, :, :N].cpu().numpy().astype(np.float64)

    kept = torch.full((H, R), -1, dtype=torch.int32, device="cuda")
    scores = torch.zeros((H, N), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    st = kvc.kvc_beacon_select_noalloc(_vp(keys), _vp(beacons), H, L, P, K, B, d, kvc.KVC_BF16,
                                       _vp(kept), _vp(scores), ctypes.c_void_p(stream.cuda_stream))
    assert st == kvc.KVC_OK, kvc.kvc_last_error(None)
    torch.cuda.synchronize()
    got_scores = scores.cpu().numpy().astype(np.float64)
    got_kept = kept.cpu().numpy()
    err = np.abs(got_scores - want_scores)
    assert np.all(err <= SCORE_ABS + SCORE_REL * np.abs(want_scores))
    for h in range(H):
        assert np.array_equal(got_kept[h, :P], np.arange(P))
        a, b = set(got_kept[h, P:].tolist()), set(want_kept[h, P:].tolist())
        assert len(a) == len(b) == M and np.all(np.diff(got_kept[h]) > 0)
        # equal selections, except positions within the threshold band
        tau = np.sort(want_scores[h])[::-1][M - 1]
        for j in a ^ b:
            assert abs(want_scores[h, j - P] - tau) <= BAND
    ctx.close()


def test_noalloc_matches_compress_two_calls_in_a_row():
    _one_case(seed=1, H=4, L=700, P=60, K=300, B=16, d=128)
    _one_case(seed=2, H=8, L=450, P=32, K=128, B=8, d=64)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    t = torch.zeros(16, dtype=torch.int32, device="cuda")
    st = kvc.kvc_beacon_select_noalloc(_vp(t), _vp(t), 64, 32768, 0, 100, 4, 128, kvc.KVC_BF16, _vp(t), None, None)
    assert st == kvc.KVC_ERR_INVALID_ARG
    assert b"scratch limit" in kvc.kvc_last_error(None)
