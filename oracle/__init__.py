"""Plain CPU oracle for the decode-time KV-cache eviction round.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product (``decode_kv_cache_paged_b200``) never imports it and
shares no code with it.

The arithmetic lives in ``oracle.c`` (single-threaded C, double precision,
full-sort selection); this module only builds it with gcc, marshals numpy
arrays through ctypes and composes the per-segment routines into a whole
round.  Sources, cited per function in ``oracle.c``:

* Random Attention article (aiinking.com/article/67532), sections
  "长推理的显存瓶颈", "Random Attention：不判断重要性，只随机保留", "发现二",
  "发现四";
* BeaconKV explainer (papers.ananclaw.com/promo/explainers__2609-04971) §3.2
  and the BeaconKV abstract (chatpaper.ai).

Parity status of each function is listed in ``PINS`` below.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# What pins each oracle function to something other than itself (tests/).
PINS = {
    "philox4x64_10": "numpy.random.Philox (independent Philox4x64-10 implementation)",
    "random_score": "numpy.random.Philox block word 0, high 32 bits",
    "retention": "hand-derived cases from the pages' serving shapes (tests/golden)",
    "select_topk": "python sorted() on (-score, pos); kept-vs-evicted dominance invariant",
    "compact_rows": "numpy.take on the kept slot list",
    "random_round": "survival (K-P)/N and geometric decay closed forms; chi^2 uniformity",
    "round_bf16": "torch fp32 -> bfloat16 conversion (round to nearest even)",
    "beacon_update": "scipy.cluster.vq.vq assignment; running mean == mean of assignment history",
    "beacon_score": "scipy.special.softmax; identical keys -> 1/L; B=1 ranking; one-hot closed form",
    "random_score_block": "numpy.random.Philox on counter (pos // block, h, l, r)",
    "hole_fill": "invariants: kept slots below R stay, holes filled in ascending order, same kept set",
    "random_round_ex": "at most one split block; sink protection = prompt protection with P = S",
    "beacon_trigger_score": "scipy.special.softmax weighted by trigger shares; one-hot trigger -> that "
                            "beacon's softmax; mass conservation sum_j = 1 (P = 0); count scaling invariance",
    "decode_attention": "scipy.special.softmax/logsumexp; L=1 -> v; q=0 -> mean of v, log L; "
                        "large-scale limit -> v of the argmax key; joint permutation invariance",
    "decode_attention_gqa": "query head hq reads KV head hq // G (marker values per KV head)",
}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _bind(L: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    i64, i32, u64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64
    L.orc_philox4x64_10.argtypes = [P, P, P]
    L.orc_philox4x64_10.restype = None
    L.orc_random_score.argtypes = [u64, u64, i64, i64, i64, i64, i32]
    L.orc_random_score.restype = ctypes.c_uint32
    L.orc_retention.argtypes = [i64, i64, i64, P, P, P]
    L.orc_retention.restype = i32
    L.orc_select_topk.argtypes = [i64, P, P, P, i64, P]
    L.orc_select_topk.restype = i64
    L.orc_compact_rows.argtypes = [i64, i64, P, i64, P, P]
    L.orc_compact_rows.restype = None
    L.orc_random_round_segment.argtypes = [u64, u64, i64, i64, i64, i32, i64, i64, i64, P, P, P]
    L.orc_random_round_segment.restype = i64
    L.orc_random_round_batch.argtypes = [u64, u64, i32, i64, P, P, i64, P, P, P]
    L.orc_random_round_batch.restype = i64
    L.orc_round_bf16.argtypes = [ctypes.c_double]
    L.orc_round_bf16.restype = ctypes.c_double
    L.orc_beacon_update.argtypes = [i64, i64, i64, P, P, P, i32, P, P]
    L.orc_beacon_update.restype = i32
    L.orc_beacon_score.argtypes = [i64, i64, i64, i64, P, P, P, P]
    L.orc_beacon_score.restype = i32
    L.orc_random_score_block.argtypes = [u64, u64, i64, i64, i64, i64, i32, i64]
    L.orc_random_score_block.restype = ctypes.c_uint32
    L.orc_hole_fill.argtypes = [i64, P, P]
    L.orc_hole_fill.restype = i64
    L.orc_random_round_segment_ex.argtypes = [u64, u64, i64, i64, i64, i32, i64, i32, i64, i64, i64, P, P]
    L.orc_random_round_segment_ex.restype = i64
    L.orc_random_round_batch_ex.argtypes = [u64, u64, i32, i64, i32, i64, P, P, i64, P, P, P]
    L.orc_random_round_batch_ex.restype = i64
    L.orc_beacon_trigger_score.argtypes = [i64, i64, i64, i64, P, P, P, P]
    L.orc_beacon_trigger_score.restype = i32
    L.orc_decode_attention.argtypes = [i64, i64, P, P, P, ctypes.c_double, P, P]
    L.orc_decode_attention.restype = None
    L.orc_decode_attention_gqa.argtypes = [i64, i64, i64, i64, P, P, P, ctypes.c_double, P, P]
    L.orc_decode_attention_gqa.restype = None
    return L


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


class use_library:
    """Context manager that swaps in another build of oracle.c (used by the
    tests that plant mistakes in a copy of the oracle to show the pins catch
    them)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = lib()
        _lib = _bind(ctypes.CDLL(self.path))
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def compile_source(src_text: str, out_path: str) -> str:
    """Compiles a (possibly modified) copy of oracle.c to out_path."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
                           "-shared", "-fPIC", "-o", out_path, c_path, "-lm"])
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- random --

def philox4x64_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(ctr, dtype=np.uint64)
    k = np.ascontiguousarray(key, dtype=np.uint64)
    out = np.zeros(4, dtype=np.uint64)
    lib().orc_philox4x64_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def random_score(seed: int, rnd: int, r: int, l: int, h: int, pos: int, shared: bool = False) -> int:
    return int(lib().orc_random_score(seed, rnd, r, l, h, pos, int(bool(shared))))


@dataclass
class Retention:
    M: int          # generated positions kept
    R: int          # new length
    noop: bool      # L <= K: nothing evicted
    over_budget: bool  # P > K: prompt alone exceeds the budget


def retention(L: int, P: int, K: int) -> Retention:
    M = np.zeros(1, np.int64)
    R = np.zeros(1, np.int64)
    f = np.zeros(1, np.int32)
    rc = lib().orc_retention(L, P, K, _ptr(M), _ptr(R), _ptr(f))
    if rc != 0:
        raise ValueError(f"invalid sizes L={L} P={P} K={K}")
    return Retention(int(M[0]), int(R[0]), bool(f[0] & 1), bool(f[0] & 2))


def select_topk(score, pos, slot, M: int) -> np.ndarray:
    """Kept slots (ascending) of the M best candidates by (score desc, pos asc)."""
    s = np.ascontiguousarray(score, dtype=np.float64)
    p = np.ascontiguousarray(pos, dtype=np.int64)
    sl = np.ascontiguousarray(slot, dtype=np.int64)
    out = np.zeros(max(M, 1), np.int64)
    got = lib().orc_select_topk(len(s), _ptr(s), _ptr(p), _ptr(sl), M, _ptr(out))
    if got != M:
        raise ValueError("select_topk failed")
    return out[:M]


def compact_rows(rows: np.ndarray, P: int, kept_generated: np.ndarray) -> np.ndarray:
    """Prompt rows [0,P) then rows[kept_generated] in order; rows is [L, ...]."""
    rows = np.ascontiguousarray(rows)
    L = rows.shape[0]
    row_bytes = rows.nbytes // max(L, 1)
    kept = np.ascontiguousarray(kept_generated, dtype=np.int64)
    out = np.zeros((P + len(kept),) + rows.shape[1:], dtype=rows.dtype)
    lib().orc_compact_rows(P, row_bytes, _ptr(rows), len(kept), _ptr(kept), _ptr(out))
    return out


def random_round_segment(seed, rnd, r, l, h, shared, P, K, pos_in):
    """Returns (kept_slots[R], pos_out[R]) for one segment."""
    pos_in = np.ascontiguousarray(pos_in, dtype=np.int32)
    L = len(pos_in)
    kept = np.zeros(max(L, 1), np.int64)
    pos_out = np.zeros(max(L, 1), np.int32)
    R = lib().orc_random_round_segment(seed, rnd, r, l, h, int(bool(shared)), L, P, K,
                                       _ptr(pos_in), _ptr(pos_out), _ptr(kept))
    if R < 0:
        raise ValueError("random_round_segment failed")
    return kept[:R], pos_out[:R]


def random_round_batch(seed, rnd, shared, rlh, lpk, pos_in):
    """Batched segments: rlh [n,3], lpk [n,3] (L,P,K), pos_in [n, stride] int32.

    Returns (pos_out [n, stride] with -1 beyond R, R [n])."""
    rlh = np.ascontiguousarray(rlh, dtype=np.int64)
    lpk = np.ascontiguousarray(lpk, dtype=np.int64)
    pos_in = np.ascontiguousarray(pos_in, dtype=np.int32)
    n, stride = pos_in.shape
    pos_out = np.full((n, stride), -1, np.int32)
    R = np.zeros(n, np.int64)
    rc = lib().orc_random_round_batch(seed, rnd, int(bool(shared)), n, _ptr(rlh), _ptr(lpk), stride,
                                      _ptr(pos_in), _ptr(pos_out), _ptr(R))
    if rc != 0:
        raise ValueError(f"random_round_batch failed at segment {rc - 1}")
    return pos_out, R


def random_score_block(seed, rnd, r, l, h, pos, shared=False, block=1) -> int:
    return int(lib().orc_random_score_block(seed, rnd, r, l, h, pos, int(bool(shared)), block))


def hole_fill(R: int, kept_slots) -> np.ndarray:
    """For each new slot s < R, the old slot whose row it holds after hole filling."""
    kept = np.ascontiguousarray(kept_slots, dtype=np.int64)
    out = np.zeros(max(R, 1), np.int64)
    if lib().orc_hole_fill(R, _ptr(kept), _ptr(out)) < 0:
        raise ValueError("hole_fill failed")
    return out[:R]


def random_round_segment_ex(seed, rnd, r, l, h, shared, block, hole_fill_mode, P, K, pos_in):
    """pos_out [R] of one segment under the extended round's options."""
    pos_in = np.ascontiguousarray(pos_in, dtype=np.int32)
    L = len(pos_in)
    pos_out = np.zeros(max(L, 1), np.int32)
    R = lib().orc_random_round_segment_ex(seed, rnd, r, l, h, int(bool(shared)), block,
                                          int(bool(hole_fill_mode)), L, P, K, _ptr(pos_in), _ptr(pos_out))
    if R < 0:
        raise ValueError("random_round_segment_ex failed")
    return pos_out[:R]


def random_round_batch_ex(seed, rnd, shared, block, hole_fill_mode, rlh, lpk, pos_in):
    rlh = np.ascontiguousarray(rlh, dtype=np.int64)
    lpk = np.ascontiguousarray(lpk, dtype=np.int64)
    pos_in = np.ascontiguousarray(pos_in, dtype=np.int32)
    n, stride = pos_in.shape
    pos_out = np.full((n, stride), -1, np.int32)
    R = np.zeros(n, np.int64)
    rc = lib().orc_random_round_batch_ex(seed, rnd, int(bool(shared)), block, int(bool(hole_fill_mode)), n,
                                         _ptr(rlh), _ptr(lpk), stride, _ptr(pos_in), _ptr(pos_out), _ptr(R))
    if rc != 0:
        raise ValueError(f"random_round_batch_ex failed at segment {rc - 1}")
    return pos_out, R


# ---------------------------------------------------------------- beacon --

def round_bf16(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    f = lib().orc_round_bf16
    return np.vectorize(lambda v: f(float(v)), otypes=[np.float64])(x) if x.size else x.copy()


def beacon_update(points, beacons, counts, init: bool, assign_override=None):
    """One periodic beacon update; returns (beacons', counts', assignment)."""
    pts = np.ascontiguousarray(points, dtype=np.float64)
    n_pts, d = pts.shape
    c = np.array(beacons, dtype=np.float64, copy=True, order="C")
    B = c.shape[0]
    if c.shape[1] != d:
        raise ValueError("dimension mismatch")
    cnt = np.array(counts, dtype=np.int64, copy=True, order="C")
    assign = np.zeros(max(n_pts, 1), np.int32)
    ov = None if assign_override is None else np.ascontiguousarray(assign_override, dtype=np.int32)
    rc = lib().orc_beacon_update(n_pts, B, d, _ptr(pts), _ptr(c), _ptr(cnt), int(bool(init)),
                                 _ptr(ov), _ptr(assign))
    if rc != 0:
        raise ValueError("beacon_update failed (n_pts < B on first update, or bad override)")
    return c, cnt, assign[:n_pts]


def beacon_score(keys, beacons_scoring, P: int):
    """Scores [L-P] (float64) and lse [B] of one segment (keys [L,d], beacons [B,d])."""
    k = np.ascontiguousarray(keys, dtype=np.float64)
    c = np.ascontiguousarray(beacons_scoring, dtype=np.float64)
    L, d = k.shape
    B = c.shape[0]
    score = np.zeros(max(L - P, 1), np.float64)
    lse = np.zeros(B, np.float64)
    rc = lib().orc_beacon_score(L, P, B, d, _ptr(k), _ptr(c), _ptr(score), _ptr(lse))
    if rc != 0:
        raise ValueError("beacon_score failed")
    return score[:L - P], lse


def segment_points(queries, h: int, G: int) -> np.ndarray:
    """Points of KV head h from a [steps, Hq, d] query window: the G query heads
    h*G .. h*G+G-1 of each step, ordered by (step, query head)."""
    q = np.asarray(queries, dtype=np.float64)
    return np.ascontiguousarray(q[:, h * G:(h + 1) * G, :].reshape(-1, q.shape[-1]))


def beacon_round_segment(keys, P: int, K: int, beacons_scoring):
    """Beacon-selector round on one segment whose slots hold positions 0..L-1 in order.

    Returns (kept_slots [R], scores float64 [L-P]).  Selection compares the
    scores after casting them to fp32, ties to the lower position."""
    L = keys.shape[0]
    ret = retention(L, P, K)
    score, _ = beacon_score(keys, beacons_scoring, P)
    if ret.noop:
        return np.arange(L, dtype=np.int64), score
    slots = np.arange(P, L, dtype=np.int64)
    s32 = score.astype(np.float32).astype(np.float64)
    kept = select_topk(s32, slots, slots, ret.M)
    return np.concatenate([np.arange(P, dtype=np.int64), kept]), score


def beacon_select_with_pos(scores32, pos, P: int, K: int):
    """Kept slots for a segment with arbitrary position map, given fp32 scores [L-P]."""
    L = len(pos)
    ret = retention(L, P, K)
    if ret.noop:
        return np.arange(L, dtype=np.int64)
    slots = np.arange(P, L, dtype=np.int64)
    kept = select_topk(np.asarray(scores32, np.float32).astype(np.float64),
                       np.asarray(pos[P:], np.int64), slots, ret.M)
    return np.concatenate([np.arange(P, dtype=np.int64), kept])


def decode_attention(q, k, v, scale=None):
    """out [d], lse of one query over rows k, v [L, d] (float64)."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64).reshape(-1, q.shape[0])
    v = np.ascontiguousarray(v, dtype=np.float64).reshape(-1, q.shape[0])
    d = q.shape[0]
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    out = np.zeros(d, np.float64)
    lse = np.zeros(1, np.float64)
    lib().orc_decode_attention(k.shape[0], d, _ptr(q), _ptr(k), _ptr(v), scale, _ptr(out), _ptr(lse))
    return out, float(lse[0])


def decode_attention_gqa(q, k, v, scale=None):
    """out [Hq, d], lse [Hq] for q [Hq, d] over k, v [Hkv, L, d] (float64)."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    Hq, d = q.shape
    Hkv, L = k.shape[0], k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    out = np.zeros((Hq, d), np.float64)
    lse = np.zeros(Hq, np.float64)
    lib().orc_decode_attention_gqa(Hq, Hkv, L, d, _ptr(q), _ptr(k), _ptr(v), scale, _ptr(out), _ptr(lse))
    return out, lse


def beacon_trigger_score(keys, beacons_scoring, trig, P: int):
    """Cluster-trigger importance [L-P] of one segment (keys [L,d], beacons [B,d], trig [B])."""
    k = np.ascontiguousarray(keys, dtype=np.float64)
    c = np.ascontiguousarray(beacons_scoring, dtype=np.float64)
    t = np.ascontiguousarray(trig, dtype=np.float64)
    L, d = k.shape
    B = c.shape[0]
    score = np.zeros(max(L - P, 1), np.float64)
    if lib().orc_beacon_trigger_score(L, P, B, d, _ptr(k), _ptr(c), _ptr(t), _ptr(score)) != 0:
        raise ValueError("beacon_trigger_score failed")
    return score[:L - P]
