"""Python binding of libkvc.so, the B200 decode-time KV-cache eviction round.

Argument marshalling only: every step of the round runs in the library's
CUDA kernels.  PyTorch supplies device memory (the K/V pools and the
workspace) and the CUDA stream.  The raw C entry points are exposed under
their C names (``kvc_create``, ``kvc_append``, ...); ``Context`` wraps them
for convenience.

The library must have been built (``python decode_kv_cache_paged_b200/build.py``);
importing this package without it raises ImportError.  There is no CPU path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvc.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python decode_kv_cache_paged_b200/build.py` "
        "(the eviction round has no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

# --------------------------------------------------------------- C types --

KVC_OK = 0
KVC_ERR_INVALID_ARG = 1
KVC_ERR_OUT_OF_PAGES = 2
KVC_ERR_STATE = 3
KVC_ERR_CUDA = 4
KVC_ERR_NAN = 5
KVC_ERR_DEVICE_CHECK = 6
KVC_ERR_DEVICE_TIMEOUT = 7
KVC_ERR_UNSUPPORTED = 8

KVC_BF16 = 0
KVC_F32 = 1

KVC_SEL_RANDOM = 0
KVC_SEL_RANDOM_SHARED = 1
KVC_SEL_BEACON = 2
KVC_SEL_BEACON_TRIGGER = 3

KVC_OPT_BEACON_SCORE_IMPL = 0
KVC_OPT_BEACON_UPDATE_IMPL = 1

KVC_COMPACT_ORDERED = 0
KVC_COMPACT_HOLE_FILL = 1
COMPACTIONS = {"ordered": KVC_COMPACT_ORDERED, "hole_fill": KVC_COMPACT_HOLE_FILL}

SELECTORS = {"random": KVC_SEL_RANDOM, "random_shared": KVC_SEL_RANDOM_SHARED,
             "beacon": KVC_SEL_BEACON, "beacon_trigger": KVC_SEL_BEACON_TRIGGER}


class kvc_config(ctypes.Structure):
    _fields_ = [("num_requests", ctypes.c_int32), ("num_layers", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("num_beacons", ctypes.c_int32),
                ("query_window", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
                ("num_pages", ctypes.c_int64)]


class kvc_round_stats(ctypes.Structure):
    _fields_ = [("round", ctypes.c_int64), ("segments", ctypes.c_int64),
                ("noop_segments", ctypes.c_int64), ("prompt_over_budget_segments", ctypes.c_int64),
                ("head_positions", ctypes.c_int64), ("candidates", ctypes.c_int64),
                ("evicted", ctypes.c_int64), ("moved_rows", ctypes.c_int64),
                ("compaction_bytes", ctypes.c_int64), ("key_bytes_scored", ctypes.c_int64),
                ("ms_score", ctypes.c_float), ("ms_select_compact", ctypes.c_float),
                ("ms_total", ctypes.c_float), ("launches", ctypes.c_int32),
                ("score_kernel", ctypes.c_int32), ("reserved", ctypes.c_int32)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_ if f != "reserved"}


class kvc_round_options(ctypes.Structure):
    _fields_ = [("sink_tokens", ctypes.c_int32), ("block", ctypes.c_int32),
                ("compaction", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class kvc_view(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("lengths", ctypes.c_void_p),
                ("prompt_lengths", ctypes.c_void_p), ("pos_map", ctypes.c_void_p),
                ("query_ring", ctypes.c_void_p), ("beacons", ctypes.c_void_p),
                ("beacons_scoring", ctypes.c_void_p), ("beacon_counts", ctypes.c_void_p),
                ("beacon_triggers", ctypes.c_void_p),
                ("max_pages_per_request", ctypes.c_int32), ("row_bytes", ctypes.c_int32),
                ("round", ctypes.c_int64)]


_P = ctypes.c_void_p
_i32, _i64, _u64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
_SIGS = {
    "kvc_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(kvc_config)]),
    "kvc_create": (_i32, [ctypes.POINTER(kvc_config), _P, _P, _P, ctypes.c_size_t, _P, ctypes.POINTER(_P)]),
    "kvc_destroy": (_i32, [_P]),
    "kvc_set_stream": (_i32, [_P, _P]),
    "kvc_set_option": (_i32, [_P, _i32, _i64]),
    "kvc_append": (_i32, [_P, _P, _i32, _i32, _P, _P, _P, _i32]),
    "kvc_update_beacons": (_i32, [_P, _P, _P]),
    "kvc_compress": (_i32, [_P, _i32, _P, _u64, _P, ctypes.POINTER(kvc_round_stats)]),
    "kvc_compress_ex": (_i32, [_P, _i32, _P, _u64, ctypes.POINTER(kvc_round_options), _P,
                               ctypes.POINTER(kvc_round_stats)]),
    "kvc_decode_attention": (_i32, [_P, _i32, _i32, _P, ctypes.c_float, _P, _P, _P]),
    "kvc_gather_view": (_i32, [_P, ctypes.POINTER(kvc_view)]),
    "kvc_get_lengths": (_i32, [_P, _P, _P]),
    "kvc_gather_dense": (_i32, [_P, _i32, _i32, _i32, _i32, _P, _P, _P]),
    "kvc_check_wait_timeout": (_i32, [_P, ctypes.c_uint32]),
    "kvc_sync": (_i32, [_P]),
    "kvc_status_string": (ctypes.c_char_p, [_i32]),
    "kvc_last_error": (ctypes.c_char_p, [_P]),
    "kvc_beacon_select_noalloc": (_i32, [_P, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _P, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args
    globals()[_name] = _f

EXPORTED = tuple(_SIGS)


class KvcError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{kvc_status_string(status).decode()}: {message}")


def _check(status: int, ctx=None):
    if status != KVC_OK:
        raise KvcError(status, kvc_last_error(ctx).decode(errors="replace"))


# --------------------------------------------------------------- Context --

def _dtype_code(dtype) -> int:
    import torch
    if dtype == torch.bfloat16:
        return KVC_BF16
    if dtype == torch.float32:
        return KVC_F32
    raise ValueError(f"unsupported cache dtype {dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@dataclass
class ContextSpec:
    num_requests: int
    num_layers: int
    num_kv_heads: int
    head_dim: int
    max_seq_len: int
    num_pages: int
    num_q_heads: int = 0
    num_beacons: int = 0
    query_window: int = 0

    def config(self, dtype_code: int) -> kvc_config:
        return kvc_config(self.num_requests, self.num_layers, self.num_kv_heads,
                          self.num_q_heads or self.num_kv_heads, self.head_dim, 16, dtype_code,
                          self.num_beacons, self.query_window, self.max_seq_len, self.num_pages)


class Context:
    """One eviction context over torch-allocated pools and workspace."""

    def __init__(self, spec: ContextSpec, dtype=None, device="cuda", stream=None):
        import torch
        dtype = dtype or torch.bfloat16
        self.spec = spec
        self.dtype = dtype
        self.device = torch.device(device)
        self.cfg = spec.config(_dtype_code(dtype))
        ws_bytes = kvc_workspace_bytes(ctypes.byref(self.cfg))
        if ws_bytes == 0:
            raise KvcError(KVC_ERR_INVALID_ARG, "invalid context configuration")
        Hq = self.cfg.num_q_heads
        shape = (spec.num_layers, spec.num_pages, spec.num_kv_heads, 16, spec.head_dim)
        self.k_pool = torch.empty(shape, dtype=dtype, device=self.device)
        self.v_pool = torch.empty(shape, dtype=dtype, device=self.device)
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=self.device)
        self.stream = stream or torch.cuda.current_stream(self.device)
        self.handle = ctypes.c_void_p()
        _check(kvc_create(ctypes.byref(self.cfg), _ptr(self.k_pool), _ptr(self.v_pool),
                          _ptr(self.workspace), ws_bytes, ctypes.c_void_p(self.stream.cuda_stream),
                          ctypes.byref(self.handle)))
        self.num_q_heads = Hq

    # -- lifecycle
    def close(self):
        if self.handle:
            kvc_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_option(self, opt: int, value: int):
        _check(kvc_set_option(self.handle, opt, value), self.handle)

    # -- calls
    def append(self, req_ids, k, v, q=None, protect: bool = False):
        ids = np.ascontiguousarray(req_ids, dtype=np.int32)
        s = self.spec
        n_tokens = int(k.shape[2])
        want = (len(ids), s.num_layers, n_tokens, s.num_kv_heads, s.head_dim)
        if tuple(k.shape) != want or tuple(v.shape) != want:
            raise ValueError(f"k and v must have shape {want}")
        if q is not None and tuple(q.shape) != (len(ids), s.num_layers, n_tokens, self.num_q_heads, s.head_dim):
            raise ValueError("q must have shape [n_req, layers, T, num_q_heads, head_dim]")
        for t in (k, v) + ((q,) if q is not None else ()):
            if not t.is_contiguous() or t.dtype != self.dtype:
                raise ValueError("k/v/q must be contiguous and of the cache dtype")
        _check(kvc_append(self.handle, ids.ctypes.data_as(_P), len(ids), n_tokens, _ptr(k), _ptr(v),
                          _ptr(q), int(bool(protect))), self.handle)

    def update_beacons(self, assign_out=None, timed: bool = False):
        ms = ctypes.c_float(0.0)
        _check(kvc_update_beacons(self.handle, _ptr(assign_out), ctypes.byref(ms) if timed else None),
               self.handle)
        return ms.value if timed else None

    def compress(self, selector, budgets, seed: int, debug_scores=None, stats: bool = False,
                 sink_tokens=None, block: int = 1, compaction="ordered"):
        """One eviction round (kvc_compress_ex).  sink_tokens None protects the
        whole prompt; block and compaction as in kvc_round_options."""
        sel = SELECTORS[selector] if isinstance(selector, str) else int(selector)
        b = np.ascontiguousarray(budgets, dtype=np.int32)
        if b.shape != (self.spec.num_requests,):
            raise ValueError("budgets must have one entry per request")
        comp = COMPACTIONS[compaction] if isinstance(compaction, str) else int(compaction)
        opts = kvc_round_options(-1 if sink_tokens is None else int(sink_tokens), int(block), comp, 0)
        st = kvc_round_stats()
        _check(kvc_compress_ex(self.handle, sel, b.ctypes.data_as(_P), ctypes.c_uint64(seed),
                               ctypes.byref(opts), _ptr(debug_scores),
                               ctypes.byref(st) if stats else None), self.handle)
        return st.as_dict() if stats else None

    def decode_attention(self, q, layer_begin: int = 0, out=None, lse=None, scale: float = 0.0,
                         with_lse: bool = True, timed: bool = False):
        """kvc_decode_attention for q [layer_count, R, Hq, d] (cache dtype, on the
        context's device).  Returns (out, lse) float32 tensors, plus the device
        time in ms when timed."""
        import torch
        s = self.spec
        if q.dim() != 4 or q.shape[1:] != (s.num_requests, s.num_q_heads, s.head_dim) or q.dtype != self.dtype:
            raise ValueError("q must be [layer_count, num_requests, num_q_heads, head_dim] in the cache dtype")
        q = q.contiguous()
        lc = q.shape[0]
        if out is None:
            out = torch.empty((lc, s.num_requests, s.num_q_heads, s.head_dim), dtype=torch.float32,
                              device=self.device)
        if lse is None and with_lse:
            lse = torch.empty((lc, s.num_requests, s.num_q_heads), dtype=torch.float32, device=self.device)
        ms = ctypes.c_float(0.0)
        _check(kvc_decode_attention(self.handle, int(layer_begin), int(lc), _ptr(q), ctypes.c_float(scale),
                                    _ptr(out), _ptr(lse), ctypes.byref(ms) if timed else None), self.handle)
        return (out, lse, ms.value) if timed else (out, lse)

    def check_wait_timeout(self, limit_ms: int = 100):
        """kvc_check_wait_timeout: raises KvcError(KVC_ERR_DEVICE_TIMEOUT) when the
        bounded-wait failure detection works."""
        _check(kvc_check_wait_timeout(self.handle, int(limit_ms)), self.handle)

    def sync(self):
        _check(kvc_sync(self.handle), self.handle)

    def lengths(self):
        R = self.spec.num_requests
        ln = np.zeros(R, np.int32)
        pr = np.zeros(R, np.int32)
        _check(kvc_get_lengths(self.handle, ln.ctypes.data_as(_P), pr.ctypes.data_as(_P)), self.handle)
        return ln, pr

    def view(self) -> kvc_view:
        v = kvc_view()
        _check(kvc_gather_view(self.handle, ctypes.byref(v)), self.handle)
        return v

    def _ws_tensor(self, ptr: int, nbytes: int, dtype, shape):
        off = ptr - self.workspace.data_ptr()
        assert 0 <= off and off + nbytes <= self.workspace.numel()
        return self.workspace[off:off + nbytes].view(dtype).view(shape)

    def state_tensors(self):
        """Torch views (no copy) of the device state in the workspace."""
        import torch
        v = self.view()
        s = self.spec
        R, Ly, H, d = s.num_requests, s.num_layers, s.num_kv_heads, s.head_dim
        B, W, Hq = s.num_beacons, s.query_window, self.num_q_heads
        es = self.k_pool.element_size()
        out = {
            "block_table": self._ws_tensor(v.block_table, R * v.max_pages_per_request * 4, torch.int32,
                                           (R, v.max_pages_per_request)),
            "lengths": self._ws_tensor(v.lengths, R * 4, torch.int32, (R,)),
            "prompt_lengths": self._ws_tensor(v.prompt_lengths, R * 4, torch.int32, (R,)),
            "pos_map": self._ws_tensor(v.pos_map, Ly * s.num_pages * H * 16 * 4, torch.int32,
                                       (Ly, s.num_pages, H, 16)),
        }
        if W:
            out["query_ring"] = self._ws_tensor(v.query_ring, R * Ly * W * Hq * d * es, self.dtype,
                                                (R, Ly, W, Hq, d))
        if B:
            out["beacons"] = self._ws_tensor(v.beacons, R * Ly * H * B * d * 4, torch.float32, (R, Ly, H, B, d))
            out["beacons_scoring"] = self._ws_tensor(v.beacons_scoring, R * Ly * H * B * d * es, self.dtype,
                                                     (R, Ly, H, B, d))
            out["beacon_counts"] = self._ws_tensor(v.beacon_counts, R * Ly * H * B * 4, torch.int32, (R, Ly, H, B))
            out["beacon_triggers"] = self._ws_tensor(v.beacon_triggers, R * Ly * H * B * 4, torch.float32,
                                                     (R, Ly, H, B))
        return out

    def gather_dense(self, layer: int, req_begin: int = 0, req_count: int | None = None, cap: int | None = None):
        """Dense copies (k, v [n, Hkv, cap, d], pos [n, Hkv, cap]) of one layer."""
        import torch
        s = self.spec
        n = s.num_requests - req_begin if req_count is None else req_count
        cap = s.max_seq_len if cap is None else cap
        k = torch.empty((n, s.num_kv_heads, cap, s.head_dim), dtype=self.dtype, device=self.device)
        v = torch.empty_like(k)
        pos = torch.empty((n, s.num_kv_heads, cap), dtype=torch.int32, device=self.device)
        _check(kvc_gather_dense(self.handle, layer, req_begin, n, cap, _ptr(k), _ptr(v), _ptr(pos)),
               self.handle)
        return k, v, pos
