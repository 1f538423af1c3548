"""The C ABI without a GPU: libkvc.so loads, exports every entry point that
include/kvc.h declares, sizes workspaces and rejects invalid configurations
(host-side logic only; no compute call)."""
import ctypes
import os
import re
import subprocess

import pytest

import decode_kv_cache_paged_b200 as kvc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(kvc_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 14
    out = subprocess.run(["nm", "-D", "--defined-only", kvc.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (kvc_\w+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(kvc._lib, n)


def test_binding_covers_header():
    assert set(declared_functions()) == set(kvc.EXPORTED) | (set(declared_functions()) - set(kvc.EXPORTED))
    assert set(kvc.EXPORTED) <= set(declared_functions())


def _cfg(**kw):
    base = dict(num_requests=4, num_layers=2, num_kv_heads=8, num_q_heads=32, head_dim=128, page_size=16,
                dtype=kvc.KVC_BF16, num_beacons=64, query_window=64, max_seq_len=2112, num_pages=600)
    base.update(kw)
    return kvc.kvc_config(**base)


def test_workspace_bytes_and_layout():
    c = _cfg()
    n = kvc.kvc_workspace_bytes(ctypes.byref(c))
    R, Ly, H, Hq, d, B, W, S = 4, 2, 8, 32, 128, 64, 64, 2112
    lower = (R * (S // 16) * 4 + Ly * 600 * H * 16 * 4 + R * Ly * W * Hq * d * 2 + R * Ly * H * B * d * 6
             + R * Ly * H * S * 4)
    assert lower <= n < lower + (1 << 24)
    assert n % 256 == 0
    # no beacons: no score scratch, no beacon state
    c2 = _cfg(num_beacons=0, query_window=0)
    assert kvc.kvc_workspace_bytes(ctypes.byref(c2)) < n - R * Ly * H * S * 4


@pytest.mark.parametrize("bad", [
    dict(page_size=32), dict(num_requests=0), dict(num_q_heads=12), dict(dtype=7), dict(head_dim=100),
    dict(head_dim=1024), dict(max_seq_len=40000), dict(max_seq_len=100), dict(num_beacons=300),
    dict(query_window=2000), dict(num_pages=0), dict(num_beacons=4, query_window=0), dict(head_dim=96),
])
def test_invalid_configs_rejected(bad):
    c = _cfg(**bad)
    assert kvc.kvc_workspace_bytes(ctypes.byref(c)) == 0
    h = ctypes.c_void_p()
    st = kvc.kvc_create(ctypes.byref(c), None, None, None, 0, None, ctypes.byref(h))
    assert st == kvc.KVC_ERR_INVALID_ARG
    assert kvc.kvc_last_error(None)
    assert not h


def test_create_rejects_host_pointers_without_gpu():
    c = _cfg()
    buf = (ctypes.c_uint8 * 4096)()
    h = ctypes.c_void_p()
    st = kvc.kvc_create(ctypes.byref(c), ctypes.addressof(buf), ctypes.addressof(buf), ctypes.addressof(buf),
                        1 << 40, None, ctypes.byref(h))
    assert st == kvc.KVC_ERR_INVALID_ARG  # not 256-aligned or not device memory


def test_status_strings_and_null_handles():
    for s in range(9):
        assert kvc.kvc_status_string(s).startswith(b"KVC_")
    assert kvc.kvc_destroy(None) == kvc.KVC_OK
    assert kvc.kvc_sync(None) == kvc.KVC_ERR_INVALID_ARG
    assert kvc.kvc_compress(None, 0, None, 0, None, None) == kvc.KVC_ERR_INVALID_ARG
    assert kvc.kvc_append(None, None, 0, 0, None, None, None, 0) == kvc.KVC_ERR_INVALID_ARG
