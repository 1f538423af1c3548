"""Seeded synthetic workloads of the pages' serving shapes.

This module draws random inputs only; it holds none of the eviction round's
arithmetic.  Both the GPU path (through tests and bench.py) and the CPU
oracle's tests consume what it generates.

Shapes come from the pages: budget K = 2048, a 1k-token protected prompt,
128 concurrent requests, a compression trigger every 64 tokens and 32k-token
generations (Random Attention article, "发现四"); compression factors 2x to
16x ("实验结果"); 64 to 256 beacons (BeaconKV explainer §3.3).  The pages
measure on public benchmarks with real models; none are available here, so
these synthetic inputs stand in for them:

* K/V rows ~ N(0, 1), with 4 channels per (layer, KV head) scaled by 8 (the
  outlier channels of real keys and values);
* decode queries from a mixture of von Mises-Fisher distributions on the unit
  sphere (per (layer, KV head) a set of component means uniform on the
  sphere; each (request, step, query head) picks a component uniformly and
  draws with concentration kappa = 20, Wood's 1994 rejection sampler), or,
  for the "sharp" test variants, the same directions scaled to norm sqrt(d)
  so that beacon scores spread far from the uniform 1/L;
* ragged lengths L_r ~ U{4096..32768} and prompts P_r ~ U{128..1536}.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np


@dataclass
class Workload:
    name: str
    num_requests: int
    num_layers: int
    num_kv_heads: int
    head_dim: int
    prompt: np.ndarray   # P_r, protected prompt length per request
    length: np.ndarray   # L_r, cache length at the trigger (before the round)
    budget: np.ndarray   # K_r
    dtype: str = "bf16"  # "bf16" or "f32"
    selectors: tuple = ("random",)
    num_q_heads: int = 0
    num_beacons: int = 0
    query_window: int = 0
    n_components: int = 0
    kappa: float = 20.0
    query_norm: float = 1.0  # queries lie on the sphere of this radius (sqrt(d) spreads the scores)
    outlier_channels: int = 4
    outlier_scale: float = 8.0
    trigger: int = 64       # tokens appended between rounds at steady state
    data_seed: int = 1000
    philox_seed: int = 0
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return (self.num_q_heads or self.num_kv_heads) // self.num_kv_heads

    @property
    def segments(self) -> int:
        return self.num_requests * self.num_layers * self.num_kv_heads

    @property
    def head_positions(self) -> int:
        return int(self.length.sum()) * self.num_layers * self.num_kv_heads

    def max_seq_len(self, headroom: int = 0) -> int:
        m = int(self.length.max()) + headroom
        return (m + 15) // 16 * 16

    def pages_needed(self, headroom: int = 0) -> int:
        return int(((self.length + headroom + 15) // 16).sum())


def _full(n, v):
    return np.full(n, v, dtype=np.int64)


def tiny() -> Workload:
    """1 request, 1 layer, 2 KV heads, d=64, fp32, 16 prompt + 240 generated, K=64;
    beacon selector with 4 beacons from the last 16 queries."""
    return Workload("tiny", 1, 1, 2, 64, _full(1, 16), _full(1, 256), _full(1, 64), dtype="f32",
                    selectors=("random", "random_shared", "beacon"), num_q_heads=2, num_beacons=4,
                    query_window=16, n_components=4, outlier_channels=0, data_seed=1000, philox_seed=0)


def random_serving(R=128, layers=36) -> Workload:
    """128 requests, 36 layers, 8 KV heads, d=128, bf16, P=1024, L=2048+64, K=2048."""
    return Workload("random_serving", R, layers, 8, 128, _full(R, 1024), _full(R, 2112), _full(R, 2048),
                    selectors=("random",), data_seed=1001, philox_seed=1)


def beacon_serving(R=128, layers=36) -> Workload:
    """As random_serving with 32 query heads (G=4), 64-component vMF(kappa=20) queries,
    64 beacons, window 64."""
    return Workload("beacon_serving", R, layers, 8, 128, _full(R, 1024), _full(R, 2112), _full(R, 2048),
                    selectors=("beacon",), num_q_heads=32, num_beacons=64, query_window=64,
                    n_components=64, data_seed=1002, philox_seed=2)


def long_trace(R=8, layers=64) -> Workload:
    """8 requests, 64 layers, P=1024 + 31744 generated compressed to 4096 in one round,
    256 beacons from a 256-component mixture; G=4 and W=256 (1024 points) by reading."""
    return Workload("long_trace", R, layers, 8, 128, _full(R, 1024), _full(R, 32768), _full(R, 4096),
                    selectors=("beacon",), num_q_heads=32, num_beacons=256, query_window=256,
                    n_components=256, data_seed=1003, philox_seed=3)


def ragged(c: int, R=64, layers=36, selectors=("random", "random_shared", "beacon"), seed=1004) -> Workload:
    """64 requests with L ~ U{4096..32768}, P ~ U{128..1536}, K = floor(L / c)."""
    rng = np.random.default_rng(seed)
    L = rng.integers(4096, 32768, R, endpoint=True)
    P = rng.integers(128, 1536, R, endpoint=True)
    K = L // c
    return Workload(f"ragged_c{c}", R, layers, 8, 128, P.astype(np.int64), L.astype(np.int64),
                    K.astype(np.int64), selectors=tuple(selectors), num_q_heads=32, num_beacons=64,
                    query_window=64, n_components=64, data_seed=seed, philox_seed=4,
                    extra={"compression": c})


def scaled(w: Workload, **kw) -> Workload:
    """A copy with some fields replaced (smaller test variants)."""
    n = kw.get("num_requests", w.num_requests)
    out = replace(w, **kw)
    if n != w.num_requests:
        out.prompt = w.prompt[:n].copy() if n <= len(w.prompt) else np.resize(w.prompt, n)
        out.length = w.length[:n].copy() if n <= len(w.length) else np.resize(w.length, n)
        out.budget = w.budget[:n].copy() if n <= len(w.budget) else np.resize(w.budget, n)
    return out


# ------------------------------------------------------------ generators --

def torch_dtype(name: str):
    import torch
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


class Generator:
    """Seeded source of K/V rows and decode queries for one workload.

    Draws happen on ``device`` with a torch.Generator; the fixed per-(layer,
    head) structure (outlier channels, mixture means) is drawn once."""

    def __init__(self, w: Workload, device="cuda"):
        import torch
        self.w = w
        self.device = torch.device(device)
        self.dtype = torch_dtype(w.dtype)
        self.gen = torch.Generator(device=self.device)
        self.gen.manual_seed(w.data_seed)
        cpu = torch.Generator().manual_seed(w.data_seed + 7919)
        Ly, H, d = w.num_layers, w.num_kv_heads, w.head_dim
        scale = torch.ones((Ly, H, d), dtype=torch.float32)
        if w.outlier_channels > 0:
            for l in range(Ly):
                for h in range(H):
                    ch = torch.randperm(d, generator=cpu)[: w.outlier_channels]
                    scale[l, h, ch] = w.outlier_scale
        self.channel_scale = scale.to(self.device).view(1, Ly, 1, H, d)
        self.means = None
        if w.n_components > 0:
            m = torch.randn((Ly, H, w.n_components, d), generator=cpu, dtype=torch.float64)
            self.means = (m / m.norm(dim=-1, keepdim=True)).to(self.device)
        self.np_rng = np.random.default_rng(w.data_seed + 104729)

    def kv(self, n_req: int, T: int):
        """K and V rows [n_req, layers, T, Hkv, d] in the cache dtype."""
        import torch
        w = self.w
        shape = (n_req, w.num_layers, T, w.num_kv_heads, w.head_dim)
        out = []
        for _ in range(2):
            x = torch.randn(shape, generator=self.gen, device=self.device, dtype=torch.float32)
            x.mul_(self.channel_scale)
            out.append(x.to(self.dtype))
        return out[0], out[1]

    def _wood_w(self, n: int) -> np.ndarray:
        """n draws of the cosine to the mean direction for vMF(kappa) in d dims (Wood 1994)."""
        kappa, p = self.w.kappa, self.w.head_dim
        b = (-2 * kappa + math.sqrt(4 * kappa * kappa + (p - 1) ** 2)) / (p - 1)
        x0 = (1 - b) / (1 + b)
        c = kappa * x0 + (p - 1) * math.log(1 - x0 * x0)
        out = np.empty(n)
        todo = np.arange(n)
        rng = self.np_rng
        while len(todo):
            z = rng.beta((p - 1) / 2, (p - 1) / 2, len(todo))
            wv = (1 - (1 + b) * z) / (1 - (1 - b) * z)
            u = rng.random(len(todo))
            ok = kappa * wv + (p - 1) * np.log(1 - x0 * wv) - c >= np.log(u)
            out[todo[ok]] = wv[ok]
            todo = todo[~ok]
        return out

    def queries(self, n_req: int, T: int, norm: float | None = None):
        """Decode queries [n_req, layers, T, Hq, d] from the vMF mixture, scaled to
        the workload's query norm unless ``norm`` is given."""
        import torch
        w = self.w
        norm = w.query_norm if norm is None else norm
        Ly, Hq, d = w.num_layers, w.num_q_heads or w.num_kv_heads, w.head_dim
        out = torch.empty((n_req, Ly, T, Hq, d), dtype=self.dtype, device=self.device)
        per_req = Ly * T * Hq * d * 8 * 4  # float64 temporaries
        step = max(1, min(n_req, (1 << 30) // per_req))
        for r0 in range(0, n_req, step):
            r1 = min(n_req, r0 + step)
            out[r0:r1] = self._queries(r1 - r0, T, norm)
        return out

    def _queries(self, n_req: int, T: int, norm: float):
        import torch
        w = self.w
        Ly, Hq, d, G = w.num_layers, w.num_q_heads or w.num_kv_heads, w.head_dim, w.G
        n = n_req * Ly * T * Hq
        comp = torch.randint(0, w.n_components, (n_req, Ly, T, Hq), generator=self.gen, device=self.device)
        kv_head = (torch.arange(Hq, device=self.device) // G).view(1, 1, 1, Hq).expand(n_req, Ly, T, Hq)
        layer = torch.arange(Ly, device=self.device).view(1, Ly, 1, 1).expand(n_req, Ly, T, Hq)
        mu = self.means[layer, kv_head, comp]  # [n_req, Ly, T, Hq, d] float64
        wv = torch.from_numpy(self._wood_w(n)).to(self.device).view(n_req, Ly, T, Hq, 1)
        v = torch.randn(mu.shape, generator=self.gen, device=self.device, dtype=torch.float64)
        v = v - (v * mu).sum(-1, keepdim=True) * mu
        v = v / v.norm(dim=-1, keepdim=True)
        x = wv * mu + torch.sqrt(torch.clamp(1 - wv * wv, min=0)) * v
        return (x * norm).to(self.dtype)


def fill(ctx, w: Workload, gen: Generator, chunk: int = 256, with_queries: bool | None = None):
    """Brings every request of ctx to the workload's pre-round state: P_r
    protected tokens then L_r - P_r generated tokens, appended in chunks.
    Queries are appended with the generated tokens when the workload has a
    query window (only the last W steps stay in the ring)."""
    with_queries = (w.query_window > 0) if with_queries is None else with_queries
    R = w.num_requests
    groups = {}
    for r in range(R):
        groups.setdefault((int(w.prompt[r]), int(w.length[r])), []).append(r)
    for (P, L), reqs in groups.items():
        ids = np.array(reqs, np.int32)
        done = 0
        while done < P:
            T = min(chunk, P - done)
            k, v = gen.kv(len(ids), T)
            ctx.append(ids, k, v, None, protect=True)
            done += T
        q_from = L - min(w.query_window, L - P) if with_queries else L
        while done < L:
            T = min(chunk if done < q_from else 16, (q_from if done < q_from else L) - done)
            k, v = gen.kv(len(ids), T)
            q = gen.queries(len(ids), T) if done >= q_from else None
            ctx.append(ids, k, v, q, protect=False)
            done += T
