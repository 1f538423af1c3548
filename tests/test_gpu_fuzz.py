"""Seeded random configurations of the random-selector round against the
oracle: request count, layers, heads, head_dim, dtype, lengths, prompts,
budgets and the round options all drawn at random, three rounds each, every
segment's position map and the K/V bytes of one layer checked exactly."""
import numpy as np
import pytest

from decode_kv_cache_paged_b200 import workloads as wl
from test_gpu_round_options import run_option_rounds

pytestmark = pytest.mark.gpu


def _config(seed: int):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 7))
    layers = int(rng.integers(1, 4))
    H = int(rng.choice([1, 2, 4]))
    d = int(rng.choice([64, 128]))
    dtype = str(rng.choice(["bf16", "f32"]))
    L = rng.integers(0, 3000, R)
    P = np.minimum(rng.integers(0, 600, R), L)
    K = rng.integers(1, 2500, R)
    w = wl.Workload(f"fuzz{seed}", R, layers, H, d, P.astype(np.int64), L.astype(np.int64), K.astype(np.int64),
                    dtype=dtype, selectors=("random",), trigger=int(rng.integers(1, 80)), data_seed=seed,
                    philox_seed=seed)
    selector = str(rng.choice(["random", "random_shared"]))
    plan = []
    for _ in range(3):
        opt = {}
        if rng.random() < 0.3:
            opt["sinks"] = int(rng.integers(0, 64))
        if rng.random() < 0.4:
            opt["block"] = int(rng.choice([2, 16, 64, 256]))
        if rng.random() < 0.4:
            opt["compaction"] = "hole_fill"
        plan.append(opt)
    return w, selector, plan


@pytest.mark.parametrize("seed", list(range(12)))
def test_random_configuration(seed):
    w, selector, plan = _config(seed)
    # requests that never evict grow by a trigger window per round: room for three
    extra = w.num_requests * (3 * w.trigger // 16 + 2) * w.num_layers
    run_option_rounds(w, selector, plan, seed=1000 + seed, kv_layers=(0,), check_scores_n=100, extra_pages=extra)


@pytest.mark.parametrize("seed", list(range(6)))
def test_attention_random_configuration(seed):
    """Decode attention after a random round, on a random configuration."""
    from test_gpu_attention import _run
    w, _, plan = _config(100 + seed)
    rng = np.random.default_rng(200 + seed)
    w.num_q_heads = w.num_kv_heads * int(rng.choice([1, 2, 4, 8]))
    w.num_beacons = 0
    w.query_window = 0
    w.budget = np.maximum(w.budget, 1)
    opts = {("sink_tokens" if k == "sinks" else k): v for k, v in plan[0].items()}
    print(_run(w, rounds=[opts], seed=seed))
