"""Plants one plausible mistake at a time in a copy of the oracle (on the CPU)
and checks that at least one pin catches it.  This shows the pins are strong
enough to fail on a dropped term, a wrong sign or index, a swapped operand."""
import pytest

import oracle
import pins

# (name, original text, mutated text, the checks expected to catch it)
MUTANTS = [
    ("philox_multiplier", "orc_mulhilo64(ORC_PHILOX_M0, x0", "orc_mulhilo64(ORC_PHILOX_M1, x0",
     [pins.check_philox]),
    ("philox_key_schedule", "if (i > 0) {", "if (i >= 0) {", [pins.check_philox]),
    ("philox_word_mix", "uint64_t y0 = hi1 ^ x1 ^ k0;", "uint64_t y0 = hi1 ^ x3 ^ k0;",
     [pins.check_philox]),
    ("score_low_bits", "return (uint32_t)(out[0] >> 32);", "return (uint32_t)(out[0]);",
     [pins.check_random_score]),
    ("counter_order", "ctr[2] = (uint64_t)l;\n  ctr[3] = (uint64_t)r;",
     "ctr[2] = (uint64_t)r;\n  ctr[3] = (uint64_t)l;", [pins.check_random_score]),
    ("noop_boundary", "if (L <= K) {", "if (L < K) {", [pins.check_retention]),
    ("over_budget_flag", "if (P > K) *flags |= 2;", "if (P >= K) *flags |= 2;",
     [pins.check_retention]),
    ("tie_break_reversed", "if (x->pos < y->pos) return -1;\n  if (x->pos > y->pos) return 1;",
     "if (x->pos < y->pos) return 1;\n  if (x->pos > y->pos) return -1;", [pins.check_select]),
    ("keep_lowest_scores", "if (x->score > y->score) return -1;\n  if (x->score < y->score) return 1;",
     "if (x->score > y->score) return 1;\n  if (x->score < y->score) return -1;",
     [pins.check_select, pins.check_random_round_invariants]),
    ("prompt_copy_short", "memcpy(rows_out, rows_in, (size_t)(P * row_bytes));",
     "memcpy(rows_out, rows_in, (size_t)((P > 0 ? P - 1 : 0) * row_bytes));", [pins.check_compact]),
    ("update_drops_history", "(n * beacons[i * d + k] + sum[i * d + k]) / (n + (double)m[i])",
     "(beacons[i * d + k] + sum[i * d + k]) / (n + (double)m[i])", [pins.check_beacon_update]),
    ("init_index", "int64_t src = (i * n_pts) / B;", "int64_t src = i;", [pins.check_beacon_update]),
    ("distance_sign", "double diff = pts[p * d + k] - beacons[i * d + k];",
     "double diff = pts[p * d + k] + beacons[i * d + k];", [pins.check_beacon_update]),
    ("scale_by_d", "double inv_sqrt_d = 1.0 / sqrt((double)d);", "double inv_sqrt_d = 1.0 / (double)d;",
     [pins.check_beacon_score]),
    ("lse_drops_max", "lse[b] = mx + log(s);", "lse[b] = log(s);", [pins.check_beacon_score]),
    ("lse_skips_prompt", "for (int64_t j = 0; j < L; ++j) s += exp(z[b * L + j] - mx);",
     "for (int64_t j = P; j < L; ++j) s += exp(z[b * L + j] - mx);", [pins.check_beacon_score]),
    ("min_over_beacons", "if (p > best) best = p;", "if (p < best || best == -INFINITY) best = p;",
     [pins.check_beacon_score]),
    ("bf16_precision", "double q = nearbyint(ldexp(m, 8));", "double q = nearbyint(ldexp(m, 9));",
     [pins.check_bf16]),
    ("bf16_truncates", "double q = nearbyint(ldexp(m, 8));", "double q = trunc(ldexp(m, 8));",
     [pins.check_bf16]),
    ("block_index_modulo", "return orc_random_score(seed, round, r, l, h, pos / (block > 0 ? block : 1), shared);",
     "return orc_random_score(seed, round, r, l, h, pos % (block > 0 ? block : 1), shared);",
     [pins.check_block_score]),
    ("hole_fill_reverse", "for (int64_t i = 0; i < R; ++i) {\n    if (kept_slots[i] < R) continue;",
     "for (int64_t i = R - 1; i >= 0; --i) {\n    if (kept_slots[i] < R) continue;", [pins.check_hole_fill]),
    ("trigger_unnormalised", "acc += (trig[b] / total) * exp(z[b * L + j] - lse[b]);",
     "acc += trig[b] * exp(z[b * L + j] - lse[b]);", [pins.check_beacon_trigger_score]),
    ("trigger_max_not_sum", "acc += (trig[b] / total) * exp(z[b * L + j] - lse[b]);",
     "acc = fmax(acc, (trig[b] / total) * exp(z[b * L + j] - lse[b]));", [pins.check_beacon_trigger_score]),
    ("trigger_lse_skips_prompt", "for (int64_t j = 0; j < L; ++j) sum += exp(z[b * L + j] - mx);",
     "for (int64_t j = P; j < L; ++j) sum += exp(z[b * L + j] - mx);", [pins.check_beacon_trigger_score]),
    ("trigger_scale_by_d", "const double rsqrt_d = 1.0 / sqrt((double)d);", "const double rsqrt_d = 1.0 / (double)d;",
     [pins.check_beacon_trigger_score]),
    ("attention_no_scale", "s[j] = scale * dot;", "s[j] = dot;", [pins.check_decode_attention]),
    ("attention_lse_drops_max", "double lse = mx + log(sum);", "double lse = log(sum);",
     [pins.check_decode_attention]),
    ("attention_weight_no_norm", "double w = exp(s[j] - lse);", "double w = exp(s[j] - mx);",
     [pins.check_decode_attention]),
    ("attention_gqa_modulo", "int64_t h = hq / G;", "int64_t h = hq % Hkv;", [pins.check_decode_attention_gqa]),
    ("attention_value_row", "out[c] += w * v[j * d + c];", "out[c] += w * v[c];", [pins.check_decode_attention]),
]


@pytest.mark.parametrize("name,old,new,checks", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new, checks):
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = oracle.compile_source(src.replace(old, new), str(tmp_path / f"mut_{name}.so"))
    caught = False
    with oracle.use_library(path):
        for check in checks:
            try:
                check()
            except (AssertionError, ValueError):
                caught = True
                break
    assert caught, f"mutant {name} survived the pins"
