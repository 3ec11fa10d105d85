"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source, builds the copy into
a temporary library on the CPU, swaps it in for the oracle, and requires that at least
one of the pins named for that case fails. A pin that cannot tell the planted mistake
from the correct oracle would leave the oracle unpinned where that mistake could hide.
"""
import ctypes
import importlib
import inspect
import os
import subprocess

import pytest

import oracle
from oracle import build as oracle_build

# (what the mistake is, text replaced, replacement, pins expected to catch it)
MUTANTS = [
    ("plan order ignores the source rank",
     "    if (a->src != b->src) return a->src < b->src ? -1 : 1;\n", "",
     ["test_oracle_plan.test_plan_hand_example", "test_oracle_plan.test_plan_exhaustive_tiny"]),
    ("home rank by modulo instead of division",
     "sl[n].rank = e / per_rank;", "sl[n].rank = e % R;",
     ["test_oracle_plan.test_plan_hand_example", "test_oracle_plan.test_plan_exhaustive_tiny"]),
    ("cut at S*K-1 rows",
     "row_rank[i] = (int32_t)(i / SK);", "row_rank[i] = (int32_t)(i / (SK - 1 > 0 ? SK - 1 : 1)) % R;",
     ["test_oracle_plan.test_plan_hand_example", "test_oracle_plan.test_plan_exhaustive_tiny"]),
    ("redundant counts every instance",
     "if (inst[e] > 1) redundant += inst[e] - 1;", "redundant += inst[e];",
     ["test_oracle_plan.test_plan_hand_example", "test_oracle_plan.test_plan_single_hot_expert_spans_every_rank"]),
    ("prefetched counts home replicas",
     "if (r != e / per_rank) prefetched += 1;", "prefetched += 1;",
     ["test_oracle_plan.test_plan_hand_example", "test_oracle_plan.test_plan_balanced_input_keeps_experts_home"]),
    ("histogram double-counts",
     "        hist[e] += 1;\n    }\n    return ORC_OK;", "        hist[e] += (e == 0) ? 2 : 1;\n    }\n    return ORC_OK;",
     ["test_oracle_plan.test_histogram_matches_bincount_and_sums_to_n"]),
    ("grouped plan keeps dropped slots",
     "                if (keep && !keep[n]) continue;\n", "",
     ["test_oracle_plan.test_grouped_plan_packs_kept_slots_by_instance"]),
    ("mapping mode 0 with a floor instead of a ceiling",
     "(world_size + c - 1) / c;", "world_size / c;",
     ["test_oracle_update_expert.test_mode0_column_never_exceeds_count",
      "test_oracle_update_expert.test_mapping_hand_example"]),
    ("mapping mode 1 by flat slot index",
     "col = (i % c) + 1;", "col = ((i * K + k) % c) + 1;",
     ["test_oracle_update_expert.test_mapping_hand_example", "test_oracle_update_expert.test_mode1_round_robin_by_token"]),
    ("mapping mode 1 without the +1",
     "col = (i % c) + 1;", "col = (i % c);",
     ["test_oracle_update_expert.test_mapping_hand_example", "test_oracle_update_expert.test_mode1_round_robin_by_token"]),
    ("pruning keeps the low scores (the literal line)",
     "!(scales[i * K + k] < v)", "(scales[i * K + k] < v)",
     ["test_oracle_update_expert.test_pruning_hand_example"]),
    ("threshold value is the last product only",
     "                v = v + prod;", "                v = prod;",
     ["test_oracle_update_expert.test_pruning_hand_example"]),
    ("quantisation rounds half away from zero",
     "float r = nearbyintf(v);", "float r = roundf(v);",
     ["test_oracle_numerics.test_quant_half_even_golden"]),
    ("quantisation scale over 128",
     "float scale = amax / 127.0f;\n    *scale_out = scale;", "float scale = amax / 128.0f;\n    *scale_out = scale;",
     ["test_oracle_numerics.test_quant_half_even_golden", "test_oracle_numerics.test_quant_properties"]),
    ("bf16 conversion truncates",
     "u = u + 0x7fffu + keep_lsb;", "u = u;",
     ["test_oracle_numerics.test_float_to_bf16_matches_torch"]),
    ("dispatch copies the wrong token",
     "const uint16_t *src = x + (n / K) * H;", "const uint16_t *src = x + (n % K) * H;",
     ["test_oracle_numerics.test_dispatch_copies_rows_to_their_positions"]),
    ("combine weights every slot by the first gate",
     "float prod = gates[g * K + k] * bf16_bits_to_float(y[p * H + h]);",
     "float prod = gates[g * K] * bf16_bits_to_float(y[p * H + h]);",
     ["test_oracle_numerics.test_combine_softmax_gates_identity_expert_returns_x",
      "test_oracle_numerics.test_combine_random_rows_within_error_bound"]),
    ("prefetch gives home replicas a slot",
     "            if (e / per_rank == r) {\n                row = e;", "            if (0) {\n                row = e;",
     ["test_oracle_prefetch.test_prefetch_hand_example",
      ("test_oracle_prefetch.test_prefetch_properties", {"name": "tiny", "B": 4})]),
    ("grad reduce adds in descending rank order",
     "        for (int64_t s = 0; s < (int64_t)R * B; s++) {\n            if (slot_expert[s] != e) continue;",
     "        for (int64_t s = (int64_t)R * B - 1; s >= 0; s--) {\n            if (slot_expert[s] != e) continue;",
     ["test_oracle_prefetch.test_grad_reduce_adds_in_ascending_rank_order"]),
    ("grad reduce leaves the slots uncleared",
     "        for (int64_t i = 0; i < D; i++) grad_slots[s * D + i] = 0.0f;\n", "",
     ["test_oracle_prefetch.test_grad_reduce_conserves_integer_gradients"]),
    ("smooth quantisation uses the first expert's scales",
     "float v = bf16_bits_to_float(row[h]) * smooth[(int64_t)e * H + h];",
     "float v = bf16_bits_to_float(row[h]) * smooth[h];",
     ["test_oracle_smooth.test_power_of_two_scales_commute_with_quantisation",
      "test_oracle_smooth.test_per_slot_bounds"]),
    ("combine skips the last slot",
     "                acc = acc + prod;", "                if (k + 1 < K) acc = acc + prod;",
     ["test_oracle_numerics.test_combine_k1_is_one_rounded_product",
      ("test_oracle_numerics.test_combine_equal_power_of_two_gates_is_exact", {"K": 4})]),
    ("dedup: a rank's row range includes the next rank's first row",
     "if (p >= rank_off[r] && p < rank_off[r + 1]) return r;",
     "if (p >= rank_off[r] && p <= rank_off[r + 1]) return r;",
     ["test_oracle_dedup.test_dedup_hand_example"]),
    ("dedup: every slot is put on the send list",
     "                if (first < 0) {\n                    first = n;",
     "                if (1) {\n                    first = n;",
     ["test_oracle_dedup.test_dedup_hand_example",
      ("test_oracle_dedup.test_dedup_balanced_plans", {"R": 4, "E": 16, "S": 37, "K": 3})]),
    ("dedup: a rank's rows in descending token order",
     "        for (int64_t g = 0; g < T; g++) {\n            int64_t first = -1;",
     "        for (int64_t g = T - 1; g >= 0; g--) {\n            int64_t first = -1;",
     ["test_oracle_dedup.test_dedup_hand_example",
      ("test_oracle_dedup.test_dedup_balanced_plans", {"R": 2, "E": 4, "S": 3, "K": 2})]),
    ("pruning ignores the active mask",
     "                out_mask[i * K + k] = (uint8_t)(act && !(scales[i * K + k] < v));",
     "                out_mask[i * K + k] = (uint8_t)(!(scales[i * K + k] < v));",
     ["test_oracle_update_expert.test_pruning_hand_example",
      "test_oracle_update_expert.test_generated_mapping_workload_properties"]),
    ("grouped plan ranks instances by modulo",
     "                sl[m].rank = key / keys_per_rank;", "                sl[m].rank = key % R;",
     ["test_oracle_plan.test_grouped_plan_packs_kept_slots_by_instance"]),
    ("dequantisation truncates to bf16",
     "            y[r * H + h] = orc_float_to_bf16(v);",
     "            { uint32_t u; memcpy(&u, &v, sizeof u); y[r * H + h] = (uint16_t)(u >> 16); }",
     ["test_oracle_numerics.test_dequantize_is_rounded_product"]),
    ("prefetch copies the first expert into every slot",
     "        for (int64_t i = 0; i < D; i++) w_slots[s * D + i] = w_home[(int64_t)e * D + i];",
     "        for (int64_t i = 0; i < D; i++) w_slots[s * D + i] = w_home[i];",
     [("test_oracle_prefetch.test_prefetch_properties", {"name": "r8", "B": 8})]),
    ("rmsnorm without eps",
     "        double r = 1.0 / sqrt(ss / (double)H + eps);",
     "        double r = 1.0 / sqrt(ss / (double)H);",
     ["test_oracle_rmsnorm.test_rmsnorm_constant_rows_closed_form",
      "test_oracle_rmsnorm.test_rmsnorm_matches_torch_float64"]),
    ("rmsnorm mean over H - 1",
     "        double r = 1.0 / sqrt(ss / (double)H + eps);",
     "        double r = 1.0 / sqrt(ss / (double)(H - 1) + eps);",
     ["test_oracle_rmsnorm.test_rmsnorm_constant_rows_closed_form",
      "test_oracle_rmsnorm.test_rmsnorm_matches_torch_float64"]),
    ("rmsnorm without gamma",
     "            double v = x[h] * r * (double)bf16_bits_to_float(gamma[h]);",
     "            double v = x[h] * r;",
     ["test_oracle_rmsnorm.test_rmsnorm_matches_torch_float64"]),
    ("rmsnorm drops the residual from x",
     "            x[h] = (double)bf16_bits_to_float(c[g * H + h]) + (double)bf16_bits_to_float(residual[g * H + h]);",
     "            x[h] = (double)bf16_bits_to_float(c[g * H + h]);",
     ["test_oracle_rmsnorm.test_rmsnorm_dropped_token_is_the_residual",
      "test_oracle_rmsnorm.test_rmsnorm_matches_torch_float64"]),
    ("binary64 to bf16 through binary32 (two roundings)",
     "        r = ldexp(nearbyint(ldexp(m, 8)), e - 8);   /* 8 significant bits */",
     "        r = ldexp(nearbyint(ldexp((double)(float)m, 8)), e - 8);",
     ["test_oracle_rmsnorm.test_double_to_bf16_single_rounding"]),
    ("expansion copies the first row's scale",
     "if (src_scale && dst_scale) dst_scale[p] = src_scale[u];",
     "if (src_scale && dst_scale) dst_scale[p] = src_scale[0];",
     ["test_oracle_dedup.test_expand_copies_rows_and_scales"]),
]


def _run_pin(pin, golden_dir):
    """Run one pin: a 'module.function' name, or (name, arguments of a parametrized pin)."""
    pin, kwargs = (pin, {}) if isinstance(pin, str) else (pin[0], dict(pin[1]))
    mod, fn = pin.split(".")
    f = getattr(importlib.import_module(mod), fn)
    if "golden_dir" in inspect.signature(f).parameters:
        kwargs["golden_dir"] = golden_dir
    f(**kwargs)


@pytest.fixture(scope="module")
def oracle_source():
    return open(oracle_build.SRC).read()


@pytest.mark.parametrize("what,find,repl,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(what, find, repl, pins, oracle_source, tmp_path, golden_dir,
                                   monkeypatch):
    assert oracle_source.count(find) == 1, f"mutation target not unique: {what}"
    # the correct oracle passes these pins
    for pin in pins:
        _run_pin(pin, golden_dir)
    src = tmp_path / "mutant.c"
    src.write_text(oracle_source.replace(find, repl))
    so = tmp_path / "mutant.so"
    subprocess.run(["gcc", *oracle_build.CFLAGS, str(src), "-o", str(so), "-lm"], check=True,
                   capture_output=True)
    monkeypatch.setattr(oracle, "_lib", oracle._configure(ctypes.CDLL(os.fspath(so))))
    caught = []
    for pin in pins:
        try:
            _run_pin(pin, golden_dir)
        except (AssertionError, oracle.OracleError):
            caught.append(pin)
    assert caught, f"no pin caught the planted mistake: {what}"
