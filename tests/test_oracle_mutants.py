"""Mutation tests of the oracle's pins, on the CPU.

Each case plants one plausible mistake in a copy of the oracle's C source
(a dropped rank, a missing 1/D, a flipped update sign, a missing bias
correction, a wrong slice index, a wrong rounding tie, a wrong pad, a reversed
gather, a wrong ledger bucket, ...), builds that copy with the oracle's flags,
swaps it in, and runs the pins of tests/test_oracle.py against it: at least one
pin must fail.  A mutant that survives means the pins do not fix that part of
the oracle."""
import os
import subprocess
import tempfile


import oracle
import test_oracle as pins
from oracle import build as obuild

SOURCE = open(obuild.SRC).read()

MUTANTS = [
    ("the last rank is dropped from the fold",
     "for (int32_t d = 1; d < D; ++d)\n            acc = acc + ",
     "for (int32_t d = 1; d < D - 1; ++d)\n            acc = acc + "),
    ("the fp32 sum is not scaled by 1/D", "return acc * inv_D;", "return acc;"),
    ("the bf16 average is not rounded to bf16",
     "return ref_f32_from_bf16(ref_bf16_from_f32(ref_f32_from_bf16(acc) * inv_D));",
     "return ref_f32_from_bf16(acc) * inv_D;"),
    ("the update is added instead of subtracted", "float p2 = p1 - delta;", "float p2 = p1 + delta;"),
    ("no first-moment bias correction", "c.step_size = (float)(hp->lr / bias_correction1);",
     "c.step_size = (float)(hp->lr / (0.0 * bias_correction1 + 1.0));"),
    ("no second-moment bias correction", "float root_hat = root * c->inv_sqrt_bc2;",
     "float root_hat = root + 0.0f * c->inv_sqrt_bc2;"),
    ("no weight decay", "float p1 = *p * c->decay;", "float p1 = *p;"),
    ("v accumulates g instead of g*g", "float v_new_part = c->omb2 * g2;",
     "float v_new_part = c->omb2 * g2 * 0.0f + c->omb2 * g;"),
    ("eps left out of the denominator", "float denom = root_hat + c->eps;", "float denom = root_hat;"),
    ("the full layout ignores the rank's offset", "return layout == 0 ? (int64_t)r * S + j : j;",
     "return layout == 0 ? (int64_t)r * S * 0 + j : j;"),
    ("ties round away from zero instead of to even",
     "if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u)))", "if (dropped >= 0x8000u)"),
    ("one extra unit of padding", "*N_pad_out = units * unit;", "*N_pad_out = units * unit + unit;"),
    ("the gather reverses the shards", "flat[(int64_t)r * S + j] = shards[r][j];",
     "flat[(int64_t)r * S + j] = shards[D - 1 - r][j];"),
    ("ZeRO-1 forgets the gradient bucket", "case 1: return optim * N / D + weights * N + grads * N;",
     "case 1: return optim * N / D + weights * N;"),
    ("the unflatten starts one element late", "out[t][k] = flat[offset[t] + k];",
     "out[t][k] = flat[offset[t] + k + (k + 1 < numel[t] ? 1 : 0)];"),
    ("the all-gather counts the device's own shard as received",
     "return (double)n_blocks * block_bytes * (double)(D - 1) / (double)D;",
     "return (double)n_blocks * block_bytes * (double)(D) / (double)D;"),
    ("the cross-node fold takes the node sums in reverse order",
     "float total = node_sums[0][i];\n"
     "        for (int32_t k = 1; k < R; ++k) {\n"
     "            total = total + node_sums[k][i];",
     "float total = node_sums[R - 1][i];\n"
     "        for (int32_t k = 1; k < R; ++k) {\n"
     "            total = total + node_sums[R - 1 - k][i];"),
    ("the cross-node fold leaves the scaled bf16 gradient unrounded",
     "        float g = total * inv_RD;\n"
     "        if (reduce_dtype == 1)\n"
     "            g = ref_f32_from_bf16(ref_bf16_from_f32(g));",
     "        float g = total * inv_RD;"),
    ("HYBRID_SHARD folds all ranks flat, ignoring the nodes",
     "float node_sum = ref_f32_from_bf16(node[0][idx]);",
     "float node_sum = k == 0 ? ref_f32_from_bf16(node[0][idx]) : total + ref_f32_from_bf16(node[0][idx]);"
     " total = 0.0f;"),
    ("HYBRID_SHARD scales by 1/D instead of 1/(R*D)", "return total * inv_RD;",
     "return total * (inv_RD * (float)R);"),
    ("HYBRID_SHARD sums the nodes in reverse order",
     "const uint16_t* const* node = contrib + (int64_t)k * D;\n            float node_sum",
     "const uint16_t* const* node = contrib + (int64_t)(R - 1 - k) * D;\n            float node_sum"),
    ("HYBRID_SHARD maps rank k*D+d to node d",
     "node_sum = node_sum + ref_f32_from_bf16(node[d][idx]);",
     "node_sum = node_sum + ref_f32_from_bf16(contrib[(int64_t)d * R + k][idx]);"),
    ("HYBRID_SHARD rounds each bf16 node sum once, at the node's end",
     "uint16_t node_sum = node[0][idx];\n"
     "            for (int32_t d = 1; d < D; ++d)\n"
     "                node_sum = ref_bf16_from_f32(ref_f32_from_bf16(node_sum) + ref_f32_from_bf16(node[d][idx]));",
     "float node_f = ref_f32_from_bf16(node[0][idx]);\n"
     "            for (int32_t d = 1; d < D; ++d)\n"
     "                node_f = node_f + ref_f32_from_bf16(node[d][idx]);\n"
     "            uint16_t node_sum = ref_bf16_from_f32(node_f);"),
    ("HYBRID_SHARD bf16 cross-node sums are kept in fp32",
     "        uint16_t total = 0;\n"
     "        for (int32_t k = 0; k < R; ++k) {\n"
     "            const uint16_t* const* node = contrib + (int64_t)k * D;\n"
     "            uint16_t node_sum = node[0][idx];\n"
     "            for (int32_t d = 1; d < D; ++d)\n"
     "                node_sum = ref_bf16_from_f32(ref_f32_from_bf16(node_sum) + ref_f32_from_bf16(node[d][idx]));\n"
     "            total = (k == 0) ? node_sum\n"
     "                             : ref_bf16_from_f32(ref_f32_from_bf16(total) + ref_f32_from_bf16(node_sum));\n"
     "        }\n"
     "        return ref_f32_from_bf16(ref_bf16_from_f32(ref_f32_from_bf16(total) * inv_RD));",
     "        float total = 0.0f;\n"
     "        for (int32_t k = 0; k < R; ++k) {\n"
     "            const uint16_t* const* node = contrib + (int64_t)k * D;\n"
     "            uint16_t node_sum = node[0][idx];\n"
     "            for (int32_t d = 1; d < D; ++d)\n"
     "                node_sum = ref_bf16_from_f32(ref_f32_from_bf16(node_sum) + ref_f32_from_bf16(node[d][idx]));\n"
     "            total = (k == 0) ? ref_f32_from_bf16(node_sum) : total + ref_f32_from_bf16(node_sum);\n"
     "        }\n"
     "        return ref_f32_from_bf16(ref_bf16_from_f32(total * inv_RD));"),
]


def golden(name):
    import json
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)) as f:
        return json.load(f)


# the pins, cheapest first; each is called with fixed arguments
PINS = [
    lambda: pins.test_reduce_scatter_worked_example(golden),
    lambda: pins.test_allgather_worked_example(golden),
    lambda: pins.test_plan_workloads_golden(golden),
    lambda: pins.test_memory_figures_golden(golden),
    lambda: pins.test_transient_and_steady_state_golden(golden),
    lambda: pins.test_allgather_volume_golden(golden),
    lambda: pins.test_adamw_step1_closed_form(),
    lambda: pins.test_adamw_zero_gradient_keeps_zero_pad(),
    lambda: pins.test_reduce_fp32_matches_torch_left_fold(8),
    lambda: pins.test_reduce_bf16_matches_torch_bf16_adds(6),   # 1/6 is inexact: the final rounding shows
    lambda: pins.test_reduce_integers_modes_agree_and_are_exact(),
    lambda: pins.test_bf16_rne_matches_torch_cast(),
    lambda: pins.test_gather_round_trip_and_unflatten(),
    lambda: pins.test_plan_invariants_brute_force(),
    lambda: pins.test_adamw_ten_steps_matches_torch_adamw_float64(),
    lambda: pins.test_reduce_adamw_composes_reduce_then_adamw(),
    lambda: pins.test_sharded_steps_equal_one_unsharded_step(4, 1, [5, 7, 1]),
    lambda: pins.test_hybrid_worked_examples(golden),
    lambda: pins.test_hybrid_integers_are_the_exact_mean(4, 8),
    lambda: pins.test_hybrid_one_node_is_the_plain_reduction(3, 0),
    lambda: pins.test_hybrid_one_node_is_the_plain_reduction(3, 1),
    lambda: pins.test_hybrid_one_rank_per_node_is_the_plain_fold_over_nodes(3, 0),
    lambda: pins.test_hybrid_one_rank_per_node_is_the_plain_fold_over_nodes(3, 1),
    lambda: pins.test_hybrid_matches_torch_two_level_fold(2, 3),
    lambda: pins.test_hybrid_worked_examples_through_the_two_parts(golden),
    lambda: pins.test_node_sums_then_fold_is_the_hybrid_step(2, 3),
    lambda: pins.test_node_sum_matches_torch_folds(5),
]


def build_mutant(src: str, out_dir: str, tag: int) -> str:
    c_path = os.path.join(out_dir, f"mutant{tag}.c")
    so_path = os.path.join(out_dir, f"libmutant{tag}.so")
    with open(c_path, "w") as f:
        f.write(src)
    subprocess.run(["gcc", *obuild.CFLAGS, c_path, "-o", so_path, "-lm"], check=True, capture_output=True)
    return so_path


def killed_by(so_path: str):
    """The index of the first pin that fails against the given library, or None."""
    previous = oracle.use_library(so_path)
    try:
        for k, pin in enumerate(PINS):
            try:
                pin()
            except (AssertionError, ValueError):
                return k
        return None
    finally:
        oracle.restore_library(previous)


def test_every_planted_mistake_fails_a_pin():
    survivors = []
    with tempfile.TemporaryDirectory() as tmp:
        for tag, (what, old, new) in enumerate(MUTANTS):
            assert SOURCE.count(old) == 1, f"mutation site not found exactly once: {what}"
            so = build_mutant(SOURCE.replace(old, new), tmp, tag)
            if killed_by(so) is None:
                survivors.append(what)
    assert not survivors, f"mutants the pins did not catch: {survivors}"


def test_the_unmutated_oracle_passes_every_pin():
    with tempfile.TemporaryDirectory() as tmp:
        assert killed_by(build_mutant(SOURCE, tmp, 99)) is None
