"""The pins reject planted mistakes in the oracle (CPU only).

Each case copies oracle/moe_oracle.c, plants one plausible mistake (a dropped
term, a wrong sign, bound or index, a swapped operand, a wrong order or
rounding), builds the copy with the oracle's own flags and runs the pin tests
named beside it against that library (MOE_ORACLE_LIB) in a child pytest. The
case passes when the child reports a failing test: some pin caught the mistake.
A control build of the unmodified source must pass the same pins, so that a
failure cannot come from the harness itself. Every planted mistake keeps all
memory accesses inside their buffers. The numpy exchange (oracle.ep_exchange)
is mutated the same way in a copy of its source, in this process.
"""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")
SRC = os.path.join(ORACLE_DIR, "moe_oracle.c")

ROUTE = ["tests/test_oracle_route.py"]
LAYOUT = ["tests/test_oracle_layout.py", "tests/test_golden.py"]
REROUTE = ["tests/test_oracle_reroute.py", "tests/test_golden.py"]
COMBINE = ["tests/test_oracle_permute_combine.py", "tests/test_golden.py"]
TP = ["tests/test_oracle_tp_fold.py"]
DEDUP = ["tests/test_oracle_dedup.py"]

# id, text in moe_oracle.c (must occur exactly once), replacement, pin files
MUTANTS = [
    ("bf16_round_half_up", "(b + 0x7FFFu + lsb) >> 16", "(b + 0x8000u) >> 16", COMBINE),
    ("bf16_truncate", "(b + 0x7FFFu + lsb) >> 16", "b >> 16", COMBINE),
    ("route_ties_to_higher_id", "if (best < 0 || l[e] > l[best])", "if (best < 0 || l[e] >= l[best])", ROUTE),
    ("route_softmax_drops_first_term", "for (int32_t e = 0; e < E; ++e)\n            s += exp",
     "for (int32_t e = 1; e < E; ++e)\n            s += exp", ROUTE),
    ("route_mask_inverted", "if (token_mask && token_mask[t])", "if (token_mask && !token_mask[t])", ROUTE),
    ("route_prob_of_wrong_expert", "pr[j] = (float)(exp((double)l[best] - m) / s);",
     "pr[j] = (float)(exp((double)l[j] - m) / s);", ROUTE),
    ("layout_ordinal_off_by_one_for_expert_0", "o->ordinal[a] = seen[q]++;",
     "o->ordinal[a] = ++seen[q] - 1 + (q == 0);", LAYOUT),
    ("layout_invalid_id_not_flagged", "            error = 1;\n", "", LAYOUT),
    ("layout_dropped_not_counted", "            ++dropped;\n", "", LAYOUT),
    ("layout_padded_counts_valid", "o->counters[ORC_PADDED] = (int32_t)(rows_max - kept);",
     "o->counters[ORC_PADDED] = (int32_t)(rows_max - valid);", LAYOUT),
    ("layout_rank_offsets_wrong_index", "o->rank_offsets[r] = o->expert_offsets[r * E_loc];",
     "o->rank_offsets[r] = o->expert_offsets[r];", LAYOUT),
    ("layout_row_slot_transposed", "o->row_slot[row] = (int32_t)(a % k);", "o->row_slot[row] = (int32_t)(a / k);",
     LAYOUT),
    ("layout_rows_not_aligned", "        while (rows % A != 0)\n            ++rows;\n", "", LAYOUT),
    ("layout_capacity_rows_from_counts",
     "int32_t rows = C > 0 ? oracle_local_capacity(p) : o->tokens_per_expert[e];",
     "int32_t rows = o->tokens_per_expert[e];", LAYOUT),
    ("layout_local_id_not_rebased", "o->local_topk[(int64_t)r * NK + a] = keep ? q - r * E_loc : -1;",
     "o->local_topk[(int64_t)r * NK + a] = keep ? q : -1;", LAYOUT),
    ("layout_row_prob_of_slot_zero", "o->row_prob[row] = topk_probs ? topk_probs[a] : 0.0f;",
     "o->row_prob[row] = topk_probs ? topk_probs[a - a % k] : 0.0f;", LAYOUT),
    ("reroute_odd_ordinals_to_master", "(o->placement[e] >= 0 && (lo % 2) == 1)",
     "(o->placement[e] >= 0 && (lo % 2) == 0)", REROUTE),
    ("reroute_hot_ties_to_higher_id", "if (!is_hot[c] && (e < 0 || o->counts_logical[c] > o->counts_logical[e]))",
     "if (!is_hot[c] && (e < 0 || o->counts_logical[c] >= o->counts_logical[e]))", REROUTE),
    ("reroute_most_loaded_rank", "(best < 0 || load[r] < load[best])", "(best < 0 || load[r] > load[best])", REROUTE),
    ("reroute_load_not_added_to_chosen_rank", "            load[best] += moved;\n", "", REROUTE),
    ("reroute_load_not_taken_from_home", "            load[home] -= moved;\n", "", REROUTE),
    ("permute_copies_next_token", "memcpy(send + (int64_t)row * H, hidden + t * H,",
     "memcpy(send + (int64_t)row * H, hidden + ((t + 1) % p->N) * H,", COMBINE),
    ("combine_slots_descending",
     "            for (int32_t j = 0; j < p->k; ++j) {\n                int32_t row = dest_row[t * p->k + j];\n"
     "                if (row < 0)\n                    continue;\n                float w = topk_probs ? topk_probs[t * p->k + j] : 1.0f;\n"
     "                acc = fmaf(w, oracle_f32_from_bf16(expert_out[(int64_t)row * H + h]), acc);\n            }\n"
     "            out[t * H + h]",
     "            for (int32_t j = p->k - 1; j >= 0; --j) {\n                int32_t row = dest_row[t * p->k + j];\n"
     "                if (row < 0)\n                    continue;\n                float w = topk_probs ? topk_probs[t * p->k + j] : 1.0f;\n"
     "                acc = fmaf(w, oracle_f32_from_bf16(expert_out[(int64_t)row * H + h]), acc);\n            }\n"
     "            out[t * H + h]", COMBINE),
    ("combine_unfused_multiply_add",
     "                acc = fmaf(w, oracle_f32_from_bf16(expert_out[(int64_t)row * H + h]), acc);\n            }\n"
     "            out[t * H + h]",
     "                acc = acc + w * oracle_f32_from_bf16(expert_out[(int64_t)row * H + h]);\n            }\n"
     "            out[t * H + h]", COMBINE),
    ("combine_weight_of_slot_zero",
     "                float w = topk_probs ? topk_probs[t * p->k + j] : 1.0f;\n"
     "                acc = fmaf(w, oracle_f32_from_bf16(expert_out[(int64_t)row * H + h]), acc);\n            }\n"
     "            out[t * H + h]",
     "                float w = topk_probs ? topk_probs[t * p->k] : 1.0f;\n"
     "                acc = fmaf(w, oracle_f32_from_bf16(expert_out[(int64_t)row * H + h]), acc);\n            }\n"
     "            out[t * H + h]", COMBINE),
    ("permute_backward_slots_descending",
     "            for (int32_t j = 0; j < p->k; ++j) {\n                int32_t row = dest_row[t * p->k + j];\n"
     "                if (row >= 0)\n                    acc = acc +",
     "            for (int32_t j = p->k - 1; j >= 0; --j) {\n                int32_t row = dest_row[t * p->k + j];\n"
     "                if (row >= 0)\n                    acc = acc +", COMBINE),
    ("combine_backward_grad_y_unweighted", "float prod = row_prob[row] * oracle_f32_from_bf16(",
     "float prod = 1.0f * oracle_f32_from_bf16(", COMBINE),
    ("combine_backward_grad_probs_wrong_token", "s += (double)oracle_f32_from_bf16(grad_out[t * H + h]) *",
     "s += (double)oracle_f32_from_bf16(grad_out[((t + 1) % p->N) * H + h]) *", COMBINE),
    ("tp_fold_ignores_peer", "o->ordinal[a] % T != p->tp_rank", "o->ordinal[a] % T != 0", TP),
    ("dedup_tokens_descending",
     "        for (int64_t t = 0; t < N; ++t) {\n            if (!o->is_token_in_rank[t * R + r]) {",
     "        for (int64_t t = N - 1; t >= 0; --t) {\n            if (!o->is_token_in_rank[t * R + r]) {", DEDUP),
    ("dedup_weight_of_slot_zero", "float w = topk_probs ? topk_probs[t * k + j] : 0.0f;",
     "float w = topk_probs ? topk_probs[t * k] : 0.0f;", DEDUP),
    ("dedup_multihot_not_set", "o->recv_routing_map[(int64_t)row * E_loc + local] = 1;",
     "o->recv_routing_map[(int64_t)row * E_loc + local] = 0;", DEDUP),
    ("dedup_partial_takes_next_rank_row", "if (d < rank_offsets[r] || d >= rank_offsets[r + 1])",
     "if (d < rank_offsets[r] || d > rank_offsets[r + 1])", DEDUP),
]


def _build(src_text, out_dir, name):
    c_path = os.path.join(out_dir, f"{name}.c")
    so_path = os.path.join(out_dir, f"lib{name}.so")
    with open(c_path, "w") as f:
        f.write(src_text)
    cmd = [os.environ.get("CC", "gcc"), "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-w", "-I", ORACLE_DIR, "-o", so_path, c_path, "-lm"]
    subprocess.run(cmd, check=True)
    return so_path


def _run_pins(so_path, files):
    env = dict(os.environ, MOE_ORACLE_LIB=so_path)
    cmd = [sys.executable, "-m", "pytest", *files, "-x", "-q", "-m", "not gpu", "-p", "no:cacheprovider"]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


def test_control_build_passes_the_pins(source, tmp_path):
    files = sorted({f for m in MUTANTS for f in m[3]})
    r = _run_pins(_build(source, str(tmp_path), "control"), files)
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_planted_mistake(source, tmp_path, mutant):
    name, old, new, files = mutant
    assert source.count(old) == 1, f"{name}: the planted text must occur exactly once"
    r = _run_pins(_build(source.replace(old, new), str(tmp_path), name), files)
    # 1 = some test failed; anything else (a crash, a collection error) is not a pin at work
    assert r.returncode == 1, f"{name}: the pins did not reject it (exit {r.returncode})\n{r.stdout[-2000:]}"


# The expert-parallel exchange of the oracle is numpy (oracle.ep_exchange): its
# planted mistakes are made in a copy of the function's source, and the exchange
# pins of tests/test_oracle_ep.py run in this process against the copy.
EP_MUTANTS = [
    ("ep_sources_descending", "            for s in range(S):", "            for s in reversed(range(S)):"),
    ("ep_experts_descending", "        for q in range(r * E_loc, (r + 1) * E_loc):",
     "        for q in reversed(range(r * E_loc, (r + 1) * E_loc)):"),
    ("ep_padding_rows_left_out",
     'lo, hi = int(layouts[s]["expert_offsets"][q]), int(layouts[s]["expert_offsets"][q + 1])',
     'lo = int(layouts[s]["expert_offsets"][q]); hi = lo + int(layouts[s]["tokens_per_expert"][q])'),
    ("ep_base_after_the_rows", "                base[s][q] = pos\n                blocks.append(sends[s][lo:hi])\n"
     "                pos += hi - lo\n",
     "                blocks.append(sends[s][lo:hi])\n                pos += hi - lo\n                base[s][q] = pos\n"),
    ("ep_expert_offsets_shifted", "            offs.append(pos)\n            for s in range(S):",
     "            for s in range(S):\n                offs.append(pos) if s == S - 1 else None"),
]


def _ep_variant(old=None, new=None):
    import inspect
    import textwrap
    import types

    import numpy as np

    import oracle

    src = textwrap.dedent(inspect.getsource(oracle.oracle.ep_exchange))
    if old is not None:
        assert src.count(old) == 1, "the planted text must occur exactly once"
        src = src.replace(old, new)
    ns = {"np": np}
    exec(compile(src, "<ep_exchange variant>", "exec"), ns)
    return types.SimpleNamespace(layout=oracle.layout, permute=oracle.permute, combine=oracle.combine,
                                 ep_exchange=ns["ep_exchange"])


def _ep_pins_fail(lib):
    import test_oracle_ep

    for case in test_oracle_ep.CASES:
        try:
            test_oracle_ep.test_exchange_delivers_every_kept_assignment_once(lib, case)
        except (AssertionError, ValueError, IndexError):  # a failed pin, as pytest would count it
            return True
    return False


def test_ep_control_passes_the_pins():
    assert not _ep_pins_fail(_ep_variant())


@pytest.mark.parametrize("mutant", EP_MUTANTS, ids=[m[0] for m in EP_MUTANTS])
def test_ep_pins_reject_planted_mistake(mutant):
    name, old, new = mutant
    assert _ep_pins_fail(_ep_variant(old, new)), f"{name}: the exchange pins did not reject it"
