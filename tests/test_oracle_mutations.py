"""Plants plausible mistakes in copies of the C oracle and checks that the pins in
test_oracle_pins.py, test_oracle_block_pins.py, test_oracle_mods_pins.py,
test_oracle_bwd_pins.py, test_oracle_block_bwd_pins.py and test_oracle_fp8_pins.py catch every one (each mutant must fail at least one pin).
Everything runs on the CPU against a temporary build; the real oracle is untouched.
Mutants that leave the mathematics unchanged (e.g. dropping the fully-masked guard,
which still yields p = 0 and log 0 = -inf) are not listed: no test could tell them apart."""
import os
import subprocess
import tempfile

import pytest
import torch

import oracle
import tests.test_oracle_block_bwd_pins as bbpins
import tests.test_oracle_block_pins as bpins
import tests.test_oracle_bwd_pins as bwpins
import tests.test_oracle_fp8_pins as f8pins
import tests.test_oracle_mods_pins as mpins
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "flex_oracle.c")

# (name, text in flex_oracle.c, replacement)
MUTANTS = [
    ("scale dropped", "  double s = J->scale * dot;\n  if (J->score_mod", "  double s = dot;\n  if (J->score_mod"),
    ("scale applied after alibi", "  double s = J->scale * dot;\n  if (J->score_mod == OR_SCORE_ALIBI) s += slope * (double)(j - i);",
     "  double s = dot;\n  if (J->score_mod == OR_SCORE_ALIBI) s += slope * (double)(j - i);\n  s *= J->scale;"),
    ("alibi sign", "s += slope * (double)(j - i);", "s += slope * (double)(i - j);"),
    ("alibi slope index", "pow(2.0, -8.0 * (double)(h + 1) / (double)H)", "pow(2.0, -8.0 * (double)h / (double)H)"),
    ("causal strict", "case OR_MASK_CAUSAL: return j <= i;", "case OR_MASK_CAUSAL: return j < i;"),
    ("window off by one", "(i - j < (int64_t)window)", "(i - j <= (int64_t)window)"),
    ("window not causal", "return (j <= i) && (i - j < (int64_t)window);", "return (i - j < (int64_t)window);"),
    ("offset sign", "return j <= i + (int64_t)offset;", "return j <= i - (int64_t)offset;"),
    ("GQA modulo mapping", "  int hk = h / G;\n  return hk;", "  int hk = h % J->Hkv;\n  return hk;"),
    ("LSE in base 2", "  J->lse[r] = M + log(l);\n}\n\nstatic void* fwd_worker", "  J->lse[r] = M + log2(l);\n}\n\nstatic void* fwd_worker"),
    ("K used for V", "o[d] += p * elem(J->v, kvbase + j * D + d, J->dtype);", "o[d] += p * elem(J->k, kvbase + j * D + d, J->dtype);"),
    ("Q index transposed", "elem(J->q, qbase + d, J->dtype) * elem(J->k, kvbase + j * D + d, J->dtype)",
     "elem(J->q, qbase + d, J->dtype) * elem(J->k, kvbase + d * J->Skv + j, J->dtype)"),
    ("decode mask scaled", "    double s = J->scale * dot;\n    if (J->mask) s += elem(J->mask, r * (int64_t)J->cap + j, J->mask_dtype);",
     "    double s = dot;\n    if (J->mask) s += elem(J->mask, r * (int64_t)J->cap + j, J->mask_dtype);\n    s *= J->scale;"),
    ("decode drops last key", "  int64_t L = J->kv_len[b];", "  int64_t L = J->kv_len[b] > 0 ? J->kv_len[b] - 1 : 0;"),
    ("decode head mapping", "  int hk = h / (J->H / J->Hkv);", "  int hk = h % J->Hkv;"),
    ("fully masked row LSE 0", "    J->lse[r] = -INFINITY;\n    if (J->probs)", "    J->lse[r] = 0.0;\n    if (J->probs)"),
    ("decode empty row LSE 0", "  if (M == -INFINITY) {   /* kv_len == 0 or every position masked */\n    J->lse[r] = -INFINITY;",
     "  if (M == -INFINITY) {   /* kv_len == 0 or every position masked */\n    J->lse[r] = 0.0;"),
    ("tile classes swapped", "(kept == total ? 1 : 2)", "(kept == total ? 2 : 1)"),
    ("tile ignores pad", "if (j < Skv && keep_rule(", "if (keep_rule("),
    ("block: full list ignored", "  if (block_listed(L->full_num, L->full_idx, tile_row, L->max_blocks, u)) return 1;\n", ""),
    ("block: partial skips mask_mod", "u)) return keep_rule(mask_mod, window, offset, C, b, i, j);", "u)) return 1;"),
    ("block: partial beats full",
     "  if (block_listed(L->full_num, L->full_idx, tile_row, L->max_blocks, u)) return 1;\n  if (block_listed(L->kv_num, L->kv_idx, tile_row, L->max_blocks, u)) return keep_rule(mask_mod, window, offset, C, b, i, j);",
     "  if (block_listed(L->kv_num, L->kv_idx, tile_row, L->max_blocks, u)) return keep_rule(mask_mod, window, offset, C, b, i, j);\n  if (block_listed(L->full_num, L->full_idx, tile_row, L->max_blocks, u)) return 1;"),
    ("block: query tile from BN", "int64_t tile_row = bh * L->n_qtiles + i / L->BM;", "int64_t tile_row = bh * L->n_qtiles + i / L->BN;"),
    ("document end inclusive", "pos < (int64_t)off[d + 1]) return d;", "pos <= (int64_t)off[d + 1]) return d;"),
    ("document causal ignored", "return mask_mod == OR_MASK_DOC || j <= i;", "return 1;"),
    ("document keys use query boundaries", "const int32_t* okv = C->off_kv + (int64_t)b", "const int32_t* okv = C->off_q + (int64_t)b"),
    ("document of batch 0 for every batch", "const int32_t* oq = C->off_q + (int64_t)b * (C->n_docs + 1);",
     "const int32_t* oq = C->off_q;"),
    ("slope table ignored", "slope = J->cap.slopes ? J->cap.slopes[h] : oracle_alibi_slope(h, J->H);",
     "slope = oracle_alibi_slope(h, J->H);"),
    ("bwd delta sign", "double ds = pij * (dp - delta);", "double ds = pij * (dp + delta);"),
    ("bwd dK without scale", "dk[d] += J->scale * ds * elem(J->q, qbase + d, J->dtype);", "dk[d] += ds * elem(J->q, qbase + d, J->dtype);"),
    ("bwd dV from dS", "dv[d] += pij * elem(W->dout, qbase + d, J->dtype);", "dv[d] += ds * elem(W->dout, qbase + d, J->dtype);"),
    ("bwd dQ from V", "dq[d] += J->scale * ds * elem(J->k, kvbase + j * D + d, J->dtype);",
     "dq[d] += J->scale * ds * elem(J->v, kvbase + j * D + d, J->dtype);"),
    ("bwd one head per group", "for (int hg = 0; hg < G; ++hg) {", "for (int hg = 0; hg < 1; ++hg) {"),
    ("bwd P unnormalised", "double pij = exp(score_ij(J, b, h, i, j) - W->M[srow]) / W->l[srow];",
     "double pij = exp(score_ij(J, b, h, i, j) - W->M[srow]);"),
    ("e4m3 exponent bias", "v = ldexp((double)(m + 8), e - 10);    /* (1 + m/8) * 2^(e-7) */",
     "v = ldexp((double)(m + 8), e - 11);    /* (1 + m/8) * 2^(e-7) */"),
    ("e4m3 subnormal scale", "v = ldexp((double)m, -9);              /* subnormal: m/8 * 2^-6 */",
     "v = ldexp((double)m, -10);              /* subnormal: m/8 * 2^-6 */"),
    ("bwd ignores the block mask", "  J->blk = blk;\n  W.dout = dout;", "  W.dout = dout;"),
    ("bf16 decoded as truncated", "  uint32_t u = ((uint32_t)b) << 16;", "  uint32_t u = ((uint32_t)(b & 0xFFF0)) << 16;"),
]

CHECKS = [
    (pins.test_no_mod_equals_torch_float64_softmax, {"dtype": torch.bfloat16}),
    (pins.test_no_mod_equals_torch_float64_softmax, {"dtype": torch.float16}),
    (pins.test_causal_equals_torch_masked_softmax, {}),
    (pins.test_two_keys_closed_form, {}),
    (pins.test_scale_then_alibi_order_and_slopes, {}),
    (pins.test_zero_query_counts, {"mask": "causal", "window": 0, "offset": 0}),
    (pins.test_zero_query_counts, {"mask": "sliding_window", "window": 5, "offset": 0}),
    (pins.test_zero_query_counts, {"mask": "kv_le_q_plus_offset", "window": 0, "offset": 3}),
    (pins.test_alibi_zero_query_closed_form, {"H": 4, "h": 3}),
    (pins.test_identities_between_masks, {}),
    (pins.test_probabilities_sum_to_one, {}),
    (pins.test_gqa_equals_repeated_kv, {}),
    (pins.test_alibi_row_shift, {}),
    (pins.test_cross_attention_fully_masked, {}),
    (pins.test_decode_equals_forward_single_row, {}),
    (pins.test_decode_mask_cutoff_equals_shorter_length, {}),
    (pins.test_decode_empty_and_all_masked, {}),
    (pins.test_decode_finite_mask_added_after_scale, {"L": 7}),
    (pins.test_tile_map_closed_forms, {}),
    (pins.test_mask_matrix_counts, {}),
    (bpins.test_block_sparse_equals_dense_masked_softmax, {"mask": "causal", "window": 0, "offset": 0, "score": "none"}),
    (bpins.test_block_sparse_equals_dense_masked_softmax, {"mask": "sliding_window", "window": 6, "offset": 0,
                                                            "score": "alibi"}),
    (bpins.test_full_block_beats_partial_and_ignores_mask_mod, {}),
    (bpins.test_every_block_full_equals_no_mask, {}),
    (bpins.test_empty_block_mask_gives_zero_rows, {}),
    (mpins.test_random_slope_table_equals_torch, {}),
    (mpins.test_document_masks_equal_torch, {"case": "packed", "causal": True}),
    (mpins.test_document_masks_equal_torch, {"case": "tail_unassigned", "causal": False}),
    (mpins.test_document_masks_equal_torch, {"case": "cross", "causal": False}),
    (mpins.test_document_mask_matrix_and_tile_map, {"causal": True}),
    (bwpins.test_bwd_equals_torch_autograd, {"mask": "causal", "window": 0, "offset": 0, "score": "alibi",
                                             "dtype": torch.bfloat16}),
    (bwpins.test_bwd_single_key_closed_form, {}),
    (bwpins.test_bwd_equals_finite_differences_of_forward, {}),
    (f8pins.test_e4m3_decode_matches_torch, {}),
    (bbpins.test_block_bwd_equals_autograd, {"mask": "causal", "window": 0, "offset": 0, "score": "alibi",
                                              "dtype": torch.bfloat16}),
]


def _caught(lib_path):
    oracle.use_library(lib_path)
    try:
        failed = []
        for fn, kw in CHECKS:
            try:
                fn(oracle_mod=oracle, **kw)
            except Exception:  # an assertion, NaN comparison, or rejected arguments
                failed.append(fn.__name__)
        return failed
    finally:
        oracle.use_library(None)


def test_pins_pass_on_the_real_oracle():
    oracle.build()
    assert _caught(oracle.build()) == []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_every_planted_mistake_fails_a_pin(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(lib), str(mutant), "-lm",
                           "-lpthread"])
    failed = _caught(str(lib))
    assert failed, f"no pin caught the mutant '{name}'"
