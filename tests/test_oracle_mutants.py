"""Plant plausible mistakes in copies of the oracle's C source (on the CPU) and
check that at least one pin catches each: a dropped term, a wrong sign or
index, a transposed operand, a wrong rounding rule, a wrong stride."""
import os
import shutil
import subprocess

import pytest

import oracle
import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "ep_oracle.c")

MUTANTS = {
    "destpe_modulo": ("if (e / nEpr != pe) continue;", "if (e % W != pe) continue;"),
    "weight_sum_dropped_term": ("if (c->useWeights) s = s + topk_w[g * k + j];",
                                "if (c->useWeights) s = topk_w[g * k + j];"),
    "unweighted_not_one": ("if (!c->useWeights) s = 1.0f;", "if (!c->useWeights) s = 0.0f + s;"),
    "meta_rank_token_swapped": ("meta[0] = (int32_t)r;\n                meta[1] = (int32_t)t;",
                                "meta[0] = (int32_t)t;\n                meta[1] = (int32_t)r;"),
    "local_id_sign": ("(int32_t)(e - pe * nEpr)", "(int32_t)(pe * nEpr - e)"),
    "masked_minus_one_routed": ("if (e < 0) continue;", "if (e < -1) continue;"),
    "slot_order_token_major": (
        "for (int64_t r = 0; r < W; ++r) {\n            for (int64_t t = 0; t < T; ++t) {",
        "for (int64_t t = 0; t < T; ++t) {\n            for (int64_t r = 0; r < W; ++r) {"),
    "combine_drops_accumulator": ("acc[i] = fmaf(w, bf16_to_f32(row[i]), acc[i]);",
                                  "acc[i] = fmaf(w, bf16_to_f32(row[i]), 0.0f);"),
    "combine_unfused": ("acc[i] = fmaf(w, bf16_to_f32(row[i]), acc[i]);",
                        "acc[i] = acc[i] + w * bf16_to_f32(row[i]);"),
    "combine_ignores_weight": ("acc[i] = fmaf(w, bf16_to_f32(row[i]), acc[i]);",
                               "acc[i] = fmaf(1.0f, bf16_to_f32(row[i]), acc[i]);"),
    "combine_wrong_stride": ("const uint16_t *row = y + (pe * R + slot) * h;",
                             "const uint16_t *row = y + (pe * T + slot) * h;"),
    "round_ties_away": ("(lower == 0x8000u && (upper & 1u))", "(lower == 0x8000u)"),
    "round_truncate": ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))",
                       "if (0)"),
    "bf16_widen_shift": ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
    "fp32_payload_two_bytes": ("return c->dtype == DT_FP32 ? 4 : c->dtype == DT_BF16 ? 2 : 1;",
                               "return c->dtype == DT_FP32 ? 2 : c->dtype == DT_BF16 ? 2 : 1;"),
    "fp4x2_combine_not_unpacked": ("return c->dtype == DT_FP4X2 ? 2 * (int64_t)c->hiddenDim : c->hiddenDim;",
                                   "return c->hiddenDim;"),
    "fp32_combine_rounded_to_bf16": ("for (int64_t i = 0; i < h; ++i) outf[g * h + i] = acc[i];",
                                     "for (int64_t i = 0; i < h; ++i) outf[g * h + i] = bf16_to_f32(f32_to_bf16_rne(acc[i]));"),
    "scale_row_of_wrong_token": ("memcpy(recv_scales + (pe * R + slot) * scale_words, scales + g * scale_words,",
                                 "memcpy(recv_scales + (pe * R + slot) * scale_words, scales + t * scale_words,"),
    "count_not_stored": ("recv_count[pe] = (int32_t)n;", "recv_count[pe] = (int32_t)n - (pe == 0);"),
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, mutant_dir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    csrc = os.path.join(mutant_dir, f"{name}.c")
    so = os.path.join(mutant_dir, f"lib{name}.so")
    with open(csrc, "w") as f:
        f.write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                           "-fPIC", "-shared", "-o", so, csrc, "-lm"])
    lib = oracle.load_library(so)
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(lib=lib)
        except (AssertionError, ValueError, IndexError) as exc:  # noqa: PERF203
            caught.append((pin.__name__, type(exc).__name__))
    assert caught, f"no pin caught the planted mistake {name}"


def test_unmutated_copy_passes(mutant_dir):
    """Control: the same build route on the unmodified source passes every pin."""
    csrc = os.path.join(mutant_dir, "control.c")
    so = os.path.join(mutant_dir, "libcontrol.so")
    shutil.copy(SRC, csrc)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                           "-fPIC", "-shared", "-o", so, csrc, "-lm"])
    lib = oracle.load_library(so)
    for pin in P.ALL_PINS:
        pin(lib=lib)
