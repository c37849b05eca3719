"""Plant one plausible mistake at a time in a copy of the CPU oracle and check
that the pins catch it (each mutant must fail at least one pin).  The copies
are compiled into a temporary directory; the committed oracle is untouched."""
import json
import os
import subprocess
import sys
import tempfile

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ep_oracle.c")

# (name, exact text in ep_oracle.c, replacement, pin-name prefixes to run against the mutant)
PLANTS = [
    ("bf16_truncates", "u += 0x7FFFu + lsb;", "u += 0u * lsb;", "pin_bf16"),
    ("e4m3_ties_away", "int m = (int)nearbyintf(q);\n    if (m == 16)", "int m = (int)roundf(q);\n    if (m == 16)", "pin_e4m3"),
    ("e4m3_no_subnormal_round", "int m = (int)nearbyintf(q);\n        return", "int m = (int)q;\n        return", "pin_e4m3"),
    ("fp8_scale_447", "float scale = amax / 448.0f;", "float scale = amax / 447.0f;", "pin_fp8"),
    ("fp8_amax_skips_last_channel", "for (int32_t i = 0; i < 128; ++i) {\n            float v = fabsf(",
     "for (int32_t i = 0; i < 127; ++i) {\n            float v = fabsf(", "pin_fp8"),
    ("fp8_inv_not_clamped", "inv = FLT_MAX;", "inv = inv;", "pin_fp8"),
    ("layout_rank_modulo", "mask |= 1u << (uint32_t)(e / per_rank);\n            } else {",
     "mask |= 1u << (uint32_t)(e % R);\n            } else {", "pin_tc_layout"),
    ("layout_slot_off_by_one", "slot[(int64_t)t * K + k] = counts[e];", "slot[(int64_t)t * K + k] = counts[e] + (t > 3);", "pin_tc_layout"),
    ("layout_last_expert_dropped", "if (e >= 0 && e < E) {\n                slot",
     "if (e >= 0 && e < E - 1) {\n                slot", "pin_tc_layout"),
    ("padded_row_shift", "row = e * (int64_t)max_tokens + s;", "row = e * (int64_t)max_tokens + s + (e & 1);", "pin_tc_dispatch"),
    ("combine_reverse_k", "        for (int32_t k = 0; k < K; ++k) {\n            int64_t e = topk_idx[(int64_t)t * K + k];\n            int32_t s = slot[(int64_t)t * K + k];\n            int64_t row = pair_row(e, s, E, offsets, mode, max_tokens, num_y_rows);",
     "        for (int32_t k = K - 1; k >= 0; --k) {\n            int64_t e = topk_idx[(int64_t)t * K + k];\n            int32_t s = slot[(int64_t)t * K + k];\n            int64_t row = pair_row(e, s, E, offsets, mode, max_tokens, num_y_rows);", "pin_tc_combine"),
    ("combine_unfused", "acc[h] = fmaf(w, oracle_bf16_to_f32(y[row * H + h]), acc[h]);",
     "acc[h] = acc[h] + w * oracle_bf16_to_f32(y[row * H + h]);", "pin_tc_combine"),
    ("combine_drops_last_k", "            float w = topk_weights[(int64_t)t * K + k];",
     "            float w = topk_weights[(int64_t)t * K + k];\n            if (k == K - 1 && K > 1) continue;", "pin_tc_c"),
    ("combine_weight_of_next_k", "            float w = topk_weights[(int64_t)t * K + k];",
     "            float w = topk_weights[(int64_t)t * K + (k + 1) % K];", "pin_tc_c"),
    ("ec_rank_of_token", "mask[t] |= 1u << (uint32_t)(e / per_rank);", "mask[t] |= 1u << (uint32_t)(t % R);", "pin_ec_layout"),
    ("ec_slots_descending", "    for (int64_t s = 0; s < S; ++s) {\n        int32_t t = token_indices[s];\n        if (t >= 0 && t < T) {\n            token_slots",
     "    for (int64_t s = S - 1; s >= 0; --s) {\n        int32_t t = token_indices[s];\n        if (t >= 0 && t < T) {\n            token_slots", "pin_ec"),
    ("ec_combine_unfused", "acc[h] = fmaf(w, oracle_bf16_to_f32(y[s * H + h]), acc[h]);",
     "acc[h] = acc[h] + w * oracle_bf16_to_f32(y[s * H + h]);", "pin_ec"),
    ("ec_dispatch_wrong_row", "memcpy(recv + s * H, x + (int64_t)t * H", "memcpy(recv + s * H, x + (int64_t)((t + 1) % T) * H", "pin_ec_dispatch"),
    ("e5m2_ties_away", "int m = (int)nearbyintf(fr * 8.0f);", "int m = (int)roundf(fr * 8.0f);", "pin_e5m2"),
    ("e5m2_bias_16", "int code = ((unb + 15) << 2) | (m - 4);", "int code = ((unb + 16) << 2) | (m - 4);", "pin_e5m2"),
    ("e5m2_subnormal_truncates", "int m = (int)nearbyintf(ldexpf(a, 16));", "int m = (int)ldexpf(a, 16);", "pin_e5m2"),
    ("e2m1_ties_away", "int m = (int)nearbyintf(fr * 4.0f);", "int m = (int)roundf(fr * 4.0f);", "pin_e2m1"),
    ("e2m1_subnormal_truncates", "int m = (int)nearbyintf(ldexpf(a, 1));", "int m = (int)ldexpf(a, 1);", "pin_e2m1"),
    ("int8_truncates", "float r = nearbyintf(f);", "float r = truncf(f);", "pin_int8"),
    ("int8_clamp_low_128", "if (r < -127.0f)\n        r = -127.0f;", "if (r < -128.0f)\n        r = -128.0f;", "pin_int8"),
    ("int8_scale_128", "*scale = amax / 127.0f;", "*scale = amax / 128.0f;", "pin_int8"),
    ("fp8_pertoken_first_group_amax", "float amax = row_amax(xrow, hidden);\n    if (amax == 0.0f) {\n        *scale = 0.0f;\n        for (int32_t i = 0; i < hidden; ++i)\n            q[i] = 0x00;",
     "float amax = row_amax(xrow, hidden < 128 ? hidden : 128);\n    if (amax == 0.0f) {\n        *scale = 0.0f;\n        for (int32_t i = 0; i < hidden; ++i)\n            q[i] = 0x00;", "pin_fp8_pertoken"),
    ("mx_exp_off_by_one", "int32_t X = (ex - 1) - emax_elem;", "int32_t X = ex - emax_elem;", "pin_mx"),
    ("mx_no_low_clamp", "if (X < -127)\n        X = -127;", "if (X < -1000)\n        X = -127;", "pin_mx"),
    ("mx_e5m2_emax_16", "dtype == OR_MXFP8_E5M2 ? 15 : 2", "dtype == OR_MXFP8_E5M2 ? 16 : 2", "pin_mx"),
    ("mx_block_amax_of_16", "float amax = row_amax(xrow + g * 32, 32);", "float amax = row_amax(xrow + g * 32, 16);", "pin_mx"),
    ("fp4_nibbles_swapped", "if (h % 2 == 0)\n                    q[h / 2] = c;\n                else\n                    q[h / 2] = (uint8_t)(q[h / 2] | (c << 4));",
     "if (h % 2 == 0)\n                    q[h / 2] = (uint8_t)(c << 4);\n                else\n                    q[h / 2] = (uint8_t)(q[h / 2] | c);", "pin_mx"),
    ("rank_rows_by_token_descending", "    for (int32_t t = 0; t < T; ++t) {\n        for (int32_t r = 0; r < R; ++r) {\n            if (is_token_in_rank[(int64_t)t * R + r]) {",
     "    for (int32_t t = T - 1; t >= 0; --t) {\n        for (int32_t r = 0; r < R; ++r) {\n            if (is_token_in_rank[(int64_t)t * R + r]) {", "pin_rank"),
    ("rank_offsets_inclusive", "rank_offsets[r + 1] = rank_offsets[r] + count[r];", "rank_offsets[r + 1] = rank_offsets[r] + count[r] + (r == 0);", "pin_rank"),
    ("rank_local_id_global", "recv_topk_idx[row * K + k] = local ? e - (int64_t)r * per_rank : -1;",
     "recv_topk_idx[row * K + k] = local ? e : -1;", "pin_rank_dispatch"),
    ("rank_weight_of_foreign_expert", "recv_topk_weights[row * K + k] = local ? topk_weights[(int64_t)t * K + k] : 0.0f;",
     "recv_topk_weights[row * K + k] = topk_weights[(int64_t)t * K + k];", "pin_rank"),
    ("rank_combine_descending", "        for (int32_t r = 0; r < R; ++r) {\n            int64_t row = rank_row[(int64_t)t * R + r];\n            if (row < 0)\n                continue;\n            for (int32_t h = 0; h < H; ++h)\n                acc[h] = acc[h] +",
     "        for (int32_t r = R - 1; r >= 0; --r) {\n            int64_t row = rank_row[(int64_t)t * R + r];\n            if (row < 0)\n                continue;\n            for (int32_t h = 0; h < H; ++h)\n                acc[h] = acc[h] +", "pin_rank"),
    ("rank_combine_skips_last_rank", "            if (row < 0)\n                continue;\n            for (int32_t h = 0; h < H; ++h)\n                acc[h] = acc[h] +",
     "            if (row < 0 || (r == R - 1 && R > 1))\n                continue;\n            for (int32_t h = 0; h < H; ++h)\n                acc[h] = acc[h] +", "pin_rank"),
    ("quant_dispatch_scale_row_shift", "memcpy((uint8_t*)recv_scales + row * scale_bytes, srow",
     "memcpy((uint8_t*)recv_scales + (row / 2 * 2) * scale_bytes, srow", "pin_quant_dispatch"),
]


def _build_mutant(src_text, tmpdir, name):
    path_c = os.path.join(tmpdir, name + ".c")
    path_so = os.path.join(tmpdir, name + ".so")
    with open(path_c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", path_so,
                           path_c, "-lm"])
    return path_so


_RUNNER = r"""
import json, sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle, pins
oracle.use(oracle.load({so!r}))
failed = []
for pin in pins.ALL_PINS:
    if not pin.__name__.startswith({prefix!r}):
        continue
    try:
        pin(oracle)
    except Exception:  # an assertion, or a check that could not even run
        failed.append(pin.__name__)
print(json.dumps(failed))
"""


def _run_plant(plant, tmpdir):
    name, old, new, prefix = plant
    text = open(SRC).read()
    if text.count(old) < 1:
        return ("anchor-missing", None)
    mutated = text.replace(old, new)
    here = os.path.dirname(os.path.abspath(__file__))
    so = _build_mutant(mutated, tmpdir, name)
    # each mutant runs in a child process so a mutant that corrupts memory
    # cannot take the test session down with it
    code = _RUNNER.format(root=os.path.dirname(here), tests=here, so=so, prefix=prefix)
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    if res.returncode != 0:
        return ("crashed", res.stderr[-2000:])
    return ("ran", json.loads(res.stdout.strip().splitlines()[-1]))


@pytest.fixture(scope="module")
def plant_results(oracle_mod):
    from concurrent.futures import ThreadPoolExecutor

    with tempfile.TemporaryDirectory() as d:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            futs = {p[0]: ex.submit(_run_plant, p, d) for p in PLANTS}
            return {k: f.result() for k, f in futs.items()}


@pytest.mark.parametrize("plant", PLANTS, ids=[p[0] for p in PLANTS])
def test_planted_mistake_is_caught(plant_results, plant):
    status, detail = plant_results[plant[0]]
    assert status == "ran", (status, detail)
    assert detail, "no pin caught the planted mistake " + plant[0]
