"""The oracle's pins catch plausible mistakes.

Each mutant is a copy of oracle/ep_oracle.c with one planted mistake -- a
dropped term, a wrong index, a transposed operand, a wrong rounding or
order.  The pin suite (tests/test_oracle.py) is run against every mutant
in a subprocess and must fail; against the unmodified oracle it must pass.
Mistakes are planted in the oracle only, on the CPU."""

import concurrent.futures
import os
import subprocess
import sys
import tempfile

import pytest

from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "bf16 ties away from even": ("(dropped == 0x8000u && (keep & 1u))", "(dropped == 0x8000u)"),
    "bf16 truncates": ("if (dropped > 0x8000u || (dropped == 0x8000u && (keep & 1u))) keep += 1u;", ""),
    "e4m3 overflow gives NaN": ("if (a >= 448.0f) return (uint8_t)(sign | 0x7E);",
                                "if (a >= 448.0f) return (uint8_t)(sign | 0x7F);"),
    "e4m3 truncates": ("float n = rintf(a / quantum);", "float n = floorf(a / quantum);"),
    "e4m3 subnormal edge": ("if (a < 0.015625f)", "if (a < 0.0078125f)"),
    "e4m3 sign dropped": ("uint8_t sign = signbit(v) ? 0x80 : 0x00;", "uint8_t sign = 0x00;"),
    "amax floor dropped": ("if (amax < AMAX_FLOOR) amax = AMAX_FLOOR;", ""),
    "scale transposed": ("*scale = amax / E4M3_MAX;", "*scale = E4M3_MAX / amax;"),
    "quantise divides by the scale": ("for (int i = 0; i < QBLOCK; ++i) q[i] = oracle_e4m3_encode(oracle_bf16_to_f32(x[i]) * inv);",
                                      "for (int i = 0; i < QBLOCK; ++i) q[i] = oracle_e4m3_encode(oracle_bf16_to_f32(x[i]) / *scale);"),
    "amax misses last value": ("for (int i = 0; i < QBLOCK; ++i) amax = fmaxf",
                               "for (int i = 0; i < QBLOCK - 1; ++i) amax = fmaxf"),
    "alignment rounds up one block too many": ("int32_t padded = (counts[e] + align - 1) / align * align;",
                                                "int32_t padded = (counts[e] + align) / align * align;"),
    "rows in reverse slot order": ("    for (int64_t s = 0; s < n; ++s) {\n        int32_t e = expert[s];\n        if (e < 0) { slot_map[s] = -1; continue; }",
                                   "    for (int64_t s = n - 1; s >= 0; --s) {\n        int32_t e = expert[s];\n        if (e < 0) { slot_map[s] = -1; continue; }"),
    "segments count slots": ("if (e >= 0 && e / per_seg == g) hit = 1;", "if (e >= 0 && e / per_seg == g) hit += 1;"),
    "bad index kept": ("if (e < -1 || e >= E) { flags |= 1u; e = -1; }", "if (e < -1 || e >= E) { flags |= 1u; e = 0; }"),
    "row weight from wrong slot": ("recv_topk_weights[row] = topk_weights ? topk_weights[s] : 0.0f;",
                                   "recv_topk_weights[row] = topk_weights ? topk_weights[s - s % k] : 0.0f;"),
    "padding not zeroed": ("memset((uint8_t*)recv_x + (size_t)row * row_bytes, 0, row_bytes);", ""),
    "scales go to the token's row": ("memcpy((uint8_t*)recv_scales + (size_t)row * scale_bytes, src_scales, scale_bytes);",
                                     "memcpy((uint8_t*)recv_scales + (size_t)t * scale_bytes, src_scales, scale_bytes);"),
    "combine sums in reverse order": ("            for (int32_t j = 0; j < k; ++j) {\n                if (sm[j] < 0) continue;",
                                      "            for (int32_t j = k - 1; j >= 0; --j) {\n                if (sm[j] < 0) continue;"),
    "combine weight of wrong slot": ("float w = weights ? weights[(int64_t)t * k + j] : 1.0f;",
                                     "float w = weights ? weights[(int64_t)t * k + (k - 1 - j)] : 1.0f;"),
    "combine rounds twice": ("acc = fmaf(w, oracle_bf16_to_f32(y[(size_t)sm[j] * H + h]), acc);",
                             "acc = w * oracle_bf16_to_f32(y[(size_t)sm[j] * H + h]) + acc;"),
    "combine truncates to bf16": ("out[(size_t)t * H + h] = oracle_f32_to_bf16(acc);",
                                  "{ uint32_t u; memcpy(&u, &acc, 4); out[(size_t)t * H + h] = (uint16_t)(u >> 16); }"),
    "backward drops the weight": ("grad_y[(size_t)row * H + h] = oracle_f32_to_bf16(w * gv);",
                                  "grad_y[(size_t)row * H + h] = oracle_f32_to_bf16(gv);"),
    "backward dot uses the token's own row": ("dot += (double)gv * (double)oracle_bf16_to_f32(y[(size_t)row * H + h]);",
                                              "dot += (double)gv * (double)oracle_bf16_to_f32(y[(size_t)t * H + h]);"),
    "backward padding not zeroed": ("if (recv_src[row] < 0) memset(grad_y + (size_t)row * H, 0, sizeof(uint16_t) * H);",
                                    "if (recv_src[row] < 0) {}"),
    "e2m1 ties away from even": ("int n = (int)rintf(a / quantum);", "int n = (int)floorf(a / quantum + 0.5f);"),
    "nvfp4 nibbles swapped": ("q[i / 2] = (uint8_t)(oracle_e2m1_encode(oracle_bf16_to_f32(x[i]) * inv) |\n                             (oracle_e2m1_encode(oracle_bf16_to_f32(x[i + 1]) * inv) << 4));",
                              "q[i / 2] = (uint8_t)(oracle_e2m1_encode(oracle_bf16_to_f32(x[i + 1]) * inv) |\n                             (oracle_e2m1_encode(oracle_bf16_to_f32(x[i]) * inv) << 4));"),
    "nvfp4 scale from amax / 4": ("*scale = oracle_e4m3_encode(amax / E2M1_MAX);", "*scale = oracle_e4m3_encode(amax / 4.0f);"),
    "nvfp4 divides by the unrounded scale": ("float inv = 1.0f / oracle_e4m3_decode(*scale);", "float inv = E2M1_MAX / amax;"),
    "fp8 combine drops the scale": ("const float v = oracle_e4m3_decode(yq[(size_t)r * H + h]) * ys[(size_t)r * B + h / 128];",
                                    "const float v = oracle_e4m3_decode(yq[(size_t)r * H + h]);"),
    "fp8 combine takes the wrong block's scale": ("ys[(size_t)r * B + h / 128]", "ys[(size_t)r * B + h % B]"),
    "fp8 combine sums in reverse order": ("            for (int32_t j = 0; j < k; ++j) {\n                const int32_t r = slot_map[(int64_t)t * k + j];",
                                          "            for (int32_t j = k - 1; j >= 0; --j) {\n                const int32_t r = slot_map[(int64_t)t * k + j];"),
    "fp8 combine rounds twice": ("sum = fmaf(wj, v, sum);", "sum = wj * v + sum;"),
    "weight gather ignores the slot map": ("(sm[j] >= 0 && recv_weights_in) ? recv_weights_in[sm[j]] : 0.0f;",
                                           "(sm[j] >= 0 && recv_weights_in) ? recv_weights_in[j] : 0.0f;"),
}


def _pins_pass(lib_path: str) -> bool:
    env = dict(os.environ, EP_ORACLE_LIB=lib_path, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle.py"), "-x", "-q",
                        "-p", "no:cacheprovider", "-m", "not gpu"], cwd=ROOT, env=env,
                       stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL, timeout=600)
    return r.returncode == 0


@pytest.fixture(scope="module")
def mutant_results():
    src = open(obuild.SRC).read()
    with tempfile.TemporaryDirectory() as d:
        libs = {}
        for i, (name, (old, new)) in enumerate(MUTANTS.items()):
            assert src.count(old) == 1, f"mutation site not unique or missing: {name}"
            p = os.path.join(d, f"m{i}.c")
            open(p, "w").write(src.replace(old, new))
            libs[name] = obuild.compile_to(p, os.path.join(d, f"m{i}.so"))
        libs["<unmodified>"] = obuild.compile_to(obuild.SRC, os.path.join(d, "orig.so"))
        with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
            res = dict(zip(libs, ex.map(_pins_pass, libs.values())))
    return res


def test_unmodified_oracle_passes_its_pins(mutant_results):
    assert mutant_results["<unmodified>"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant_results, name):
    assert not mutant_results[name], f"no pin caught: {name}"
