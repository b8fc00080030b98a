"""The oracle's pins catch plausible mistakes.  Each case plants one mistake
in a copy of the oracle's C source (on the CPU), builds it, and runs the pin
tests against it in a subprocess: at least one pin must fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "pa_oracle.c")

MUTANTS = {
    "gqa_modulo": ("int32_t h = j / group;", "int32_t h = j % num_kv_heads;"),
    "table_index_off_by_one": ("[(int64_t)s * max_blocks_per_seq + t / block_size]",
                               "[(int64_t)s * max_blocks_per_seq + (t + 1) / block_size]"),
    "block_offset_swapped": ("(blk * block_size + t % block_size) * num_kv_heads + h",
                             "(blk * block_size + t / block_size) * num_kv_heads + h"),
    "scale_dropped": ("z[t] = scale * acc;", "z[t] = acc;"),
    "k_and_v_swapped": ("acc += bf16_to_double(qr[d]) * kk[t * head_dim + d];",
                        "acc += bf16_to_double(qr[d]) * vv[t * head_dim + d];"),
    "softmax_sign": ("z[t] = exp(z[t] - zmax);", "z[t] = exp(zmax - z[t]);"),
    "last_token_dropped": ("        for (int64_t t = 0; t < n; ++t)\n                acc += z[t] * vv[t * head_dim + d];",
                           "        for (int64_t t = 0; t < n - 1; ++t)\n                acc += z[t] * vv[t * head_dim + d];"),
    "write_skips_slot_zero": ("if (slot < 0)\n            continue;", "if (slot <= 0)\n            continue;"),
    "write_k_into_v": ("v_cache[slot * row_elems + e] = v[i * row_elems + e];",
                       "v_cache[slot * row_elems + e] = k[i * row_elems + e];"),
    "copy_in_place_chain": ("    /* gather */", "    goto scatter_now;\n    /* gather */"),
    "copy_wrong_direction": ("k_cache[d * block_elems + e] = tmp[(2 * p) * block_elems + e];",
                             "k_cache[pairs[2 * p] * block_elems + e] = tmp[(2 * p) * block_elems + e];"),
    "attn_no_causal_mask": ("const int64_t visible = n - q_len + i + 1;", "const int64_t visible = n;"),
    "attn_top_left_causal": ("const int64_t visible = n - q_len + i + 1;", "const int64_t visible = i + 1;"),
    "attn_excludes_own_token": ("const int64_t visible = n - q_len + i + 1;", "const int64_t visible = n - q_len + i;"),
    "attn_rows_reversed": ("const uint16_t *qr = q + ((row0 + i) * num_q_heads + j) * head_dim;",
                           "const uint16_t *qr = q + ((row0 + q_len - 1 - i) * num_q_heads + j) * head_dim;"),
    "attn_gqa_modulo": ("for (int32_t j = h * group; j < (h + 1) * group; ++j) {",
                        "for (int32_t j = h; j < num_q_heads; j += num_kv_heads) {"),
    "e4m3_bias_8": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_ties_away": ("    if (r - x == 0.5 && fmod(r, 2.0) != 0.0)\n        r -= 1.0;", ""),
    "e4m3_no_saturation": ("    if (a >= 448.0)\n        return (uint8_t)(sign | 0x7E);", "    if (a >= 480.0)\n        return 0x7F;"),
    "fp8_write_multiplies": ("oracle_e4m3_from_float(kx / k_scale)", "oracle_e4m3_from_float(kx * k_scale)"),
    "fp8_v_scale_dropped": ("vv[t * head_dim + d] = oracle_e4m3_to_double(v_cache[row * head_dim + d]) * v_scale;",
                            "vv[t * head_dim + d] = oracle_e4m3_to_double(v_cache[row * head_dim + d]);"),
}
PINS = ["tests/test_oracle_decode.py", "tests/test_oracle_formulas.py", "tests/test_oracle_fp8.py",
        "tests/test_oracle_attention.py"]


def _build(name, tmp_path):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, name
    mutated = src.replace(old, new, 1)  # the first occurrence: the bf16 functions
    if name == "copy_in_place_chain":
        # read-modify-write pair by pair instead of reading all sources first
        mutated = mutated.replace("    /* scatter */", "scatter_now:\n    /* scatter */")
        mutated = mutated.replace(
            "k_cache[d * block_elems + e] = tmp[(2 * p) * block_elems + e];",
            "k_cache[d * block_elems + e] = k_cache[pairs[2 * p] * block_elems + e];")
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    so = _build(name, tmp_path)
    env = dict(os.environ, ORACLE_LIB=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"no pin failed for mutant {name}:\n{r.stdout[-2000:]}"


def test_unmutated_copy_passes(tmp_path):
    """Control: the same harness with the oracle as written passes."""
    c = tmp_path / "same.c"
    so = tmp_path / "same.so"
    c.write_text(open(SRC).read())
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS],
                       cwd=ROOT, env=dict(os.environ, ORACLE_LIB=str(so)), capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]
