"""Mutation check of the oracle's pins: each seeded mistake below, planted in a copy of oracle.c
(built into a temporary library, never the real one), must make at least one oracle test fail.

The mistakes are the plausible ones: a sign, an index, a dropped term, the wrong operand, the wrong
rounding or constant, a missing step of the append rule or of the copy. One planted mistake is
expected to survive: clamping INT8 codes at -128 instead of -127 cannot show, because every scale
is derived from an absmax, so |x / s| <= 127 holds for every value quantized with it.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from oracle import build as oracle_build  # noqa: E402

PIN_TESTS = ["tests/test_oracle_store.py", "tests/test_oracle_decode.py", "tests/test_oracle_copy.py",
             "tests/test_oracle_fp8.py", "tests/test_oracle_prefill.py"]
EXPECTED_SURVIVORS = {"clamp128"}

MUTANTS = {
    "zp_sign": ("((double)get_nibble(r, j) - (double)c->v_zp[meta])", "((double)get_nibble(r, j) + (double)c->v_zp[meta])"),
    "gqa_mod": ("const int g = h / G;", "const int g = h % H;"),
    "trunc": ("float r = rintf(x / s);   /* R1 */", "float r = truncf(x / s);"),
    "scale128": ("float s = m_new / 127.0f;", "float s = m_new / 128.0f;"),
    "no_smscale": ("z[t] = (double)softmax_scale * dot;", "z[t] = dot;"),
    "offset_idx": ("dequant(c, 0, block, g, t % bs, j)", "dequant(c, 0, block, g, t / bs, j)"),
    "zp_derive_sign": ("float z = rintf(-lo / s);", "float z = rintf(lo / s);"),
    "nibble_order": ("return (dim % 2 == 0) ? (byte & 0xF) : (byte >> 4);", "return (dim % 2 == 0) ? (byte >> 4) : (byte & 0xF);"),
    "no_requant_old": ("for (int i = 0; i < n_old; ++i) tile[i] = quant_sym(xh[i], s);", ""),
    "fit_sign": ("fits = (r <= 127.0f && r >= -127.0f);", "fits = (r <= 127.0f);"),
    "int4_range_no0": ("float lo_new = 0.0f, hi_new = 0.0f;", "float lo_new = 1e30f, hi_new = -1e30f;"),
    "v_uses_k": ("o[j] += w * dequant(c, 1, block, g, t % bs, j);", "o[j] += w * dequant(c, 0, block, g, t % bs, j);"),
    "clamp128": ("if (r < -127.0f) r = -127.0f; /* R4 */", "if (r < -128.0f) r = -128.0f;"),
    "vscale_kscale": ("double s = which_v ? (double)c->v_scale[meta] : (double)c->k_scale[meta];", "double s = (double)c->k_scale[meta];"),
    "asym_plus_zp_missing": ("float r = rintf(x / s + (float)zp);", "float r = rintf(x / s);"),
    "fp8_ties_odd": ("if (d < best_d || (d == best_d && (c & 1) == 0)) {", "if (d < best_d || (d == best_d && (c & 1) == 1)) {"),
    "fp8_ties_up": ("if (d < best_d || (d == best_d && (c & 1) == 0)) {", "if (d <= best_d) {"),
    "fp8_exp_bias": ("else v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */", "else v = ldexp((double)(8 + m), e - 9);"),
    "fp8_subnormal": ("if (e == 0) v = ldexp((double)m, -9);", "if (e == 0) v = ldexp((double)m, -10);"),
    "fp8_scale480": ("float s = m_new / 448.0f;", "float s = m_new / 480.0f;"),
    "fp8_fit_480": ("else fits = (fabsf(new_x[i] / s_old) <= 448.0f);", "else fits = (fabsf(new_x[i] / s_old) <= 480.0f);"),
    "fp8_no_requant_old": ("for (int i = 0; i < n_old; ++i) tile[i] = quant_fp8(xh[i], s);", ""),
    "fp8_sign": ("uint8_t sign = signbit(x) ? 0x80 : 0x00;", "uint8_t sign = 0x00;"),
    "prefill_causal_off_by_one": ("int L = context_lens[s] - q_len + i + 1; /* causal: positions 0 .. p */", "int L = context_lens[s] - q_len + i;"),
    "prefill_not_causal": ("int L = context_lens[s] - q_len + i + 1; /* causal: positions 0 .. p */", "int L = context_lens[s];"),
    "prefill_wrong_seq": ("while (s + 1 < num_seqs && cu_q_lens[s + 1] <= row) ++s;", "while (s + 1 < num_seqs && cu_q_lens[s + 1] < row) ++s;"),
    "copy_scales_missing": ("memcpy(c->k_scale + (size_t)dst * H, c->k_scale + (size_t)src * H, sizeof(float) * H);", ";"),
}


def _run_pins_against(name, a, b, src, tmp):
    c_path = os.path.join(tmp, f"{name}.c")
    so_path = os.path.join(tmp, f"{name}.so")
    with open(c_path, "w") as f:
        f.write(src.replace(a, b, 1))
    subprocess.run(["gcc", *oracle_build.FLAGS, "-I", os.path.join(ROOT, "oracle"), "-o", so_path, c_path, "-lm"],
                   check=True)
    env = dict(os.environ, PKV_ORACLE_LIB=so_path)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_TESTS],
                       cwd=ROOT, env=env, capture_output=True, text=True)
    return name, r.returncode != 0


def test_pins_catch_planted_mistakes():
    src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    for name, (a, _) in MUTANTS.items():
        assert a in src, f"mutant {name}: its target text is no longer in oracle.c"
    with tempfile.TemporaryDirectory() as tmp, cf.ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        killed = dict(ex.map(lambda kv: _run_pins_against(kv[0], *kv[1], src, tmp), MUTANTS.items()))
    survivors = {n for n, k in killed.items() if not k}
    assert survivors == EXPECTED_SURVIVORS, f"planted mistakes not caught: {sorted(survivors - EXPECTED_SURVIVORS)}"
