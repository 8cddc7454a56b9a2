"""The pins must catch plausible mistakes: each case below plants one slip in
a copy of the oracle's C source (on the CPU), builds it, and requires the pin
suite to fail against it."""
import os
import subprocess
import sys

import pytest

from oracle import oracle as O

MUTANTS = {
    "drop_zero_point": ("pvi[c] += 8 * (int64_t)colsum", "pvi[c] += 0 * (int64_t)colsum"),
    "swap_scale_index": ("qs[i / QK_BLOCK] * ks[n / QK_BLOCK]", "qs[n / QK_BLOCK] * ks[i / QK_BLOCK]"),
    "rope_sign": ("y[o + 2 * j] = a0 - a1;", "y[o + 2 * j] = a0 + a1;"),
    "interleaved_sign": ("z[o + 2 * j + 1] = b0 - b1;", "z[o + 2 * j + 1] = b0 + b1;"),
    "half_partner": ("float a = y[o + i], b = y[o + i + h];", "float a = y[o + i], b = y[o + h - 1 - i];"),
    "p_scale_16": ("nearbyintf(15.0f * P) - 8", "nearbyintf(16.0f * P) - 8"),
    "global_not_running_max": ("float m_new = m > tmax ? m : tmax;", "float m_new = tmax > m ? tmax : tmax;"),
    "rescale_sign": ("exp((double)m - (double)m_new)", "exp((double)m_new - (double)m)"),
    "qk_scale_8": ("float s = amax / 7.0f;", "float s = amax / 8.0f;"),
    "rope_freq": ("-(double)(2 * j) / (double)p->split[s]", "-(double)(j) / (double)p->split[s]"),
    "token_order": ("pos[1] = (n / p->W) % p->Hh;", "pos[1] = (n / p->Hh) % p->W;"),
    "v_scale_per_tensor": ("sv[c] = amax / 7.0f;", "sv[c] = (amax > sv[0] ? amax : sv[0]) / 7.0f;"),
    "softmax_scale": ("(float)(1.0 / sqrt((double)d))", "(float)(1.0 / (double)d)"),
    "normaliser_exact_p": ("Li += code + zp;", "Li += 15;"),
    "blocks_merge_sign": ("m01 = (float)(R[1] * ca - R[0] * sa)", "m01 = (float)(R[1] * ca + R[0] * sa)"),
    "blocks_half_transposed": ("r10 = (float)R[2], r11 = (float)R[3];", "r10 = (float)R[1], r11 = (float)R[3];"),
    "v_hadamard_not_undone": ("if (p->v_rot) hadamard_f64(orow, d);", "if (0) hadamard_f64(orow, d);"),
    "v_hadamard_f64_sign": ("                y[k + w] = u - t;", "                y[k + w] = t - u;"),
    "hadamard_sign": ("                y[k + h] = a - b;", "                y[k + h] = b - a;"),
    "hadamard_skips_stride_1": ("for (int h = 1; h < d; h <<= 1)", "for (int h = 2; h < d; h <<= 1)"),
    "p_sym_scale_8": ("nearbyintf(7.0f * P)", "nearbyintf(8.0f * P)"),
    "sym_keeps_zero_point": ("const int zp = quant_p == 2 ? 0 : 8;", "const int zp = 8;"),
    # the quantised path's exponent in log2 units
    "log2_scale_index": ("(float)acc_s * (kq * ks[n / QK_BLOCK])", "(float)acc_s * (kq * ks[i / QK_BLOCK])"),
    "exponent_scale_index": ("fmaf((float)S[n - n0], kq * ks[n / QK_BLOCK], -m_new)",
                             "fmaf((float)S[n - n0], kq * ks[n0 / QK_BLOCK], -m_new)"),
    "natural_not_log2": ("const float log2e_f = (float)M_LOG2E", "const float log2e_f = 1.0f"),
    "log2_softmax_scale": ("const float K_log2 = log2e_f / sqrt_d_f;", "const float K_log2 = log2e_f / (float)d;"),
    "exponent_drops_max": ("fmaf((float)S[n - n0], kq * ks[n / QK_BLOCK], -m_new)",
                           "fmaf((float)S[n - n0], kq * ks[n / QK_BLOCK], -m)"),
    "rescale_sign_log2": ("exp2((double)m - (double)m_new)", "exp2((double)m_new - (double)m)"),
    "p_weight_levels_16": ("const int levels = quant_p == 2 ? 7 : 15;", "const int levels = quant_p == 2 ? 7 : 16;"),
    "amb_weight_floor": ("    return (int)rint(v);", "    return (int)floor(v);"),
    "amb_window_absolute": ("*amb = dist <= v * ORC_EX2_REL;", "*amb = dist <= ORC_EX2_REL;"),
    "flip_same_side": ("return v >= (double)w ? w + 1 : w - 1;", "return v >= (double)w ? w - 1 : w + 1;"),
    "p_weight_floor": ("(int)rint((double)levels * exp2((double)x))", "(int)floor((double)levels * exp2((double)x))"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(O.SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    mlib = str(tmp_path / "libmutant.so")
    O.compile_oracle(str(msrc), mlib)
    env = dict(os.environ, RA_ORACLE_LIB=mlib)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(root, "tests", "test_oracle_pins.py")],
                       cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
