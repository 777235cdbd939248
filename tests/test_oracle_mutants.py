"""Planted mistakes in copies of the oracle must each fail at least one pin (CPU only).

Each mutant is the oracle's C source with one plausible mistake substituted in
(a swapped nibble, a wrong shift or index, a dropped term, a flipped sign, a
changed tie rule), compiled into a temporary library; the real oracle is never
modified.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    "scale_min_swapped": ("int scale = scales[sb] & 0xF;", "int scale = scales[sb] >> 4;"),
    "shift_by_half": ("(qs[32 * h + l] >> (2 * j))", "(qs[32 * h + l] >> (2 * h))"),
    "byte_stride_16": ("(qs[32 * h + l] >> (2 * j))", "(qs[16 * h + l % 16] >> (2 * j))"),
    "subblock_by_32": ("int sb = i / 16;", "int sb = i / 32;"),
    "min_term_dropped": ("w[i] = d * scale * q - dmin * mn;", "w[i] = d * scale * q;"),
    "min_sign_flipped": ("w[i] = d * scale * q - dmin * mn;", "w[i] = d * scale * q + dmin * mn;"),
    "d_dmin_swapped": ("double d = ora_f16_to_double((uint16_t)(blk[80] | (blk[81] << 8)));",
                       "double d = ora_f16_to_double((uint16_t)(blk[82] | (blk[83] << 8)));"),
    "d_big_endian": ("double d = ora_f16_to_double((uint16_t)(blk[80] | (blk[81] << 8)));",
                     "double d = ora_f16_to_double((uint16_t)(blk[81] | (blk[80] << 8)));"),
    "softplus_naive_sign": ("return fmax(l, 0.0) + log1p(exp(-fabs(l)));",
                            "return fmax(l, 0.0) + log1p(exp(fabs(l)));"),
    "score_no_sqrt": ("return sqrt(ora_softplus(l));", "return ora_softplus(l);"),
    "ties_to_higher": ("(best < 0 || lg[e] > lg[best])", "(best < 0 || lg[e] >= lg[best])"),
    "weights_unnormalised": ("wts[j] = ssum > 0.0 ? s[j] / ssum : 1.0 / k;", "wts[j] = s[j];"),
    "bias_dropped": ("        acc += (double)*bias_e;", "        acc += 0.0;"),
    "silu_sign": ("return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));"),
    "swiglu_swapped": ("h[r] = ora_silu(g) * u;\n        if (g_out)", "h[r] = g * ora_silu(u);\n        if (g_out)"),
    "down_uses_gate_rowlen": ("o_out[c] = ora_q2k_row_dot(down + c * row_d, I, h);",
                              "o_out[c] = ora_q2k_row_dot(down + c * row_d / 2, I, h);"),
    "perm_fill_preinc": ("int pos = offsets[e] + fill[e]++;", "int pos = offsets[e] + ++fill[e] - (fill[e] > 1);"),
    "shared_dropped": ("                yt[c] += s[c];\n        }\n        if (idx_out)",
                       "                yt[c] += 0.0 * s[c];\n        }\n        if (idx_out)"),
    "renorm_no_eps_mean": ("double denom = sqrt(ss / H + 1e-6);", "double denom = sqrt(ss + 1e-6);"),
    "bf16_truncates": ("double r = nearbyint(ldexp(m, 8));", "double r = trunc(ldexp(m, 8));"),
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("mutants")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, mutant_dir):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "ds4moe_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, "mutation anchor not found: " + name
    msrc = src.replace(old, new, 1)
    cpath = os.path.join(str(mutant_dir), name + ".c")
    with open(cpath, "w") as f:
        f.write(msrc)
    so = oracle.build(force=True, src=cpath, out=os.path.join(str(mutant_dir), name + ".so"))
    mo = oracle.Oracle(oracle.load(so))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mo)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, "no pin caught the planted mistake " + name
