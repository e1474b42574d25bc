"""Planted mistakes: each mutant is oracle.cpp with one plausible error (a
dropped term, a wrong sign, a wrong index or partner, a transposed operand, a
wrong rounding rule). Each is built on the CPU into a temporary library and
must fail at least one pin. This shows the pins bite, not only that the real
oracle passes them."""

import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as obuild
import pins

MUTANTS = {
    "dropped_term": ("for (int q = first + 1; q < first + count; ++q)",
                     "for (int q = first + 2; q < first + count; ++q)"),
    "descending_order": (
        "float acc = E::widen(in_ptr<E>(in, first)[i]);\n"
        "    for (int q = first + 1; q < first + count; ++q) acc = add32(acc, E::widen(in_ptr<E>(in, q)[i]));",
        "float acc = E::widen(in_ptr<E>(in, first + count - 1)[i]);\n"
        "    for (int q = first + count - 2; q >= first; --q) acc = add32(acc, E::widen(in_ptr<E>(in, q)[i]));"),
    "subtract": ("acc = add32(acc, E::widen(in_ptr<E>(in, q)[i]));",
                 "acc = add32(acc, -E::widen(in_ptr<E>(in, q)[i]));"),
    "round_half_away": ("u += 0x7FFFu + keep_lsb;", "u += 0x8000u + 0u * keep_lsb;"),
    "truncate": ("u += 0x7FFFu + keep_lsb;", "u += 0u * keep_lsb;"),
    "widen_shift": ("static_cast<uint32_t>(h) << 16", "static_cast<uint32_t>(h) << 15"),
    "rd_cyclic_partner": ("const int q = p ^ dist;", "const int q = (p + dist) % ranks;"),
    "rd_in_place": ("next[p][i] = E::narrow(add32(E::widen(v[p][i]), E::widen(v[q][i])));",
                    "v[p][i] = E::narrow(add32(E::widen(v[p][i]), E::widen(v[q][i])));"),
    "rd_dropped_step": ("for (int dist = 1; dist < ranks; dist <<= 1)",
                        "for (int dist = 1; 2 * dist < ranks; dist <<= 1)"),
    "twostage_write_owner_only": ("for (int r = 0; r < P; ++r) out_ptr<E>(out, r)[i] = v;",
                                  "out_ptr<E>(out, c)[i] = v;"),
    "hier_interleaved_groups": ("part[g * L + l][i] = reduce_ranks<E>(in, g * L, L, i);",
                                "part[g * L + l][i] = reduce_ranks<E>(in, g, L, i);"),
    "twostage_pull_wrong_owner": ("if (c == r) continue;", "if (c != r) continue;"),
    "all_gather_transposed": ("out_ptr<E>(out, p)[c * m + j] = in_ptr<E>(in, c)[j];",
                              "out_ptr<E>(out, p)[j * P + c] = in_ptr<E>(in, c)[j];"),
    "reduce_scatter_strided": ("reduce_ranks<E>(in, 0, P, p * m + j);", "reduce_ranks<E>(in, 0, P, j * P + p);"),
    "fp64_scale_signed": ("a += x < 0 ? -x : x;", "a += x;"),
    "half_round_half_away": ("if (rest > 0x1000u || (rest == 0x1000u && (keep & 1u))) keep += 1;",
                             "if (rest >= 0x1000u) keep += 1;"),
    "half_subnormal_truncate": ("if (rest > 0.5f || (rest == 0.5f && (i & 1u))) i += 1;",
                                "if (rest > 2.0f) i += 1;"),
    "fp32wire_hier_rounds_group_sum": (
        "part[g * L + l][i] = reduce_ranks_f32<E>(in, g * L, L, i);",
        "part[g * L + l][i] = E::widen(reduce_ranks<E>(in, g * L, L, i));"),
    "half_widen_bias": ("return bits_to_f32(sign | ((exp + 112u) << 23) | (frac << 13));",
                        "return bits_to_f32(sign | ((exp + 111u) << 23) | (frac << 13));"),
    "e4m3_round_half_away": ("if (frac > 0.5f || (frac == 0.5f && std::fmod(r, 2.0f) != 0.0f)) r += 1.0f;",
                             "if (frac >= 0.5f) r += 1.0f;"),
    "e4m3_truncate": ("if (frac > 0.5f || (frac == 0.5f && std::fmod(r, 2.0f) != 0.0f)) r += 1.0f;",
                      "if (frac > 2.0f) r += 1.0f;"),
    "e4m3_flush_subnormals": ("ulp = 0.001953125f;   /* 2^-9 */", "ulp = 0.015625f;"),
    "e4m3_no_saturation": ("if (q > 448.0f) q = 448.0f;", ""),
    "fp8_scale_fnuz_max": ("volatile float s = amax / 448.0f;", "volatile float s = amax / 240.0f;"),
    "fp8_amax_signed": ("const float a = x[i] < 0.0f ? -x[i] : x[i];\n        if (a > amax) amax = a;",
                        "const float a = x[i];\n        if (a > amax) amax = a;"),
    "fp8_groups_of_4": ("for (int64_t g = 0; g < n; g += 8) fp8_group_qdq(v.data() + g, static_cast<int>(n - g < 8 ? n - g : 8));",
                        "for (int64_t g = 0; g < n; g += 4) fp8_group_qdq(v.data() + g, static_cast<int>(n - g < 4 ? n - g : 4));"),
    "twostage_fp8_single_wire": ("    fp8_wire(sum);\n", ""),
}


def _build_mutant(name, tmpdir):
    src = open(obuild.SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation anchor for {name} not found in oracle.cpp"
    src = src.replace(old, new)
    cpp = os.path.join(tmpdir, f"{name}.cpp")
    lib = os.path.join(tmpdir, f"lib{name}.so")
    with open(cpp, "w") as f:
        f.write(src)
    cmd = ["g++", *obuild.FLAGS, "-w", "-o", lib, cpp]
    subprocess.run(cmd, check=True, capture_output=True)
    return oracle.Oracle(lib)


# Smaller integer sweep for mutants, to keep the CPU suite fast.
def _pins_for_mutants():
    out = []
    for p in pins.ALL_PINS:
        if p is pins.pin_integer_sums:
            out.append(lambda o: pins.pin_integer_sums(o, n_values=(1, 3, 8, 9, 17), P_values=(2, 3, 4, 8, 32)))
        else:
            out.append(p)
    return out


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    with tempfile.TemporaryDirectory() as d:
        o = _build_mutant(name, d)
        failures = 0
        for pin in _pins_for_mutants():
            try:
                pin(o)
            except (AssertionError, ValueError):
                failures += 1
        assert failures > 0, f"mutant {name} passed every pin"
