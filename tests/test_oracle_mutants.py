"""Plant plausible mistakes in copies of the C oracle (CPU only) and require that
each copy fails at least one pin.  This shows the pins are strong enough that
the oracle cannot be wrong in one of these ways and still pass."""
import os
import shutil

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "sherry_ref.c")
HDR = os.path.join(os.path.dirname(oracle.__file__), "sherry_ref.h")

MUTANTS = {
    "tie_zeroes_last_index": ("if (a[i] < a[z]) z = i;", "if (a[i] <= a[z]) z = i;"),
    "negative_zero_is_negative": ("s[i] = (w[i] >= 0.0f) ? 1 : -1;", "s[i] = signbit(w[i]) ? -1 : 1;"),
    "d1_d2_swapped": ("*nibble = 4u * (unsigned)z + 2u * d1 + d2;", "*nibble = 4u * (unsigned)z + 2u * d2 + d1;"),
    "global_sign_from_second": ("unsigned G = (s[p[0]] < 0) ? 1u : 0u;", "unsigned G = (s[p[1]] < 0) ? 1u : 0u;"),
    "group_denominator_L": ("float D = (float)((double)group / 4.0 * 3.0);", "float D = (float)group;"),
    "channel_denominator_L": ("float D = (float)((double)K / 4.0 * 3.0);", "float D = (float)K;"),
    "tensor_denominator_L": ("double Dd = (double)L / 4.0 * 3.0;", "double Dd = (double)L;"),
    "no_max_one_clause": ("if (Dd < 1.0) Dd = 1.0;", ""),
    "sum_includes_zeroed": ("mag[i] = (i == z) ? 0.0f : a[i];", "mag[i] = a[i];"),
    "strided_tree": ("buf[i] = buf[2 * i] + buf[2 * i + 1];", "buf[i] = buf[i] + buf[h + i];"),
    "decode_d1_inverted": ("t[p[1]] = d1 ? -first : first;", "t[p[1]] = d1 ? first : -first;"),
    "scale_index_no_row": ("return n * (K / group) + k / group;", "return n + k / group;"),
    "linear_row_dropped": ("acc += (double)bf16_bits_to_f32(X[m * K + k]) * (double)wrow[k];",
                           "acc += (double)bf16_bits_to_f32(X[k]) * (double)wrow[k];"),
    "channel_sum_short": ("scales[n] = sherry_ref_pairsum(&mag[n * K], K) / D;",
                          "scales[n] = sherry_ref_pairsum(&mag[n * K], K - 32) / D;"),
    "bf16_round_half_up": ("u += 0x7FFFu + lsb;", "u += 0x8000u;"),
    "bf16_truncate": ("u += 0x7FFFu + lsb;", "u += 0u * lsb;"),
    "nibble_order_reversed": ("idx[n * words + b / 8] |= (uint32_t)nib << (4 * (b % 8));",
                              "idx[n * words + b / 8] |= (uint32_t)nib << (4 * (7 - b % 8));"),
    "sign_bit_order_reversed": ("sgn[n * words + b / 8] |= (uint8_t)(g << (b % 8));",
                                "sgn[n * words + b / 8] |= (uint8_t)(g << (7 - b % 8));"),
    "pad_with_one": ("buf[i] = (i < L) ? v[i] : 0.0f;", "buf[i] = (i < L) ? v[i] : 1.0f;"),
    "group_error_not_checked": ("(group % 32) != 0 || ", ""),
    "arenas_residual_unscaled": ("Y[m * N + n] = yt + (double)lambda * yw;", "Y[m * N + n] = yt + yw;"),
    "arenas_linear_schedule": ("return lambda0 * 0.5 * (1.0 + cos(3.14159265358979323846 * s / (double)total));",
                               "return lambda0 * (1.0 - s / (double)total);"),
    "tequila_dead_from_first_weight": ("const float dead = eps * wv[nib >> 2];", "const float dead = eps * wv[0];"),
    "tequila_sign_of_zero_positive": ("const double sx = (x > 0.0f) ? 1.0 : ((x < 0.0f) ? -1.0 : 0.0);",
                                      "const double sx = (x >= 0.0f) ? 1.0 : -1.0;"),
    "tequila_zero_position_low_bits": ("const unsigned z = (idx[n * words + b / 8] >> (4 * (b % 8) + 2)) & 3u;",
                                       "const unsigned z = (idx[n * words + b / 8] >> (4 * (b % 8))) & 3u;"),
    "fake_quant_zero_keeps_sign": ("sgn[n * K + 4 * b + i] = (int8_t)((i == z) ? 0 : ((wv[i] >= 0.0f) ? 1 : -1));",
                                   "sgn[n * K + 4 * b + i] = (int8_t)((wv[i] >= 0.0f) ? 1 : -1);"),
    "fake_quant_scale_from_next_domain": ("for (int64_t k = j * L; k < j * L + L; ++k) Wq[n * K + k] = (float)sgn[n * K + k] * a;",
                                          "for (int64_t k = j * L; k < j * L + L; ++k) Wq[n * K + (k + L) % K] = (float)sgn[n * K + (k + L) % K] * a;"),
    "fake_quant_bf16_truncated": ("if (Wb)\n        for (int64_t i = 0; i < N * K; ++i) Wb[i] = f32_to_bf16_rne(Wq[i]);",
                                  "if (Wb)\n        for (int64_t i = 0; i < N * K; ++i) Wb[i] = (uint16_t)(f32_to_bf16_rne(Wq[i]) & 0xFFFEu);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not unique"
    src = tmp_path / "sherry_ref.c"
    src.write_text(text.replace(old, new))
    shutil.copy(HDR, tmp_path / "sherry_ref.h")
    so = str(tmp_path / "libmutant.so")
    oracle.build(src=str(src), out=so, force=True)
    mutant = oracle.Oracle(oracle.load_so(so))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
