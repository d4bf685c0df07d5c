"""Plants plausible mistakes in copies of the oracle and checks that the pins catch each.

Every mutant is a text substitution applied to oracle.c, compiled with gcc
into a temporary library; the committed oracle is never touched.  Several
mutants change encoder and decoder together (a consistent misreading of the
format), which a plain round trip cannot see: the golden streams and the
independent numpy reader have to catch those.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# name -> list of (old, new, count) substitutions; count None = replace all occurrences
MUTANTS = {
    "tie_break_larger_value": [("(hist[u] == hist[v] && u < v)", "(hist[u] == hist[v] && u > v)", 1)],
    "least_frequent_first": [("if (hist[u] > hist[v] ||", "if (hist[u] < hist[v] ||", 1)],
    "codebook_of_14": [("#define ORC_CODES 15u", "#define ORC_CODES 14u", 1)],
    "nibble_order_swapped": [("(4 * (i % 2))", "(4 * (1 - i % 2))", None)],
    "sign_in_low_bit": [("(uint8_t)((s << 7) | m)", "(uint8_t)((m << 1) | s)", 1),
                        ("s = sm >> 7;", "s = sm & 1u;", 1),
                        ("m = sm & 0x7Fu;", "m = sm >> 1;", 1)],
    "block_of_2048": [("#define ORC_BLOCK 4096u", "#define ORC_BLOCK 2048u", 1)],
    "escape_payload_inverted": [("out[L.esc + k] = (uint8_t)e;", "out[L.esc + k] = (uint8_t)(e ^ 0xFFu);", 1),
                                ("e = comp[L.esc + k];", "e = comp[L.esc + k] ^ (exponent_values(dtype) - 1u);", 1)],
    "n_and_E_swapped": [("put_u64(out + 8, n);", "put_u64(out + 16, n);", 1),
                        ("put_u64(out + 16, E);", "put_u64(out + 8, E);", 1),
                        ("*n = get_u64(comp + 8);", "*n = get_u64(comp + 16);", 1),
                        ("*E = get_u64(comp + 16);", "*E = get_u64(comp + 8);", 1)],
    "align_128": [("return (x + 255u) / 256u * 256u;", "return (x + 127u) / 128u * 128u;", 1)],
    "e5m2_one_mantissa_bit": [("bits & 0x3u", "bits & 0x1u", 1)],
    "e5m2_exponent_shift": [("(bits >> 2) & 0x1Fu", "(bits >> 3) & 0x1Fu", 1)],
    "bf16_exponent_7_bits": [("(bits >> 7) & 0xFFu", "(bits >> 7) & 0x7Fu", 1)],
    "first_element_not_counted": [("hist[exponent_of(dtype, element_bits(dtype, in, i))] += 1;",
                                   "hist[exponent_of(dtype, element_bits(dtype, in, i))] += (i > 0);", 1)],
    "no_zero_fill": [("memset(out, 0, L.total);", "", 1)],
    "inclusive_offsets": [("if (i % ORC_BLOCK == 0) put_u32(out + 64 + 4 * (i / ORC_BLOCK), (uint32_t)k);",
                           "if (i % ORC_BLOCK == 0 && i > 0) put_u32(out + 64 + 4 * (i / ORC_BLOCK - 1), (uint32_t)k);", 1),
                          ("put_u32(out + 64 + 4 * L.nb, (uint32_t)k);",
                           "put_u32(out + 64 + 4 * (L.nb ? L.nb - 1 : 0), (uint32_t)k);", 1),
                          ("if (i % ORC_BLOCK == 0 && get_u32(comp + 64 + 4 * (i / ORC_BLOCK)) != k)",
                           "if (0)", 1),
                          ("if (get_u32(comp + 64 + 4 * L.nb) != E) return ORC_ERR_CORRUPT;", "", 1)],
    "escape_counter_not_advanced": [("            k++;\n        }\n    }\n    put_u32", "        }\n    }\n    put_u32", 1)],
    "table_one_entry_short": [("64u + 4u * (L.nb + 1u)", "64u + 4u * L.nb", 1)],
    "given_codebook_duplicates_accepted": [("if (cb[d] == cb[c]) return -ORC_ERR_ARG;", "(void)d;", 1)],
    "given_codebook_replaced_by_own": [
        ("    uint64_t E = 0;\n    uint64_t nb = ceil_div(n, ORC_BLOCK);",
         "    uint64_t own_h[256];\n    uint8_t own_cb2[ORC_CODES];\n"
         "    orc_histogram(dtype, in, n, own_h);\n    orc_codebook(dtype, own_h, own_cb2);\n    cb = own_cb2;\n"
         "    uint64_t E = 0;\n    uint64_t nb = ceil_div(n, ORC_BLOCK);", 1)],
    # raw blocks
    "raw_threshold_strict": [("return escapes >= raw_block_bytes(dtype, m);",
                              "return escapes > raw_block_bytes(dtype, m);", 1)],
    "raw_blocks_never_taken": [("    if (!(flags & ORC_FLAG_RAW_BLOCKS)) return 0;\n", "    return 0;\n", 1)],
    "raw_flag_not_written": [("out[39] = (uint8_t)flags;", "out[39] = 0;", 1)],
    "raw_high_nibbles_swapped": [("(4 * (j % 2))", "(4 * (1 - j % 2))", None)],
    "raw_e5m2_bitmap_msb_first": [("(j % 8)", "(7 - j % 8)", None)],
    "raw_low_bits_shifted": [("unsigned c = raw ? (e & 0xFu) : code_of(cb, e);",
                              "unsigned c = raw ? ((e >> 1) & 0xFu) : code_of(cb, e);", 1),
                             ("e = (high << 4) | c;", "e = (high << 4) | (c << 1);", 1)],
    "raw_block_bytes_bf16_quarter": [("return dtype == ORC_BF16 ? ceil_div(m, 2) : ceil_div(m, 8);",
                                      "return dtype == ORC_BF16 ? ceil_div(m, 4) : ceil_div(m, 8);", 1)],
}


def _build_mutant(name, tmp_path):
    src = open(SRC).read()
    for old, new, count in MUTANTS[name]:
        found = src.count(old)
        assert found >= 1, "mutation %s no longer applies: %r not in oracle.c" % (name, old)
        src = src.replace(old, new) if count is None else src.replace(old, new, count)
    c = tmp_path / ("%s.c" % name)
    so = tmp_path / ("%s.so" % name)
    c.write_text(src)
    subprocess.run(["gcc", "-O2", "-std=c11", "-w", "-shared", "-fPIC", "-o", str(so), str(c)], check=True)
    return oracle.Oracle(str(so))


def _pins_fail(orc):
    failures = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, IndexError):
            failures.append(pin.__name__)
    return failures


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    orc = _build_mutant(name, tmp_path)
    failures = _pins_fail(orc)
    assert failures, "mutant %s passed every pin" % name


def test_unmutated_copy_passes(tmp_path):
    src = open(SRC).read()
    c = tmp_path / "same.c"
    so = tmp_path / "same.so"
    c.write_text(src)
    subprocess.run(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", str(so), str(c)], check=True)
    assert _pins_fail(oracle.Oracle(str(so))) == []
