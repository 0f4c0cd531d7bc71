"""Planted mistakes: each plausible slip in the oracle must fail one of its pins.

Every mutant is a one-line edit of a temporary copy of oracle/qsgd_oracle.c,
compiled on the CPU.  The battery below re-runs the pins (Philox known answers,
textbook omega codewords, omega round trip, hand-derived golden streams, the
decode-accumulate hand values, unbiasedness on a small sweep).
"""

import os
import shutil

import numpy as np
import pytest

import oracle as oracle_mod
from helpers import (bits_to_words, fixture_decoded, fixture_vector, load_kat,
                     load_omega_codewords, load_streams, words_to_bits)
import stats_common as sc

SRC = os.path.join(os.path.dirname(oracle_mod.__file__), "qsgd_oracle.c")

MUTANTS = {
    "philox_swap_hi_lo": ("uint32_t y1 = lo1;", "uint32_t y1 = hi1;"),
    "philox_no_key_bump": ("k1 += W1;", ""),
    "philox_wrong_multiplier_operand": ("(uint64_t)M1 * (uint64_t)x2", "(uint64_t)M1 * (uint64_t)x1"),
    "random_word_wrong_lane": ("return out[i % 4];", "return out[(i + 1) % 4];"),
    "uniform_wrong_shift": ("(float)(r >> 9) * 0x1p-23f", "(float)(r >> 8) * 0x1p-23f"),
    "omega_len_off_by_one": ("len += b;", "len += b - 1;"),
    "omega_groups_reversed": ("for (int g = ngroups - 1; g >= 0; --g) {", "for (int g = 0; g < ngroups; ++g) {"),
    "omega_get_group_width": ("for (uint64_t t = 0; t < value; ++t) {", "for (uint64_t t = 1; t < value; ++t) {"),
    "round_up_direction": ("if (u < p) k += 1;", "if (u > p) k += 1;"),
    "round_to_nearest": ("float l = floorf(t);", "float l = roundf(t);"),
    "scale_inverted": ("float sinv = (float)s / norm;", "float sinv = norm / (float)s;"),
    "l1_norm": ("sum += (double)v[i] * (double)v[i];", "sum += fabs((double)v[i]);"),
    "gap_origin_zero": ("int64_t prev = -1;\n    for (uint64_t i = 0; i < m && err == 0; ++i) {",
                        "int64_t prev = 0;\n    for (uint64_t i = 0; i < m && err == 0; ++i) {"),
    "gap_not_updated": ("prev = (int64_t)i;\n        uint32_t k", "uint32_t k"),
    "sign_inverted": ("put_bit(words, cap_words, pos, levels[i] < 0);",
                      "put_bit(words, cap_words, pos, levels[i] > 0);"),
    "fields_swapped": ("err |= qo_omega_put(words, cap_words, pos, gap);\n        err |= put_bit(words, cap_words, pos, levels[i] < 0);\n        err |= qo_omega_put(words, cap_words, pos, k);",
                       "err |= qo_omega_put(words, cap_words, pos, k);\n        err |= put_bit(words, cap_words, pos, levels[i] < 0);\n        err |= qo_omega_put(words, cap_words, pos, gap);"),
    "bit_order_lsb_first": ("if (bit) words[w] |= (uint32_t)1u << (31 - (unsigned)(*pos % 32));",
                            "if (bit) words[w] |= (uint32_t)1u << ((unsigned)(*pos % 32));"),
    "decode_scale_inverted": ("float scale = norm / (float)s;", "float scale = (float)s / norm;"),
    "decode_sign_dropped": ("if (q < 0) value = -value;", ""),
    "accumulate_overwrites": ("out[i] = out[i] + q[i];", "out[i] = q[i];"),
    "decode_index_not_advanced": ("idx += (int64_t)gap;", "idx += 1;"),
    # fixed-width b-bit variant
    "bbit_sign_in_low_bit": ("uint32_t code = ((levels[i] < 0 ? 1u : 0u) << (b - 1)) | k;",
                             "uint32_t code = (k << 1) | (levels[i] < 0 ? 1u : 0u);"),
    "bbit_levels_full_width": ("(1u << (b - 1)) - 1u : 0u;", "(1u << b) - 1u : 0u;"),
    "bbit_decode_sign_dropped": ("if (sign) value = -value;", ""),
    "bbit_decode_scale_inverted": ("float bscale = norm / (float)s;", "float bscale = (float)s / norm;"),
    "bbit_sign_on_zero_accepted": ("if (sign) bad = 1; /* a sign on a zero level: no encoder writes it */", ""),
    "bbit_accumulate_overwrites": ("out[i] += q[i];", "out[i] = q[i];"),
    # max-norm (QSGDinf) scale
    "maxnorm_drops_nan": ("if (isnan(v[i])) return NAN;", ""),
    "maxnorm_signed": ("if (fabsf(v[i]) > mx) mx = fabsf(v[i]);", "if (v[i] > mx) mx = v[i];"),
    # error feedback
    "ef_residual_sign": ("e[i] = q[i] != 0.0f ? p[i] - q[i] : p[i];", "e[i] = q[i] != 0.0f ? q[i] - p[i] : p[i];"),
    "ef_forgets_memory": ("p[i] = e[i] + g[i];", "p[i] = g[i];"),
    "ef_drops_unsent": ("e[i] = q[i] != 0.0f ? p[i] - q[i] : p[i];", "e[i] = q[i] != 0.0f ? p[i] - q[i] : 0.0f;"),
    # mean of K streams
    "mean_not_divided": ("if (qo_decode_accumulate(words, offsets, K, n, d, s, out, status) != 0) return -1;\n    for (uint64_t i = 0; i < n; ++i) out[i] = out[i] / (float)K;",
                         "if (qo_decode_accumulate(words, offsets, K, n, d, s, out, status) != 0) return -1;"),
    "mean_wrong_count": ("if (qo_decode_accumulate(words, offsets, K, n, d, s, out, status) != 0) return -1;\n    for (uint64_t i = 0; i < n; ++i) out[i] = out[i] / (float)K;",
                         "if (qo_decode_accumulate(words, offsets, K, n, d, s, out, status) != 0) return -1;\n    for (uint64_t i = 0; i < n; ++i) out[i] = out[i] / (float)(K + 1);"),
    "bbit_mean_not_divided": ("if (qo_bbit_decode_accumulate(norms, codes, K, n, d, b, out, status) != 0) return -1;\n    for (uint64_t i = 0; i < n; ++i) out[i] = out[i] / (float)K;",
                              "if (qo_bbit_decode_accumulate(norms, codes, K, n, d, b, out, status) != 0) return -1;"),
    "bbit_code_shifted": ("uint64_t pos = (base + i) * b;\n            put_bits_msb_first",
                          "uint64_t pos = (base + i) * b + 1;\n            put_bits_msb_first"),
}


# Survives every CPU pin: all CPU pins use seeds below 2^32 and no published
# known-answer vector has a non-zero key with counter (j, 0, 0, 0).  It is caught
# by the GPU test that runs curand's Philox4_32_10 generator
# (tests/test_gpu_philox_curand.py).
GPU_PINNED_MUTANTS = {
    "random_word_key_halves_swapped": (
        "uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};",
        "uint32_t key[2] = {(uint32_t)(seed >> 32), (uint32_t)(seed & 0xFFFFFFFFu)};"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    d = tmp_path / name
    d.mkdir()
    shutil.copy(os.path.join(os.path.dirname(SRC), "qsgd_oracle.h"), d / "qsgd_oracle.h")
    (d / "qsgd_oracle.c").write_text(src.replace(old, new))
    out = oracle_mod.build(force=True, src=str(d / "qsgd_oracle.c"), out=str(d / "lib.so"))
    return oracle_mod.Oracle(oracle_mod.load(out))


def pin_battery(o) -> list:
    """Names of the pins that fail for oracle o."""
    failed = []
    for ctr, key, expect in load_kat():
        if [int(x) for x in o.philox(ctr, key)] != expect:
            failed.append("philox_kat")
            break
    for N, code in load_omega_codewords():
        if o.omega_bits(N) != code or o.omega_len(N) != len(code):
            failed.append("omega_textbook")
            break
    vals = np.arange(1, 4097, dtype=np.uint64)
    try:
        words, nbits = o.omega_put_many(vals)
        dec, pos = o.omega_get_many(words, len(vals), nbits)
        if pos != nbits or list(dec) != [int(x) for x in vals]:
            failed.append("omega_round_trip")
    except (ValueError, AssertionError):
        failed.append("omega_round_trip")
    for case in load_streams():
        v = fixture_vector(case["v"])
        bits = "".join(case["bits"]).replace(" ", "")
        try:
            w, off, _, st = o.encode(v, case["d"], case["s"], case["seed"])
            ok = ([int(x) for x in off] == case["offsets"] and words_to_bits(w, len(bits)) == bits
                  and st == case["status"])
        except RuntimeError:
            ok = False
        if not ok:
            failed.append("golden_encode")
            break
    for case in load_streams():
        out, st = o.decode(bits_to_words("".join(case["bits"]).replace(" ", "")),
                           np.array(case["offsets"], np.uint64), len(case["v"]), case["d"], case["s"])
        if out.view(np.uint32).tolist() != fixture_decoded(case["decoded"]).view(np.uint32).tolist():
            failed.append("golden_decode")
            break
    a = bits_to_words("01000000101000000000000000000000" + "00110" + "00101000")
    b = bits_to_words("01000000000000000000000000000000" + "100" + "1" + "0")
    out = np.array([0.5, -0.0], dtype=np.float32)
    o.decode_accumulate([(a, np.array([0, 45], np.uint64)), (b, np.array([0, 37], np.uint64))],
                        2, 2, 5, out)
    f = np.float32
    expect = np.array([f(f(0.5) + f(3)) + f(0), f(f(-0.0) + f(4)) + f(-0.4)], np.float32)
    if out.view(np.uint32).tolist() != expect.view(np.uint32).tolist():
        failed.append("accumulate_hand")
    from quantized_gradient_compression_b200 import workloads

    # b-bit variant: hand-derived words, the Elias path's levels, malformed codes,
    # decode-accumulate
    try:
        for bw, vv, dd, words_expect in [(4, [2, -3, 6, 0, 0, 0, 0, 0], 8, [0x2B600000]),
                                          (4, [0, 14, 0, 0, 0, 0, 0, 0], 8, [0x07000000]),
                                          (2, [0, -1, 0, 0], 4, [0x30000000]),
                                          (4, [0, 0, 7, 0, 0, -7, 0, 0], 4, [0x00700F00])]:
            vv = np.array(vv, np.float32)
            codes, nrm, _ = o.bbit_encode(vv, dd, bw, 3)
            dec, st = o.bbit_decode(nrm, codes, vv.size, dd, bw)
            if [int(x) for x in codes] != words_expect or st != 0 or not np.array_equal(dec, vv):
                failed.append("bbit_golden")
                break
        vv = workloads.normal(300, 5)
        lv, _, _ = o.quantize(vv, 100, 7, 2)
        codes, nrm, _ = o.bbit_encode(vv, 100, 4, 2)
        bits = np.unpackbits(codes.astype(">u4").view(np.uint8))[:1200].reshape(300, 4)
        code = (bits * np.array([8, 4, 2, 1])).sum(axis=1)
        if not (np.array_equal(code & 7, np.abs(lv)) and np.array_equal(code >> 3, (lv < 0).astype(int))):
            failed.append("bbit_levels")
        _, st = o.bbit_decode(np.array([7.0], np.float32), np.array([0x2B680000], np.uint32), 8, 8, 4)
        if not st & oracle_mod.ST_BAD_STREAM:
            failed.append("bbit_malformed")
        acc = np.array([0.25] * 8, np.float32)
        c1, n1, _ = o.bbit_encode(np.array([2, -3, 6, 0, 0, 0, 0, 0], np.float32), 8, 4, 1)
        o.bbit_decode_accumulate([(n1, c1), (n1, c1)], 8, 8, 4, acc)
        if acc.tolist() != [4.25, -5.75, 12.25, 0.25, 0.25, 0.25, 0.25, 0.25]:
            failed.append("bbit_accumulate")
    except (ValueError, AssertionError):
        failed.append("bbit")
    # max-norm scale: numpy's max |v| per bucket, NaN propagated
    vm = workloads.normal(1000, 4)
    ref = np.array([np.max(np.abs(vm[b * 100:(b + 1) * 100])) for b in range(10)], np.float32)
    vn = vm.copy()
    vn[5] = np.nan
    if not (np.array_equal(o.maxnorms(vm, 100), ref) and np.isnan(o.maxnorms(vn, 100)[0])):
        failed.append("maxnorm")
    # error feedback: an exact step, the two outcomes of a fractional one, e = 0
    try:
        g = np.array([1, 4, 0, 0, 0, 0, 0, 0], np.float32)
        e = np.array([2, 0, 0, 0, 0, 0, 0, 0], np.float32)
        w, off, _, _, e_new = o.encode_ef(g, e, 8, 5, 1)
        pw, _, _, _ = o.encode(g + e, 8, 5, 1)
        if not (np.array_equal(w, pw) and e_new.view(np.uint32).tolist() == [0] * 8):
            failed.append("ef_exact")
        for seed in range(40):
            _, _, _, _, e_new = o.encode_ef(np.array([-3, 4, 0, 0], np.float32), np.zeros(4, np.float32),
                                            4, 1, seed)
            if e_new[0] not in (-3.0, 2.0) or e_new[1] not in (4.0, -1.0):
                failed.append("ef_outcomes")
                break
        g = workloads.normal(300, 12)
        _, _, _, _, e_new = o.encode_ef(g, np.zeros(300, np.float32), 100, 2, 4)
        w, off, _, _ = o.encode(g, 100, 2, 4)
        q, _ = o.decode(w, off, 300, 100, 2)
        if not np.array_equal(e_new[q == 0], g[q == 0]):
            failed.append("ef_unsent")
    except (RuntimeError, ValueError, AssertionError):
        failed.append("ef")
    # mean of K streams: hand values, and two equal b-bit streams give their decode
    mo, _ = o.decode_mean([(a, np.array([0, 45], np.uint64)), (b, np.array([0, 37], np.uint64))], 2, 2, 5)
    if mo.tolist() != [1.5, float(np.float32(np.float32(4) + np.float32(-0.4)) / np.float32(2))]:
        failed.append("mean_hand")
    try:
        c1, n1, _ = o.bbit_encode(np.array([2, -3, 6, 0, 0, 0, 0, 0], np.float32), 8, 4, 1)
        bm, _ = o.bbit_decode_mean([(n1, c1), (n1, c1)], 8, 8, 4)
        if bm.tolist() != [2, -3, 6, 0, 0, 0, 0, 0]:
            failed.append("bbit_mean")
    except (ValueError, AssertionError):
        failed.append("bbit_mean")
    # small unbiasedness sweep: 4096 N(0,1) coordinates, s = 8, 400 seeds
    v = workloads.normal(4096, 1)
    sums = sc.Sums(v.size)
    v64 = v.astype(np.float64)
    for seed in range(400):
        levels, norms, _ = o.quantize(v, v.size, 8, seed)
        sums.add_levels(v64, levels, norms[0], 8)
    try:
        sc.check_unbiased(v, 8, sums, max_beyond_4se=10)
    except AssertionError:
        failed.append("unbiased")
    return failed


def test_unmutated_oracle_passes_battery(tmp_path):
    o = _build_mutant(tmp_path, "identity", "int qo_omega_len(uint64_t N) {", "int qo_omega_len(uint64_t N) {")
    assert pin_battery(o) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    o = _build_mutant(tmp_path, name, old, new)
    failed = pin_battery(o)
    assert failed, "mutant %s survived every pin" % name
