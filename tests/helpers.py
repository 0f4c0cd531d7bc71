"""Small helpers shared by the tests (bit-string packing, fixture loading)."""

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def bits_to_words(bits: str) -> np.ndarray:
    """Packs a '0'/'1' string MSB-first into uint32 words (zero-padded)."""
    bits = bits.replace(" ", "")
    nwords = (len(bits) + 31) // 32
    bits = bits.ljust(nwords * 32, "0")
    return np.array([int(bits[32 * w:32 * w + 32], 2) for w in range(nwords)], dtype=np.uint32)


def words_to_bits(words: np.ndarray, nbits: int) -> str:
    s = "".join(format(int(w), "032b") for w in np.asarray(words, dtype=np.uint32))
    return s[:nbits]


def load_streams():
    with open(os.path.join(GOLDEN, "qsgd_streams.json")) as f:
        return json.load(f)["cases"]


def fixture_vector(vals) -> np.ndarray:
    return np.array([float(x) for x in vals], dtype=np.float32)


def fixture_decoded(vals) -> np.ndarray:
    out = []
    for x in vals:
        if isinstance(x, str) and x.startswith("0x"):
            out.append(np.array([int(x, 16)], dtype=np.uint32).view(np.float32)[0])
        else:
            out.append(np.float32(x))
    return np.array(out, dtype=np.float32)


def load_kat():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            left, right = line.split("|")
            a = [int(x, 16) for x in left.split()]
            b = [int(x, 16) for x in right.split()]
            rows.append((a[:4], a[4:6], b))
    return rows


def load_omega_codewords():
    rows = []
    with open(os.path.join(GOLDEN, "elias_omega_codewords.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            n, code = line.split()
            rows.append((int(n), code))
    return rows
