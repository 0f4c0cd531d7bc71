"""Hand-derived golden bitstreams (tests/golden/qsgd_streams.json) pin the oracle."""

import numpy as np
import pytest

from helpers import bits_to_words, fixture_decoded, fixture_vector, load_streams, words_to_bits

CASES = load_streams()


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_golden_encode(oracle_lib, case):
    v = fixture_vector(case["v"])
    words, offsets, norms, status = oracle_lib.encode(v, case["d"], case["s"], case["seed"])
    expect_bits = "".join(case["bits"]).replace(" ", "")
    assert [int(x) for x in offsets] == case["offsets"]
    assert len(expect_bits) == case["offsets"][-1]
    assert words_to_bits(words, len(expect_bits)) == expect_bits
    assert np.array_equal(words, bits_to_words(expect_bits))
    assert status == case["status"]


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_golden_decode(oracle_lib, case):
    bits = "".join(case["bits"]).replace(" ", "")
    words = bits_to_words(bits)
    offsets = np.array(case["offsets"], dtype=np.uint64)
    n = len(case["v"])
    out, status = oracle_lib.decode(words, offsets, n, case["d"], case["s"])
    expect = fixture_decoded(case["decoded"])
    assert out.view(np.uint32).tolist() == expect.view(np.uint32).tolist()
    assert status == 0
