"""Pin of the oracle's binary16 decoder against numpy's, over all 65536 bit patterns."""
import numpy as np

import oracle


def test_all_half_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    # signs of zeros and infinities
    assert np.signbit(got[0x8000]) and not np.signbit(got[0x0000])
    assert got[0x7C00] == np.inf and got[0xFC00] == -np.inf
    assert got[0x0001] == 2.0 ** -24 and got[0x7BFF] == 65504.0
