"""bitssm_check_packed on host memory (no GPU): a matrix packed by the
oracle's encoding is valid; a planted code 3, or a padding element that is
not code 1, is counted."""

import numpy as np
import pytest

from oracle import bitssm_oracle as O
from tests.test_abi_exports import ensure_built


def test_valid_and_invalid_codes_are_counted():
    ensure_built()
    from ternary_weight_selective_b200 import bitssm as abi
    Wq = np.random.default_rng(0).integers(-1, 2, size=(7, 30)).astype(np.int8)
    packed = O.pack_ternary(Wq)                      # 30 = 7 bytes + 2 padding codes per row
    assert abi.bitssm_check_packed(packed, 7, 30) == 0
    bad = packed.copy()
    bad[3, 2] |= 0b11 << 4                            # element (3, 10) := code 3
    assert abi.bitssm_check_packed(bad, 7, 30) == 1
    pad = packed.copy()
    pad[5, 7] &= 0b11001111                          # padding element (5, 30) := code 0
    assert abi.bitssm_check_packed(pad, 7, 30) == 1
    everything = np.full_like(packed, 0xFF)
    assert abi.bitssm_check_packed(everything, 7, 30) == 7 * 32


def test_argument_errors():
    ensure_built()
    from ternary_weight_selective_b200 import bitssm as abi
    with pytest.raises(abi.BitssmError):
        abi.bitssm_check_packed(np.zeros((1, 1), np.uint8), 0, 4)
