"""Host-side argument checks of ssd_scan_forward on a machine without a GPU
(every case returns its status before anything is launched)."""

import pytest

from tests.test_abi_exports import ensure_built

FAKE = 0x10000  # a non-null placeholder address, never read


@pytest.mark.parametrize("H,P,G,N,status", [
    (4, 32, 3, 16, "ERR_INVALID_ARG"),          # heads do not split over the groups
    (4, 32, 2, 24, "ERR_UNSUPPORTED_SHAPE"),    # N not 16 * 2^k
    (4, 32, 2, 48, "ERR_UNSUPPORTED_SHAPE"),
    (4, 8, 2, 16, "ERR_UNSUPPORTED_SHAPE"),     # P * N / 16 not a multiple of 32
    (4, 128, 2, 256, "ERR_UNSUPPORTED_SHAPE"),  # more than 1024 threads
    (4, 32, 2, 1024, "ERR_UNSUPPORTED_SHAPE"),  # N above 512
    (0, 32, 1, 16, "ERR_INVALID_ARG"),
])
def test_ssd_argument_errors(H, P, G, N, status):
    ensure_built()
    from ternary_weight_selective_b200 import bitssm as abi
    with pytest.raises(abi.BitssmError) as e:
        abi.ssd_scan_forward(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None,
                             2, 8, H, P, G, N)
    assert e.value.status == getattr(abi, status)


def test_ssd_null_pointers_and_empty_batch():
    ensure_built()
    from ternary_weight_selective_b200 import bitssm as abi
    with pytest.raises(abi.BitssmError) as e:
        abi.ssd_scan_forward(None, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None,
                             2, 8, 4, 32, 2, 16)
    assert e.value.status == abi.ERR_INVALID_ARG
    with pytest.raises(abi.BitssmError) as e:
        abi.ssd_scan_forward(FAKE, FAKE, None, FAKE, FAKE, None, None, FAKE, None,
                             2, 8, 4, 32, 2, 16)
    assert e.value.status == abi.ERR_INVALID_ARG
    # an empty batch is a no-op that launches nothing
    abi.ssd_scan_forward(None, None, FAKE, None, None, None, None, None, None, 0, 8, 4, 32, 2, 16)
