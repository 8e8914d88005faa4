"""Host-side checks of the block form (d_conv != 0) through the C ABI, on a
machine without a GPU: argument validation, workspace layout and launch
counts.  The layer's device pointers are placeholders that these calls never
dereference."""

import pytest

from tests.test_abi_exports import ensure_built

FAKE = 0x10000  # a non-null placeholder address, never read


def _layer(abi, d=256, E=512, N=16, R=16, d_conv=4):
    tw = lambda n, k: abi.bitssm_tw(FAKE, FAKE, n, k, 0)
    L = abi.bitssm_layer(tw(E, d), tw(R, E), tw(N, E), tw(N, E), tw(E, R), tw(d, E),
                         FAKE, FAKE, FAKE, d, E, N, R, None, 0)
    if d_conv:
        L.z_proj = tw(E, d)
        L.conv_w = FAKE
        L.conv_b = None
        L.d_conv = d_conv
    return L


def test_block_layout_sizes_and_launches():
    ensure_built()
    from ternary_weight_selective_b200 import bitssm as abi
    B, L = 64, 256
    T = B * L
    blk = _layer(abi)
    mix = _layer(abi, d_conv=0)
    v = abi.bitssm_workspace_layout(blk, B, L, abi.BF16, abi.A8)
    none = 2**64 - 1
    assert v.u_pre != none and v.z != none and v.u_dtype == abi.F32
    regions = sorted((getattr(v, n), n) for n in ("u_pre", "z", "u", "y") if getattr(v, n) != none)
    for (o0, _), (o1, _) in zip(regions, regions[1:]):
        assert o1 - o0 >= T * 512 * 4            # float [T, E] regions do not overlap
    vm = abi.bitssm_workspace_layout(mix, B, L, abi.BF16, abi.A8)
    assert vm.u_pre == none and vm.z == none
    assert abi.bitssm_workspace_size(blk, B, L, abi.BF16, abi.A8) > \
        abi.bitssm_workspace_size(mix, B, L, abi.BF16, abi.A8)
    assert abi.bitssm_forward_launches(blk, B, L, abi.A8) == 9
    blk.prepared = FAKE
    assert abi.bitssm_forward_launches(blk, B, L, abi.A8) == 8
    # the prepared block holds the expanded z_proj after the six mixer matrices
    assert abi.bitssm_prepared_size(blk, abi.A8) == \
        abi.bitssm_prepared_size(mix, abi.A8) + 512 * 256


@pytest.mark.parametrize("d_conv,act,status", [(5, "A8", "ERR_INVALID_ARG"),
                                               (-1, "A8", "ERR_INVALID_ARG"),
                                               (4, "A16", "ERR_UNSUPPORTED_SHAPE")])
def test_block_argument_errors(d_conv, act, status):
    ensure_built()
    from ternary_weight_selective_b200 import bitssm as abi
    lay = _layer(abi, d_conv=d_conv)
    with pytest.raises(abi.BitssmError) as e:
        abi.bitssm_workspace_size(lay, 2, 8, abi.BF16, getattr(abi, act))
    assert e.value.status == getattr(abi, status)


def test_block_rejects_missing_pieces_and_carried_state():
    ensure_built()
    from ternary_weight_selective_b200 import bitssm as abi
    lay = _layer(abi)
    lay.conv_w = None
    with pytest.raises(abi.BitssmError) as e:
        abi.bitssm_workspace_size(lay, 2, 8, abi.BF16, abi.A8)
    assert e.value.status == abi.ERR_INVALID_ARG
    lay = _layer(abi)
    lay.z_proj.n_out = 256                      # z_proj must be [d_inner, d_model]
    with pytest.raises(abi.BitssmError) as e:
        abi.bitssm_workspace_size(lay, 2, 8, abi.BF16, abi.A8)
    assert e.value.status == abi.ERR_INVALID_ARG
    # a carried state is refused before anything is queued
    lay = _layer(abi)
    with pytest.raises(abi.BitssmError) as e:
        abi.bitssm_forward_state(lay, FAKE, FAKE, None, FAKE, 2, 8, abi.BF16, abi.A8, FAKE, 1 << 30)
    assert e.value.status == abi.ERR_UNSUPPORTED_SHAPE
