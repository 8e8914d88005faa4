"""The C-ABI library loads on a machine without a GPU and exports every
entry point that include/bitssm.h declares (no compute call is made)."""

import ctypes
import os
import re
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitssm.h")
LIB = os.path.join(ROOT, "ternary_weight_selective_b200", "libbitssm.so")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?(?:int|char|size_t|void)\s*\**\s*(\w+)\s*\(", src, re.M)
    return sorted(set(names))


def ensure_built():
    from ternary_weight_selective_b200 import build
    build.build()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("bitssm_forward", "bitlinear_forward", "selective_scan_forward",
              "bitssm_workspace_size", "bitssm_pack_ternary", "bitssm_status_string",
              "bitssm_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    ensure_built()
    lib = ctypes.CDLL(LIB)
    for n in declared_functions():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(declared_functions()) <= exported


def test_binding_names_match_header_and_host_calls():
    ensure_built()
    from ternary_weight_selective_b200 import bitssm as abi
    assert set(abi.EXPORTS) == set(declared_functions())
    assert abi.bitssm_version() == 2
    assert abi.bitssm_status_string(abi.ERR_WORKSPACE).startswith("workspace")
    # host-only argument checks return statuses without touching a device
    import pytest
    with pytest.raises(abi.BitssmError) as e:
        abi.bitssm_pack_workspace_size(0, 4, 0)
    assert e.value.status == abi.ERR_INVALID_ARG
    assert abi.bitssm_pack_workspace_size(16, 64, 0) >= 8
    tw = abi.bitssm_tw(None, None, 16, 64, 0)
    with pytest.raises(abi.BitssmError) as e:
        abi.bitlinear_workspace_size(tw, 8, abi.A8)
    assert e.value.status == abi.ERR_INVALID_ARG
    with pytest.raises(abi.BitssmError) as e:
        abi.selective_scan_forward(None, None, None, None, None, None, None, None, None, None,
                                   1, 4, 16, 8, abi.F32)
    assert e.value.status == abi.ERR_UNSUPPORTED_SHAPE
