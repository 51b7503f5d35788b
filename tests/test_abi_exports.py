"""The C-ABI library loads on a machine without a GPU and exports every
function include/amk.h declares; host-only entry points answer."""
import ctypes
import os
import re

import pytest

import persistent_megakernel_decode_cta_b200 as amk
from persistent_megakernel_decode_cta_b200 import abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "amk.h")).read()
    return sorted(set(re.findall(r"AMK_API[^;(]*?\b(amk_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 18
    lib = ctypes.CDLL(abi.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    # the binding knows every declared function, and nothing else
    assert sorted(abi.SIGNATURES) == names


def test_only_declared_symbols_are_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines()
                       if " T " in ln and ln.split()[-1].startswith("amk_")})
    assert exported == declared_functions()


def test_host_only_entry_points():
    assert "sm_100a" in amk.version()
    lib = abi.lib()
    assert lib.amk_strerror(-3).decode().startswith("schedule rejected")
    o = amk.default_options()
    assert o.ring_stages == 0 and o.stage_bytes == 0  # resolved per weight format
    assert o.debug_skip_signal_task == -1
    assert lib.amk_default_options(None) == abi.ERR["AMK_ERR_INVALID_ARG"]
    assert lib.amk_validate_graph(None, None) == abi.ERR["AMK_ERR_INVALID_ARG"]


def test_create_without_device_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    import synth_inputs as si
    cfg = si.get_config("tiny")
    w = abi.Weights()
    h = ctypes.c_void_p()
    rc = abi.lib().amk_create(ctypes.byref(amk.make_config(cfg)), ctypes.byref(w), None, None,
                              ctypes.byref(h))
    assert rc == abi.ERR["AMK_ERR_NO_DEVICE"]
    assert not h.value


def test_read_ceiling_rejects_small_buffers_on_the_host():
    """Arguments are checked before any device work: a buffer smaller than
    1 GiB (L2 could hold it) is refused."""
    import ctypes
    from persistent_megakernel_decode_cta_b200 import abi
    g = ctypes.c_double(0.0)
    rc = abi.lib().amk_read_ceiling(ctypes.c_void_p(1 << 20), 1 << 20, 148, 32768, 3, 1, None,
                                    ctypes.byref(g))
    assert rc == abi.ERR["AMK_ERR_INVALID_ARG"]
