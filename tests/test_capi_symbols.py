"""The C-ABI library loads and exports every function include/*.h declares;
host-side argument checks that need no GPU answer as documented."""
import ctypes
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^WKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)
    return names


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("wkv_forward", "wkv_forward_bf16", "diag_scan", "wkv_device_status",
                     "wkv_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol():
    import rwkv_wkv_mixing_b200 as wkv
    lib = ctypes.CDLL(wkv.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert missing == []


def test_host_side_argument_errors():
    import rwkv_wkv_mixing_b200 as wkv
    lib = wkv.lib
    # negative sizes are rejected before any CUDA call
    assert lib.wkv_forward(-1, 4, 4, None, None, None, None, None, None) == wkv.WKV_ERR_INVALID_ARG
    assert "negative" in wkv.wkv_last_error()
    assert lib.diag_scan(2, -3, 4, None, None, None, None, None) == wkv.WKV_ERR_INVALID_ARG
    # empty tensors are a no-op
    assert lib.wkv_forward(0, 4, 4, None, None, None, None, None, None) == wkv.WKV_OK
    assert lib.wkv_forward_bf16(3, 0, 4, None, None, None, None, None, None) == wkv.WKV_OK
    assert lib.diag_scan(1, 1, 0, None, None, None, None, None) == wkv.WKV_OK
    assert lib.wkv_forward_state(-2, 1, 4, None, None, None, None, None, None, None, None) == \
        wkv.WKV_ERR_INVALID_ARG
    assert lib.wkv_forward_bf16_state(2, 0, 4, None, None, None, None, None, None, None,
                                      None) == wkv.WKV_OK
    # sizes beyond the int32 range of one dimension
    assert lib.wkv_forward(1, 1 << 31, 1, None, None, None, None, None, None) == \
        wkv.WKV_ERR_INVALID_ARG
    # tile-length knob
    assert lib.wkv_set_tile_steps(100) == wkv.WKV_ERR_INVALID_ARG
    assert lib.wkv_set_tile_steps(64) == wkv.WKV_OK and lib.wkv_get_tile_steps() == 64
    assert lib.wkv_set_tile_steps(256) == wkv.WKV_OK and lib.wkv_get_tile_steps() == 256
    assert lib.wkv_tile_steps_for(8, 1024, 768, 4) == 256
    assert lib.wkv_set_tile_steps(0) == wkv.WKV_OK and lib.wkv_get_tile_steps() == 0
    # automatic: 128 steps, 256 for long sequences over few tiles per segment
    assert lib.wkv_tile_steps_for(8, 1024, 768, 4) == 128
    assert lib.wkv_tile_steps_for(1, 131072, 1024, 4) == 256
    assert lib.wkv_tile_steps_for(8, 4096, 2560, 2) == 128
    assert lib.wkv_tile_steps_for(0, 1, 1, 4) == 0


def test_product_path_has_no_cpu_fallback():
    """The package never imports the oracle and fails loudly without its .so."""
    pkg = os.path.join(ROOT, "rwkv_wkv_mixing_b200")
    for f in glob.glob(os.path.join(pkg, "**", "*.py"), recursive=True):
        src = open(f).read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", src, flags=re.M), f
    init = open(os.path.join(pkg, "__init__.py")).read()
    assert "raise ImportError" in init
