"""The C ABI library loads and exports every symbol include/kvc.h declares (CPU only).

No compute call is made here: without a GPU only loading, symbol lookup and
the pure KV-bytes formula are exercised.
"""
import re
from pathlib import Path

import pytest

import kv_cache_decode_03_b200 as kvc
from kv_cache_decode_03_b200 import build as kvc_build
from tests import oracle_pins

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "kvc.h"


@pytest.fixture(scope="module")
def lib():
    if not kvc_build.up_to_date():
        kvc_build.build()
    return kvc.library()


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b(kvc_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("kvc_create", "kvc_append", "kvc_attend", "kvc_bytes", "kvc_destroy",
                     "kvc_get_error"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_kv_bytes_formula_matches_the_worked_example(lib):
    for layers, heads, dim, T, e, batch, want in oracle_pins.golden_kv_bytes():
        assert kvc.kvc_bytes_formula(layers, heads, dim, T, e, batch) == want


def test_status_strings(lib):
    assert kvc.kvc_status_string(kvc.KVC_OK) == "KVC_OK"
    assert kvc.kvc_status_string(kvc.KVC_ERR_BOUNDS) == "KVC_ERR_BOUNDS"
    assert kvc.kvc_status_string(kvc.KVC_ERR_TIMEOUT) == "KVC_ERR_TIMEOUT"


def test_create_rejects_bad_arguments_before_touching_a_device(lib):
    # argument checks run before any CUDA call, so these hold without a GPU
    for args in [(0, 8, 128, 16, "bf16", 0, 1, 0),      # B = 0
                 (1, 8, 128, 16, "bf16", 16, 1, 0),     # paged without pages
                 (1, 8, 128, 16, "bf16", 0, 1, 5),      # pages on a contiguous cache
                 (1, 8, 128, 16, "bf16", 12, 1, 4)]:    # page size not a power of two
        with pytest.raises(kvc.KvcError) as e:
            kvc.kvc_create(*args)
        assert e.value.status == kvc.KVC_ERR_INVALID_ARG
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_create(1, 8, 96, 16, "bf16", 0, 1, 0)
    assert e.value.status == kvc.KVC_ERR_UNSUPPORTED


def test_null_handle_calls_fail_cleanly(lib):
    assert lib.kvc_append(None, 0, None, None, 1, None, 0, None, None) == kvc.KVC_ERR_INVALID_ARG
    assert lib.kvc_attend(None, 0, None, 8, 1, None, 0, None, 1.0, None, None) == \
        kvc.KVC_ERR_INVALID_ARG
    assert lib.kvc_get_error(None) == kvc.KVC_ERR_INVALID_ARG
    assert kvc.kvc_bytes(0) == 0
    assert lib.kvc_destroy(None) == kvc.KVC_OK


def test_missing_library_fails_loudly():
    """Without libkvc.so the product path raises; there is no fallback."""
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from pathlib import Path\n"
        "import kv_cache_decode_03_b200 as k\n"
        "k.LIB_PATH = Path('/nonexistent/libkvc.so'); k._lib = None\n"
        "try:\n"
        "    k.KVCache(1, 1, 64, 8, 'bf16')\n"
        "except ImportError as e:\n"
        "    print('raised:', e)\n"
    ) % str(ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert "raised:" in out.stdout, out.stdout + out.stderr


def test_package_does_not_load_the_oracle():
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, %r)\n"
            "import kv_cache_decode_03_b200\n"
            "print('oracle' in sys.modules)\n") % str(ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert out.stdout.strip() == "False", out.stdout + out.stderr
