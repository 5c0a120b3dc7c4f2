"""The C-ABI library loads and exports every symbol include/bsa.h declares.
No compute call is made: only calls that return before touching a device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def bsa():
    import top_block_sparse_bsa_b200 as m   # conftest has built libbsa.so
    return m


def test_header_declares_the_six_calls():
    names = _declared()
    for call in ("bsa_score_blocks", "bsa_topk_select", "bsa_sparse_attn_prefill", "bsa_sparse_attn_decode",
                 "bsa_gated_attn_fwd", "bsa_gist_expand_decode"):
        assert call in names


def test_library_exports_every_declared_symbol(bsa):
    lib = ctypes.CDLL(bsa.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", bsa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (bsa_\w+)", out))
    assert set(_declared()) <= exported
    assert set(bsa.EXPORTED_SYMBOLS) == set(_declared())


def test_binding_names_match_the_abi(bsa):
    for name in _declared():
        assert callable(getattr(bsa, name)), name


def test_status_strings_and_version(bsa):
    assert bsa.bsa_version() == 100
    assert bsa.bsa_status_string(0) == "BSA_OK"
    assert bsa.bsa_status_string(1) == "BSA_ERR_INVALID_ARG"
    assert bsa.bsa_status_string(2) == "BSA_ERR_UNSUPPORTED"
    assert bsa.bsa_status_string(4) == "BSA_ERR_TIMEOUT"


def test_host_checks_reject_before_any_launch(bsa):
    # malformed arguments are refused on the host, before any device work
    lib = bsa.lib
    assert lib.bsa_topk_select(None, 4, 8, 0, 2, None, 3, None, None) == 1
    bad = bsa.make_shape(1, 4, 3, 64, 64, 128, 64, 1)          # Hq % Hkv != 0
    assert lib.bsa_score_blocks(ctypes.byref(bad), 0, ctypes.c_void_p(16), None, None, None, None,
                                ctypes.c_void_p(16), None) == 1
    bad2 = bsa.make_shape(1, 4, 1, 64, 100, 128, 64, 1)        # Nk % block != 0
    assert lib.bsa_sparse_attn_prefill(ctypes.byref(bad2), None, None, None, None, 3, ctypes.c_float(0.1),
                                       None, None, None) == 1
    assert lib.bsa_gated_attn_fwd(ctypes.byref(bad2), None, None, None, None, 3, None, ctypes.c_float(0.1),
                                  None, None, None) == 1


def test_decode_rejects_groups_wider_than_the_mma_tile(bsa):
    # the decode kernels hold at most 16 query heads of a group (MMA N = 16):
    # 17..32 heads per KV group are refused on the host as unsupported
    lib = bsa.lib
    p = ctypes.c_void_p(4096)   # aligned stand-in pointers; nothing is dereferenced
    for hq in (17 * 2, 32 * 2):
        shape = bsa.make_shape(1, hq, 2, 1, 4096, 128, 64, bsa.BSA_BF16)
        assert lib.bsa_sparse_attn_decode(ctypes.byref(shape), p, p, p, p, 8, ctypes.c_float(0.1), p,
                                          ctypes.c_size_t(1 << 30), p, None, None) == 2
        assert lib.bsa_gist_expand_decode(ctypes.byref(shape), p, p, p, p, p, 4, None, None, ctypes.c_float(0.1),
                                          p, ctypes.c_size_t(1 << 30), p, None, None) == 2


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "top_block_sparse_bsa_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "bsa_oracle" not in src, f


def test_build_compiles_every_kernel_source():
    """libbsa.so is linked from exactly the .cu files under csrc/ (a source
    left out would only show as an undefined symbol when the library loads)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("_bsa_build_under_test",
                                                  os.path.join(ROOT, "top_block_sparse_bsa_b200", "_build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    on_disk = sorted(f for f in os.listdir(mod.CSRC) if f.endswith(".cu"))
    assert sorted(mod.SOURCES) == on_disk
    headers = sorted(f for f in os.listdir(mod.CSRC) if f.endswith((".cuh", ".h")))
    assert sorted(mod.HEADERS) == headers


def test_library_has_no_undefined_bsa_symbols():
    lib = os.path.join(ROOT, "top_block_sparse_bsa_b200", "libbsa.so")
    out = subprocess.run(["nm", "-D", "--undefined-only", lib], capture_output=True, text=True, check=True).stdout
    missing = [line for line in out.splitlines() if "bsa" in line]
    assert not missing, missing
