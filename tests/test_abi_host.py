"""Host-side checks of the C ABI (no GPU needed).

* libbsa.so loads and exports every function ``include/bsa.h`` declares;
* the library's Gilbert table equals the oracle's bit for bit (two
  independent implementations of the same construction: the oracle
  enumerates the curve recursively, the library locates each position by
  descent);
* argument validation rejects bad calls before anything is launched.
"""
import ctypes
import os
import random
import re

import numpy as np
import pytest

import block_sparse_kv_bsa_b200 as bsa
from oracle.gilbert import gilbert_perm as oracle_perm

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "bsa.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(bsa_\w+)\s*\(", text, flags=re.M)))


def test_header_lists_every_binding_export():
    assert header_functions() == sorted(bsa.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(bsa.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {bsa.LIB_PATH}").read()
    for name in header_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_abi_version_and_status_strings():
    assert bsa.abi_version() == 2
    for code, name in bsa.STATUS_NAMES.items():
        assert bsa.status_string(code) == name


@pytest.mark.parametrize("grid", [(2, 8, 16), (4, 16, 32), (5, 30, 52), (4, 30, 52),
                                  (4, 32, 32), (1, 1, 1), (3, 5, 7), (2, 2, 2)])
def test_gilbert_table_matches_oracle(grid):
    assert np.array_equal(bsa.bsa_gilbert_perm(*grid), oracle_perm(*grid))


def test_gilbert_table_matches_oracle_random_shapes():
    rnd = random.Random(99)
    for _ in range(40):
        grid = (rnd.randint(1, 6), rnd.randint(1, 33), rnd.randint(1, 41))
        assert np.array_equal(bsa.bsa_gilbert_perm(*grid), oracle_perm(*grid)), grid


def test_gilbert_perm_rejects_bad_args():
    lib = bsa.lib()
    buf = np.zeros(8, dtype=np.int32)
    p = buf.ctypes.data_as(ctypes.c_void_p)
    assert lib.bsa_gilbert_perm(0, 2, 2, p) == 1
    assert lib.bsa_gilbert_perm(2, 2, 2, None) == 1
    assert lib.bsa_gilbert_perm(1 << 10, 1 << 10, 1 << 10, p) == 2


def test_workspace_size_formula():
    n = bsa.bsa_route_workspace_size(1, 24, 128, 49, 2303)
    qm = -(-4 * 24 * 49 * 128 // 256) * 256
    s = -(-4 * 24 * 49 * 2304 // 256) * 256     # score rows padded to 32 floats
    assert n == qm + s
    with pytest.raises(bsa.BsaError):
        bsa.bsa_route_workspace_size(1, 24, 96, 49, 10)


def test_calls_validate_before_launch():
    lib = bsa.lib()
    c = bsa.CCache(None, None, None, 1, 2, 128, 10, 0)
    # Null pointers are rejected with BSA_ERR_INVALID_ARG, nothing is launched.
    assert lib.bsa_kv_append(ctypes.byref(c), None, None, 2, 8, 16, None, None, None) == 1
    assert lib.bsa_attn(None, ctypes.byref(c), None, None, None, 1, 1, 0.1, None, None,
                        None, None) == 1
    assert lib.bsa_route(None, ctypes.byref(c), None, 0, 0, 1, None, 2.0, 0.2, 0.1, 1,
                         None, None, 1, None, 0, None, None) == 1
    assert lib.bsa_tokens_to_blocks(None, None, 1, 1, 128, 1, 1, 1, None, None, None) == 1
    assert lib.bsa_check_device_error(None, None, None) == 1
