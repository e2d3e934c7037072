"""CPU checks of the C-ABI library: it is built for sm_100a, loads, exports every
function include/hisa.h declares, and rejects bad host arguments before touching a GPU."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hisa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_top_hisa_b200 import build
    build.build()
    from sparse_attention_top_hisa_b200 import binding
    return binding.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("hisa_pool_blocks", "hisa_append_keys", "hisa_select", "dsa_flat_select",
              "hisa_sparse_attention"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from sparse_attention_top_hisa_b200 import binding
    names = declared_functions()
    assert sorted(binding.EXPORTED) == names
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(l.split()[-1] for l in out.splitlines() if l.strip())
    for n in names:
        assert n in exported, n
        assert getattr(lib, n) is not None


def test_status_strings(lib):
    for code in range(8):
        assert lib.hisa_status_string(code)
    assert lib.hisa_status_string(0) == b"ok"
    assert lib.hisa_version() >= 100


def test_host_validation_needs_no_gpu(lib):
    P = ctypes.c_void_p
    dummy = P(4096)  # never dereferenced: validation fails first
    # B other than 128
    assert lib.hisa_pool_blocks(dummy, dummy, None, 1, 128, 64, dummy, None) == 1
    assert lib.hisa_select(dummy, dummy, dummy, dummy, dummy, None, 1, 4, 128, 64, 8, 16, dummy,
                           None, None, dummy, 1 << 20, None) == 1
    # m and k out of range
    assert lib.hisa_select(dummy, dummy, dummy, dummy, dummy, None, 1, 4, 128, 128, 0, 16, dummy,
                           None, None, dummy, 1 << 20, None) == 1
    assert lib.hisa_select(dummy, dummy, dummy, dummy, dummy, None, 1, 4, 128, 128, 8, 4096,
                           dummy, None, None, dummy, 1 << 20, None) == 1
    assert lib.dsa_flat_select(dummy, dummy, dummy, dummy, None, 1, 4, 128, 0, dummy, None, dummy,
                               1 << 20, None) == 1
    # empty problems are a no-op
    assert lib.hisa_select(None, None, None, None, None, None, 0, 0, 0, 128, 8, 16, None, None,
                           None, None, 0, None) == 0
    # sparse attention: heads and k out of range, unaligned, empty
    F = ctypes.c_float
    assert lib.hisa_sparse_attention(dummy, dummy, dummy, dummy, dummy, dummy, 1, 4, 0, 16, F(0.1),
                                     dummy, None, None) == 1
    assert lib.hisa_sparse_attention(dummy, dummy, dummy, dummy, dummy, dummy, 1, 4, 33, 16,
                                     F(0.1), dummy, None, None) == 1
    assert lib.hisa_sparse_attention(dummy, dummy, dummy, dummy, dummy, dummy, 1, 4, 8, 0, F(0.1),
                                     dummy, None, None) == 1
    assert lib.hisa_sparse_attention(P(4096 + 2), dummy, dummy, dummy, dummy, dummy, 1, 4, 8, 16,
                                     F(0.1), dummy, None, None) == 2
    assert lib.hisa_sparse_attention(None, None, None, None, None, None, 0, 0, 8, 16, F(0.1), None,
                                     None, None) == 0
    # unaligned pointers
    odd = P(4096 + 2)
    assert lib.hisa_select(odd, dummy, dummy, dummy, dummy, None, 1, 4, 128, 128, 8, 16, dummy,
                           None, None, dummy, 1 << 20, None) == 2
    # missing workspace
    assert lib.hisa_select(dummy, dummy, dummy, dummy, dummy, None, 1, 4, 128, 128, 8, 16, dummy,
                           None, None, None, 0, None) == 3
    assert lib.dsa_flat_select(dummy, dummy, dummy, dummy, None, 1, 4, 128, 16, dummy, None, None,
                               0, None) == 3
    # negative counts
    assert lib.hisa_append_keys(dummy, dummy, dummy, dummy, dummy, -1, 1, 128, None) == 1


def test_workspace_sizes_grow(lib):
    a = lib.hisa_select_workspace_size(4096, 1, 4096, 128, 8, 256)
    b = lib.hisa_select_workspace_size(32768, 1, 32768, 128, 64, 2048)
    assert 0 < a < b
    assert lib.dsa_flat_workspace_size(4096, 1, 4096, 256) > 0


def test_no_cpu_fallback():
    """The product path has no CPU route: host tensors are refused, and a missing
    library is an error at the first call, not a silent fallback."""
    import sys

    import torch

    import sparse_attention_top_hisa_b200 as H
    k = torch.zeros(256, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 256], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        H.hisa_pool_blocks(k, cu, None, 256)
    script = (
        "import sys; sys.path.insert(0, %r)\n"
        "import sparse_attention_top_hisa_b200.binding as b\n"
        "b.LIB_PATH = '/nonexistent/libhisa.so'\n"
        "try:\n"
        "    b.lib()\n"
        "except ImportError as e:\n"
        "    print('refused:', e)\n"
        "else:\n"
        "    raise SystemExit('loaded a library that does not exist')\n"
    ) % ROOT
    p = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True,
                       timeout=120)
    assert p.returncode == 0, p.stderr[-1500:]
    assert "refused:" in p.stdout and "is missing" in p.stdout
