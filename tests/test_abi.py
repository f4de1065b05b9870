"""C-ABI library: loads, exports every symbol include/*.h declares, and
rejects bad arguments on the host (no GPU needed: nothing is launched)."""
import ctypes
import glob
import os
import re

import pytest

from tests.conftest import ROOT

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"ROSA_API\s+[\w\s\*]*?\b(rosa_\w+)\s*\(", src)
    return names


@pytest.fixture(scope="module")
def lib():
    from suffix_automaton_retrieval_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("rosa_discretize", "rosa_match", "rosa_gather", "rosa_match_workspace_size",
                 "rosa_status_string", "rosa_match_device_status"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    lib.rosa_status_string.restype = ctypes.c_char_p
    assert lib.rosa_status_string(0) == b"ROSA_OK"
    assert lib.rosa_status_string(2) == b"ROSA_ERR_WORKSPACE"
    assert lib.rosa_status_string(99) == b"ROSA_ERR_UNKNOWN"


def test_workspace_size(lib):
    f = lib.rosa_match_workspace_size
    f.argtypes = [ctypes.c_int] * 3
    f.restype = ctypes.c_size_t
    a = f(1, 4096, 2)
    b = f(128, 131072, 256)
    assert 0 < a < b
    assert b % 256 == 0
    assert f(-1, 10, 2) == 0 and f(1, 10, 0) == 0 and f(1, 10, 257) == 0
    assert f(1 << 15, 1 << 16, 4) == 0   # item count beyond int32


def test_host_argument_errors(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.rosa_match.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.rosa_discretize.argtypes = [vp, i, i, i, i, vp, vp]
    lib.rosa_gather.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, vp, i, i, i, i, vp, vp]
    fake = vp(0x10000)   # never dereferenced: every call below fails its host checks
    # g < 1, K out of range, NULL pointers, missing or short workspace
    assert lib.rosa_match(fake, fake, None, 1, 8, 2, 0, fake, fake, fake, fake, 1 << 20, None) == 1
    assert lib.rosa_match(fake, fake, None, 1, 8, 300, 2, fake, fake, fake, fake, 1 << 20, None) == 1
    assert lib.rosa_match(None, fake, None, 1, 8, 2, 2, fake, fake, fake, fake, 1 << 20, None) == 1
    assert lib.rosa_match(fake, fake, None, 1, 8, 2, 2, fake, fake, fake, None, 1 << 20, None) == 2
    assert lib.rosa_match(fake, fake, None, 1, 8, 2, 2, fake, fake, fake, fake, 16, None) == 2
    assert lib.rosa_match(fake, fake, None, 1, 8, 2, 2, fake, fake, fake, vp(0x10008), 1 << 20, None) == 2
    # discretize: M out of range, C % M != 0
    assert lib.rosa_discretize(fake, 1, 4, 8, 9, fake, None) == 1
    assert lib.rosa_discretize(fake, 1, 4, 6, 4, fake, None) == 1
    # gather: route slice beyond the row, d < 1
    assert lib.rosa_gather(fake, 16, 8, fake, 1, 3, 4, 8, fake, None) == 1
    assert lib.rosa_gather(fake, 16, 8, fake, 1, 2, 4, 0, fake, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    from suffix_automaton_retrieval_b200 import binding
    with pytest.raises(ValueError):
        binding.match(torch.zeros((1, 4), dtype=torch.uint8))
    with pytest.raises(ValueError):
        binding.discretize(torch.zeros((1, 4, 8), dtype=torch.bfloat16), 4)
