"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/csa.h declares, and rejects bad arguments with the
documented error codes before touching a device."""
import ctypes
import os
import re

import pytest

import compressed_sparse_attention_16_b200 as csa
from compressed_sparse_attention_16_b200 import Dims

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "csa.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*?\**\s*\**\s*([a-z_][a-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(n for n in names if n.startswith(("csa_", "hca_"))))


def test_header_symbols_are_exported():
    lib = csa.lib()
    declared = _declared_functions()
    assert "csa_compress" in declared and "hca_attend" in declared
    assert set(declared) == set(csa.SYMBOLS)
    for name in declared:
        assert hasattr(lib, name), name


def test_version_and_error_string():
    assert csa.version() == 100
    assert isinstance(csa.lib().csa_last_error(), bytes)


def test_dims_struct_layout_matches_c_compiler(tmp_path):
    """The ctypes mirror of csa_dims has the C compiler's size and offsets."""
    import subprocess
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "csa.h"\n'
                   'int main(void){printf("%zu %zu %zu %zu %zu", sizeof(csa_dims),'
                   ' offsetof(csa_dims, n_entries), offsetof(csa_dims, entry_cap),'
                   ' offsetof(csa_dims, win_cap), offsetof(csa_dims, softmax_scale));return 0;}')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    assert got == [ctypes.sizeof(Dims), Dims.n_entries.offset, Dims.entry_cap.offset,
                   Dims.win_cap.offset, Dims.softmax_scale.offset]


def test_workspace_sizes_are_host_only():
    d = Dims(B=2, Tq=3, H=4, D=64, HI=2, dI=32, K=16, W=8, m=4, n_entries=10)
    assert csa.index_topk_workspace(d) >= 0
    assert csa.attend_workspace(d) >= 0 and csa.attend_workspace(d, dense=True) >= 0


def _rc(fn, *args):
    rc = fn(*args)
    return rc, csa.lib().csa_last_error().decode()


def test_compress_rejects_bad_arguments():
    L = csa.lib()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails first
    rc, msg = _rc(L.csa_compress, fake, fake, 1, 8, 6, 4, 48, fake, fake, 0, 2, 0, None, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED and "D=6" in msg
    rc, msg = _rc(L.csa_compress, fake, fake, 1, 8, 64, 0, 512, fake, fake, 0, 2, 0, None, None)
    assert rc == csa.CSA_ERR_INVALID
    rc, msg = _rc(L.csa_compress, None, fake, 1, 8, 64, 4, 512, fake, fake, 0, 2, 0, None, None)
    assert rc == csa.CSA_ERR_INVALID and "NULL" in msg
    rc, msg = _rc(L.csa_compress, ctypes.c_void_p((1 << 20) + 4), fake, 1, 8, 64, 4, 512, fake, fake,
                  0, 2, 0, None, None)
    assert rc == csa.CSA_ERR_INVALID and "misaligned" in msg
    # T < m and B == 0 are no-ops that succeed without a device
    assert L.csa_compress(fake, fake, 1, 3, 64, 4, 192, fake, fake, 0, 1, 0, None, None) == 0
    assert L.csa_compress(fake, fake, 0, 8, 64, 4, 512, fake, fake, 0, 2, 0, None, None) == 0


def test_index_topk_rejects_bad_arguments():
    L = csa.lib()
    fake = ctypes.c_void_p(1 << 20)
    d = Dims(B=1, Tq=1, HI=4, dI=48, K=4, m=4, n_entries=8)
    rc, msg = _rc(L.csa_index_topk, fake, fake, fake, fake, ctypes.byref(d), fake, None, None, 0, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED
    d = Dims(B=1, Tq=1, HI=4, dI=64, K=4096, m=4, n_entries=8)
    rc, _ = _rc(L.csa_index_topk, fake, fake, fake, fake, ctypes.byref(d), fake, None, None, 0, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED
    d = Dims(B=1, Tq=1, HI=4, dI=64, K=4, m=4, n_entries=8, entry_cap=4)
    rc, _ = _rc(L.csa_index_topk, fake, fake, fake, fake, ctypes.byref(d), fake, None, None, 0, None)
    assert rc == csa.CSA_ERR_INVALID
    d = Dims(B=1, Tq=1, HI=4, dI=64, K=4, m=4, n_entries=8)
    if csa.index_topk_workspace(d):
        rc, msg = _rc(L.csa_index_topk, fake, fake, fake, fake, ctypes.byref(d), fake, None, None, 0, None)
        assert rc == csa.CSA_ERR_WORKSPACE and "workspace" in msg
    rc, _ = _rc(L.csa_index_topk, fake, fake, fake, fake, None, fake, None, None, 0, None)
    assert rc == csa.CSA_ERR_INVALID


def test_attend_rejects_bad_arguments():
    L = csa.lib()
    fake = ctypes.c_void_p(1 << 20)
    d = Dims(B=1, Tq=1, H=4, D=96, K=4, W=8, m=4, n_entries=8)
    rc, msg = _rc(L.csa_attend, fake, fake, fake, fake, fake, fake, fake, ctypes.byref(d), fake, None,
                  None, 0, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED and "D=96" in msg
    d = Dims(B=1, Tq=1, H=4, D=64, K=4, W=8, m=4, n_entries=8, win_cap=4)
    rc, msg = _rc(L.csa_attend, fake, fake, fake, fake, fake, fake, fake, ctypes.byref(d), fake, None,
                  None, 0, None)
    assert rc == csa.CSA_ERR_INVALID and "win_cap" in msg
    d = Dims(B=1, Tq=1, H=4, D=64, K=4, W=8, m=4, n_entries=8)
    rc, msg = _rc(L.csa_attend, fake, fake, fake, None, fake, fake, fake, ctypes.byref(d), fake, None,
                  None, 0, None)
    assert rc == csa.CSA_ERR_INVALID and "hca_attend" in msg


def test_binding_requires_cuda_tensors():
    import torch
    x = torch.zeros(1, 8, 64)
    with pytest.raises(ValueError):
        csa.compress(x, x, 4, torch.zeros(1, 2, 64, dtype=torch.uint8), torch.zeros(1, 2))


def test_quantize_mxfp4_rejects_bad_arguments():
    L = csa.lib()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails first
    rc, msg = _rc(L.csa_quantize_mxfp4, fake, 4, 48, fake, fake, None)
    assert rc == csa.CSA_ERR_INVALID and "multiple of 32" in msg
    rc, _ = _rc(L.csa_quantize_mxfp4, fake, -1, 64, fake, fake, None)
    assert rc == csa.CSA_ERR_INVALID
    rc, msg = _rc(L.csa_quantize_mxfp4, None, 4, 64, fake, fake, None)
    assert rc == csa.CSA_ERR_INVALID and "NULL" in msg
    rc, msg = _rc(L.csa_quantize_mxfp4, ctypes.c_void_p((1 << 20) + 8), 4, 64, fake, fake, None)
    assert rc == csa.CSA_ERR_INVALID and "misaligned" in msg
    rc, msg = _rc(L.csa_quantize_mxfp4, fake, 4, 64, ctypes.c_void_p((1 << 20) + 2), fake, None)
    assert rc == csa.CSA_ERR_INVALID and "misaligned" in msg
    # no rows is a no-op that succeeds without a device
    assert L.csa_quantize_mxfp4(fake, 0, 64, fake, fake, None) == 0
