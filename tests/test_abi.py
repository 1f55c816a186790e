"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

import compressed_sparse_attention_09_b200 as csa
from compressed_sparse_attention_09_b200 import capi

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "csa.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(csa_[a-z_0-9]+)\s*\(", src, flags=re.M)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(capi.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = csa.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_debug_build_exports_every_declared_symbol():
    """libcsa_debug.so (device-side index checks) is built beside libcsa.so
    with the same entry points, and each reports which build it is."""
    debug = ctypes.CDLL(os.path.join(capi.PKG, "libcsa_debug.so"))
    for name in declared_functions():
        assert hasattr(debug, name), name
    debug.csa_debug_build.restype = ctypes.c_int
    assert debug.csa_debug_build() == 1
    release = ctypes.CDLL(os.path.join(capi.PKG, "libcsa.so"))
    release.csa_debug_build.restype = ctypes.c_int
    assert release.csa_debug_build() == 0
    debug.csa_status_string.restype = ctypes.c_char_p
    assert b"debug-build" in debug.csa_status_string(8)


def test_no_python_fallback_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(capi, "_lib", None)
    monkeypatch.setattr(capi, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        capi.lib()


TINY = csa.Dims(d=256, c=64, m=4, cI=32, nhI=4, nh=8, dc=128, topk=16, dtype=csa.CSA_F32)


def test_sizes_and_strings():
    assert csa.csa_packed_weights_bytes(TINY) > 0
    assert csa.csa_forward_workspace_bytes(TINY, 256, 1) > 0
    assert csa.csa_ring_row_elems(TINY) == 4 * 64 + 4 * 32
    assert csa.csa_decode_workspace_bytes(TINY, 3, 40) > 0
    assert csa.status_string(0) == "ok"
    bad = csa.Dims(d=256, c=63, m=4, cI=32, nhI=4, nh=8, dc=128, topk=16, dtype=csa.CSA_F32)
    assert csa.csa_packed_weights_bytes(bad) == 0
    assert csa.csa_forward_workspace_bytes(csa.Dims(0, 64, 4, 32, 4, 8, 128, 16, 0), 256, 1) == 0


@pytest.mark.parametrize("dims,status", [
    (csa.Dims(d=256, c=64, m=3, cI=32, nhI=4, nh=8, dc=128, topk=16, dtype=0), 2),    # m outside {1,2,4,8}
    (csa.Dims(d=256, c=96, m=4, cI=32, nhI=4, nh=8, dc=128, topk=16, dtype=0), 2),    # c not a power of 2
    (csa.Dims(d=256, c=64, m=4, cI=32, nhI=4, nh=8, dc=128, topk=0, dtype=0), 1),     # k = 0
    (csa.Dims(d=256, c=64, m=4, cI=32, nhI=4, nh=8, dc=128, topk=16, dtype=7), 1),    # bad dtype
])
def test_host_validation_before_any_launch(dims, status):
    L = csa.lib()
    dummy = ctypes.c_void_p(1 << 20)
    rc = L.csa_forward(ctypes.byref(dims.c_struct()), dummy, dummy, dummy, dummy, 1, 256, 64, 256, dummy,
                       None, None, None, dummy, 1 << 30, None)
    assert rc == status


def test_null_pointers_rejected():
    L = csa.lib()
    d = ctypes.byref(TINY.c_struct())
    assert L.csa_forward(d, None, None, None, None, 1, 256, 64, 256, None, None, None, None, None, 0, None) == 1
    assert L.csa_compress(d, None, None, None, None, 64, None, None, 64, None, None, 1, 256, 64, None, None) == 1
    assert L.csa_decode(d, None, None, None, None, None, None, None, 10, 1, None, None, None, 0, None) == 1


def test_workspace_too_small_rejected():
    L = csa.lib()
    d = ctypes.byref(TINY.c_struct())
    p = ctypes.c_void_p(1 << 20)   # 1024-aligned fake address; nothing is launched
    need = csa.csa_forward_workspace_bytes(TINY, 256, 1)
    assert L.csa_forward(d, p, p, p, p, 1, 256, 64, 256, p, None, None, None, p, need - 1, None) == 7


def test_misaligned_workspace_rejected():
    L = csa.lib()
    d = ctypes.byref(TINY.c_struct())
    p = ctypes.c_void_p(1 << 20)
    q = ctypes.c_void_p((1 << 20) + 128)
    assert L.csa_forward(d, p, p, p, p, 1, 256, 64, 256, p, None, None, None, q, 1 << 30, None) == 1


def test_every_stage_rejects_null_pointers_before_any_launch():
    """Each stage entry checks its pointers on the host: a null buffer is
    CSA_ERR_INVALID_ARG and nothing is launched."""
    L = csa.lib()
    d = ctypes.byref(TINY.c_struct())
    n0 = csa.csa_launch_count()
    assert L.csa_pack_weights(d, None, None, 0, None) == 1
    assert L.csa_project_hidden(d, None, None, 64, None, None, None) == 1
    assert L.csa_project_query(d, None, None, 128, 64, None, None) == 1
    assert L.csa_compress_kv(d, None, None, 64, None, None, 1, 16, None, None, None) == 1
    assert L.csa_indexer_topk(d, None, 128, None, 4, None, None, None, 1, 256, 64, 256, None, None, 0, None) == 1
    assert L.csa_indexer_topk_noalloc(d, None, 128, None, 4, None, None, None, 1, 256, 64, 256, None, None) == 1
    assert L.csa_sparse_mqa(d, None, 512, None, None, None, None, 1, 256, 64, None, None) == 1
    assert L.csa_cache_append(d, None, None, None, None, None, None, None, 10, 1, None) == 1
    assert csa.csa_launch_count() == n0


def test_decode_workspace_too_small_rejected():
    L = csa.lib()
    d = ctypes.byref(TINY.c_struct())
    p = ctypes.c_void_p(1 << 20)   # 1024-aligned fake address; nothing is launched
    need = csa.csa_decode_workspace_bytes(TINY, 3, 40)
    n0 = csa.csa_launch_count()
    assert L.csa_decode(d, p, p, p, p, p, p, p, 40, 3, p, None, p, need - 1, None) == 7
    assert csa.csa_launch_count() == n0


def test_indexer_row_limit_refused_before_any_launch():
    """The CUDA-core indexer (fp32 here) keeps a query's candidate scores in
    shared memory.  A forward whose longest sequence, a decode step whose cache
    capacity, or a context-parallel chunk whose prefix needs more than one
    block's shared memory is refused with CSA_ERR_UNSUPPORTED before anything
    is launched: in particular before the decode append changes a cache.
    (Only refusals are exercised: the addresses are fake.)"""
    L = csa.lib()
    d = ctypes.byref(TINY.c_struct())
    p = ctypes.c_void_p(1 << 20)
    n0 = csa.csa_launch_count()
    T = 300_000            # 75000 blocks of fp32 scores: more than 227 KB
    ws = csa.csa_forward_workspace_bytes(TINY, T, 1)
    assert L.csa_forward(d, p, p, p, p, 1, T, T // 4, T, p, None, None, None, p, ws, None) == 2
    cap = 100_000
    ws = csa.csa_decode_workspace_bytes(TINY, 3, cap)
    assert L.csa_decode(d, p, p, p, p, p, p, p, cap, 3, p, None, p, ws, None) == 2
    ws = csa.csa_cp_workspace_bytes(TINY, 4096, T)
    assert ws > 0
    assert L.csa_cp_queries(d, p, p, p, 4096, T - 4096, p, p, T // 4, p, None, p, ws, None) == 2
    assert csa.csa_launch_count() == n0


def test_decode_workspace_holds_scores_and_split_sums():
    """The decode workspace covers the [B, cap] fp32 scores and the four fp32
    K-slices of the hidden-side projection ([slice][token][feature], features
    padded to 128)."""
    dims = csa.Dims(d=4096, c=512, m=4, cI=128, nhI=64, nh=128, dc=1536, topk=2048, dtype=csa.CSA_BF16)
    B, cap = 64, 16384
    n1 = 4 * dims.c + 4 * dims.cI + dims.dc + dims.nhI
    n1p = (n1 + 127) // 128 * 128
    assert csa.csa_decode_workspace_bytes(dims, B, cap) >= B * cap * 4 + 4 * n1p * B * 4
    assert csa.csa_decode_workspace_bytes(dims, 2 * B, cap) > csa.csa_decode_workspace_bytes(dims, B, cap)
