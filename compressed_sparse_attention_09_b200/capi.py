"""ctypes binding of libcsa.so (include/csa.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors (their ``data_ptr()`` is passed), plain ints or None (NULL), and
raises ``CsaError`` when the call returns a status other than CSA_OK.  No
step of the computation happens in Python.  Loading fails loudly if the
library has not been built; there is no fallback.  CSA_DEBUG=1 in the
environment loads the debug build, libcsa_debug.so, instead (device-side
index checks; see csa_debug_build in include/csa.h).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libcsa_debug.so" if os.environ.get("CSA_DEBUG") == "1" else "libcsa.so")

CSA_F32, CSA_BF16 = 0, 1
STATUS = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED", 3: "CSA_ERR_CUDA",
          4: "CSA_ERR_DEVICE_TIMEOUT", 5: "CSA_ERR_BAD_INDEX", 6: "CSA_ERR_BAD_METADATA",
          7: "CSA_ERR_WORKSPACE", 8: "CSA_ERR_DEVICE_BOUNDS"}

# every symbol include/csa.h declares
EXPORTS = (
    "csa_packed_weights_bytes", "csa_pack_weights", "csa_compress", "csa_compress_kv", "csa_indexer_topk",
    "csa_sparse_mqa", "csa_forward_workspace_bytes", "csa_forward", "csa_ring_row_elems",
    "csa_cache_append", "csa_decode_workspace_bytes", "csa_decode", "csa_get_device_status",
    "csa_status_string", "csa_hidden_row_elems", "csa_query_row_elems", "csa_project_hidden",
    "csa_project_query", "csa_launch_count", "csa_indexer_workspace_bytes", "csa_indexer_topk_noalloc",
    "csa_set_wait_limit_ns", "csa_check_wait_timeout", "csa_forward_staged", "csa_decode_staged",
    "csa_project_compress_workspace_bytes", "csa_project_hidden_compress", "csa_cp_workspace_bytes",
    "csa_cp_compress", "csa_cp_queries", "csa_quantize_keys_e4m3", "csa_decode_q8", "csa_decode_q8_staged",
    "csa_debug_build",
)


class CsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status_string(status)})")


class csa_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("d", "c", "m", "cI", "nhI", "nh", "dc", "topk", "dtype")]


_WEIGHT_FIELDS = ("W_aKV", "W_bKV", "W_aZ", "W_bZ", "B_a", "B_b", "W_aKV_I", "W_bKV_I", "W_aZ_I",
                  "W_bZ_I", "B_a_I", "B_b_I", "W_DQ", "W_IUQ", "W_UQ", "W_w")


class csa_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _WEIGHT_FIELDS]


@dataclass(frozen=True)
class Dims:
    d: int
    c: int
    m: int
    cI: int
    nhI: int
    nh: int
    dc: int
    topk: int
    dtype: int = CSA_BF16

    def c_struct(self) -> csa_dims:
        return csa_dims(self.d, self.c, self.m, self.cI, self.nhI, self.nh, self.dc, self.topk, self.dtype)


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libcsa.so (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        D = ctypes.POINTER(csa_dims)
        sig = {
            "csa_packed_weights_bytes": (sz, [D]),
            "csa_pack_weights": (i, [D, ctypes.POINTER(csa_weights), vp, sz, vp]),
            "csa_compress": (i, [D, vp, vp, vp, vp, i, vp, vp, i, vp, vp, i, i, i, vp, vp]),
            "csa_compress_kv": (i, [D, vp, vp, i, vp, vp, i, i, vp, vp, vp]),
            "csa_indexer_topk": (i, [D, vp, i, vp, i, vp, vp, vp, i, i, i, i, vp, vp, sz, vp]),
            "csa_indexer_workspace_bytes": (sz, [D, i, i, i]),
            "csa_indexer_topk_noalloc": (i, [D, vp, i, vp, i, vp, vp, vp, i, i, i, i, vp, vp]),
            "csa_sparse_mqa": (i, [D, vp, i, vp, vp, vp, vp, i, i, i, vp, vp]),
            "csa_forward_workspace_bytes": (sz, [D, i, i]),
            "csa_forward": (i, [D, vp, vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp, sz, vp]),
            "csa_ring_row_elems": (i, [D]),
            "csa_cache_append": (i, [D, vp, vp, vp, vp, vp, vp, vp, i, i, vp]),
            "csa_decode_workspace_bytes": (sz, [D, i, i]),
            "csa_decode": (i, [D, vp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, sz, vp]),
            "csa_get_device_status": (i, [vp]),
            "csa_status_string": (ctypes.c_char_p, [i]),
            "csa_hidden_row_elems": (i, [D]),
            "csa_query_row_elems": (i, [D]),
            "csa_project_hidden": (i, [D, vp, vp, i, vp, vp, vp]),
            "csa_project_query": (i, [D, vp, vp, i, i, vp, vp]),
            "csa_launch_count": (ctypes.c_uint64, []),
            "csa_set_wait_limit_ns": (i, [ctypes.c_ulonglong]),
            "csa_project_compress_workspace_bytes": (sz, [D, i]),
            "csa_cp_workspace_bytes": (sz, [D, i, i]),
            "csa_quantize_keys_e4m3": (i, [vp, ctypes.c_longlong, i, i, vp, vp, vp]),
            "csa_decode_q8": (i, [D, vp, vp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, sz, vp]),
            "csa_decode_q8_staged": (i, [D, vp, vp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, sz, vp, vp]),
            "csa_cp_compress": (i, [D, vp, vp, i, i, vp, vp, vp, vp, vp, sz, vp]),
            "csa_cp_queries": (i, [D, vp, vp, vp, i, i, vp, vp, i, vp, vp, vp, sz, vp]),
            "csa_project_hidden_compress": (i, [D, vp, vp, i, vp, vp, i, i, vp, vp, vp, vp, vp, sz, vp]),
            "csa_forward_staged": (i, [D, vp, vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp, sz, vp, vp]),
            "csa_decode_staged": (i, [D, vp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, sz, vp, vp]),
            "csa_check_wait_timeout": (i, [vp, vp]),
            "csa_debug_build": (i, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _p(x):
    """Pointer of a tensor (or an int address / None)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise CsaError(status, where)


def status_string(status: int) -> str:
    return lib().csa_status_string(status).decode()


def _d(dims: Dims):
    return ctypes.byref(dims.c_struct())


# ---------------------------------------------------------------- entry points

def csa_packed_weights_bytes(dims: Dims) -> int:
    return lib().csa_packed_weights_bytes(_d(dims))


def csa_pack_weights(dims: Dims, weights: dict, packed, stream=None):
    w = csa_weights(*[_p(weights[n]) for n in _WEIGHT_FIELDS])
    _check(lib().csa_pack_weights(_d(dims), ctypes.byref(w), _p(packed),
                                  packed.numel() * packed.element_size(), _stream(stream)),
           "csa_pack_weights")


def csa_compress(dims: Dims, Ca, Cb, Za, Zb, ld, Ba, Bb, width, cu_seqlens, cu_blocks, nseq,
                 total_tokens, total_blocks, out, stream=None):
    _check(lib().csa_compress(_d(dims), _p(Ca), _p(Cb), _p(Za), _p(Zb), ld, _p(Ba), _p(Bb), width,
                              _p(cu_seqlens), _p(cu_blocks), nseq, total_tokens, total_blocks, _p(out),
                              _stream(stream)), "csa_compress")


def csa_compress_kv(dims: Dims, packed, Y1, T, cu_seqlens, cu_blocks, nseq, total_blocks, Ccomp, KIcomp,
                    stream=None):
    _check(lib().csa_compress_kv(_d(dims), _p(packed), _p(Y1), T, _p(cu_seqlens), _p(cu_blocks), nseq,
                                 total_blocks, _p(Ccomp), _p(KIcomp), _stream(stream)), "csa_compress_kv")


def csa_indexer_workspace_bytes(dims: Dims, total_tokens: int, nseq: int, max_seqlen: int) -> int:
    return lib().csa_indexer_workspace_bytes(_d(dims), total_tokens, nseq, max_seqlen)


def csa_indexer_topk(dims: Dims, qI, ld_qI, wI, ld_wI, KI, cu_seqlens, cu_blocks, nseq, total_tokens,
                     total_blocks, max_seqlen, idx, ws=None, stream=None):
    _check(lib().csa_indexer_topk(_d(dims), _p(qI), ld_qI, _p(wI), ld_wI, _p(KI), _p(cu_seqlens),
                                  _p(cu_blocks), nseq, total_tokens, total_blocks, max_seqlen, _p(idx),
                                  _p(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                  _stream(stream)), "csa_indexer_topk")


def csa_indexer_topk_noalloc(dims: Dims, qI, ld_qI, wI, ld_wI, KI, cu_seqlens, cu_blocks, nseq, total_tokens,
                             total_blocks, max_seqlen, idx, stream=None):
    """csa_indexer_topk without a workspace argument (see include/csa.h)."""
    _check(lib().csa_indexer_topk_noalloc(_d(dims), _p(qI), ld_qI, _p(wI), ld_wI, _p(KI), _p(cu_seqlens),
                                          _p(cu_blocks), nseq, total_tokens, total_blocks, max_seqlen, _p(idx),
                                          _stream(stream)), "csa_indexer_topk_noalloc")


def csa_sparse_mqa(dims: Dims, q, ld_q, Ccomp, idx, cu_seqlens, cu_blocks, nseq, total_tokens,
                   total_blocks, O, stream=None):
    _check(lib().csa_sparse_mqa(_d(dims), _p(q), ld_q, _p(Ccomp), _p(idx), _p(cu_seqlens), _p(cu_blocks),
                                nseq, total_tokens, total_blocks, _p(O), _stream(stream)),
           "csa_sparse_mqa")


def csa_forward_workspace_bytes(dims: Dims, total_tokens: int, nseq: int) -> int:
    return lib().csa_forward_workspace_bytes(_d(dims), total_tokens, nseq)


def csa_forward(dims: Dims, packed, H, cu_seqlens, cu_blocks, nseq, total_tokens, total_blocks,
                max_seqlen, O, Ccomp_out=None, KI_out=None, idx_out=None, ws=None, stream=None):
    _check(lib().csa_forward(_d(dims), _p(packed), _p(H), _p(cu_seqlens), _p(cu_blocks), nseq,
                             total_tokens, total_blocks, max_seqlen, _p(O), _p(Ccomp_out), _p(KI_out),
                             _p(idx_out), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "csa_forward")


def csa_ring_row_elems(dims: Dims) -> int:
    return lib().csa_ring_row_elems(_d(dims))


def csa_cache_append(dims: Dims, packed, rows, pos, ring, Ccache, KIcache, cache_len, cap, B, stream=None):
    _check(lib().csa_cache_append(_d(dims), _p(packed), _p(rows), _p(pos), _p(ring), _p(Ccache),
                                  _p(KIcache), _p(cache_len), cap, B, _stream(stream)), "csa_cache_append")


def csa_decode_workspace_bytes(dims: Dims, B: int, cap: int) -> int:
    return lib().csa_decode_workspace_bytes(_d(dims), B, cap)


def csa_decode(dims: Dims, packed, h, pos, ring, Ccache, KIcache, cache_len, cap, B, O, idx_out=None,
               ws=None, stream=None):
    _check(lib().csa_decode(_d(dims), _p(packed), _p(h), _p(pos), _p(ring), _p(Ccache), _p(KIcache),
                            _p(cache_len), cap, B, _p(O), _p(idx_out), _p(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "csa_decode")


def csa_hidden_row_elems(dims: Dims) -> int:
    return lib().csa_hidden_row_elems(_d(dims))


def csa_query_row_elems(dims: Dims) -> int:
    return lib().csa_query_row_elems(_d(dims))


def csa_project_hidden(dims: Dims, packed, H, T, Y1, wI, stream=None):
    _check(lib().csa_project_hidden(_d(dims), _p(packed), _p(H), T, _p(Y1), _p(wI), _stream(stream)),
           "csa_project_hidden")


def csa_project_query(dims: Dims, packed, cQ, ld_cQ, T, Y2, stream=None):
    _check(lib().csa_project_query(_d(dims), _p(packed), _p(cQ), ld_cQ, T, _p(Y2), _stream(stream)),
           "csa_project_query")


def csa_debug_build() -> int:
    return lib().csa_debug_build()


def csa_launch_count() -> int:
    return lib().csa_launch_count()


def csa_get_device_status(stream=None) -> int:
    """Status code (0 = CSA_OK) of the conditions kernels recorded; syncs the stream."""
    return lib().csa_get_device_status(_stream(stream))


def csa_set_wait_limit_ns(ns: int):
    """Limit of every bounded device wait on the current device (ns)."""
    _check(lib().csa_set_wait_limit_ns(int(ns)), "csa_set_wait_limit_ns")


def csa_check_wait_timeout(out, stream=None):
    """Enqueues the bounded-wait self-check kernel; out: 3 x int64 on the device."""
    _check(lib().csa_check_wait_timeout(_p(out), _stream(stream)), "csa_check_wait_timeout")


def _event_array(events):
    """ctypes array of cudaEvent_t handles from torch.cuda.Event objects (each
    recorded once beforehand, so that its handle exists)."""
    arr = (ctypes.c_void_p * len(events))()
    for k, e in enumerate(events):
        arr[k] = e.cuda_event if hasattr(e, "cuda_event") else int(e)
    return arr


def csa_forward_staged(dims: Dims, packed, H, cu_seqlens, cu_blocks, nseq, total_tokens, total_blocks, max_seqlen,
                       O, Ccomp_out, KI_out, idx_out, ws, events, stream=None):
    """csa_forward recording events[0..5] around its five stages."""
    _check(lib().csa_forward_staged(_d(dims), _p(packed), _p(H), _p(cu_seqlens), _p(cu_blocks), nseq,
                                    total_tokens, total_blocks, max_seqlen, _p(O), _p(Ccomp_out), _p(KI_out),
                                    _p(idx_out), _p(ws), ws.numel() * ws.element_size(), _event_array(events),
                                    _stream(stream)), "csa_forward_staged")


def csa_decode_staged(dims: Dims, packed, h, pos, ring, Ccache, KIcache, cache_len, cap, B, O, idx_out, ws, events,
                      stream=None):
    """csa_decode recording events[0..6] around its stages."""
    _check(lib().csa_decode_staged(_d(dims), _p(packed), _p(h), _p(pos), _p(ring), _p(Ccache), _p(KIcache),
                                   _p(cache_len), cap, B, _p(O), _p(idx_out), _p(ws), ws.numel() * ws.element_size(),
                                   _event_array(events), _stream(stream)), "csa_decode_staged")


def csa_project_compress_workspace_bytes(dims: Dims, T) -> int:
    return lib().csa_project_compress_workspace_bytes(_d(dims), T)


def csa_project_hidden_compress(dims: Dims, packed, H, T, cu_seqlens, cu_blocks, nseq, total_blocks, Y1, wI, Ccomp,
                                KIcomp, ws, stream=None):
    """A1 with A3 in its epilogue (C^Comp, K^IComp, the c^Q columns of Y1, w^I)."""
    _check(lib().csa_project_hidden_compress(_d(dims), _p(packed), _p(H), T, _p(cu_seqlens), _p(cu_blocks), nseq,
                                             total_blocks, _p(Y1), _p(wI), _p(Ccomp), _p(KIcomp), _p(ws),
                                             ws.numel() * ws.element_size(), _stream(stream)),
           "csa_project_hidden_compress")


def csa_cp_workspace_bytes(dims: Dims, T, ctx) -> int:
    return lib().csa_cp_workspace_bytes(_d(dims), T, ctx)


def csa_cp_compress(dims: Dims, packed, H, T, pos0, Y1, wI, Ccomp_chunk, KIcomp_chunk, ws, stream=None):
    """Context-parallel step 1: A1 (+A3) over a chunk of T tokens at position pos0 (H: the m rows
    before the chunk when pos0 > 0, then the chunk)."""
    _check(lib().csa_cp_compress(_d(dims), _p(packed), _p(H), T, pos0, _p(Y1), _p(wI), _p(Ccomp_chunk),
                                 _p(KIcomp_chunk), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "csa_cp_compress")


def csa_cp_queries(dims: Dims, packed, Y1, wI, T, pos0, Ccomp, KIcomp, total_blocks, O, idx_out, ws, stream=None):
    """Context-parallel step 3: A2, A4, A5 for a chunk's queries over the whole sequence's entries."""
    _check(lib().csa_cp_queries(_d(dims), _p(packed), _p(Y1), _p(wI), T, pos0, _p(Ccomp), _p(KIcomp), total_blocks,
                                _p(O), _p(idx_out), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "csa_cp_queries")


def csa_quantize_keys_e4m3(KI, ld, n, w, codes, scales, stream=None):
    """bf16 rows [n, w] (row stride ld) to E4M3 codes [n, w] and fp32 scales [n]."""
    _check(lib().csa_quantize_keys_e4m3(_p(KI), ld, n, w, _p(codes), _p(scales), _stream(stream)),
           "csa_quantize_keys_e4m3")


def csa_decode_q8(dims: Dims, packed, h, pos, ring, Ccache, KIcodes, KIscale, cache_len, cap, B, O, idx_out=None,
                  ws=None, stream=None):
    """csa_decode with the indexer-key cache as E4M3 codes + per-entry scales."""
    _check(lib().csa_decode_q8(_d(dims), _p(packed), _p(h), _p(pos), _p(ring), _p(Ccache), _p(KIcodes), _p(KIscale),
                               _p(cache_len), cap, B, _p(O), _p(idx_out), _p(ws), ws.numel() * ws.element_size(),
                               _stream(stream)), "csa_decode_q8")


def csa_decode_q8_staged(dims: Dims, packed, h, pos, ring, Ccache, KIcodes, KIscale, cache_len, cap, B, O, idx_out,
                         ws, events, stream=None):
    _check(lib().csa_decode_q8_staged(_d(dims), _p(packed), _p(h), _p(pos), _p(ring), _p(Ccache), _p(KIcodes),
                                      _p(KIscale), _p(cache_len), cap, B, _p(O), _p(idx_out), _p(ws),
                                      ws.numel() * ws.element_size(), _event_array(events), _stream(stream)),
           "csa_decode_q8_staged")
