"""B200 (sm_100a) forward path of Compressed Sparse Attention.

The computation lives in libcsa.so (C ABI: include/csa.h); ``capi`` binds it
with ctypes under the same names.  PyTorch is used by callers only for device
memory and streams.
"""
from .capi import (CSA_BF16, CSA_F32, CsaError, Dims, csa_cache_append, csa_compress,  # noqa: F401
                   csa_decode, csa_decode_workspace_bytes, csa_forward, csa_forward_workspace_bytes,
                   csa_get_device_status, csa_indexer_topk, csa_pack_weights, csa_packed_weights_bytes,
                   csa_ring_row_elems, csa_sparse_mqa, lib, status_string,
                   csa_hidden_row_elems, csa_query_row_elems, csa_project_hidden, csa_project_query,
                   csa_launch_count, csa_indexer_workspace_bytes,
                   csa_indexer_topk_noalloc, csa_compress_kv, csa_set_wait_limit_ns,
                   csa_check_wait_timeout, csa_forward_staged, csa_decode_staged,
                   csa_project_compress_workspace_bytes, csa_project_hidden_compress,
                   csa_cp_workspace_bytes, csa_cp_compress, csa_cp_queries, csa_quantize_keys_e4m3,
                   csa_decode_q8, csa_decode_q8_staged, csa_debug_build)
from .meta import cu_from_lengths  # noqa: F401
