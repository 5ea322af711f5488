"""B200 (sm_100a) implementation of the HHR decode-time retrieval path.

HHR ("Hierarchical Hash Retrieval for Efficient LLM Generation", arXiv
2610.01230) prunes KV-cache pages with rotated per-page min/max logit bounds
(GKR) and then ranks the keys of the kept pages by the Hamming distance of
learned sign codes (LHP) before attending over the selected keys.

The C ABI is ``include/hhr.h``; ``libhhr.so`` implements it with hand-written
CUDA kernels.  This package is its ctypes binding (same function names) plus
``HHRCache``, which owns torch device buffers and forwards to the library.
"""
from ._binding import (HHR_ERR_CUDA, HHR_ERR_INVALID_ARG, HHR_ERR_TIMEOUT, HHR_ERR_UNSUPPORTED,
                       HHR_ERR_WORKSPACE, HHR_FLAG_GQA_SUM, HHR_FLAG_META_F32, HHR_FLAG_SIMT_BOUNDS,
                       HHR_MAX_PAGES,
                       HHR_OK, HhrError, hhr_decode_step, hhr_decode_step_host, hhr_dense_attend,
                       hhr_decode_step_noalloc, hhr_dims, hhr_encode_keys, hhr_encode_status,
                       hhr_noalloc_read_status, hhr_read_status, hhr_select, hhr_sparse_attend,
                       hhr_status_string, hhr_test_arm_timeout, hhr_version, hhr_workspace_size,
                       lib, make_dims)
from .cache import HHRCache

__all__ = [
    "HHR_OK", "HHR_ERR_INVALID_ARG", "HHR_ERR_UNSUPPORTED", "HHR_ERR_WORKSPACE", "HHR_ERR_CUDA",
    "HHR_ERR_TIMEOUT", "HHR_MAX_PAGES", "HHR_FLAG_META_F32", "HHR_FLAG_GQA_SUM", "HHR_FLAG_SIMT_BOUNDS", "HhrError", "hhr_dims", "make_dims", "lib", "hhr_version",
    "hhr_status_string", "hhr_encode_keys", "hhr_encode_status", "hhr_workspace_size", "hhr_select",
    "hhr_sparse_attend", "hhr_dense_attend", "hhr_decode_step", "hhr_decode_step_host", "hhr_decode_step_noalloc", "hhr_noalloc_read_status", "hhr_read_status", "hhr_test_arm_timeout", "HHRCache",
]
