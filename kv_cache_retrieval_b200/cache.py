"""A KV cache with HHR retrieval state, held in torch device tensors.

``HHRCache`` owns the device buffers the C ABI works on (keys, values, codes,
page metadata, R, W, decode outputs and workspace) and forwards every
operation to libhhr.so.  torch provides memory and streams only.
"""
from __future__ import annotations

import math

import torch

from . import _binding as B


class HHRCache:
    def __init__(self, *, batch, q_heads, kv_heads, capacity, bits=128, page=16, head_dim=128,
                 P=512, k=4096, device="cuda", flags=0):
        """flags: HHR_FLAG_META_F32 (float32 page metadata) and / or
        HHR_FLAG_GQA_SUM (summed group distances); 0 for the defaults."""
        self.dims = B.make_dims(batch, q_heads, kv_heads, head_dim, bits, page, capacity, flags)
        self.device = torch.device(device)
        self.P, self.k = P, k
        n_pages = (capacity + page - 1) // page
        dev = self.device
        self.K = torch.zeros(batch, kv_heads, capacity, head_dim, dtype=torch.bfloat16, device=dev)
        self.V = torch.zeros_like(self.K)
        self.codes = torch.zeros(batch, kv_heads, capacity, bits // 32, dtype=torch.int32, device=dev)
        meta_dtype = torch.float32 if flags & B.HHR_FLAG_META_F32 else torch.bfloat16
        self.meta = torch.zeros(batch, kv_heads, n_pages, 2, head_dim, dtype=meta_dtype, device=dev)
        self.R = torch.zeros(kv_heads, head_dim, head_dim, dtype=torch.float32, device=dev)
        self.W = torch.zeros(kv_heads, head_dim, bits, dtype=torch.float32, device=dev)
        self.page_idx = torch.empty(batch, kv_heads, P, dtype=torch.int32, device=dev)
        self.tok_idx = torch.empty(batch, kv_heads, k, dtype=torch.int32, device=dev)
        self.n_sel = torch.empty(batch, kv_heads, dtype=torch.int32, device=dev)
        self.out = torch.empty(batch, q_heads, head_dim, dtype=torch.float32, device=dev)
        ws = B.hhr_workspace_size(self.dims, P, k)
        if ws == 0:
            raise B.HhrError(B.HHR_ERR_INVALID_ARG, "hhr_workspace_size")
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=dev)
        self.scale = 1.0 / math.sqrt(head_dim)

    # -- key encoding -------------------------------------------------------
    def encode(self, n_begin, n_end, stream=None):
        B.hhr_encode_keys(self.dims, self.K, self.R, self.W, n_begin, n_end, self.codes,
                          self.meta, stream)

    # -- decode -------------------------------------------------------------
    def select(self, q, n_valid, dbg_U=None, dbg_D=None, stream=None):
        B.hhr_select(self.dims, q, self.R, self.W, self.codes, self.meta, n_valid, self.P,
                     self.k, self.page_idx, self.tok_idx, self.n_sel, dbg_U, dbg_D,
                     self.workspace, None, stream)

    def attend(self, q, tok_idx=None, n_sel=None, out=None, stream=None):
        B.hhr_sparse_attend(self.dims, q, self.K, self.V,
                            self.tok_idx if tok_idx is None else tok_idx,
                            self.n_sel if n_sel is None else n_sel, self.k, self.scale,
                            self.out if out is None else out, self.workspace, None, stream)

    def decode_step(self, q, n_valid, stream=None):
        B.hhr_decode_step(self.dims, q, self.R, self.W, self.codes, self.meta, self.K, self.V,
                          n_valid, self.P, self.k, self.scale, self.page_idx, self.tok_idx,
                          self.n_sel, self.out, self.workspace, None, stream)
        return self.out

    def dense_attend(self, q, n_valid, out=None, stream=None):
        """Dense attention over every valid key (the comparator of the sparse
        step)."""
        B.hhr_dense_attend(self.dims, q, self.K, self.V, n_valid, self.scale,
                           self.out if out is None else out, self.workspace, None, stream)
        return self.out if out is None else out

    def status(self, stream=None) -> int:
        return B.hhr_read_status(self.workspace, stream)
