"""The allocation-free decode entry point against the workspace one.

hhr_decode_step_noalloc serves callers that cannot allocate device memory for
a workspace; it keeps its scratch in a fixed array inside the library.  Two
calls in a row (the second one reusing whatever the first left in that
array) must give what hhr_decode_step gives on the same inputs.  This file
is collected last so that a failure here does not hide any other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import kv_cache_retrieval_b200 as hhr
from kv_cache_retrieval_b200 import _binding as Bnd
from gpu_harness import ATTN_TOL, Dev
from workloads import get, make_inputs, scaled

pytestmark = pytest.mark.gpu


def test_noalloc_step_matches_workspace_step_twice():
    w = scaled(get("llama8b_32k"), N=20003)
    inp = make_inputs(w)
    d = Dev(inp)
    assert hhr.hhr_workspace_size(d.dims, d.P, d.k) <= Bnd.HHR_NOALLOC_SCRATCH_BYTES
    d.encode(0, w.N)
    page_idx = torch.full_like(d.page_idx, -7)
    tok_idx = torch.full_like(d.tok_idx, -7)
    n_sel = torch.full_like(d.n_sel, -7)
    out = torch.full_like(d.out, float("nan"))
    for step in range(2):
        d.decode(0)
        Bnd.hhr_decode_step_noalloc(d.dims, d.q[0], d.R, d.W, d.codes, d.meta, d.K, d.V, w.N, d.P,
                                    d.k, d.scale, page_idx, tok_idx, n_sel, out)
        torch.cuda.synchronize()
        assert d.status() == hhr.HHR_OK
        assert torch.equal(page_idx, d.page_idx), f"call {step}: page_idx differs"
        assert torch.equal(tok_idx, d.tok_idx), f"call {step}: tok_idx differs"
        assert torch.equal(n_sel, d.n_sel), f"call {step}: n_sel differs"
        err = float((out - d.out).abs().max().item())
        assert err <= ATTN_TOL, f"call {step}: max abs difference {err}"
        assert hhr.hhr_noalloc_read_status() == hhr.HHR_OK
    # a rejected call reports the error and leaves the scratch alone
    st = Bnd.lib().hhr_decode_step_noalloc(C.byref(d.dims), None, d.R.data_ptr(), d.W.data_ptr(),
                                           d.codes.data_ptr(), d.meta.data_ptr(), d.K.data_ptr(),
                                           d.V.data_ptr(), w.N, d.P, d.k, d.scale,
                                           page_idx.data_ptr(), tok_idx.data_ptr(),
                                           n_sel.data_ptr(), out.data_ptr(), None)
    assert st == hhr.HHR_ERR_INVALID_ARG
    assert hhr.hhr_noalloc_read_status() == hhr.HHR_OK


def test_noalloc_rejects_sizes_beyond_its_scratch():
    w = get("batch8_64k_b256")
    dims = hhr.make_dims(w.B, w.Hq, w.Hkv, w.d, w.bits, w.page, w.n_cap)
    assert hhr.hhr_workspace_size(dims, w.P, w.k) > Bnd.HHR_NOALLOC_SCRATCH_BYTES
    FAKE = 1 << 20
    st = Bnd.lib().hhr_decode_step_noalloc(C.byref(dims), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                           w.N, w.P, w.k, 0.1, FAKE, FAKE, FAKE, FAKE, None)
    assert st == hhr.HHR_ERR_UNSUPPORTED
