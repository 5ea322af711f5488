"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Small cases span several CTAs per unit and ragged
tails; the full-size workloads run in the benchmark's launch configuration
and are checked on sampled (sequence, KV head) units."""
import numpy as np
import pytest
import torch

import kv_cache_retrieval_b200 as hhr
from gpu_harness import (Dev, bits_host, compare_encode, compare_out, compare_select, u32_host)
from oracle import oracle as O
from workloads import get, make_inputs, scaled

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_4k": get("tiny_4k"),
    "llama_20k_ragged": scaled(get("llama8b_32k"), N=20003),
    "b256_s32": scaled(get("batch8_64k_b256"), B=2, N=9001, P=64, k=1024),
    "rope_appends": scaled(get("qwen8b_128k_rope"), B=2, N=7000, P=64, k=512, appends=4),
    "page1": scaled(get("llama8b_32k"), Hq=8, Hkv=2, N=700, page=1, P=100, k=50, planted=4),
    "page64": scaled(get("llama8b_32k"), Hq=8, Hkv=2, N=5000, page=64, P=20, k=300, planted=4),
    "gqa2": scaled(get("llama8b_32k"), Hq=16, Hkv=8, N=3000, P=40, k=200, planted=8),
    "gqa8": scaled(get("llama8b_32k"), Hq=32, Hkv=4, N=3000, P=40, k=200, planted=8),
    # r = 8 with 256-bit codes: the widest GQA-sum histogram (r b + 1 = 2049 bins)
    "gqa8_b256": scaled(get("batch8_64k_b256"), B=1, Hq=32, Hkv=4, N=3000, P=40, k=200, planted=8),
}

_cache = {}


def case(name):
    if name not in _cache:
        w = SMALL[name]
        inp = make_inputs(w)
        codes, meta, _ = O.encode_all(inp, n_end=w.N)
        _cache[name] = (inp, codes, meta)
    return _cache[name]


def all_units(w):
    return [(b, g) for b in range(w.B) for g in range(w.Hkv)]


@pytest.mark.parametrize("name", list(SMALL))
def test_encode_matches_oracle(name):
    inp, _, _ = case(name)
    w = inp.w
    d = Dev(inp)
    d.encode(0, w.N)
    torch.cuda.synchronize()
    rep = compare_encode(inp, u32_host(d.codes), bits_host(d.meta), all_units(w), w.N)
    print(name, rep)


def test_append_encoding_matches_oracle():
    inp, _, _ = case("llama_20k_ragged")
    w = inp.w
    d = Dev(inp)
    n = w.N
    d.encode(0, n - 9)
    for a, b in [(n - 9, n - 8), (n - 8, n - 5), (n - 5, n - 4), (n - 4, n)]:
        d.encode(a, b)
    torch.cuda.synchronize()
    compare_encode(inp, u32_host(d.codes), bits_host(d.meta), all_units(w), n)


def _host(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("name", list(SMALL))
def test_select_matches_oracle(name):
    inp, codes, meta = case(name)
    w = inp.w
    step = inp.steps - 1
    ores = O.decode_all(inp, codes, meta, step=step, attend_too=False)
    d = Dev(inp)
    d.load_state(codes, meta)
    d.select(step=step)
    assert d.status() == hhr.HHR_OK
    rep = compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), all_units(w),
                         dbg_U=_host(d.dbg_U), dbg_D=_host(d.dbg_D), name=f"select {name}")
    print(name, rep)


@pytest.mark.parametrize("name", list(SMALL))
def test_attend_matches_oracle_on_oracle_indices(name):
    inp, codes, meta = case(name)
    w = inp.w
    ores = O.decode_all(inp, codes, meta)
    d = Dev(inp)
    tok = torch.from_numpy(ores["tok_idx"]).cuda()
    nsel = torch.from_numpy(ores["n_sel"]).cuda()
    d.attend(0, tok, nsel)
    assert d.status() == hhr.HHR_OK
    err = compare_out(w, ores["out"], _host(d.out), all_units(w))
    print(name, "max abs err", err)


@pytest.mark.parametrize("name", list(SMALL))
def test_fused_decode_matches_oracle(name):
    inp, codes, meta = case(name)
    w = inp.w
    ores = O.decode_all(inp, codes, meta)
    d = Dev(inp)
    d.load_state(codes, meta)
    d.decode(0)
    assert d.status() == hhr.HHR_OK
    rep = compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), all_units(w),
                         inp=inp, step=0, out_g=_host(d.out), name=f"fused {name}")
    print(name, rep)


@pytest.mark.parametrize("name", ["tiny_4k", "llama_20k_ragged", "b256_s32"])
def test_gpu_encode_then_decode_matches_oracle(name):
    inp, codes, meta = case(name)
    w = inp.w
    ores = O.decode_all(inp, codes, meta)
    d = Dev(inp)
    d.encode(0, w.N)
    d.decode(0)
    assert d.status() == hhr.HHR_OK
    rep = compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), all_units(w),
                         inp=inp, step=0, out_g=_host(d.out), name=f"gpu-encoded {name}")
    print(name, rep)


def test_rope_appends_each_step():
    """Encode the context, then per decode step append one key and decode."""
    inp, _, _ = case("rope_appends")
    w = inp.w
    d = Dev(inp)
    d.encode(0, w.N)
    codes = np.zeros((w.B, w.Hkv, w.n_cap, w.words), np.uint32)
    meta = np.zeros((w.B, w.Hkv, w.np_cap, 2, w.d), np.uint16)
    O.encode_all(inp, 0, w.N, codes=codes, meta=meta)
    for step in range(w.appends):
        d.encode(w.N + step, w.N + step + 1)
        O.encode_all(inp, w.N + step, w.N + step + 1, codes=codes, meta=meta)
        d.decode(step)
        ores = O.decode_all(inp, codes, meta, step=step)
        compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), all_units(w),
                       inp=inp, step=step, out_g=_host(d.out), name=f"rope appends step {step}")
    torch.cuda.synchronize()
    compare_encode(inp, u32_host(d.codes), bits_host(d.meta), all_units(w), w.n_cap)
    assert d.status() == hhr.HHR_OK


# ------------------------------------------------------------------ variants

VARIANTS = {
    "meta_f32": hhr.HHR_FLAG_META_F32,
    "gqa_sum": hhr.HHR_FLAG_GQA_SUM,
    "both": hhr.HHR_FLAG_META_F32 | hhr.HHR_FLAG_GQA_SUM,
    "simt_bounds": hhr.HHR_FLAG_SIMT_BOUNDS,
}
_vcache = {}


def variant_state(name, f32):
    """Oracle-encoded codes and metadata of a small case (float32 metadata
    with f32)."""
    key = (name, f32)
    if key not in _vcache:
        inp, _, _ = case(name)
        codes, meta, _ = O.encode_all(inp, n_end=inp.w.N, meta_f32=f32)
        _vcache[key] = (codes, meta)
    return _vcache[key]


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("name", ["llama_20k_ragged", "b256_s32", "gqa8", "gqa8_b256", "page1", "tiny_4k"])
def test_variant_matches_oracle(name, variant):
    """HHR_FLAG_META_F32 (float32 page metadata) and HHR_FLAG_GQA_SUM (summed
    group distances) against the oracle's variants: the GPU encode, the
    selection with its debug bounds / distances on the oracle's state, and
    the fused step on the GPU-encoded state."""
    inp, _, _ = case(name)
    w = inp.w
    flags = VARIANTS[variant]
    f32 = bool(flags & hhr.HHR_FLAG_META_F32)
    gsum = bool(flags & hhr.HHR_FLAG_GQA_SUM)
    codes, meta = variant_state(name, f32)
    d = Dev(inp, flags=flags)
    d.encode(0, w.N)
    torch.cuda.synchronize()
    compare_encode(inp, u32_host(d.codes), d.meta_host(), all_units(w), w.N)
    ores = O.decode_all(inp, codes, meta, gqa_sum=gsum)
    s = Dev(inp, flags=flags)
    s.load_state(codes, meta)
    s.select(step=0)
    assert s.status() == hhr.HHR_OK
    compare_select(w, ores, _host(s.page_idx), _host(s.tok_idx), _host(s.n_sel), all_units(w),
                   dbg_U=_host(s.dbg_U), dbg_D=_host(s.dbg_D), name=f"select {variant} {name}")
    d.decode(0)
    assert d.status() == hhr.HHR_OK
    compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), all_units(w),
                   inp=inp, step=0, out_g=_host(d.out), name=f"fused {variant} {name}")


def test_variant_flags_are_validated():
    inp, _, _ = case("tiny_4k")
    w = inp.w
    d = Dev(inp)
    bad = hhr.make_dims(w.B, w.Hq, w.Hkv, w.d, w.bits, w.page, w.n_cap, 8)
    with pytest.raises(hhr.HhrError) as e:
        hhr.hhr_encode_keys(bad, d.K, d.R, d.W, 0, w.N, d.codes, d.meta)
    assert e.value.status == hhr.HHR_ERR_INVALID_ARG
    # the summed distances need wider histograms: a larger workspace
    sumd = hhr.make_dims(w.B, w.Hq, w.Hkv, w.d, w.bits, w.page, w.n_cap, hhr.HHR_FLAG_GQA_SUM)
    assert hhr.hhr_workspace_size(sumd, w.P, w.k) >= hhr.hhr_workspace_size(d.dims, w.P, w.k)


# --------------------------------------------------------- dense comparator

def _dense_ref(inp, units, n_valid, step=0):
    w = inp.w
    r = w.r
    out = np.zeros((w.B, w.Hq, w.d), np.float32)
    for (b, g) in units:
        out[b, g * r:(g + 1) * r] = O.attend(inp.q[step, b, g * r:(g + 1) * r], inp.K[b, g], inp.V[b, g],
                                             np.arange(n_valid, dtype=np.int32), 1.0 / np.sqrt(w.d))
    return out


@pytest.mark.parametrize("name,n_valid", [("tiny_4k", 4096), ("llama_20k_ragged", 20003),
                                          ("gqa8", 3000), ("gqa2", 2999), ("b256_s32", 9001),
                                          ("tiny_4k", 0), ("tiny_4k", 1), ("tiny_4k", 17)])
def test_dense_attend_matches_oracle(name, n_valid):
    """hhr_dense_attend = softmax attention over every valid key (the oracle's
    attention with the full index list)."""
    inp, _, _ = case(name)
    w = inp.w
    d = Dev(inp)
    hhr.hhr_dense_attend(d.dims, d.q[0], d.K, d.V, n_valid, d.scale, d.out, d.ws)
    assert d.status() == hhr.HHR_OK
    err = compare_out(w, _dense_ref(inp, all_units(w), n_valid), _host(d.out), all_units(w))
    print(name, n_valid, "dense max abs err", err)


# ------------------------------------------------------------------ edge cases

@pytest.mark.parametrize("n_valid", [0, 1, 5, 16, 17, 333, 4096])
def test_edge_context_lengths(n_valid):
    inp, codes, meta = case("tiny_4k")
    w = inp.w
    d = Dev(inp)
    d.load_state(codes, meta)
    # oracle on the (possibly truncated) context of the single unit
    res = O.decode_unit(inp.q[0, 0, 0:1], inp.R[0], inp.W[0], codes[0, 0], meta[0, 0],
                        inp.K[0, 0], inp.V[0, 0], n_valid, w.page, w.P, w.k, d.scale)
    ores = dict(page_idx=res["page_idx"][None, None], tok_idx=res["tok_idx"][None, None],
                n_sel=np.array([[res["n_sel"]]]), out=res["out"][None],
                D=res["D"][None, None], q_ambiguous=np.array([[res["q_ambiguous"]]]),
                U={(0, 0): res["U"]})
    d.decode(0, n_valid=n_valid)
    assert d.status() == hhr.HHR_OK
    compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), [(0, 0)],
                   inp=inp, step=0, out_g=_host(d.out), name=f"context {n_valid}")
    d.select(0, n_valid=n_valid)
    compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), [(0, 0)],
                   dbg_U=_host(d.dbg_U), dbg_D=_host(d.dbg_D), name=f"context {n_valid} select")


@pytest.mark.parametrize("P,k", [(10_000, 128), (32, 100_000), (10_000, 100_000), (1, 1)])
def test_budget_extremes(P, k):
    inp, codes, meta = case("llama_20k_ragged")
    w = inp.w
    ores = O.decode_all(inp, codes, meta, P=P, k=k)
    d = Dev(inp, P=P, k=k)
    d.load_state(codes, meta)
    d.decode(0)
    assert d.status() == hhr.HHR_OK
    compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), all_units(w),
                   P=P, k=k, inp=inp, step=0, out_g=_host(d.out), name=f"budgets P={P} k={k}")


def test_degenerate_all_equal_scores():
    """Zero keys: every page bound is equal and every code is zero, so the
    selection is decided by the index tie-breaks alone."""
    w = scaled(get("llama8b_32k"), Hq=8, Hkv=2, N=3000, P=50, k=300, planted=0)
    inp = make_inputs(w)
    inp.K[:] = 0
    codes, meta, _ = O.encode_all(inp)
    ores = O.decode_all(inp, codes, meta)
    d = Dev(inp)
    d.encode(0, w.N)
    d.decode(0)
    assert d.status() == hhr.HHR_OK
    rep = compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), all_units(w),
                         inp=inp, step=0, out_g=_host(d.out), name="all-equal scores")
    assert rep["units_exact"] == rep["units"]        # no near-cutoff freedom: every tie is by index
    assert _host(d.page_idx)[0, 0].tolist() == list(range(50))


def test_workspace_is_reusable_and_results_repeat():
    inp, codes, meta = case("llama_20k_ragged")
    d = Dev(inp)
    d.load_state(codes, meta)
    outs = []
    for _ in range(3):
        d.decode(0)
        outs.append((_host(d.tok_idx).copy(), _host(d.out).copy()))
    assert d.status() == hhr.HHR_OK
    for t, o in outs[1:]:
        assert np.array_equal(t, outs[0][0]) and np.array_equal(o, outs[0][1])
    # the per-unit counters (4 bytes each, at offset 256) are back to zero
    units = inp.w.B * inp.w.Hkv
    assert int(d.ws[256:256 + 4 * units].sum().item()) == 0


@pytest.mark.parametrize("where", [1, 2])
def test_decode_unit_barrier_timeout(where):
    """The decode kernel's own inter-CTA wait (after the page bounds, or after
    the distances) is made unmeetable through the test hook: every CTA of
    every unit gives up after a short spin, the status word says so, and the
    next call, on a zero-filled workspace, is correct."""
    inp, codes, meta = case("llama_20k_ragged")
    w = inp.w
    d = Dev(inp)
    d.load_state(codes, meta)
    hhr.hhr_test_arm_timeout(where, 200_000)
    d.decode(0)
    torch.cuda.synchronize()                            # the kernel has ended
    assert d.status() == hhr.HHR_ERR_TIMEOUT
    d.ws.zero_()
    d.decode(0)
    assert d.status() == hhr.HHR_OK
    ores = O.decode_all(inp, codes, meta)
    compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), all_units(w),
                   inp=inp, step=0, out_g=_host(d.out), name=f"after barrier-{where} timeout")


def test_encode_pipeline_timeout():
    """The key-encoding kernel's pipeline wait is made unmeetable through the
    test hook: the kernel gives up, leaves no MMA in flight, frees its tensor
    memory and reports HHR_ERR_TIMEOUT once; the next encoding is correct."""
    inp, _, _ = case("tiny_4k")
    w = inp.w
    d = Dev(inp)
    assert hhr.hhr_encode_status() == hhr.HHR_OK
    hhr.hhr_test_arm_timeout(3, 200_000)
    d.encode(0, w.N)
    torch.cuda.synchronize()
    assert hhr.hhr_encode_status() == hhr.HHR_ERR_TIMEOUT
    assert hhr.hhr_encode_status() == hhr.HHR_OK         # cleared by the read
    d.encode(0, w.N)
    torch.cuda.synchronize()
    assert hhr.hhr_encode_status() == hhr.HHR_OK
    compare_encode(inp, u32_host(d.codes), bits_host(d.meta), all_units(w), w.N)


def test_timeout_hook_rejects_unknown_site():
    with pytest.raises(hhr.HhrError):
        hhr.hhr_test_arm_timeout(7, 1000)


def test_host_buffer_step_matches_device_step():
    """hhr_decode_step_host (pinned host query in, host output back, blocking)
    gives what hhr_decode_step gives, through a prepared call."""
    from kv_cache_retrieval_b200 import _binding as Bnd
    inp, codes, meta = case("llama_20k_ragged")
    w = inp.w
    d = Dev(inp)
    d.load_state(codes, meta)
    d.decode(0)
    ref_out, ref_tok = _host(d.out).copy(), _host(d.tok_idx).copy()
    q_pin = d.q[0].cpu().pin_memory()
    out_pin = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(d.q[0])
    d.out.fill_(float("nan"))
    call = Bnd.prepare("hhr_decode_step_host", d.dims, q_pin, q_dev, d.R, d.W, d.codes, d.meta, d.K,
                       d.V, w.N, d.P, d.k, d.scale, d.page_idx, d.tok_idx, d.n_sel, d.out, out_pin,
                       d.ws, d.ws.numel(), torch.cuda.current_stream().cuda_stream)
    for _ in range(3):   # the first call runs on the stream, the others replay its graph
        call()
        assert np.array_equal(out_pin.numpy(), ref_out)
        assert np.array_equal(_host(d.tok_idx), ref_tok)
    # a new query in the same pinned buffer: the replay copies what is there now
    q2 = torch.roll(d.q[0], shifts=1, dims=1).contiguous()
    hhr.hhr_decode_step(d.dims, q2, d.R, d.W, d.codes, d.meta, d.K, d.V, w.N, d.P, d.k, d.scale,
                        d.page_idx, d.tok_idx, d.n_sel, d.out, d.ws)
    ref2 = _host(d.out).copy()
    assert not np.array_equal(ref2, ref_out)
    q_pin.copy_(q2.cpu())
    call()
    assert np.array_equal(out_pin.numpy(), ref2)
    assert d.status() == hhr.HHR_OK


# -------------------------------------------------------------- full sizes

FULL_SAMPLES = {
    "llama8b_32k": [(0, 0), (0, 5)],
    "llama8b_128k": [(0, 3), (0, 7)],
    "batch8_64k_b256": [(0, 0), (5, 2), (7, 7)],
    "qwen8b_128k_rope": [(1, 4), (3, 0)],
    "llama8b_128k_paper": [(0, 1), (0, 6)],
}


@pytest.mark.slow
@pytest.mark.parametrize("name", list(FULL_SAMPLES))
def test_full_size_sampled_units(name):
    w = get(name)
    inp = make_inputs(w)
    units = FULL_SAMPLES[name]
    d = Dev(inp)
    d.encode(0, w.N)
    codes = np.zeros((w.B, w.Hkv, w.n_cap, w.words), np.uint32)
    meta = np.zeros((w.B, w.Hkv, w.np_cap, 2, w.d), np.uint16)
    O.encode_all(inp, 0, w.N, codes=codes, meta=meta, units=units)
    steps = [0] if not w.appends else list(range(w.appends))
    for step in steps:
        if w.appends:
            d.encode(w.N + step, w.N + step + 1)
            O.encode_all(inp, w.N + step, w.N + step + 1, codes=codes, meta=meta, units=units)
        d.decode(step)
        if step in (0, steps[-1]):
            ores = O.decode_all(inp, codes, meta, step=step, units=units)
            rep = compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), units,
                                 inp=inp, step=step, out_g=_host(d.out), name=f"full {name} step {step}")
            print(name, step, rep)
            # the attention kernel alone, on the oracle's own indices, in the
            # launch configuration of this workload
            tok = torch.from_numpy(ores["tok_idx"]).cuda()
            nsel = torch.from_numpy(ores["n_sel"]).cuda()
            d.attend(step, tok, nsel)
            err = compare_out(w, ores["out"], _host(d.out), units)
            print(name, step, "attention on oracle indices, max abs err", err)
    assert d.status() == hhr.HHR_OK
    torch.cuda.synchronize()
    rep = compare_encode(inp, u32_host(d.codes), bits_host(d.meta), units, inp.n_valid(steps[-1]))
    print(name, rep)


@pytest.mark.slow
@pytest.mark.parametrize("variant", ["meta_f32", "gqa_sum"])
def test_full_size_variants_sampled_units(variant):
    """The variants at 128K in the launch configuration the benchmark times,
    on sampled units (GPU encode, fused step)."""
    w = get("llama8b_128k")
    inp = make_inputs(w)
    units = [(0, 2), (0, 5)]
    flags = VARIANTS[variant]
    f32 = bool(flags & hhr.HHR_FLAG_META_F32)
    d = Dev(inp, flags=flags)
    d.encode(0, w.N)
    d.decode(0)
    codes, meta, _ = O.encode_all(inp, 0, w.N, units=units, meta_f32=f32)
    ores = O.decode_all(inp, codes, meta, units=units, gqa_sum=bool(flags & hhr.HHR_FLAG_GQA_SUM))
    rep = compare_select(w, ores, _host(d.page_idx), _host(d.tok_idx), _host(d.n_sel), units,
                         inp=inp, step=0, out_g=_host(d.out), name=f"full {variant} llama8b_128k")
    print(variant, rep)
    assert d.status() == hhr.HHR_OK
    torch.cuda.synchronize()
    compare_encode(inp, u32_host(d.codes), d.meta_host(), units, w.N)


@pytest.mark.slow
def test_full_size_dense_attend_sampled_units():
    """The dense comparator at 128K in the launch configuration the benchmark
    times (every unit runs; two are checked)."""
    w = get("llama8b_128k")
    inp = make_inputs(w)
    units = [(0, 1), (0, 6)]
    d = Dev(inp)
    hhr.hhr_dense_attend(d.dims, d.q[0], d.K, d.V, w.N, d.scale, d.out, d.ws)
    assert d.status() == hhr.HHR_OK
    err = compare_out(w, _dense_ref(inp, units, w.N), _host(d.out), units)
    print("dense 128K max abs err", err)
