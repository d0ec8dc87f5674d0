"""GPU test of pkv_decode_noalloc, the decode entry point for callers that
cannot allocate device memory (it keeps its split-KV scratch in a fixed array
inside the library instead of a caller-allocated workspace).

It is called through the C ABI and compared with the regular path
(pkv_plan_create / pkv_plan_upload / pkv_run) on the same inputs, within the
tolerances the parity tests use, on two calls in a row with different batches:
the second call reuses the scratch the first one left behind, so stale partial
states would show up as a mismatch. This file is collected last so a run that
stops at its first failure has run every other test already; it also passes on
its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_attention_38_b200 as pkv
from paged_kv_attention_38_b200 import workloads as W

pytestmark = pytest.mark.gpu

ATOL_O, RTOL_O, ATOL_LSE = 1e-2, 1e-2, 1e-3


def _noalloc_fn():
    lib = pkv.load_library()
    fn = lib.pkv_decode_noalloc
    P = ctypes.c_void_p
    i32 = ctypes.c_int32
    fn.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, ctypes.c_float, P, P, P]
    fn.restype = ctypes.c_int
    return lib, fn


def _regular(p, dev):
    idx = torch.from_numpy(p.kv_indices.astype(np.int32)).to(dev)
    pl = pkv.plan(p.qo_indptr, p.kv_indptr, idx, p.kv_last_page_len, p.num_qo_heads, p.num_kv_heads,
                  p.head_dim, p.page_size, False, p.sm_scale)
    assert pl.kind == pkv.KIND_DECODE
    return pkv.run(pl, p.q.to(dev), p.k_cache.to(dev), p.v_cache.to(dev))


def _noalloc(p, dev, max_kv_len):
    lib, fn = _noalloc_fn()
    q, k, v = p.q.to(dev), p.k_cache.to(dev), p.v_cache.to(dev)
    indptr = torch.from_numpy(p.kv_indptr.astype(np.int32)).to(dev)
    idx = torch.from_numpy(p.kv_indices.astype(np.int32)).to(dev)
    last = torch.from_numpy(p.kv_last_page_len.astype(np.int32)).to(dev)
    o = torch.full((p.batch, p.num_qo_heads, p.head_dim), 7.0, dtype=torch.bfloat16, device=dev)
    lse = torch.full((p.batch, p.num_qo_heads), 7.0, dtype=torch.float32, device=dev)
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), indptr.data_ptr(), idx.data_ptr(), last.data_ptr(),
            p.batch, p.num_qo_heads, p.num_kv_heads, p.head_dim, p.page_size, max_kv_len, p.sm_scale,
            o.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == pkv.PKV_OK, lib.pkv_last_error().decode()
    return o, lse


def _close(o, lse, o_ref, lse_ref):
    o, o_ref = o.float().cpu().double().numpy(), o_ref.float().cpu().double().numpy()
    assert np.all(np.abs(o - o_ref) <= ATOL_O + RTOL_O * np.abs(o_ref)), np.abs(o - o_ref).max()
    l, l_ref = lse.cpu().double().numpy(), lse_ref.cpu().double().numpy()
    assert np.array_equal(np.isneginf(l), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    assert np.all(np.abs(l[fin] - l_ref[fin]) <= ATOL_LSE), np.abs(l[fin] - l_ref[fin]).max()


def test_noalloc_decode_matches_regular_path_twice():
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    # call 1: few long requests, so the KV of each (request, kv head) is split
    p1 = W.make_problem("noalloc_a", [1] * 3, [3000, 1000, 77], num_qo_heads=32, num_kv_heads=8,
                        head_dim=128, page_size=16, causal=False, seed=501)
    # call 2: another batch and shape; reads only what it wrote itself
    p2 = W.make_problem("noalloc_b", [1] * 5, [1900, 5, 640, 1, 1300], num_qo_heads=16, num_kv_heads=4,
                        head_dim=128, page_size=1, causal=False, seed=502)
    for p, max_kv in ((p1, 3000), (p2, 1900)):
        o_ref, lse_ref = _regular(p, dev)
        o, lse = _noalloc(p, dev, max_kv)
        torch.cuda.synchronize()
        _close(o, lse, o_ref, lse_ref)


def test_noalloc_rejects_unsupported_shapes_before_launch():
    """Shapes it does not handle are refused on the host; no kernel is launched."""
    lib, fn = _noalloc_fn()
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    ptr = dummy.data_ptr()
    # 32 query heads per kv head (above 16)
    st = fn(ptr, ptr, ptr, ptr, ptr, ptr, 1, 64, 2, 128, 16, 64, 0.1, ptr, ptr, None)
    assert st == pkv.PKV_EUNSUPPORTED and "16" in lib.pkv_last_error().decode()
    # page size not a power of two
    st = fn(ptr, ptr, ptr, ptr, ptr, ptr, 1, 8, 2, 128, 24, 64, 0.1, ptr, ptr, None)
    assert st == pkv.PKV_EUNSUPPORTED
