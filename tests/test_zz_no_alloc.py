"""GPU tests of pkv_decode_noalloc, the decode entry point for callers that
cannot allocate device memory (it keeps its split-KV scratch in a fixed array
inside the library instead of a caller-allocated workspace).

Every call goes through the C ABI. Results are compared with the float64
oracle and with the regular path (pkv_plan_create / pkv_plan_upload /
pkv_run) on the same inputs, within the tolerances the parity tests use. The
first test makes two calls in a row with different batches: the second call
reuses the scratch the first one left behind, so stale partial states would
show up as a mismatch. This file is collected last so a run that stops at its
first failure has run every other test already; it also passes on its own in
a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
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


def _noalloc(p, dev, max_kv_len, with_lse=True):
    lib, fn = _noalloc_fn()
    q, k, v = p.q.to(dev), p.k_cache.to(dev), p.v_cache.to(dev)
    indptr = torch.from_numpy(p.kv_indptr.astype(np.int32)).to(dev)
    idx = torch.from_numpy(p.kv_indices.astype(np.int32)).to(dev)
    last = torch.from_numpy(p.kv_last_page_len.astype(np.int32)).to(dev)
    o = torch.full((p.batch, p.num_qo_heads, p.head_dim), 7.0, dtype=torch.bfloat16, device=dev)
    lse = torch.full((p.batch, p.num_qo_heads), 7.0, dtype=torch.float32, device=dev) if with_lse else None
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), indptr.data_ptr(), idx.data_ptr(), last.data_ptr(),
            p.batch, p.num_qo_heads, p.num_kv_heads, p.head_dim, p.page_size, max_kv_len, p.sm_scale,
            o.data_ptr(), lse.data_ptr() if with_lse else None, torch.cuda.current_stream().cuda_stream)
    assert st == pkv.PKV_OK, lib.pkv_last_error().decode()
    return o, lse


def _close(o, lse, o_ref, lse_ref):
    o = o.float().cpu().double().numpy()
    o_ref = o_ref.float().cpu().double().numpy() if hasattr(o_ref, "cpu") else o_ref
    assert np.all(np.isfinite(o))
    assert np.all(np.abs(o - o_ref) <= ATOL_O + RTOL_O * np.abs(o_ref)), np.abs(o - o_ref).max()
    if lse is None:
        return
    l = lse.cpu().double().numpy()
    l_ref = lse_ref.cpu().double().numpy() if hasattr(lse_ref, "cpu") else lse_ref
    assert np.array_equal(np.isneginf(l), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    assert np.all(np.abs(l[fin] - l_ref[fin]) <= ATOL_LSE), np.abs(l[fin] - l_ref[fin]).max()


def _oracle(p):
    return oracle.paged_attention(p.q, p.k_cache, p.v_cache, p.qo_indptr, p.kv_indptr, p.kv_indices,
                                  p.kv_last_page_len, p.page_size, False, p.sm_scale)


def _decode_problem(name, kv, hq, hk, d, ps, seed):
    return W.make_problem(name, [1] * len(kv), kv, num_qo_heads=hq, num_kv_heads=hk, head_dim=d, page_size=ps,
                          causal=False, seed=seed)


def test_noalloc_decode_matches_regular_path_twice():
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    # call 1: few long requests, so the KV of each (request, kv head) is split
    p1 = _decode_problem("noalloc_a", [3000, 1000, 77], 32, 8, 128, 16, 501)
    # call 2: another batch and shape; reads only what it wrote itself
    p2 = _decode_problem("noalloc_b", [1900, 5, 640, 1, 1300], 16, 4, 128, 1, 502)
    for p, max_kv in ((p1, 3000), (p2, 1900)):
        o_ref, lse_ref = _regular(p, dev)
        o, lse = _noalloc(p, dev, max_kv)
        torch.cuda.synchronize()
        _close(o, lse, o_ref, lse_ref)
        _close(o, lse, *_oracle(p))


def test_noalloc_kv_len_above_max_kv_len():
    """max_kv_len only sizes the split: keys past it go to the last chunk, exactly."""
    p = _decode_problem("noalloc_long", [3000, 2100, 9], 16, 2, 128, 16, 503)
    o, lse = _noalloc(p, torch.device("cuda", 0), 700)
    torch.cuda.synchronize()
    _close(o, lse, *_oracle(p))


def test_noalloc_single_chunk_head_dim_64_without_lse():
    """max_kv_len <= 256 gives one chunk: O is written directly, no merge, no scratch;
    head_dim 64 and a NULL lse."""
    p = _decode_problem("noalloc_one", [256, 1, 100, 0], 12, 4, 64, 4, 504)
    o, _ = _noalloc(p, torch.device("cuda", 0), 256, with_lse=False)
    torch.cuda.synchronize()
    _close(o, None, *_oracle(p))


def test_noalloc_largest_scratch_use():
    """The split rule's largest scratch use on this GPU: just under four CTAs per SM
    worth of (request, kv head) pairs, each split in two (group 16, head_dim 128)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    hk = 3
    batch = (4 * sms - 1) // hk
    rng = np.random.default_rng(505)
    kv = rng.integers(300, 600, batch).tolist()
    p = _decode_problem("noalloc_big", kv, 16 * hk, hk, 128, 16, 505)
    o, lse = _noalloc(p, torch.device("cuda", 0), 600)
    torch.cuda.synchronize()
    _close(o, lse, *_oracle(p))


def test_noalloc_rejects_unsupported_shapes_before_launch():
    """Shapes and pointers it does not handle are refused on the host; no kernel is launched."""
    lib, fn = _noalloc_fn()
    dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
    ptr = dummy.data_ptr()
    # 32 query heads per kv head (above 16)
    st = fn(ptr, ptr, ptr, ptr, ptr, ptr, 1, 64, 2, 128, 16, 64, 0.1, ptr, ptr, None)
    assert st == pkv.PKV_EUNSUPPORTED and "16" in lib.pkv_last_error().decode()
    # page size not a power of two
    st = fn(ptr, ptr, ptr, ptr, ptr, ptr, 1, 8, 2, 128, 24, 64, 0.1, ptr, ptr, None)
    assert st == pkv.PKV_EUNSUPPORTED
    # q not 16-byte aligned
    st = fn(ptr + 8, ptr, ptr, ptr, ptr, ptr, 1, 8, 2, 128, 16, 64, 0.1, ptr, ptr, None)
    assert st == pkv.PKV_EINVAL and "aligned" in lib.pkv_last_error().decode()
    # a batch beyond the launch grid's limit
    st = fn(ptr, ptr, ptr, ptr, ptr, ptr, 70000, 8, 2, 128, 16, 64, 0.1, ptr, ptr, None)
    assert st == pkv.PKV_EUNSUPPORTED and "65535" in lib.pkv_last_error().decode()
    torch.cuda.synchronize()
    assert torch.all(dummy == 0)
