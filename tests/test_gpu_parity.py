"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Tolerances (stated numbers for this path): bf16 O elementwise
|o - ref| <= 1e-2 + 1e-2 |ref|; fp32 base-2 LSE |lse - ref| <= 1e-3; rows that
see no key must give O = 0 and LSE = -inf exactly.
"""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
import paged_kv_attention_38_b200 as pkv
from paged_kv_attention_38_b200 import workloads as W

pytestmark = pytest.mark.gpu

ATOL_O, RTOL_O, ATOL_LSE = 1e-2, 1e-2, 1e-3


def assert_parity(o, lse, o_ref, lse_ref, what=""):
    o = o.float().cpu().double().numpy() if hasattr(o, "cpu") else o
    lse = lse.float().cpu().double().numpy() if hasattr(lse, "cpu") else lse
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite O"
    err = np.abs(o - o_ref)
    bad = err > ATOL_O + RTOL_O * np.abs(o_ref)
    assert not bad.any(), (f"{what}: O mismatch at {np.argwhere(bad)[:5].tolist()}, max abs err "
                           f"{err.max():.3e}, ref there {o_ref[bad][:3]}")
    ninf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf_ref), f"{what}: -inf LSE rows differ"
    fin = ~ninf_ref
    lerr = np.abs(lse[fin] - lse_ref[fin]) if fin.any() else np.zeros(1)
    assert lerr.max() <= ATOL_LSE, f"{what}: LSE max abs err {lerr.max():.3e}"


def to_dev(p: W.PagedProblem):
    d = {}
    for name in ("q", "k_cache", "v_cache", "q_nope", "q_pe", "ckv_cache", "kpe_cache"):
        t = getattr(p, name)
        if t is not None:
            d[name] = t.cuda()
    d["kv_indices"] = torch.from_numpy(p.kv_indices.astype(np.int32)).cuda()
    return d


def gpu_run(p: W.PagedProblem, **plan_kw):
    d = to_dev(p)
    pl = pkv.plan(p.qo_indptr, p.kv_indptr, d["kv_indices"], p.kv_last_page_len, p.num_qo_heads,
                  p.num_kv_heads, p.head_dim, p.page_size, p.causal, p.sm_scale, **plan_kw)
    o, lse = pkv.run(pl, d["q"], d["k_cache"], d["v_cache"])
    torch.cuda.synchronize()
    assert pkv.device_status(pl) == 0
    return o, lse, pl


def oracle_run(p: W.PagedProblem):
    return oracle.paged_attention(p.q, p.k_cache, p.v_cache, p.qo_indptr, p.kv_indptr, p.kv_indices,
                                  p.kv_last_page_len, p.page_size, p.causal, p.sm_scale)


# --------------------------------------------------------------------------- prefill

def test_tiny_prefill():
    p = W.tiny_prefill()
    o, lse, pl = gpu_run(p)
    assert pl.kind == pkv.KIND_PREFILL
    assert_parity(o, lse, *oracle_run(p), what="tiny")


SWEEP = [
    # qo_lens, kv_lens, hq, hk, d, page, causal
    ([1, 127, 128, 129, 300], [1, 127, 128, 129, 300], 4, 4, 64, 16, True),
    ([200, 33], [200, 33], 16, 1, 128, 64, True),
    ([70, 250], [70, 250], 8, 2, 128, 1, True),
    ([64, 190], [64, 190], 4, 1, 128, 2, True),
    ([37, 100], [137, 400], 4, 2, 128, 16, True),     # chunked prefill: qo < kv (bottom-right)
    ([90, 5], [60, 5], 2, 1, 64, 8, True),            # qo > kv: first rows see no key
    ([50, 0, 80], [50, 30, 0], 4, 1, 64, 4, True),    # a request with no queries, one with no keys
    ([45, 160], [300, 160], 8, 8, 128, 32, False),    # non-causal MHA
    ([130], [130], 128, 1, 64, 16, True),             # group of 128 heads: one token per tile
]


@pytest.mark.parametrize("case", SWEEP, ids=lambda c: f"q{sum(c[0])}_h{c[2]}_{c[3]}_d{c[4]}_p{c[5]}_c{int(c[6])}")
def test_prefill_sweep(case):
    qo, kv, hq, hk, d, ps, causal = case
    p = W.make_problem("sweep", qo, kv, num_qo_heads=hq, num_kv_heads=hk, head_dim=d, page_size=ps,
                       causal=causal, seed=zlib.crc32(str(case).encode()) % 10000, pool_pages=None)
    o, lse, _ = gpu_run(p)
    assert_parity(o, lse, *oracle_run(p), what=str(case))


# Shapes the header admits beyond the powers of two above. Groups that do not
# divide the 128-row tile run the cp.async Q loader (packed rows cross token
# boundaries inside a tile); page sizes 128 and 256 run the TMA path whose box
# covers a whole KV tile inside one page (page_size >= tile).
WIDE = [
    # qo_lens, kv_lens, hq, hk, d, page, causal, forced kv chunk (0 = planner's)
    ([300, 77], [300, 77], 24, 8, 128, 16, True, 0),        # group 3, ragged tails
    ([150, 41, 9], [150, 41, 9], 40, 8, 128, 64, True, 0),  # group 5
    ([100, 260], [100, 260], 12, 1, 64, 8, True, 0),         # group 12 on one kv head
    ([70, 333], [170, 333], 24, 8, 128, 16, True, 128),     # group 3, chunked prefill, split KV
    ([1, 1, 1], [500, 33, 2000], 20, 1, 128, 16, False, 0), # group 20 decode batch: the prefill kernel
    ([200, 37], [200, 300], 16, 4, 128, 128, True, 0),      # page_size 128: one page per KV tile
    ([300, 129], [300, 129], 16, 4, 128, 256, True, 0),     # page_size 256: two KV tiles per page
    ([90, 250], [700, 250], 8, 2, 64, 256, True, 128),      # page_size 256, chunks starting mid-page
    ([160], [160], 12, 4, 128, 128, False, 0),              # group 3 with page_size 128, non-causal
    ([200, 45], [200, 45], 24, 8, 128, 1, True, 0),         # group 3, page_size 1: cp.async Q + row gather
    ([120, 300], [220, 300], 20, 4, 64, 2, True, 128),      # group 5, page_size 2, chunked, split KV (fp32 partials)
]


@pytest.mark.parametrize("case", WIDE, ids=lambda c: f"h{c[2]}_{c[3]}_d{c[4]}_p{c[5]}_c{int(c[6])}_k{c[7]}")
def test_prefill_wide_shapes(case):
    qo, kv, hq, hk, d, ps, causal, chunk = case
    p = W.make_problem("wide", qo, kv, num_qo_heads=hq, num_kv_heads=hk, head_dim=d, page_size=ps,
                       causal=causal, seed=zlib.crc32(str(case).encode()) % 10000)
    o, lse, pl = gpu_run(p, **({"kv_chunk": chunk} if chunk else {}))
    assert pl.kind == pkv.KIND_PREFILL
    if chunk:
        assert pl.num_merges > 0
    assert_parity(o, lse, *oracle_run(p), what=str(case))


@pytest.mark.parametrize("chunk", [128, 384])
def test_prefill_split_kv_matches(chunk):
    p = W.make_problem("split", [300, 40], [900, 700], num_qo_heads=8, num_kv_heads=2, head_dim=128,
                       page_size=16, causal=True, seed=77)
    o, lse, pl = gpu_run(p, kv_chunk=chunk)
    assert pl.num_merges > 0
    assert_parity(o, lse, *oracle_run(p), what=f"split {chunk}")


def test_output_guard_regions():
    """Writes stay inside o / lse: guard rows before and after are untouched."""
    p = W.make_problem("guard", [33, 100], [33, 100], num_qo_heads=4, num_kv_heads=1, head_dim=64,
                       page_size=16, causal=True, seed=5)
    d = to_dev(p)
    pl = pkv.plan(p.qo_indptr, p.kv_indptr, d["kv_indices"], p.kv_last_page_len, 4, 1, 64, 16, True, p.sm_scale,
                  kv_chunk=128)
    tq, g = p.total_q, 7
    o_buf = torch.full((tq + 2 * g, 4, 64), 123.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((tq + 2 * g, 4), 77.0, dtype=torch.float32, device="cuda")
    pkv.run(pl, d["q"], d["k_cache"], d["v_cache"], o=o_buf[g:g + tq], lse=l_buf[g:g + tq])
    torch.cuda.synchronize()
    assert torch.all(o_buf[:g] == 123.0) and torch.all(o_buf[g + tq:] == 123.0)
    assert torch.all(l_buf[:g] == 77.0) and torch.all(l_buf[g + tq:] == 77.0)
    assert_parity(o_buf[g:g + tq], l_buf[g:g + tq], *oracle_run(p), what="guard")


def test_pool_permutation_bitwise_on_gpu():
    """The physical page order does not change the GPU result at all."""
    p = W.make_problem("perm", [150, 260], [150, 260], num_qo_heads=8, num_kv_heads=2, head_dim=128,
                       page_size=1, causal=True, seed=9)
    o1, l1, _ = gpu_run(p)
    n = p.k_cache.shape[0]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(3))
    p2 = W.PagedProblem(**{**p.__dict__})
    p2.k_cache = torch.empty_like(p.k_cache)
    p2.v_cache = torch.empty_like(p.v_cache)
    p2.k_cache[perm] = p.k_cache
    p2.v_cache[perm] = p.v_cache
    p2.kv_indices = perm.numpy()[p.kv_indices].astype(np.int32)
    o2, l2, _ = gpu_run(p2)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.slow
def test_gqa_prefill_full_size_sampled():
    """h16/kv1/d128/ps64 at full size, in the launch configuration the bench times;
    checked on sampled rows (first, last, page-boundary and random tokens)."""
    p = W.gqa_prefill()
    o, lse, _ = gpu_run(p)
    rng = np.random.default_rng(0)
    for b in range(p.batch):
        L = int(p.qo_lens[b])
        pos = sorted({0, 1, 63, 64, L // 2, L - 2, L - 1, *rng.integers(0, L, 3).tolist()})
        o_r, l_r = oracle.paged_attention_rows(p.q, p.k_cache, p.v_cache, p.qo_indptr, p.kv_indptr,
                                               p.kv_indices, p.kv_last_page_len, p.page_size, True,
                                               p.sm_scale, b, pos)
        rows = [int(p.qo_indptr[b]) + x for x in pos]
        assert_parity(o[rows], lse[rows], o_r, l_r, what=f"req {b}")


@pytest.mark.slow
@pytest.mark.parametrize("bl", [(16, 2048), (1, 8192)])
def test_sparse_vs_dense_sampled(bl):
    B, L = bl
    sp = W.sparse_vs_dense(B, L, contiguous=False)
    o, lse, _ = gpu_run(sp)
    rng = np.random.default_rng(1)
    for b in rng.choice(B, size=min(B, 2), replace=False).tolist():
        pos = sorted({0, L - 1, *rng.integers(0, L, 4).tolist()})
        o_r, l_r = oracle.paged_attention_rows(sp.q, sp.k_cache, sp.v_cache, sp.qo_indptr, sp.kv_indptr,
                                               sp.kv_indices, sp.kv_last_page_len, 1, True, sp.sm_scale, b, pos)
        rows = [int(sp.qo_indptr[b]) + x for x in pos]
        assert_parity(o[rows], lse[rows], o_r, l_r, what=f"sparse {bl} req {b}")
    # the dense (contiguous) layout of the same keys and values gives the same result
    de = W.sparse_vs_dense(B, L, contiguous=True)
    hk, d = sp.k_cache.shape[2], sp.k_cache.shape[3]
    idx_s = torch.from_numpy(sp.kv_indices.astype(np.int64))
    k = torch.empty_like(de.k_cache)
    v = torch.empty_like(de.v_cache)
    k.view(-1, hk, d)[:len(idx_s)] = sp.k_cache.view(-1, hk, d)[idx_s]
    v.view(-1, hk, d)[:len(idx_s)] = sp.v_cache.view(-1, hk, d)[idx_s]
    de.k_cache, de.v_cache, de.q = k, v, sp.q
    o2, l2, _ = gpu_run(de)
    assert_parity(o2, l2, o.float().cpu().double().numpy(), lse.cpu().double().numpy(), what="dense vs sparse")


# --------------------------------------------------------------------------- decode

DECODE_SWEEP = [
    # kv_lens, hq, hk, d, page
    ([1, 63, 64, 65, 3000], 32, 8, 128, 16),
    ([500, 1], 16, 1, 128, 64),
    ([129, 700], 8, 8, 64, 1),
    ([2000, 333, 4], 64, 4, 128, 2),
    ([1, 300, 1000], 24, 8, 128, 16),       # group 3
    ([77, 513, 2], 40, 8, 64, 128),         # group 5, page_size 128
    ([2000, 5], 12, 1, 128, 256),           # group 12, page_size 256
    ([900, 130], 6, 1, 128, 1),             # group 6, vector sparse
]


@pytest.mark.parametrize("case", DECODE_SWEEP, ids=lambda c: f"h{c[1]}_{c[2]}_d{c[3]}_p{c[4]}")
@pytest.mark.parametrize("split", [False, True])
def test_decode_sweep(case, split):
    kv, hq, hk, d, ps = case
    p = W.make_problem("dec", [1] * len(kv), kv, num_qo_heads=hq, num_kv_heads=hk, head_dim=d, page_size=ps,
                       causal=False, seed=sum(kv) % 997)
    o, lse, pl = gpu_run(p, **({"kv_chunk": 128} if split else {"disable_split_kv": True}))
    assert pl.kind == pkv.KIND_DECODE
    if split and max(kv) > 128:
        assert pl.num_merges > 0
    assert_parity(o, lse, *oracle_run(p), what=f"decode {case}")


@pytest.mark.slow
def test_decode_full_size():
    """b128/h32/kv8/d128/ps16, kv_len 1024..8192, the planner's default plan (the bench's launch
    configuration; it does not split this batch): every row."""
    p = W.paged_decode()
    o, lse, pl = gpu_run(p)
    assert pl.kind == pkv.KIND_DECODE
    assert_parity(o, lse, *oracle_run(p), what="decode full")


# --------------------------------------------------------------------------- FP8 E4M3 KV decode

def gpu_run_fp8(p: W.PagedProblem, k_scale=True, v_scale=True, **plan_kw):
    d = to_dev(p)
    plan_kw.setdefault("kv_fp8", True)
    pl = pkv.plan(p.qo_indptr, p.kv_indptr, d["kv_indices"], p.kv_last_page_len, p.num_qo_heads,
                  p.num_kv_heads, p.head_dim, p.page_size, p.causal, p.sm_scale, **plan_kw)
    ks = p.meta["k_scale"].cuda() if k_scale else None
    vs = p.meta["v_scale"].cuda() if v_scale else None
    o, lse = pkv.run_fp8_kv(pl, d["q"], d["k_cache"], d["v_cache"], ks, vs)
    torch.cuda.synchronize()
    assert pkv.device_status(pl) == 0
    return o, lse, pl


def oracle_fp8(p: W.PagedProblem, k_scale=True, v_scale=True):
    one = torch.ones(p.num_kv_heads)
    return oracle.paged_attention_quantized_kv(p.q, p.k_cache, p.v_cache, p.meta["k_scale"] if k_scale else one,
                                               p.meta["v_scale"] if v_scale else one, p.qo_indptr, p.kv_indptr,
                                               p.kv_indices, p.kv_last_page_len, p.page_size, p.causal, p.sm_scale)


FP8_DECODE = [
    # kv_lens, hq, hk, d, page, forced kv chunk (0 = planner's)
    ([1, 63, 64, 65, 700, 3000], 32, 8, 128, 16, 0),   # ragged tails, the longest request split
    ([0, 5, 129, 1000], 8, 8, 64, 1, 64),              # MHA, page_size 1, an empty request, all split
    ([300, 17], 16, 1, 128, 4, 0),                     # group 16 on one kv head
]


@pytest.mark.parametrize("case", FP8_DECODE, ids=lambda c: f"h{c[1]}_{c[2]}_d{c[3]}_p{c[4]}_k{c[5]}")
def test_fp8_kv_decode(case):
    kv, hq, hk, d, ps, chunk = case
    p = W.make_fp8_kv_problem("fp8dec", [1] * len(kv), kv, num_qo_heads=hq, num_kv_heads=hk, head_dim=d,
                              page_size=ps, seed=zlib.crc32(str(case).encode()) % 10000)
    o, lse, pl = gpu_run_fp8(p, **({"kv_chunk": chunk} if chunk else {}))
    assert pl.kind == pkv.KIND_DECODE
    if chunk:
        assert pl.num_merges > 0
    assert_parity(o, lse, *oracle_fp8(p), what=f"fp8 decode {case}")


def test_fp8_kv_decode_unit_scales():
    """NULL scales read as 1.0."""
    p = W.make_fp8_kv_problem("fp8dec1", [1, 1], [90, 400], num_qo_heads=8, num_kv_heads=2, head_dim=128,
                              page_size=16, seed=3)
    o, lse, _ = gpu_run_fp8(p, k_scale=False, v_scale=False)
    assert_parity(o, lse, *oracle_fp8(p, k_scale=False, v_scale=False), what="fp8 decode unit scales")


@pytest.mark.parametrize("qmul", [1e5, 1e-6])
def test_fp8_kv_decode_query_range(qmul):
    """Queries far outside the f16 range (|q| up to ~5e5, where f16 overflows) and
    deep in its subnormals (|q| ~ 1e-6): the kernel scales Q by a power of two
    before the f16 rounding. O is checked at the stated tolerance; with |q| ~ 1e5
    the LSE is ~1e5 and fp32 resolves it to ~1e-2, so there it is checked to
    1e-6 relative."""
    p = W.make_fp8_kv_problem("fp8range", [1, 1, 1], [300, 77, 1000], num_qo_heads=16, num_kv_heads=2,
                              head_dim=128, page_size=16, seed=int(qmul < 1) + 41)
    p.q = (p.q.float() * qmul).to(torch.bfloat16)
    o, lse, _ = gpu_run_fp8(p)
    o_ref, l_ref = oracle_fp8(p)
    if qmul > 1:
        assert np.all(np.isfinite(lse.cpu().numpy()))
        err = np.abs(lse.cpu().double().numpy() - l_ref)
        assert np.all(err <= 1e-3 + 1e-6 * np.abs(l_ref)), err.max()
        assert_parity(o, np.nan_to_num(l_ref), o_ref, np.nan_to_num(l_ref), what=f"fp8 q x {qmul}")
    else:
        assert_parity(o, lse, o_ref, l_ref, what=f"fp8 q x {qmul}")


def test_fp8_kv_prefill_needs_kv_fp8_plan():
    p = W.make_fp8_kv_problem("fp8pre", [4, 2], [40, 9], num_qo_heads=4, num_kv_heads=2, head_dim=128,
                              page_size=16, seed=4, causal=True)
    d = to_dev(p)
    pl = pkv.plan(p.qo_indptr, p.kv_indptr, d["kv_indices"], p.kv_last_page_len, 4, 2, 128, 16, True, p.sm_scale)
    with pytest.raises(Exception, match="kv_fp8"):
        pkv.run_fp8_kv(pl, d["q"], d["k_cache"], d["v_cache"])


FP8_PREFILL = [
    # qo_lens, kv_lens, hq, hk, d, page, causal, forced kv chunk (0 = planner's)
    ([70, 200], [70, 200], 8, 2, 128, 16, True, 0),        # page TMA path, causal GQA
    ([90, 33], [150, 33], 16, 1, 64, 1, True, 0),          # row gather, chunked prefill (qo < kv)
    ([45, 160], [300, 160], 8, 8, 128, 64, False, 128),    # MHA, non-causal, split KV
    ([100, 0, 64], [100, 20, 0], 12, 4, 128, 16, True, 0), # group 3 (cp.async Q), no queries / no keys
]


@pytest.mark.parametrize("case", FP8_PREFILL, ids=lambda c: f"h{c[2]}_{c[3]}_d{c[4]}_p{c[5]}_c{int(c[6])}_k{c[7]}")
def test_fp8_kv_prefill(case):
    """Prefill over the FP8 cache: the pages expanded to bf16 in the workspace, the
    tensor-core prefill on the copy with the per-head scales applied."""
    qo, kv, hq, hk, d, ps, causal, chunk = case
    p = W.make_fp8_kv_problem("fp8pre", qo, kv, num_qo_heads=hq, num_kv_heads=hk, head_dim=d, page_size=ps,
                              seed=zlib.crc32(str(case).encode()) % 10000, causal=causal)
    o, lse, pl = gpu_run_fp8(p, **({"kv_chunk": chunk} if chunk else {}))
    assert pl.kind == pkv.KIND_PREFILL
    if chunk:
        assert pl.num_merges > 0
    assert_parity(o, lse, *oracle_fp8(p), what=f"fp8 prefill {case}")


@pytest.mark.parametrize("qo", [[60, 1], [1, 1]], ids=["prefill", "decode"])
def test_fp8_kv_nan_codes_outside_the_keys(qo):
    """NaN codes in slots past a request's last key (in its last page and in pages
    no request lists) never reach the output."""
    p = W.make_fp8_kv_problem("fp8nan", qo, [60, 37], num_qo_heads=8, num_kv_heads=2, head_dim=128, page_size=16,
                              seed=21, causal=qo[0] > 1, pool_pages=12)
    valid = W._valid_slot_mask(p.kv_indptr, p.kv_indices, p.kv_last_page_len, p.page_size, p.num_pages)
    p.k_cache[~valid] = 0x7F
    p.v_cache[~valid] = 0xFF
    o, lse, _ = gpu_run_fp8(p)
    assert_parity(o, lse, *oracle_fp8(p), what=f"fp8 nan slots {qo}")


@pytest.mark.slow
def test_fp8_kv_decode_full_size_sampled():
    """The full FP8 decode batch (b128/h32/kv8/d128/ps16, kv_len U[1024, 8192]) in
    the bench's launch configuration; 12 requests checked against the oracle on a
    pool cut down to their own pages."""
    p = W.paged_decode_fp8()
    o, lse, pl = gpu_run_fp8(p)
    rng = np.random.default_rng(9)
    reqs = sorted({0, p.batch - 1, *rng.integers(0, p.batch, 10).tolist()})
    pages = [p.kv_indices[p.kv_indptr[b]:p.kv_indptr[b + 1]] for b in reqs]
    ids = np.concatenate(pages)
    sub_indptr = np.concatenate([[0], np.cumsum([len(x) for x in pages])]).astype(np.int32)
    sub_q = torch.stack([p.q[int(p.qo_indptr[b])] for b in reqs])
    o_ref, l_ref = oracle.paged_attention_quantized_kv(
        sub_q, p.k_cache[torch.from_numpy(ids.astype(np.int64))], p.v_cache[torch.from_numpy(ids.astype(np.int64))],
        p.meta["k_scale"], p.meta["v_scale"], np.arange(len(reqs) + 1, dtype=np.int32), sub_indptr,
        np.arange(len(ids), dtype=np.int32), p.kv_last_page_len[reqs], p.page_size, False, p.sm_scale)
    rows = [int(p.qo_indptr[b]) for b in reqs]
    assert_parity(o[rows], lse[rows], o_ref, l_ref, what="fp8 decode full")


# --------------------------------------------------------------------------- merge

def test_merge_state_kernels():
    g = torch.Generator().manual_seed(0)
    rows, dim = 300, 96
    oa = torch.randn(rows, dim, generator=g)
    ob = torch.randn(rows, dim, generator=g)
    la = torch.randn(rows, generator=g) * 4
    lb = torch.randn(rows, generator=g) * 4
    la[0] = -math.inf
    la[1] = lb[1] = -math.inf
    o, l = pkv.merge_state(oa.cuda(), la.cuda(), ob.cuda(), lb.cuda())
    o_ref, l_ref = oracle.merge_state(oa.numpy(), la.numpy(), ob.numpy(), lb.numpy())
    np.testing.assert_allclose(o.cpu().double().numpy(), o_ref, rtol=1e-5, atol=1e-5)
    assert np.array_equal(np.isneginf(l.cpu().numpy()), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    np.testing.assert_allclose(l.cpu().double().numpy()[fin], l_ref[fin], atol=1e-5)
    # n-way merge to bf16
    n = 5
    parts = torch.randn(n, rows, dim, generator=g)
    lses = torch.randn(n, rows, generator=g) * 3
    lses[:, 7] = -math.inf
    ob16, l16 = pkv.merge_states(parts.cuda(), lses.cuda())
    o_ref, l_ref = oracle.merge_states(list(parts.numpy()), list(lses.numpy()))
    assert_parity(ob16, l16, o_ref, l_ref, what="merge_states")


# --------------------------------------------------------------------------- MLA

def gpu_run_mla(p: W.PagedProblem, **plan_kw):
    d = to_dev(p)
    pl = pkv.plan_mla(p.qo_indptr, p.kv_indptr, d["kv_indices"], p.kv_last_page_len, p.num_qo_heads, 512, 64,
                      p.page_size, p.causal, p.sm_scale, **plan_kw)
    o, lse = pkv.run_mla(pl, d["q_nope"], d["q_pe"], d["ckv_cache"], d["kpe_cache"])
    torch.cuda.synchronize()
    assert pkv.device_status(pl) == 0
    return o, lse, pl


def oracle_mla(p: W.PagedProblem):
    return oracle.mla_paged_attention(p.q_nope, p.q_pe, p.ckv_cache, p.kpe_cache, p.qo_indptr, p.kv_indptr,
                                      p.kv_indices, p.kv_last_page_len, p.page_size, p.causal, p.sm_scale)


MLA_SWEEP = [
    # qo_lens, kv_lens, heads, page, causal
    ([7, 33], [7, 33], 16, 1, True),
    ([64, 130, 1], [64, 130, 1], 16, 1, True),
    ([40, 9], [100, 9], 16, 16, True),      # chunked prefill: qo < kv
    ([5, 3], [3, 0], 8, 1, True),           # qo > kv (rows with no key) and an empty request
    ([17, 80], [200, 80], 4, 4, False),
]


@pytest.mark.parametrize("case", MLA_SWEEP, ids=lambda c: f"q{sum(c[0])}_h{c[2]}_p{c[3]}_c{int(c[4])}")
def test_mla_sweep(case):
    qo, kv, h, ps, causal = case
    p = W.make_mla_problem("mla", qo, kv, num_heads=h, page_size=ps, causal=causal,
                           seed=zlib.crc32(str(case).encode()) % 10000)
    o, lse, pl = gpu_run_mla(p)
    assert pl.kind == pkv.KIND_MLA
    assert_parity(o, lse, *oracle_mla(p), what=f"mla {case}")


def test_mla_split_kv():
    p = W.make_mla_problem("mla_split", [30, 200], [700, 200], num_heads=16, page_size=1, causal=True, seed=12)
    o, lse, pl = gpu_run_mla(p, kv_chunk=128)
    assert pl.num_merges > 0
    assert_parity(o, lse, *oracle_mla(p), what="mla split")


MLA_DECODE = [
    # kv_lens, heads, page, forced kv chunk (0 = planner's)
    ([1, 63, 64, 65, 700, 3000], 16, 1, 0),   # ragged, the longest request split
    ([0, 5, 129, 1000], 8, 1, 64),            # fewer heads than MMA rows, an empty request, every request split
    ([40, 300], 16, 16, 0),                   # page_size 16
]


@pytest.mark.parametrize("case", MLA_DECODE, ids=lambda c: f"h{c[1]}_p{c[2]}_k{c[3]}")
def test_mla_decode_small(case):
    """MLA decode (one query token per request, non-causal) through the decode kernel."""
    kv, h, ps, chunk = case
    p = W.make_mla_problem("mla_dec", [1] * len(kv), kv, num_heads=h, page_size=ps, causal=False,
                           seed=zlib.crc32(str(case).encode()) % 10000)
    o, lse, pl = gpu_run_mla(p, **({"kv_chunk": chunk} if chunk else {}))
    assert pl.kind == pkv.KIND_MLA_DECODE
    if chunk:
        assert pl.num_merges > 0
    assert_parity(o, lse, *oracle_mla(p), what=f"mla decode {case}")


@pytest.mark.slow
def test_mla_decode_full_size():
    """h16/ckv512/kpe64/ps1 decode, batch 64, kv_len U[1024, 8192], in the bench's launch
    configuration: every row (64 tokens x 16 heads) against the oracle."""
    p = W.mla_decode()
    o, lse, _ = gpu_run_mla(p)
    assert_parity(o, lse, *oracle_mla(p), what="mla decode full")


@pytest.mark.slow
def test_mla_full_size_sampled():
    """h16/ckv512/kpe64/ps1, batch 4, lengths U[256, 2048]: sampled rows of every request."""
    p = W.mla_prefill()
    o, lse, _ = gpu_run_mla(p)
    rng = np.random.default_rng(2)
    for b in range(p.batch):
        L = int(p.qo_lens[b])
        pos = sorted({0, 1, 63, 64, L - 1, *rng.integers(0, L, 3).tolist()})
        o_r, l_r = oracle.mla_paged_attention_rows(p.q_nope, p.q_pe, p.ckv_cache, p.kpe_cache, p.qo_indptr,
                                                   p.kv_indptr, p.kv_indices, p.kv_last_page_len, 1, True,
                                                   p.sm_scale, b, pos)
        rows = [int(p.qo_indptr[b]) + x for x in pos]
        assert_parity(o[rows], lse[rows], o_r, l_r, what=f"mla req {b}")


# --------------------------------------------------------------------------- paged KV append

APPEND = [
    # kv lengths after the append, new rows per request, kv heads, head dims (k, v), page size
    ([37, 1, 130, 16, 0], [5, 1, 130, 16, 0], 2, (128, 128), 16),   # prefill-sized and decode-sized appends
    ([9, 300], [1, 77], 8, (64, 64), 1),                             # vector-sparse pool
    ([200, 65], [1, 1], 1, (512, 64), 1),                            # MLA latent rows: k = ckv, v = kpe
]


@pytest.mark.parametrize("case", APPEND, ids=lambda c: f"hk{c[2]}_d{c[3][0]}_p{c[4]}")
def test_append_kv_bitwise(case):
    kv_after, n_new, hk, (dk, dv), ps = case
    g = np.random.default_rng(zlib.crc32(str(case).encode()))
    kv_after, n_new = np.array(kv_after), np.array(n_new)
    n_pages = (kv_after + ps - 1) // ps
    pool = int(n_pages.sum()) + 5
    kv_indptr = np.concatenate([[0], np.cumsum(n_pages)]).astype(np.int32)
    kv_indices = g.permutation(pool)[: int(n_pages.sum())].astype(np.int32)
    last = np.where(n_pages > 0, kv_after - (n_pages - 1) * ps, 0).astype(np.int32)
    append_indptr = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    nnz = int(n_new.sum())
    k_cache = torch.from_numpy(g.standard_normal((pool, ps, hk, dk))).to(torch.bfloat16)
    v_cache = torch.from_numpy(g.standard_normal((pool, ps, hk, dv))).to(torch.bfloat16)
    k_new = torch.from_numpy(g.standard_normal((nnz, hk, dk))).to(torch.bfloat16)
    v_new = torch.from_numpy(g.standard_normal((nnz, hk, dv))).to(torch.bfloat16)
    k_ref, v_ref = oracle.append_paged_kv(k_cache, v_cache, k_new, v_new, append_indptr, kv_indptr, kv_indices,
                                          last, ps)
    kd, vd = k_cache.cuda(), v_cache.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ii = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    pkv.append_kv(k_new.cuda(), v_new.cuda(), ii(append_indptr), ii(kv_indptr), ii(kv_indices), ii(last), kd, vd,
                  status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(kd.cpu(), k_ref) and torch.equal(vd.cpu(), v_ref)


def test_append_kv_reports_rows_without_slot():
    """A request given more new rows than its table holds: those rows are
    skipped and reported, every other row is written."""
    ps, hk, d = 16, 1, 64
    kv_after, n_new = np.array([20, 3]), np.array([2, 5])   # request 1 holds 3 positions, gets 5 rows
    n_pages = (kv_after + ps - 1) // ps
    kv_indptr = np.concatenate([[0], np.cumsum(n_pages)]).astype(np.int32)
    kv_indices = np.arange(int(n_pages.sum()), dtype=np.int32)
    last = (kv_after - (n_pages - 1) * ps).astype(np.int32)
    append_indptr = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    k_cache = torch.zeros(int(n_pages.sum()), ps, hk, d, dtype=torch.bfloat16, device="cuda")
    v_cache = torch.zeros_like(k_cache)
    k_new = torch.ones(7, hk, d, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ii = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    pkv.append_kv(k_new, k_new, ii(append_indptr), ii(kv_indptr), ii(kv_indices), ii(last), k_cache, v_cache,
                  status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    assert int(k_cache.float().sum().item()) == (2 + 3) * hk * d     # request 0's two rows + request 1's three


# --------------------------------------------------------------------------- cascade (shared prefix)

def test_merge_state_bf16_kernel():
    g = torch.Generator().manual_seed(1)
    rows, dim = 200, 128
    oa = torch.randn(rows, dim, generator=g).to(torch.bfloat16)
    ob = torch.randn(rows, dim, generator=g).to(torch.bfloat16)
    la = torch.randn(rows, generator=g) * 4
    lb = torch.randn(rows, generator=g) * 4
    la[0] = -math.inf
    la[1] = lb[1] = -math.inf
    o, l = pkv.merge_state(oa.cuda(), la.cuda(), ob.cuda(), lb.cuda())
    o_ref, l_ref = oracle.merge_state(oa.float().numpy(), la.numpy(), ob.float().numpy(), lb.numpy())
    assert_parity(o, l, o_ref, l_ref, what="merge_state bf16")


def test_cascade_shared_prefix():
    """Three requests share a 32-key prefix (two pages) and each has its own
    suffix, its queries being its last suffix tokens. Prefix pass (all queries,
    non-causal) + suffix pass (causal) merged by LSE equals attention over
    each request's full page list, prefix pages first."""
    ps, hq, hk, d = 16, 8, 2, 128
    g = np.random.default_rng(5)
    suffix, qo = np.array([20, 45, 7]), np.array([20, 10, 7])
    pre_pages = 2
    suf_pages = (suffix + ps - 1) // ps
    pool = pre_pages + int(suf_pages.sum()) + 3
    perm = g.permutation(pool).astype(np.int32)
    prefix_ids, rest = perm[:pre_pages], perm[pre_pages:]
    suf_ids = np.split(rest[: int(suf_pages.sum())], np.cumsum(suf_pages)[:-1])
    k = torch.from_numpy(g.standard_normal((pool, ps, hk, d))).to(torch.bfloat16)
    v = torch.from_numpy(g.standard_normal((pool, ps, hk, d))).to(torch.bfloat16)
    total_q = int(qo.sum())
    q = torch.from_numpy(g.standard_normal((total_q, hq, d))).to(torch.bfloat16)
    qo_indptr = np.concatenate([[0], np.cumsum(qo)]).astype(np.int32)
    scale = 1.0 / math.sqrt(d)
    last_suf = (suffix - (suf_pages - 1) * ps).astype(np.int32)
    # the oracle: each request's full table = prefix pages + its own pages
    full_indptr = np.concatenate([[0], np.cumsum(pre_pages + suf_pages)]).astype(np.int32)
    full_ids = np.concatenate([np.concatenate([prefix_ids, s]) for s in suf_ids]).astype(np.int32)
    o_ref, l_ref = oracle.paged_attention(q, k, v, qo_indptr, full_indptr, full_ids, last_suf, ps, True, scale)
    # GPU: prefix pass as one request holding every query, suffix pass per request
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    pre_plan = pkv.plan(np.array([0, total_q], np.int32), np.array([0, pre_pages], np.int32), dev(prefix_ids),
                        np.array([ps], np.int32), hq, hk, d, ps, False, scale)
    suf_indptr = np.concatenate([[0], np.cumsum(suf_pages)]).astype(np.int32)
    suf_plan = pkv.plan(qo_indptr, suf_indptr, dev(np.concatenate(suf_ids)), last_suf, hq, hk, d, ps, True, scale)
    o, l = pkv.cascade_run(pre_plan, suf_plan, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert_parity(o, l, o_ref, l_ref, what="cascade")


# --------------------------------------------------------------------------- HND page layout

HND = [
    # qo_lens, kv_lens, hq, hk, d, page, causal
    ([70, 200], [70, 200], 8, 2, 128, 16, True),    # page TMA path, boxes of one kv head's 16 slots
    ([130, 33], [130, 33], 4, 4, 64, 64, True),
    ([90, 257], [90, 257], 8, 2, 128, 1, True),     # row gather (vector sparsity)
    ([40, 100], [140, 100], 4, 2, 128, 4, True),    # chunked prefill, row gather
    ([1, 1, 1], [70, 300, 5], 8, 2, 128, 16, False),  # decode kernel
    ([70, 300], [70, 300], 8, 2, 128, 128, True),   # page_size 128: one kv head's 128 slots per box
    ([1, 1], [600, 90], 24, 8, 64, 256, False),     # decode, group 3, page_size 256
    ([100, 64], [100, 64], 12, 4, 128, 4, True),    # row gather with group 3 (cp.async Q)
]


@pytest.mark.parametrize("case", HND, ids=lambda c: f"h{c[2]}_{c[3]}_d{c[4]}_p{c[5]}_q{max(c[0])}")
def test_hnd_layout(case):
    """Pools laid out [page, kv head, slot, D] (HND) give the oracle's result on
    the same pools in NHD order, and bit for bit the NHD run's result."""
    qo, kv, hq, hk, d, ps, causal = case
    p = W.make_problem("hnd", qo, kv, num_qo_heads=hq, num_kv_heads=hk, head_dim=d, page_size=ps, causal=causal,
                       seed=zlib.crc32(str(case).encode()) % 10000)
    o_n, l_n, _ = gpu_run(p)
    d_ = to_dev(p)
    pl = pkv.plan(p.qo_indptr, p.kv_indptr, d_["kv_indices"], p.kv_last_page_len, hq, hk, d, ps, causal, p.sm_scale,
                  kv_layout=1)
    k_h = d_["k_cache"].permute(0, 2, 1, 3).contiguous()
    v_h = d_["v_cache"].permute(0, 2, 1, 3).contiguous()
    o_h, l_h = pkv.run(pl, d_["q"], k_h, v_h)
    torch.cuda.synchronize()
    assert pkv.device_status(pl) == 0
    assert_parity(o_h, l_h, *oracle_run(p), what=f"hnd {case}")
    assert torch.equal(o_h, o_n) and torch.equal(l_h, l_n)


def test_append_kv_hnd():
    """Append into HND pools equals the oracle's NHD append, transposed."""
    ps, hk, d = 16, 4, 128
    g = np.random.default_rng(11)
    kv_after, n_new = np.array([40, 3, 17]), np.array([40, 1, 2])
    n_pages = (kv_after + ps - 1) // ps
    pool = int(n_pages.sum()) + 2
    kv_indptr = np.concatenate([[0], np.cumsum(n_pages)]).astype(np.int32)
    kv_indices = g.permutation(pool)[: int(n_pages.sum())].astype(np.int32)
    last = (kv_after - (n_pages - 1) * ps).astype(np.int32)
    append_indptr = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    nnz = int(n_new.sum())
    k = torch.from_numpy(g.standard_normal((pool, ps, hk, d))).to(torch.bfloat16)
    kn = torch.from_numpy(g.standard_normal((nnz, hk, d))).to(torch.bfloat16)
    k_ref, _ = oracle.append_paged_kv(k, k, kn, kn, append_indptr, kv_indptr, kv_indices, last, ps)
    kh = k.permute(0, 2, 1, 3).contiguous().cuda()
    vh = kh.clone()
    ii = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    pkv.append_kv(kn.cuda(), kn.cuda(), ii(append_indptr), ii(kv_indptr), ii(kv_indices), ii(last), kh, vh,
                  kv_layout=1)
    torch.cuda.synchronize()
    assert torch.equal(kh.cpu(), k_ref.permute(0, 2, 1, 3).contiguous())
    assert torch.equal(vh.cpu(), k_ref.permute(0, 2, 1, 3).contiguous())
