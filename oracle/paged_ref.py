"""Float64 CPU oracle for batched attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY. It exists to check the CUDA path. Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and reference
legs) may import it; the library ``paged_kv_attention_38_b200`` never does,
and this module imports nothing from that library.

It is written for a reader checking it against the pages by eye, not for
speed: NumPy float64, one query head at a time, one library matmul per step.
The only blocking is over independent query rows (to bound memory); every
reduction over keys is done whole.

What it computes, and where the pages say so
--------------------------------------------
* Page table (flashinfer-trace discussion #15, "Notes on fa3_gqa_prefill_v1";
  FlashInfer 0.7.4 documentation, "KV-Cache Layout in FlashInfer" /
  "Page Table Layout"): request ``b`` owns pages
  ``kv_indices[kv_indptr[b]:kv_indptr[b+1]]``; every page is full except the
  last, which holds ``kv_last_page_len[b]`` valid slots.
* ``page_size`` is the column count of one sparse block; ``page_size=1`` is
  vector sparsity (FlashInfer 0.2 release, "FlashAttention-3 template with
  block/vector sparsity").
* Ragged queries ``[total_q, num_qo_heads, head_dim]`` cut by ``qo_indptr``
  (discussion #15, same notes; documentation "Ragged Tensor").
* The stored LSE is base 2: the natural-log LSE divided by ln 2 (discussion
  #15, same notes: the FA3 bridge converts FA3's natural-log LSE to base 2).
* MLA with matrix absorption (FlashInfer 0.2 release, "Fused MLA decode
  kernel"; definition ``mla_paged_prefill_causal_h16_ckv512_kpe64_ps1``):
  all heads share one latent KV row ``[ckv | kpe]``; scores are
  ``q_nope . ckv + q_pe . kpe`` and the output is ``P . ckv``.
* Merging attention states (documentation, "Attention States and Recursive
  Attention", "Merge Attention States"): two partial results over disjoint key
  sets combine by their log-sum-exp.
* Appending new K/V rows to the paged cache (FlashInfer 0.2 release, "KV-Cache
  append optimization"; documentation, ``get_batch_indices_positions``): the
  page table given is the one after the append, so request ``b``'s ``n`` new
  rows take its last ``n`` positions ``kv_len - n .. kv_len - 1``.
* A per-head-scale quantised KV cache ("[Roadmap] FlashInfer v0.2 to v0.3",
  milestone "Per Head Scale Quantized KV-Cache"; the documentation lists FP8
  KV-cache writers such as ``cake_fused_qk_rope_fp8_append``): the pools hold
  FP8 E4M3 codes and every kv head ``h`` has one fp32 scale for K and one for
  V; the cache's value is ``decode(code) * scale[h]`` (reading 6).

Readings where the pages are silent (each pinned by a test)
------------------------------------------------------------
1. The attention itself is the textbook ``softmax(sm_scale * Q K^T) V`` with the
   natural exponential; base 2 applies only to the stored LSE.
2. Causal alignment is bottom-right: query ``i`` of a request with ``qo_len``
   queries and ``kv_len`` keys sees key ``j`` iff ``j <= i + kv_len - qo_len``.
3. GQA: query head ``h`` reads kv head ``h // (num_qo_heads // num_kv_heads)``.
4. A query row that sees no key (empty request, or causal with
   ``qo_len > kv_len``) has output 0 and LSE ``-inf``.
5. Decode is the same function with one query per request and ``causal=False``.
6. The quantised cache's codes are FP8 E4M3 as the OCP 8-bit floating-point
   specification defines it (1 sign bit, 4 exponent bits with bias 7, 3
   mantissa bits; exponent field 0 is subnormal, ``m/8 * 2^-6``; no
   infinities; ``S.1111.111`` is NaN; largest finite value 448), and attention
   over it is reading 1 applied to the dequantised K and V.
"""
from __future__ import annotations

import numpy as np

LN2 = float(np.log(2.0))
ROW_BLOCK = 256


def _f64(x) -> np.ndarray:
    """bf16/fp32 torch tensor or array -> float64 ndarray (exact for bf16)."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def kv_lengths(kv_indptr, kv_last_page_len, page_size: int) -> np.ndarray:
    """KV length of every request: full pages except the last (Page Table Layout)."""
    n_pages = np.diff(np.asarray(kv_indptr, dtype=np.int64))
    last = np.asarray(kv_last_page_len, dtype=np.int64)
    return np.where(n_pages > 0, (n_pages - 1) * page_size + last, 0)


def gather_pages(cache, kv_indptr, kv_indices, kv_last_page_len, page_size: int, b: int) -> np.ndarray:
    """The KV rows of request ``b`` in logical order: ``[kv_len, ...]`` float64.

    ``cache`` is a page pool ``[num_pages, page_size, ...]``; the rows are the
    pages listed for ``b``, concatenated, cut after the last page's valid slots.
    """
    lo, hi = int(kv_indptr[b]), int(kv_indptr[b + 1])
    pool = _f64(cache)
    tail = pool.shape[2:]
    if hi == lo:
        return np.zeros((0,) + tail)
    pages = np.asarray(kv_indices[lo:hi], dtype=np.int64)
    rows = pool[pages].reshape((-1,) + tail)
    kv_len = (hi - lo - 1) * page_size + int(kv_last_page_len[b])
    return rows[:kv_len]


def visible(qo_len: int, kv_len: int, causal: bool, q_pos=None) -> np.ndarray:
    """Bool ``[n_rows, kv_len]``: which keys each query row sees (reading 2)."""
    q_pos = np.arange(qo_len) if q_pos is None else np.asarray(q_pos)
    j = np.arange(kv_len)[None, :]
    if not causal:
        return np.ones((len(q_pos), kv_len), dtype=bool)
    return j <= (q_pos[:, None] + (kv_len - qo_len))


def softmax_rows(s: np.ndarray, mask: np.ndarray):
    """Masked softmax of score rows: returns (weights, natural-log LSE).

    Rows with no visible key get all-zero weights and LSE -inf (reading 4).
    """
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True) if s.shape[1] else np.full((s.shape[0], 1), -np.inf)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.where(mask, np.exp(s - m_safe), 0.0)
    l = e.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        w = np.where(empty, 0.0, e / np.where(empty, 1.0, l))
        lse = np.where(empty[:, 0], -np.inf, (m_safe + np.log(np.where(empty, 1.0, l)))[:, 0])
    return w, lse


def attend(q, k, v, causal: bool, sm_scale: float, q_pos=None, qo_len=None):
    """Attention of one request.

    ``q [n, Hq, D]``, ``k [kv_len, Hk, D]``, ``v [kv_len, Hk, Dv]`` (float64).
    ``q_pos`` are the positions of the given rows among the request's
    ``qo_len`` queries (default: all of them, in order).
    Returns ``o [n, Hq, Dv]`` and base-2 ``lse2 [n, Hq]``.
    """
    n, hq, _ = q.shape
    kv_len, hk = k.shape[0], k.shape[1]
    dv = v.shape[2]
    qo_len = n if qo_len is None else qo_len
    q_pos = np.arange(n) if q_pos is None else np.asarray(q_pos)
    group = hq // hk
    o = np.zeros((n, hq, dv))
    lse2 = np.full((n, hq), -np.inf)
    for r0 in range(0, n, ROW_BLOCK):
        rows = slice(r0, min(n, r0 + ROW_BLOCK))
        mask = visible(qo_len, kv_len, causal, q_pos[rows])
        for h in range(hq):
            g = h // group                                  # reading 3
            s = sm_scale * (q[rows, h, :] @ k[:, g, :].T)   # [rows, kv_len]
            w, lse = softmax_rows(s, mask)
            o[rows, h, :] = w @ v[:, g, :]
            lse2[rows, h] = lse / LN2                        # base-2 LSE
    return o, lse2


def paged_attention(q, k_cache, v_cache, qo_indptr, kv_indptr, kv_indices, kv_last_page_len,
                    page_size: int, causal: bool, sm_scale: float, requests=None):
    """Batched attention over a paged KV cache (GQA / MHA / MQA, prefill or decode).

    Returns ``o [total_q, Hq, Dv]`` and ``lse2 [total_q, Hq]`` in float64; rows of
    requests not listed in ``requests`` (default: all) are left at 0 / -inf.
    """
    qf = _f64(q)
    kp, vp = _f64(k_cache), _f64(v_cache)
    total_q, hq, _ = qf.shape
    dv = vp.shape[-1]
    o = np.zeros((total_q, hq, dv))
    lse2 = np.full((total_q, hq), -np.inf)
    batch = len(kv_last_page_len)
    for b in (range(batch) if requests is None else requests):
        q0, q1 = int(qo_indptr[b]), int(qo_indptr[b + 1])
        k = gather_pages(kp, kv_indptr, kv_indices, kv_last_page_len, page_size, b)
        v = gather_pages(vp, kv_indptr, kv_indices, kv_last_page_len, page_size, b)
        o[q0:q1], lse2[q0:q1] = attend(qf[q0:q1], k, v, causal, sm_scale)
    return o, lse2


def paged_attention_rows(q, k_cache, v_cache, qo_indptr, kv_indptr, kv_indices, kv_last_page_len,
                         page_size: int, causal: bool, sm_scale: float, b: int, q_pos):
    """Selected query rows of request ``b`` (positions ``q_pos``), all heads.

    Used to check full-size runs on a sample of rows.
    """
    q0, q1 = int(qo_indptr[b]), int(qo_indptr[b + 1])
    q_pos = np.asarray(q_pos, dtype=np.int64)
    qf = _f64(q[q0:q1])[q_pos]
    k = gather_pages(k_cache, kv_indptr, kv_indices, kv_last_page_len, page_size, b)
    v = gather_pages(v_cache, kv_indptr, kv_indices, kv_last_page_len, page_size, b)
    return attend(qf, k, v, causal, sm_scale, q_pos=q_pos, qo_len=q1 - q0)


def mla_attend(q_nope, q_pe, ckv, kpe, causal: bool, sm_scale: float, q_pos=None, qo_len=None):
    """Absorbed MLA for one request: ``q_nope [n, H, Dc]``, ``q_pe [n, H, Dr]``,
    ``ckv [kv_len, Dc]``, ``kpe [kv_len, Dr]`` -> ``o [n, H, Dc]``, ``lse2 [n, H]``.

    Score ``s_j = sm_scale * (q_nope . ckv_j + q_pe . kpe_j)``; output ``sum_j p_j ckv_j``.
    """
    n, heads, dc = q_nope.shape
    kv_len = ckv.shape[0]
    qo_len = n if qo_len is None else qo_len
    q_pos = np.arange(n) if q_pos is None else np.asarray(q_pos)
    o = np.zeros((n, heads, dc))
    lse2 = np.full((n, heads), -np.inf)
    for r0 in range(0, n, ROW_BLOCK):
        rows = slice(r0, min(n, r0 + ROW_BLOCK))
        mask = visible(qo_len, kv_len, causal, q_pos[rows])
        for h in range(heads):
            s = sm_scale * (q_nope[rows, h, :] @ ckv.T + q_pe[rows, h, :] @ kpe.T)
            w, lse = softmax_rows(s, mask)
            o[rows, h, :] = w @ ckv
            lse2[rows, h] = lse / LN2
    return o, lse2


def mla_paged_attention(q_nope, q_pe, ckv_cache, kpe_cache, qo_indptr, kv_indptr, kv_indices,
                        kv_last_page_len, page_size: int, causal: bool, sm_scale: float,
                        requests=None):
    """Batched absorbed-MLA attention over paged latent caches
    ``ckv_cache [num_pages, P, Dc]`` and ``kpe_cache [num_pages, P, Dr]``."""
    qn, qp = _f64(q_nope), _f64(q_pe)
    cp, kp = _f64(ckv_cache), _f64(kpe_cache)
    total_q, heads, dc = qn.shape
    o = np.zeros((total_q, heads, dc))
    lse2 = np.full((total_q, heads), -np.inf)
    batch = len(kv_last_page_len)
    for b in (range(batch) if requests is None else requests):
        q0, q1 = int(qo_indptr[b]), int(qo_indptr[b + 1])
        ckv = gather_pages(cp, kv_indptr, kv_indices, kv_last_page_len, page_size, b)
        kpe = gather_pages(kp, kv_indptr, kv_indices, kv_last_page_len, page_size, b)
        o[q0:q1], lse2[q0:q1] = mla_attend(qn[q0:q1], qp[q0:q1], ckv, kpe, causal, sm_scale)
    return o, lse2


def mla_paged_attention_rows(q_nope, q_pe, ckv_cache, kpe_cache, qo_indptr, kv_indptr, kv_indices,
                             kv_last_page_len, page_size: int, causal: bool, sm_scale: float,
                             b: int, q_pos):
    """Selected query rows of request ``b`` for absorbed MLA (all heads)."""
    q0, q1 = int(qo_indptr[b]), int(qo_indptr[b + 1])
    q_pos = np.asarray(q_pos, dtype=np.int64)
    qn = _f64(q_nope[q0:q1])[q_pos]
    qp = _f64(q_pe[q0:q1])[q_pos]
    ckv = gather_pages(ckv_cache, kv_indptr, kv_indices, kv_last_page_len, page_size, b)
    kpe = gather_pages(kpe_cache, kv_indptr, kv_indices, kv_last_page_len, page_size, b)
    return mla_attend(qn, qp, ckv, kpe, causal, sm_scale, q_pos=q_pos, qo_len=q1 - q0)


def merge_state(o_a, lse_a, o_b, lse_b):
    """Merge two attention states over disjoint key sets (base-2 LSE).

    ``lse = log2(2^lse_a + 2^lse_b)``; ``o = 2^(lse_a - lse) o_a + 2^(lse_b - lse) o_b``.
    A state with LSE -inf (no keys) contributes nothing; two empty states stay empty.
    """
    o_a, o_b = _f64(o_a), _f64(o_b)
    lse_a, lse_b = _f64(lse_a), _f64(lse_b)
    m = np.maximum(lse_a, lse_b)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    wa = np.where(np.isfinite(lse_a), np.exp2(lse_a - m_safe), 0.0)
    wb = np.where(np.isfinite(lse_b), np.exp2(lse_b - m_safe), 0.0)
    tot = wa + wb
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(empty, -np.inf, m_safe + np.log2(np.where(empty, 1.0, tot)))
        fa = np.where(empty, 0.0, wa / np.where(empty, 1.0, tot))
        fb = np.where(empty, 0.0, wb / np.where(empty, 1.0, tot))
    o = fa[..., None] * o_a + fb[..., None] * o_b
    return o, lse


def merge_states(os, lses):
    """Merge any number of states by folding ``merge_state`` left to right."""
    o, lse = _f64(os[0]), _f64(lses[0])
    for o_i, l_i in zip(os[1:], lses[1:]):
        o, lse = merge_state(o, lse, o_i, l_i)
    return o, lse


def append_paged_kv(k_cache, v_cache, k_new, v_new, append_indptr, kv_indptr, kv_indices, kv_last_page_len,
                    page_size: int):
    """Return copies of the K and V pools with the new rows written in.

    ``k_new``/``v_new`` ``[nnz, Hk, D]`` hold request ``b``'s new rows at
    ``append_indptr[b]:append_indptr[b+1]``. With the page table after the
    append, request ``b`` has ``kv_len`` positions and its ``n`` new rows are
    positions ``kv_len - n + i``; position ``p`` lives in page
    ``kv_indices[kv_indptr[b] + p // page_size]``, slot ``p % page_size``.
    Plain loops, one row at a time; values are copied unchanged.
    """
    k_out = k_cache.clone() if hasattr(k_cache, "clone") else np.array(k_cache, copy=True)
    v_out = v_cache.clone() if hasattr(v_cache, "clone") else np.array(v_cache, copy=True)
    kv_len = kv_lengths(kv_indptr, kv_last_page_len, page_size)
    for b in range(len(kv_last_page_len)):
        a0, a1 = int(append_indptr[b]), int(append_indptr[b + 1])
        n = a1 - a0
        assert 0 <= n <= kv_len[b], "more new rows than the request's length"
        for i in range(n):
            pos = int(kv_len[b]) - n + i
            page = int(kv_indices[int(kv_indptr[b]) + pos // page_size])
            slot = pos % page_size
            k_out[page, slot] = k_new[a0 + i]
            v_out[page, slot] = v_new[a0 + i]
    return k_out, v_out


def e4m3_to_f64(codes) -> np.ndarray:
    """FP8 E4M3 codes (uint8) -> float64 values (reading 6), field by field."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 0xF) & (c & 0x7 == 0x7), np.nan, mag)
    return sign * mag


def dequantize_kv(codes, scale) -> np.ndarray:
    """A quantised pool ``[pages, page_size, Hk, D]`` of E4M3 codes with one scale
    per kv head -> its float64 values, ``decode(code) * scale[h]``."""
    c = codes.detach().cpu().numpy() if hasattr(codes, "detach") else np.asarray(codes)
    vals = e4m3_to_f64(c.view(np.uint8) if c.dtype != np.uint8 else c)
    sc = _f64(scale).reshape(-1)
    assert sc.shape[0] == vals.shape[2], "one scale per kv head"
    return vals * sc[None, None, :, None]


def paged_attention_quantized_kv(q, k_codes, v_codes, k_scale, v_scale, qo_indptr, kv_indptr, kv_indices,
                                 kv_last_page_len, page_size: int, causal: bool, sm_scale: float, requests=None):
    """Paged attention over a per-head-scale FP8 E4M3 KV cache (NHD pools):
    the dequantised pools through ``paged_attention``."""
    return paged_attention(q, dequantize_kv(k_codes, k_scale), dequantize_kv(v_codes, v_scale), qo_indptr,
                           kv_indptr, kv_indices, kv_last_page_len, page_size, causal, sm_scale, requests)
