"""Pins for the float64 oracle, each independent of the oracle's own code.

* hand-worked golden examples (tests/golden/hand_worked.json), exact answers;
* brute force with plain Python loops over the page table on tiny inputs;
* a library special case: torch's float64 scaled_dot_product_attention
  (top-left / bottom-right causal masks from torch itself, torch's GQA head
  mapping) and torch.logsumexp;
* closed forms (one key, sm_scale = 0, constant V, identical keys);
* invariants (page_size=1 equals the dense ragged layout, permuting the pool,
  cross page-size, split + merge, causal row 0, MLA reduced to GQA).

The mutation tests at the end plant plausible mistakes in a copy of the oracle's
arithmetic and check that the pins catch each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import paged_ref
from paged_kv_attention_38_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _arr(x):
    return np.asarray(x, dtype=np.float64)


def _i32(x):
    return np.asarray(x, dtype=np.int32)


# ---------------------------------------------------------------------------
# golden
# ---------------------------------------------------------------------------

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_golden_hand_worked(case):
    if case["kind"] == "paged":
        o, lse = oracle.paged_attention(_arr(case["q"]), _arr(case["k_cache"]), _arr(case["v_cache"]),
                                        _i32(case["qo_indptr"]), _i32(case["kv_indptr"]),
                                        _i32(case["kv_indices"]), _i32(case["kv_last_page_len"]),
                                        case["page_size"], case["causal"], case["sm_scale"])
    elif case["kind"] == "mla":
        o, lse = oracle.mla_paged_attention(_arr(case["q_nope"]), _arr(case["q_pe"]),
                                            _arr(case["ckv_cache"]), _arr(case["kpe_cache"]),
                                            _i32(case["qo_indptr"]), _i32(case["kv_indptr"]),
                                            _i32(case["kv_indices"]), _i32(case["kv_last_page_len"]),
                                            case["page_size"], case["causal"], case["sm_scale"])
    else:
        o, lse = oracle.merge_state(_arr(case["o_a"]), _arr(case["lse_a"]),
                                    _arr(case["o_b"]), _arr(case["lse_b"]))
    np.testing.assert_allclose(o, _arr(case["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, _arr(case["lse2"]), rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# brute force: plain loops over the page table, math module only
# ---------------------------------------------------------------------------

def brute_force(q, k_cache, v_cache, qo_indptr, kv_indptr, kv_indices, last, page_size, causal, scale):
    total_q, hq, d = q.shape
    hk, dv = k_cache.shape[2], v_cache.shape[3]
    group = hq // hk
    o = np.zeros((total_q, hq, dv))
    lse2 = np.full((total_q, hq), -math.inf)
    for b in range(len(last)):
        n_pages = int(kv_indptr[b + 1] - kv_indptr[b])
        kv_len = 0 if n_pages == 0 else (n_pages - 1) * page_size + int(last[b])
        qo_len = int(qo_indptr[b + 1] - qo_indptr[b])
        for i in range(qo_len):
            t = int(qo_indptr[b]) + i
            for h in range(hq):
                g = h // group
                scores, vals = [], []
                for j in range(kv_len):
                    if causal and j > i + kv_len - qo_len:
                        continue
                    page = int(kv_indices[int(kv_indptr[b]) + j // page_size])
                    slot = j % page_size
                    s = 0.0
                    for x in range(d):
                        s += float(q[t, h, x]) * float(k_cache[page, slot, g, x])
                    scores.append(s * scale)
                    vals.append([float(v_cache[page, slot, g, y]) for y in range(dv)])
                if not scores:
                    continue
                mx = max(scores)
                ex = [math.exp(s - mx) for s in scores]
                tot = sum(ex)
                for y in range(dv):
                    o[t, h, y] = sum(e * vv[y] for e, vv in zip(ex, vals)) / tot
                lse2[t, h] = (mx + math.log(tot)) / math.log(2.0)
    return o, lse2


def _small(seed, qo_lens, kv_lens, hq, hk, d, p, causal, dv=None, pool_extra=3):
    n_pages = sum((int(k) + p - 1) // p for k in kv_lens)
    return W.make_problem("small", qo_lens, kv_lens, num_qo_heads=hq, num_kv_heads=hk, head_dim=d,
                          head_dim_v=dv, page_size=p, causal=causal, seed=seed,
                          pool_pages=n_pages + pool_extra)


def _run_oracle(pb, **kw):
    return oracle.paged_attention(pb.q, pb.k_cache, pb.v_cache, pb.qo_indptr, pb.kv_indptr,
                                  pb.kv_indices, pb.kv_last_page_len, pb.page_size, pb.causal,
                                  pb.sm_scale, **kw)


def _f64(t):
    return t.float().double().numpy()


BRUTE_CASES = [
    # seed, qo_lens, kv_lens, hq, hk, d, page, causal, dv
    (1, [5, 9], [5, 9], 2, 1, 8, 4, True, None),
    (2, [3, 1, 6], [7, 1, 6], 4, 2, 6, 3, True, 5),     # chunked (qo < kv), last page 1 slot
    (3, [4, 4], [6, 11], 3, 3, 4, 1, False, None),      # MHA, page_size 1, non-causal
    (4, [1, 1, 1], [9, 16, 3], 4, 1, 8, 8, False, None),  # decode shape
    (5, [6, 2], [4, 2], 2, 1, 4, 2, True, None),        # qo > kv: first rows see nothing
    (6, [0, 3], [5, 3], 2, 2, 4, 2, True, None),        # a request with no queries
]


@pytest.mark.parametrize("case", BRUTE_CASES, ids=lambda c: f"seed{c[0]}")
def test_brute_force(case):
    seed, qo, kv, hq, hk, d, p, causal, dv = case
    pb = _small(seed, qo, kv, hq, hk, d, p, causal, dv)
    o, lse = _run_oracle(pb)
    ob, lb = brute_force(_f64(pb.q), _f64(pb.k_cache), _f64(pb.v_cache), pb.qo_indptr, pb.kv_indptr,
                         pb.kv_indices, pb.kv_last_page_len, pb.page_size, pb.causal, pb.sm_scale)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    assert np.array_equal(np.isinf(lse), np.isinf(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)


def test_empty_request_and_no_visible_key():
    # request 1 has no page at all; in request 0 (qo 6 > kv 4) rows 0, 1 see no key
    pb = _small(7, [6, 2], [4, 0], 2, 1, 4, 2, True)
    o, lse = _run_oracle(pb)
    assert np.all(o[0:2] == 0) and np.all(np.isneginf(lse[0:2]))
    assert np.all(o[6:8] == 0) and np.all(np.isneginf(lse[6:8]))
    assert np.all(np.isfinite(lse[2:6]))


# ---------------------------------------------------------------------------
# library special case: torch float64 SDPA
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("hq,hk,qo,kv,causal", [(4, 4, 37, 37, True), (8, 2, 29, 29, True),
                                                 (6, 3, 19, 45, True), (4, 1, 1, 50, False),
                                                 (2, 1, 23, 23, False)])
def test_torch_sdpa(hq, hk, qo, kv, causal):
    from torch.nn.attention import SDPBackend, sdpa_kernel
    from torch.nn.attention.bias import causal_lower_right
    pb = _small(11 + hq + qo, [qo], [kv], hq, hk, 16, 8, causal)
    o, lse = _run_oracle(pb)
    q = torch.from_numpy(_f64(pb.q)).permute(1, 0, 2)[None]                # [1, Hq, qo, D]
    k = torch.from_numpy(oracle.gather_pages(pb.k_cache, pb.kv_indptr, pb.kv_indices,
                                             pb.kv_last_page_len, pb.page_size, 0)).permute(1, 0, 2)[None]
    v = torch.from_numpy(oracle.gather_pages(pb.v_cache, pb.kv_indptr, pb.kv_indices,
                                             pb.kv_last_page_len, pb.page_size, 0)).permute(1, 0, 2)[None]
    mask = None
    if causal:
        mask = causal_lower_right(qo, kv) if qo != kv else None
    # torch's math backend (its plain matmul / softmax composition): the fused
    # CPU flash kernel it would otherwise pick failed this comparison now and
    # then in long test runs, far beyond any rounding difference
    with sdpa_kernel(SDPBackend.MATH):
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, attn_mask=mask, is_causal=(causal and qo == kv), scale=pb.sm_scale,
            enable_gqa=(hq != hk))
    np.testing.assert_allclose(o, ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    # LSE from torch.logsumexp of the masked logits, with torch's own causal masks
    kr = k.repeat_interleave(hq // hk, dim=1)
    logits = (q @ kr.transpose(-1, -2)) * pb.sm_scale
    if causal:
        bias = torch.zeros(qo, kv, dtype=torch.float64)
        bias = causal_lower_right(qo, kv)._materialize().to(torch.bool) if qo != kv else \
            torch.ones(qo, kv, dtype=torch.bool).tril()
        logits = logits.masked_fill(~bias, -math.inf)
    lse_ref = torch.logsumexp(logits, dim=-1)[0].T / math.log(2.0)
    np.testing.assert_allclose(lse, lse_ref.numpy(), rtol=0, atol=1e-12)


def test_oracle_is_deterministic():
    """The oracle is a pure function of its inputs: two runs on the same seeded
    problem, one of them after other NumPy work, give bitwise equal results
    (a nondeterministic oracle, e.g. through threaded BLAS reductions, would make
    every comparison against it noisy)."""
    pb = _small(41, [37, 5, 64], [37, 50, 64], 8, 2, 16, 8, True)
    o1, l1 = _run_oracle(pb)
    np.linalg.svd(np.random.default_rng(0).standard_normal((300, 300)))  # other BLAS work in between
    o2, l2 = _run_oracle(pb)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2, equal_nan=True)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def test_closed_form_one_key():
    pb = _small(21, [1, 1], [1, 1], 4, 2, 16, 4, True)
    o, lse = _run_oracle(pb)
    for b in range(2):
        k = oracle.gather_pages(pb.k_cache, pb.kv_indptr, pb.kv_indices, pb.kv_last_page_len, 4, b)
        v = oracle.gather_pages(pb.v_cache, pb.kv_indptr, pb.kv_indices, pb.kv_last_page_len, 4, b)
        q = _f64(pb.q)[b]
        for h in range(4):
            s = pb.sm_scale * float(np.dot(q[h], k[0, h // 2]))
            np.testing.assert_allclose(o[b, h], v[0, h // 2], rtol=0, atol=1e-15)
            assert abs(lse[b, h] - s / math.log(2.0)) < 1e-13


def test_closed_form_zero_scale_is_mean_of_visible():
    pb = _small(22, [13], [13], 2, 1, 8, 4, True)
    pb.sm_scale = 0.0
    o, lse = _run_oracle(pb)
    v = oracle.gather_pages(pb.v_cache, pb.kv_indptr, pb.kv_indices, pb.kv_last_page_len, 4, 0)
    for i in range(13):
        np.testing.assert_allclose(o[i, 0], v[: i + 1, 0].mean(axis=0), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[i], math.log2(i + 1), rtol=0, atol=1e-13)


def test_closed_form_constant_v_and_identical_keys():
    pb = _small(23, [9], [9], 2, 1, 8, 2, True)
    pool_v = torch.ones_like(pb.v_cache)
    o, _ = oracle.paged_attention(pb.q, pb.k_cache, pool_v, pb.qo_indptr, pb.kv_indptr, pb.kv_indices,
                                  pb.kv_last_page_len, 2, True, pb.sm_scale)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)
    # identical keys -> uniform weights, LSE = s + log2(n_visible)
    k_same = pb.k_cache.clone()
    k_same[:] = pb.k_cache[int(pb.kv_indices[0]), 0]
    o, lse = oracle.paged_attention(pb.q, k_same, pb.v_cache, pb.qo_indptr, pb.kv_indptr, pb.kv_indices,
                                    pb.kv_last_page_len, 2, True, pb.sm_scale)
    v = oracle.gather_pages(pb.v_cache, pb.kv_indptr, pb.kv_indices, pb.kv_last_page_len, 2, 0)
    kk = _f64(k_same)[0, 0, 0]
    for i in range(9):
        s = pb.sm_scale * float(np.dot(_f64(pb.q)[i, 1], kk))
        np.testing.assert_allclose(o[i, 1], v[: i + 1, 0].mean(axis=0), rtol=0, atol=1e-13)
        assert abs(lse[i, 1] - (s / math.log(2.0) + math.log2(i + 1))) < 1e-12


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

def test_vector_sparse_equals_dense_ragged():
    sp = W.make_problem("s", [17, 40], [17, 40], num_qo_heads=4, num_kv_heads=2, head_dim=16,
                        page_size=1, causal=True, seed=31)
    de = W.make_problem("d", [17, 40], [17, 40], num_qo_heads=4, num_kv_heads=2, head_dim=16,
                        page_size=1, causal=True, seed=31, contiguous=True)
    # same tensors drawn; the dense problem lays its slots out in order, so move rows accordingly
    k_dense = torch.empty_like(de.k_cache)
    v_dense = torch.empty_like(de.v_cache)
    k_dense[torch.from_numpy(de.kv_indices.astype(np.int64))] = sp.k_cache[torch.from_numpy(sp.kv_indices.astype(np.int64))]
    v_dense[torch.from_numpy(de.kv_indices.astype(np.int64))] = sp.v_cache[torch.from_numpy(sp.kv_indices.astype(np.int64))]
    o1, l1 = _run_oracle(sp)
    o2, l2 = oracle.paged_attention(sp.q, k_dense, v_dense, de.qo_indptr, de.kv_indptr, de.kv_indices,
                                    de.kv_last_page_len, 1, True, sp.sm_scale)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_pool_permutation_invariance():
    pb = _small(41, [12, 30], [12, 30], 4, 1, 8, 4, True, pool_extra=5)
    o1, l1 = _run_oracle(pb)
    n = pb.k_cache.shape[0]
    perm = np.random.default_rng(0).permutation(n)
    inv = np.argsort(perm)
    # new pool slot perm[x] holds old page x
    k2 = torch.empty_like(pb.k_cache)
    v2 = torch.empty_like(pb.v_cache)
    k2[torch.from_numpy(perm)] = pb.k_cache
    v2[torch.from_numpy(perm)] = pb.v_cache
    idx2 = perm[pb.kv_indices].astype(np.int32)
    o2, l2 = oracle.paged_attention(pb.q, k2, v2, pb.qo_indptr, pb.kv_indptr, idx2,
                                    pb.kv_last_page_len, 4, True, pb.sm_scale)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    assert inv[perm[3]] == 3


def _repage(pb, new_p, seed):
    """The same logical K/V rows laid out in a pool with another page size."""
    kv_lens = pb.kv_lens
    rows_k = [oracle.gather_pages(pb.k_cache, pb.kv_indptr, pb.kv_indices, pb.kv_last_page_len,
                                  pb.page_size, b) for b in range(pb.batch)]
    rows_v = [oracle.gather_pages(pb.v_cache, pb.kv_indptr, pb.kv_indices, pb.kv_last_page_len,
                                  pb.page_size, b) for b in range(pb.batch)]
    indptr, indices, last, pool = W.page_table(kv_lens, new_p, W._gen(seed))
    hk, d = pb.k_cache.shape[2], pb.k_cache.shape[3]
    k = np.zeros((pool, new_p, hk, d))
    v = np.full((pool, new_p, hk, pb.v_cache.shape[3]), 7.0)
    for b in range(pb.batch):
        for j in range(int(kv_lens[b])):
            page = indices[indptr[b] + j // new_p]
            k[page, j % new_p] = rows_k[b][j]
            v[page, j % new_p] = rows_v[b][j]
    return k, v, indptr, indices, last


@pytest.mark.parametrize("new_p", [1, 16, 64])
def test_cross_page_size(new_p):
    pb = _small(51, [70, 33], [70, 33], 4, 2, 8, 16, True)
    o1, l1 = _run_oracle(pb)
    k, v, indptr, indices, last = _repage(pb, new_p, 99)
    o2, l2 = oracle.paged_attention(pb.q, k, v, pb.qo_indptr, indptr, indices, last, new_p, True,
                                    pb.sm_scale)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.parametrize("cut", [1, 7, 20, 38])
def test_split_kv_merge_reproduces_full(cut):
    """Attention over keys [0, cut) and [cut, kv_len) merged by base-2 LSE equals the whole."""
    pb = _small(61, [1], [39], 8, 2, 16, 4, False)
    o, lse = _run_oracle(pb)
    k = oracle.gather_pages(pb.k_cache, pb.kv_indptr, pb.kv_indices, pb.kv_last_page_len, 4, 0)
    v = oracle.gather_pages(pb.v_cache, pb.kv_indptr, pb.kv_indices, pb.kv_last_page_len, 4, 0)
    q = _f64(pb.q)
    oa, la = oracle.attend(q, k[:cut], v[:cut], False, pb.sm_scale)
    ob, lb = oracle.attend(q, k[cut:], v[cut:], False, pb.sm_scale)
    om, lm = oracle.merge_state(oa, la, ob, lb)
    np.testing.assert_allclose(om, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lm, lse, rtol=0, atol=1e-12)
    # three-way fold, and merging with an empty state is the identity
    oc, lc = oracle.merge_states([oa, ob[..., :], np.zeros_like(oa)], [la, lb, np.full_like(la, -np.inf)])
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lc, lse, rtol=0, atol=1e-12)


def test_causal_row_zero_sees_only_key_zero():
    pb = _small(71, [10], [10], 2, 1, 8, 4, True)
    o1, l1 = _run_oracle(pb)
    k2, v2 = pb.k_cache.clone(), pb.v_cache.clone()
    first = int(pb.kv_indices[0])
    keep_k, keep_v = k2[first, 0].clone(), v2[first, 0].clone()
    k2.normal_(generator=torch.Generator().manual_seed(3))
    v2.normal_(generator=torch.Generator().manual_seed(4))
    k2[first, 0], v2[first, 0] = keep_k, keep_v
    o2, l2 = oracle.paged_attention(pb.q, k2, v2, pb.qo_indptr, pb.kv_indptr, pb.kv_indices,
                                    pb.kv_last_page_len, 4, True, pb.sm_scale)
    assert np.array_equal(o1[0], o2[0]) and np.array_equal(l1[0], l2[0])
    assert not np.allclose(o1[1:], o2[1:])


def test_gqa_head_permutation():
    """Swapping kv heads and the matching groups of query heads swaps the outputs."""
    pb = _small(81, [11], [11], 4, 2, 8, 4, True)
    o1, l1 = _run_oracle(pb)
    q2 = pb.q[:, [2, 3, 0, 1]].contiguous()
    k2 = pb.k_cache[:, :, [1, 0]].contiguous()
    v2 = pb.v_cache[:, :, [1, 0]].contiguous()
    o2, l2 = oracle.paged_attention(q2, k2, v2, pb.qo_indptr, pb.kv_indptr, pb.kv_indices,
                                    pb.kv_last_page_len, 4, True, pb.sm_scale)
    assert np.array_equal(o1[:, [2, 3, 0, 1]], o2) and np.array_equal(l1[:, [2, 3, 0, 1]], l2)


def test_mla_reduces_to_gqa():
    """With q_pe = kpe = 0, absorbed MLA is single-kv-head attention with K = V = ckv."""
    mp = W.make_mla_problem("m", [9, 14], [9, 14], num_heads=3, head_dim_ckv=16, head_dim_kpe=4,
                            seed=91)
    qpe = torch.zeros_like(mp.q_pe)
    kpe = torch.zeros_like(mp.kpe_cache)
    o1, l1 = oracle.mla_paged_attention(mp.q_nope, qpe, mp.ckv_cache, kpe, mp.qo_indptr, mp.kv_indptr,
                                        mp.kv_indices, mp.kv_last_page_len, 1, True, mp.sm_scale)
    kc = mp.ckv_cache[:, :, None, :]
    o2, l2 = oracle.paged_attention(mp.q_nope, kc, kc, mp.qo_indptr, mp.kv_indptr, mp.kv_indices,
                                    mp.kv_last_page_len, 1, True, mp.sm_scale)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_mla_brute_force():
    mp = W.make_mla_problem("m", [4, 6], [4, 6], num_heads=2, head_dim_ckv=6, head_dim_kpe=3, seed=92)
    o, lse = oracle.mla_paged_attention(mp.q_nope, mp.q_pe, mp.ckv_cache, mp.kpe_cache, mp.qo_indptr,
                                        mp.kv_indptr, mp.kv_indices, mp.kv_last_page_len, 1, True,
                                        mp.sm_scale)
    qn, qp, ckv, kpe = _f64(mp.q_nope), _f64(mp.q_pe), _f64(mp.ckv_cache), _f64(mp.kpe_cache)
    for b in range(2):
        q0, q1 = int(mp.qo_indptr[b]), int(mp.qo_indptr[b + 1])
        n = q1 - q0
        for i in range(n):
            for h in range(2):
                sc, rows = [], []
                for j in range(i + 1):
                    pg = int(mp.kv_indices[int(mp.kv_indptr[b]) + j])
                    s = sum(qn[q0 + i, h, x] * ckv[pg, 0, x] for x in range(6))
                    s += sum(qp[q0 + i, h, x] * kpe[pg, 0, x] for x in range(3))
                    sc.append(s * mp.sm_scale)
                    rows.append(ckv[pg, 0])
                mx = max(sc)
                ex = [math.exp(s - mx) for s in sc]
                ref = sum(e * r for e, r in zip(ex, rows)) / sum(ex)
                np.testing.assert_allclose(o[q0 + i, h], ref, rtol=0, atol=1e-12)
                assert abs(lse[q0 + i, h] - (mx + math.log(sum(ex))) / math.log(2)) < 1e-12


def test_rows_helper_matches_full():
    pb = _small(95, [20, 31], [20, 31], 4, 2, 8, 4, True)
    o, lse = _run_oracle(pb)
    pos = [0, 5, 30]
    o_r, l_r = oracle.paged_attention_rows(pb.q, pb.k_cache, pb.v_cache, pb.qo_indptr, pb.kv_indptr,
                                           pb.kv_indices, pb.kv_last_page_len, 4, True, pb.sm_scale,
                                           1, pos)
    q0 = int(pb.qo_indptr[1])
    np.testing.assert_allclose(o_r, o[[q0 + p for p in pos]], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_r, lse[[q0 + p for p in pos]], rtol=0, atol=1e-13)


def test_workload_shapes():
    t = W.tiny_prefill()
    assert list(t.qo_lens) == [7, 33] and list(t.kv_last_page_len) == [7, 1]
    assert t.k_cache.shape == (16, 16, 1, 64) and len(t.kv_indices) == 4
    assert len(set(t.kv_indices.tolist())) == 4
    g = W.gqa_prefill()
    assert g.batch == 8 and g.q.shape[1:] == (16, 128) and g.page_size == 64
    assert np.all((g.qo_lens >= 512) & (g.qo_lens <= 4096))
    assert sorted(g.kv_indices.tolist()) == list(range(g.num_pages))
    f = W.gqa_prefill_fp8()
    assert f.is_fp8_kv and f.causal and list(f.qo_lens) == list(g.qo_lens) and list(f.kv_lens) == list(g.kv_lens)
    assert f.k_cache.dtype == torch.uint8 and f.k_cache.shape[1:] == (64, 1, 128)


# ---------------------------------------------------------------------------
# mutation tests: plant mistakes in a copy of the oracle, check a pin fails
# ---------------------------------------------------------------------------

def _mutant_attend(kind):
    def attend(q, k, v, causal, sm_scale, q_pos=None, qo_len=None):
        n, hq, _ = q.shape
        kv_len, hk = k.shape[0], k.shape[1]
        qo_len = n if qo_len is None else qo_len
        q_pos = np.arange(n) if q_pos is None else np.asarray(q_pos)
        group = hq // hk
        o = np.zeros((n, hq, v.shape[2]))
        lse2 = np.full((n, hq), -np.inf)
        mask = paged_ref.visible(qo_len, kv_len, causal, q_pos)
        if kind == "causal_off_by_one":
            mask = paged_ref.visible(qo_len, kv_len, causal, q_pos + 1) if causal else mask
        if kind == "top_left_causal" and causal:
            mask = np.arange(kv_len)[None, :] <= q_pos[:, None]
        for h in range(hq):
            g = (h % hk) if kind == "gqa_modulo" else h // group
            kk = k[:, g, :]
            s = sm_scale * (q[:, h, :] @ (kk[:, ::-1] if kind == "reversed_dim" else kk).T)
            w, lse = paged_ref.softmax_rows(s, mask)
            o[:, h, :] = w @ v[:, g, :]
            lse2[:, h] = lse if kind == "natural_lse" else lse / paged_ref.LN2
        return o, lse2
    return attend


@pytest.mark.parametrize("kind", ["causal_off_by_one", "top_left_causal", "gqa_modulo",
                                  "reversed_dim", "natural_lse"])
def test_pins_catch_planted_mistakes(kind, monkeypatch):
    monkeypatch.setattr(paged_ref, "attend", _mutant_attend(kind))
    caught = False
    for case in BRUTE_CASES:
        try:
            test_brute_force(case)
        except AssertionError:
            caught = True
            break
    assert caught, f"brute-force pins did not catch mutant {kind}"


def test_merge_pin_catches_natural_log_merge(monkeypatch):
    def bad(o_a, lse_a, o_b, lse_b):
        m = np.maximum(lse_a, lse_b)
        lse = m + np.log(np.exp(lse_a - m) + np.exp(lse_b - m))
        wa, wb = np.exp(lse_a - lse), np.exp(lse_b - lse)
        return wa[..., None] * o_a + wb[..., None] * o_b, lse
    monkeypatch.setattr(oracle, "merge_state", bad)
    case = [c for c in _golden_cases() if c["kind"] == "merge"][0]
    with pytest.raises(AssertionError):
        test_golden_hand_worked(case)


# --------------------------------------------------------------------------- paged KV append

def _append_case(seed, page_size=4, hk=2, d=8):
    """Lengths after the append, new-row counts, a permuted pool with spare pages."""
    g = np.random.default_rng(seed)
    kv_after = np.array([5, 1, 9, 12, 0], dtype=np.int64)
    n_new = np.array([2, 1, 9, 3, 0], dtype=np.int64)
    n_pages = (kv_after + page_size - 1) // page_size
    kv_indptr = np.concatenate([[0], np.cumsum(n_pages)]).astype(np.int32)
    pool = int(n_pages.sum()) + 3
    kv_indices = g.permutation(pool)[: int(n_pages.sum())].astype(np.int32)
    last = np.where(n_pages > 0, kv_after - (n_pages - 1) * page_size, 0).astype(np.int32)
    append_indptr = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    nnz = int(n_new.sum())
    k_new = torch.from_numpy(g.standard_normal((nnz, hk, d))).to(torch.bfloat16)
    v_new = torch.from_numpy(g.standard_normal((nnz, hk, d))).to(torch.bfloat16)
    return dict(kv_after=kv_after, n_new=n_new, kv_indptr=kv_indptr, kv_indices=kv_indices, last=last,
                append_indptr=append_indptr, k_new=k_new, v_new=v_new, pool=pool, page_size=page_size, hk=hk, d=d)


def test_append_round_trip_through_gather():
    """Append into an all-zero pool, then read each request back in order with
    gather_pages (a separate, pinned path): positions kv_len - n .. kv_len - 1
    hold the new rows in order, every other position is still zero."""
    c = _append_case(1)
    z = torch.zeros((c["pool"], c["page_size"], c["hk"], c["d"]), dtype=torch.bfloat16)
    k, v = oracle.append_paged_kv(z, z, c["k_new"], c["v_new"], c["append_indptr"], c["kv_indptr"],
                                  c["kv_indices"], c["last"], c["page_size"])
    for b, (L, n) in enumerate(zip(c["kv_after"], c["n_new"])):
        for cache, new in ((k, c["k_new"]), (v, c["v_new"])):
            rows = oracle.gather_pages(cache, c["kv_indptr"], c["kv_indices"], c["last"], c["page_size"], b)
            assert rows.shape[0] == L
            a0 = int(c["append_indptr"][b])
            assert np.array_equal(rows[L - n:], new[a0:a0 + n].float().numpy())
            assert not np.any(rows[:L - n])


def test_append_in_two_steps_equals_one():
    """Appending the new rows in two batches (page table growing in between)
    writes the same pool as one append of all of them."""
    c = _append_case(2)
    P = c["page_size"]
    base = torch.from_numpy(np.random.default_rng(9).standard_normal(
        (c["pool"], P, c["hk"], c["d"]))).to(torch.bfloat16)
    k1, _ = oracle.append_paged_kv(base, base, c["k_new"], c["v_new"], c["append_indptr"], c["kv_indptr"],
                                   c["kv_indices"], c["last"], P)
    # first step: each request gets the first half of its rows, with the table truncated accordingly
    first = c["n_new"] // 2
    second = c["n_new"] - first
    mid_len = c["kv_after"] - second
    mid_pages = (mid_len + P - 1) // P
    mid_indptr = np.concatenate([[0], np.cumsum(mid_pages)]).astype(np.int32)
    mid_indices = np.concatenate([c["kv_indices"][c["kv_indptr"][b]:c["kv_indptr"][b] + mid_pages[b]]
                                  for b in range(len(mid_len))]).astype(np.int32)
    mid_last = np.where(mid_pages > 0, mid_len - (mid_pages - 1) * P, 0).astype(np.int32)
    sel1 = np.concatenate([np.arange(c["append_indptr"][b], c["append_indptr"][b] + first[b])
                           for b in range(len(first))]).astype(np.int64)
    sel2 = np.concatenate([np.arange(c["append_indptr"][b] + first[b], c["append_indptr"][b + 1])
                           for b in range(len(first))]).astype(np.int64)
    ind1 = np.concatenate([[0], np.cumsum(first)]).astype(np.int32)
    ind2 = np.concatenate([[0], np.cumsum(second)]).astype(np.int32)
    ka, _ = oracle.append_paged_kv(base, base, c["k_new"][sel1], c["v_new"][sel1], ind1, mid_indptr, mid_indices,
                                   mid_last, P)
    kb, _ = oracle.append_paged_kv(ka, ka, c["k_new"][sel2], c["v_new"][sel2], ind2, c["kv_indptr"],
                                   c["kv_indices"], c["last"], P)
    assert torch.equal(k1, kb)


def test_append_touches_only_new_slots():
    """Slots outside the appended positions keep their old bytes (unused pool
    pages included)."""
    c = _append_case(3)
    P = c["page_size"]
    base = torch.full((c["pool"], P, c["hk"], c["d"]), 7.0, dtype=torch.bfloat16)
    k, _ = oracle.append_paged_kv(base, base, c["k_new"], c["v_new"], c["append_indptr"], c["kv_indptr"],
                                  c["kv_indices"], c["last"], P)
    written = np.zeros((c["pool"], P), dtype=bool)
    for b, (L, n) in enumerate(zip(c["kv_after"], c["n_new"])):
        for pos in range(L - n, L):
            written[c["kv_indices"][c["kv_indptr"][b] + pos // P], pos % P] = True
    assert int(written.sum()) == int(c["n_new"].sum())
    assert torch.all(k[torch.from_numpy(~written)] == 7.0)


def test_append_pin_catches_off_by_one(monkeypatch):
    """A planted off-by-one in the oracle's position rule fails the round-trip pin."""
    real = paged_ref.kv_lengths
    monkeypatch.setattr(paged_ref, "kv_lengths", lambda *a: real(*a) + 1)
    with pytest.raises(AssertionError):
        try:
            test_append_round_trip_through_gather()
        except IndexError as e:  # a shifted position may also run off the page list
            raise AssertionError(str(e))


def test_cascade_identity():
    """Shared-prefix (cascade) decomposition: a non-causal pass of every query
    over the shared prefix merged with a causal pass over each request's own
    pages equals attention over prefix + own pages (queries are the last tokens
    of their suffix, so the whole prefix is visible to them)."""
    ps, hq, hk, d = 16, 8, 2, 32
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
    scale = 1 / math.sqrt(d)
    last_suf = (suffix - (suf_pages - 1) * ps).astype(np.int32)
    full_indptr = np.concatenate([[0], np.cumsum(pre_pages + suf_pages)]).astype(np.int32)
    full_ids = np.concatenate([np.concatenate([prefix_ids, s]) for s in suf_ids]).astype(np.int32)
    o_ref, l_ref = oracle.paged_attention(q, k, v, qo_indptr, full_indptr, full_ids, last_suf, ps, True, scale)
    o1, l1 = oracle.paged_attention(q, k, v, np.array([0, total_q], np.int32), np.array([0, pre_pages], np.int32),
                                    prefix_ids, np.array([ps], np.int32), ps, False, scale)
    suf_indptr = np.concatenate([[0], np.cumsum(suf_pages)]).astype(np.int32)
    o2, l2 = oracle.paged_attention(q, k, v, qo_indptr, suf_indptr, np.concatenate(suf_ids), last_suf, ps, True,
                                    scale)
    o, lse = oracle.merge_state(o1, l1, o2, l2)
    assert np.abs(o - o_ref).max() < 1e-12 and np.abs(lse - l_ref).max() < 1e-12


# ---------------------------------------------------------------------------
# per-head-scale FP8 E4M3 KV cache
# ---------------------------------------------------------------------------

def test_e4m3_decode_against_format_and_library():
    """Every one of the 256 codes against torch's float8_e4m3fn (a library
    decoder) and a few values fixed by the format itself."""
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    assert np.isnan(ours).sum() == 2  # S.1111.111 only
    ok = ~np.isnan(lib)
    assert np.array_equal(ours[ok], lib[ok])
    fixed = {0x00: 0.0, 0x38: 1.0, 0xB8: -1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9,
             0x08: 2.0 ** -6, 0x3C: 1.5, 0x40: 2.0, 0xC4: -3.0}
    for c, val in fixed.items():
        assert ours[c] == val, hex(c)


def _fp8_codes(shape, gen):
    """E4M3 codes of N(0, 1) values (no NaN codes), as uint8."""
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def test_quantized_kv_brute_force_per_head_scales():
    """Distinct per-head scales: the oracle against plain loops that decode each
    code with torch and multiply by its own head's scale."""
    gen = torch.Generator().manual_seed(7)
    hq, hk, d, p = 4, 2, 8, 4
    qo, kv = [1, 1, 1], [9, 4, 13]
    pb = _small(11, qo, kv, hq, hk, d, p, False)
    kc = _fp8_codes(tuple(pb.k_cache.shape), gen)
    vc = _fp8_codes(tuple(pb.v_cache.shape), gen)
    ks = torch.tensor([0.5, 3.0], dtype=torch.float32)
    vs = torch.tensor([2.0, 0.25], dtype=torch.float32)
    kd = kc.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vd = vc.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    k_ref, v_ref = np.zeros(kd.shape), np.zeros(vd.shape)
    for pg in range(kd.shape[0]):
        for s in range(p):
            for h in range(hk):
                for x in range(d):
                    k_ref[pg, s, h, x] = kd[pg, s, h, x] * float(ks[h])
                    v_ref[pg, s, h, x] = vd[pg, s, h, x] * float(vs[h])
    o_bf, l_bf = brute_force(_f64(pb.q), k_ref, v_ref, pb.qo_indptr, pb.kv_indptr, pb.kv_indices,
                             pb.kv_last_page_len, p, False, pb.sm_scale)
    o, lse = oracle.paged_attention_quantized_kv(pb.q, kc, vc, ks, vs, pb.qo_indptr, pb.kv_indptr, pb.kv_indices,
                                                 pb.kv_last_page_len, p, False, pb.sm_scale)
    assert np.abs(o - o_bf).max() < 1e-12 and np.abs(lse - l_bf).max() < 1e-12


def test_quantized_kv_scale_laws():
    """A V scale multiplies O and leaves the LSE; a K scale acts as a factor on
    sm_scale; unit scales reduce to attention over the decoded codes."""
    gen = torch.Generator().manual_seed(8)
    pb = _small(12, [1, 1], [37, 5], 8, 2, 16, 16, False)
    kc = _fp8_codes(tuple(pb.k_cache.shape), gen)
    vc = _fp8_codes(tuple(pb.v_cache.shape), gen)
    one = torch.ones(2)
    args = (pb.qo_indptr, pb.kv_indptr, pb.kv_indices, pb.kv_last_page_len, 16, False)
    o1, l1 = oracle.paged_attention_quantized_kv(pb.q, kc, vc, one, one, *args, pb.sm_scale)
    o2, l2 = oracle.paged_attention_quantized_kv(pb.q, kc, vc, one, torch.tensor([3.0, 3.0]), *args, pb.sm_scale)
    assert np.abs(o2 - 3.0 * o1).max() < 1e-12 and np.abs(l2 - l1).max() == 0.0
    o3, l3 = oracle.paged_attention_quantized_kv(pb.q, kc, vc, torch.tensor([0.75, 0.75]), one, *args, pb.sm_scale)
    o4, l4 = oracle.paged_attention_quantized_kv(pb.q, kc, vc, one, one, *args, pb.sm_scale * 0.75)
    assert np.abs(o3 - o4).max() < 1e-12 and np.abs(l3 - l4).max() < 1e-12
    kd = kc.view(torch.float8_e4m3fn).to(torch.float64)
    vd = vc.view(torch.float8_e4m3fn).to(torch.float64)
    o5, l5 = oracle.paged_attention(pb.q, kd, vd, *args, pb.sm_scale)
    assert np.abs(o5 - o1).max() < 1e-12 and np.abs(l5 - l1).max() < 1e-12


@pytest.mark.parametrize("kind", ["bias8", "subnormal_as_normal", "scale_by_slot"])
def test_quantized_pins_catch_planted_mistakes(kind, monkeypatch):
    """Plausible mistakes planted in a copy of the dequantisation fail a pin."""
    good_decode, good_dequant = paged_ref.e4m3_to_f64, paged_ref.dequantize_kv

    def decode(codes):
        c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
        e, m = (c >> 3) & 0xF, (c & 7) / 8.0
        sign = np.where(c >> 7, -1.0, 1.0)
        bias = 8.0 if kind == "bias8" else 7.0
        sub = (1.0 + m) * 2.0 ** (1.0 - bias) if kind == "subnormal_as_normal" else m * 2.0 ** (1.0 - bias)
        return sign * np.where(e == 0, sub, (1.0 + m) * np.exp2(e - bias))

    def dequant(codes, scale):
        vals = good_decode(np.asarray(codes))
        sc = np.asarray(scale, dtype=np.float64)
        return vals * sc[np.arange(vals.shape[1]) % len(sc)][None, :, None, None]  # by slot, not head

    if kind == "scale_by_slot":
        monkeypatch.setattr(paged_ref, "dequantize_kv", dequant)
        test = test_quantized_kv_brute_force_per_head_scales
    else:
        monkeypatch.setattr(paged_ref, "e4m3_to_f64", decode)
        monkeypatch.setattr(oracle, "e4m3_to_f64", decode)
        test = test_e4m3_decode_against_format_and_library
    with pytest.raises(AssertionError):
        test()
    assert paged_ref.dequantize_kv is (dequant if kind == "scale_by_slot" else good_dequant)
