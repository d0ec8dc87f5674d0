"""CPU tests of the C ABI library: it loads, exports every symbol include/pkv.h
declares, rejects malformed input with the documented status codes, and its
host planner covers every (request, kv head, query row, key) exactly once.

No GPU is needed: only host entry points are called (planning without upload).
"""
import ctypes
import os
import re

import numpy as np
import pytest

import paged_kv_attention_38_b200 as pkv
from oracle import paged_ref
from paged_kv_attention_38_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not os.path.exists(pkv.lib_path):
        from paged_kv_attention_38_b200 import build
        build.build()


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    lib = pkv.load_library()
    syms = _declared_symbols()
    assert len(syms) >= 14
    for s in syms:
        assert hasattr(lib, s), f"libpkv.so does not export {s}"
    assert lib.pkv_version().decode().startswith("pkv")


def test_no_hidden_symbol_leaks():
    """Only the pkv_ C ABI is exported (internal C++ symbols stay hidden)."""
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", pkv.lib_path], capture_output=True, text=True).stdout
    names = [l.split()[-1] for l in out.splitlines() if " T " in l]
    ours = [n for n in names if n.startswith("pkv_")]
    assert set(_declared_symbols()) <= set(ours)


def _plan(p: W.PagedProblem, **kw):
    kw.setdefault("num_sms", 148)
    return pkv.plan(p.qo_indptr, p.kv_indptr, None, p.kv_last_page_len, p.num_qo_heads, p.num_kv_heads,
                    p.head_dim, p.page_size, p.causal, p.sm_scale, upload=False, **kw)


def _lengths_problem(qo, kv, hq=4, hk=1, d=64, ps=16, causal=True):
    kv_indptr, kv_indices, last, _ = W.page_table(np.asarray(kv), ps, W._gen(5))
    qo_indptr = np.concatenate([[0], np.cumsum(qo)]).astype(np.int32)
    return W.PagedProblem("lens", qo_indptr, kv_indptr, kv_indices, last, ps, hq, hk, d, d, causal,
                          1.0 / np.sqrt(d))


def _check_coverage(p: W.PagedProblem, pl: pkv.Plan):
    """Every packed row of every (request, kv head) is covered; its units' key
    ranges partition [0, need) where need bounds the keys any row of the tile sees."""
    G = p.num_qo_heads // p.num_kv_heads
    units = pl.work_units()
    merges = pl.merge_tasks()
    rows_per = pl.info(4)
    tiles = {}
    for u in units:
        req, g, row0, rows, lo, hi, part, _ = u.tolist()
        tiles.setdefault((req, g, row0, rows), []).append((lo, hi, part))
    kv_lens, qo_lens = p.kv_lens, p.qo_lens
    slots_seen = set()
    for b in range(p.batch):
        packed = int(qo_lens[b]) * G
        for g in range(p.num_kv_heads):
            r = 0
            while r < packed:
                rows = min(rows_per, packed - r)
                key = (b, g, r, rows)
                assert key in tiles, f"missing tile {key}"
                t_first, t_last = r // G, (r + rows - 1) // G
                vis = paged_ref.visible(int(qo_lens[b]), int(kv_lens[b]), p.causal,
                                        np.arange(t_first, t_last + 1))
                need = int(vis.any(axis=0).nonzero()[0].max() + 1) if vis.any() else 0
                chunks = sorted(tiles.pop(key))
                assert chunks[0][0] == 0 and chunks[-1][1] == need
                for (a_lo, a_hi, _), (b_lo, _, _) in zip(chunks, chunks[1:]):
                    assert a_hi == b_lo
                if len(chunks) == 1:
                    assert chunks[0][2] == -1
                else:
                    parts = [c[2] for c in chunks]
                    assert all(x >= 0 for x in parts)
                    slots_seen.update(parts)
                    m = [t for t in merges.tolist() if t[:4] == [b, g, r, rows]]
                    assert len(m) == 1 and m[0][5] == len(chunks)
                    assert sorted(parts) == list(range(m[0][4], m[0][4] + m[0][5]))
                r += rows
    assert not tiles, f"extra tiles {list(tiles)[:3]}"
    assert len(slots_seen) == pl.info(3)


@pytest.mark.parametrize("maker", [W.tiny_prefill, W.gqa_prefill, W.paged_decode])
def test_planner_covers_workloads(maker):
    p = maker()
    _check_coverage(p, _plan(p))


@pytest.mark.parametrize("chunk", [128, 256, 1000])
def test_planner_forced_split(chunk):
    p = _lengths_problem([40, 1, 300], [40, 1300, 300], hq=8, hk=2)
    pl = _plan(p, kv_chunk=chunk)
    _check_coverage(p, pl)
    assert pl.num_merges > 0


@pytest.mark.parametrize("kv_fp8", [False, True])
@pytest.mark.parametrize("kv", [[10000, 20000, 5, 7], [100000], [512] * 4, [1, 63, 64, 65, 700, 3000],
                                [1024 + 61 * i for i in range(128)]])
def test_planner_decode_split_choice(kv, kv_fp8):
    """The decode split search: whatever chunk it picks is a multiple of the 64-key
    tile, at least 256 keys, shorter than the longest request (else no split), and
    the schedule covers every key exactly once."""
    p = _lengths_problem([1] * len(kv), kv, hq=32, hk=8, d=128, ps=16, causal=False)
    pl = _plan(p, kv_fp8=kv_fp8)
    assert pl.kind == pkv.KIND_DECODE
    c = pl.kv_chunk
    assert c == 0 or (c % 64 == 0 and 256 <= c < max(kv)), c
    assert (pl.num_merges > 0) == (c > 0 and max(kv) > c)
    _check_coverage(p, pl)


def test_planner_decode_split_balances_few_long_requests():
    """Eight (request, kv head) tiles of 100k keys cannot fill 148 SMs: the plan
    splits them into enough chunks for every SM."""
    p = _lengths_problem([1], [100000], hq=32, hk=8, d=128, ps=16, causal=False)
    pl = _plan(p)
    assert pl.num_units >= 148 and pl.num_merges == 8
    _check_coverage(p, pl)


def test_planner_disable_split_kv():
    p = _lengths_problem([1] * 4, [10000, 20000, 5, 7], hq=8, hk=2, ps=16, causal=False)
    pl = _plan(p, disable_split_kv=True)
    assert pl.num_merges == 0 and pl.kind == pkv.KIND_DECODE
    _check_coverage(p, pl)
    pl2 = _plan(p)
    assert pl2.num_merges > 0
    _check_coverage(p, pl2)


def test_planner_edge_cases():
    # empty request, qo_len > kv_len (rows with no key), qo_len = 0
    p = _lengths_problem([5, 0, 9, 3], [0, 4, 4, 3], hq=4, hk=2, ps=2)
    pl = _plan(p)
    _check_coverage(p, pl)
    # empty batch
    p0 = _lengths_problem([], [], hq=4, hk=1)
    pl0 = _plan(p0)
    assert pl0.num_units == 0


def test_planner_kinds():
    assert _plan(W.paged_decode()).kind == pkv.KIND_DECODE
    assert _plan(W.gqa_prefill()).kind == pkv.KIND_PREFILL
    m = W.mla_prefill()
    pl = pkv.plan_mla(m.qo_indptr, m.kv_indptr, None, m.kv_last_page_len, 16, 512, 64, 1, True,
                      m.sm_scale, upload=False, num_sms=148)
    assert pl.kind == pkv.KIND_MLA
    d = W.mla_decode()
    pl = pkv.plan_mla(d.qo_indptr, d.kv_indptr, None, d.kv_last_page_len, 16, 512, 64, 1, False,
                      d.sm_scale, upload=False, num_sms=148)
    assert pl.kind == pkv.KIND_MLA_DECODE and pl.info(4) == 16  # 16 rows (heads) per partial slot


def test_longest_units_first():
    """Decode CTAs run one unit each, handed out in index order: longest first."""
    pl = _plan(W.paged_decode())
    assert pl.cta_units().size == 0 and pl.num_ctas == pl.num_units
    u = pl.work_units()
    lens = u[:, 5] - u[:, 4]
    assert np.all(np.diff(lens) <= 0)


@pytest.mark.parametrize("maker,banded", [(W.gqa_prefill, False), (lambda: W.sparse_vs_dense(16, 2048, True), True),
                                          (W.tiny_prefill, False), (W.mla_prefill, False)])
def test_persistent_prefill_schedule(maker, banded):
    """Prefill: min(SMs, units) persistent CTAs; every unit in exactly one CTA's
    list and the greedy balance bound: the loads (KV tiles + 1 per unit)
    differ by at most one unit's cost. Each CTA's list is longest first; when
    the batch's K/V exceeds the L2 band size (16 x 2048 tokens x 8 kv heads:
    134 MB) it is instead ordered band by band, i.e. by (request, kv head)
    group, so that concurrently running units share groups."""
    p = maker()
    if p.is_mla:
        pl = pkv.plan_mla(p.qo_indptr, p.kv_indptr, None, p.kv_last_page_len, p.num_qo_heads, 512, 64, p.page_size,
                          p.causal, p.sm_scale, upload=False, num_sms=148)
    else:
        pl = _plan(p)
    tile = 64 if p.is_mla else 128
    u = pl.work_units()
    ptr = pl.cta_units()
    assert pl.num_ctas == min(148, len(u)) == len(ptr) - 1
    assert ptr[0] == 0 and ptr[-1] == len(u) and np.all(np.diff(ptr) >= 1)
    cost = (u[:, 5] - u[:, 4] + tile - 1) // tile + 1
    loads = np.array([cost[a:b].sum() for a, b in zip(ptr[:-1], ptr[1:])])
    group = u[:, 0].astype(np.int64) * p.num_kv_heads + u[:, 1]
    # bands: whole groups in (request, kv head) order, cut once a band holds >= 148 units
    per_group = np.bincount(group, minlength=int(group.max()) + 1)
    band_of, band, run = np.zeros(len(per_group), np.int64), 0, 0
    for g_, n in enumerate(per_group):
        band_of[g_] = band
        run += n
        if run >= 148:
            band, run = band + 1, 0
    band_u = band_of[group]
    for a, b in zip(ptr[:-1], ptr[1:]):
        if banded:
            assert np.all(np.diff(band_u[a:b]) >= 0)
        else:
            assert np.all(np.diff(u[a:b, 5] - u[a:b, 4]) <= 0)
    assert loads.max() - loads.min() <= cost.max()
    assert loads.sum() == cost.sum()
    # coverage: every (req, head, row block, kv range) exactly once
    assert len({tuple(r) for r in u[:, :6].tolist()}) == len(u)


@pytest.mark.parametrize("mutate,status", [
    (lambda a: a["qo"].__setitem__(1, -3), pkv.PKV_EINVAL),            # qo_indptr decreasing
    (lambda a: a["kv"].__setitem__(0, 1), pkv.PKV_EINVAL),             # kv_indptr not starting at 0
    (lambda a: a["last"].__setitem__(0, 0), pkv.PKV_EINVAL),           # last_page_len 0 with pages
    (lambda a: a["last"].__setitem__(0, 17), pkv.PKV_EINVAL),          # last_page_len > page_size
    (lambda a: a.__setitem__("ps", 24), pkv.PKV_EUNSUPPORTED),         # page size not a power of two
    (lambda a: a.__setitem__("d", 96), pkv.PKV_EUNSUPPORTED),          # unsupported head_dim
    (lambda a: a.__setitem__("hk", 3), pkv.PKV_EINVAL),                # hq % hk != 0
    (lambda a: a.__setitem__("scale", float("nan")), pkv.PKV_EINVAL),  # sm_scale not finite
    (lambda a: a.__setitem__("scale", 0.0), pkv.PKV_EUNSUPPORTED),     # sm_scale must be positive
])
def test_error_codes(mutate, status):
    a = dict(qo=np.array([0, 5, 9], np.int32), kv=np.array([0, 1, 2], np.int32),
             last=np.array([5, 4], np.int32), ps=16, d=64, hk=1, scale=0.125)
    mutate(a)
    with pytest.raises(pkv.PkvError) as e:
        pkv.plan(a["qo"], a["kv"], None, a["last"], 4, a["hk"], a["d"], a["ps"], True, a["scale"],
                 upload=False, num_sms=148)
    assert e.value.status == status
    assert len(pkv.load_library().pkv_last_error()) > 0


def test_upload_rejects_bad_workspace():
    lib = pkv.load_library()
    p = _lengths_problem([5], [5])
    pl = _plan(p)
    assert lib.pkv_plan_upload(pl.handle, None, 0, None) == pkv.PKV_EINVAL
    assert lib.pkv_plan_upload(pl.handle, 256, 1, None) == pkv.PKV_ENOSPACE
    assert lib.pkv_plan_upload(pl.handle, 257, 1 << 20, None) == pkv.PKV_EINVAL
    # run before upload is refused before any launch
    assert lib.pkv_run(pl.handle, 16, 16, 16, 1, 16, 16, None) == pkv.PKV_EINVAL
    assert lib.pkv_merge_state(None, None, None, None, None, None, 4, 0, None) == pkv.PKV_EINVAL
    assert lib.pkv_merge_states(None, None, 0, 4, 8, None, None, None) == pkv.PKV_EINVAL


def test_append_host_validation():
    """pkv_append_kv rejects bad arguments on the host, before any launch."""
    lib = pkv.load_library()
    one = ctypes.c_int32(0)
    p = ctypes.cast(ctypes.pointer(one), ctypes.c_void_p)  # a host address: never dereferenced on these paths
    args = lambda nnz, hk, d, dv, ps, pages, ptr, lay=0: (ptr, ptr, ptr, nnz, ptr, ptr, ptr, 1, hk, d, dv, ps, pages,
                                                          lay, ptr, ptr, None, None)
    assert lib.pkv_append_kv(*args(0, 1, 64, 64, 16, 4, p)) == pkv.PKV_OK            # nothing to append
    assert lib.pkv_append_kv(*args(-1, 1, 64, 64, 16, 4, p)) == pkv.PKV_EINVAL
    assert lib.pkv_append_kv(*args(4, 1, 12, 64, 16, 4, p)) == pkv.PKV_EUNSUPPORTED  # head_dim not a multiple of 8
    assert lib.pkv_append_kv(*args(4, 1, 64, 64, 0, 4, p)) == pkv.PKV_EINVAL         # page_size 0
    assert lib.pkv_append_kv(*args(4, 1, 64, 64, 16, 4, p, 2)) == pkv.PKV_EINVAL     # unknown layout
    assert lib.pkv_append_kv(*args(4, 1, 64, 64, 16, 4, None)) == pkv.PKV_EINVAL     # NULL pointers
    assert b"NULL" in lib.pkv_last_error()


def test_kv_layout_option():
    """kv_layout 0 (NHD) and 1 (HND) plan the same schedule; other values are rejected."""
    p = W.gqa_prefill()
    a = _plan(p)
    b = pkv.plan(p.qo_indptr, p.kv_indptr, None, p.kv_last_page_len, p.num_qo_heads, p.num_kv_heads, p.head_dim,
                 p.page_size, p.causal, p.sm_scale, upload=False, num_sms=148, kv_layout=1)
    assert np.array_equal(a.work_units(), b.work_units())
    with pytest.raises(pkv.PkvError):
        pkv.plan(p.qo_indptr, p.kv_indptr, None, p.kv_last_page_len, p.num_qo_heads, p.num_kv_heads, p.head_dim,
                 p.page_size, p.causal, p.sm_scale, upload=False, num_sms=148, kv_layout=2)


@pytest.mark.parametrize("trial", range(40))
def test_planner_random_batches(trial):
    """Seeded random batches over every plan kind (GQA prefill, decode, MLA
    prefill, MLA decode), page sizes, causal flags, SM counts and forced KV
    chunks: the work list covers every packed row exactly once with key ranges
    that partition what the rows can see, the merge list matches the split
    units, and persistent plans deal every unit to exactly one CTA within the
    greedy balance bound."""
    g = np.random.default_rng(1000 + trial)
    kind = trial % 4
    batch = int(g.integers(1, 7))
    ps = int(2 ** g.integers(0, 7))
    causal = bool(g.integers(0, 2))
    sms = int(g.choice([1, 7, 64, 148]))
    chunk = int(g.choice([0, 0, 64, 200, 777]))
    kv = g.integers(0, 900, size=batch)
    if kind in (1, 3):  # one query token per request
        qo = np.ones(batch, dtype=np.int64)
        causal = False
    else:
        qo = np.minimum(g.integers(0, 300, size=batch), np.maximum(kv, 1)) if causal else g.integers(0, 300, size=batch)
    if kind >= 2:
        p = W.make_mla_problem("rnd", qo, kv, num_heads=int(g.choice([4, 8, 16])), page_size=ps, causal=causal,
                               seed=trial)
        pl = pkv.plan_mla(p.qo_indptr, p.kv_indptr, None, p.kv_last_page_len, p.num_qo_heads, 512, 64, ps, causal,
                          p.sm_scale, upload=False, num_sms=sms, kv_chunk=chunk)
        assert pl.kind == (pkv.KIND_MLA_DECODE if kind == 3 else pkv.KIND_MLA)
    else:
        hk = int(g.choice([1, 2, 4]))
        hq = hk * int(g.choice([1, 2, 4, 8] if kind == 1 else [1, 3, 4, 16]))
        p = _lengths_problem(qo, kv, hq=hq, hk=hk, ps=ps, causal=causal)
        pl = _plan(p, num_sms=sms, kv_chunk=chunk)
        assert pl.kind == (pkv.KIND_DECODE if kind == 1 else pkv.KIND_PREFILL)
    _check_coverage(p, pl)
    ptr = pl.cta_units()
    if pl.kind in (pkv.KIND_PREFILL, pkv.KIND_MLA) and pl.num_units > 0:
        u = pl.work_units()
        assert len(ptr) == pl.num_ctas + 1 == min(sms, len(u)) + 1
        assert ptr[0] == 0 and ptr[-1] == len(u) and np.all(np.diff(ptr) >= 1)
        tile = 64 if pl.kind == pkv.KIND_MLA else 128
        cost = (u[:, 5] - u[:, 4] + tile - 1) // tile + 1
        loads = np.array([cost[a:b].sum() for a, b in zip(ptr[:-1], ptr[1:])])
        assert loads.max() - loads.min() <= cost.max()
    else:
        assert ptr.size == 0 and pl.num_ctas == pl.num_units


def test_fp8_kv_workload_and_host_checks():
    """The FP8-KV decode workload (codes, masked slots, per-head scales), the
    bench's byte count for it, and the binding's host-side argument checks."""
    import torch
    import bench
    p = W.make_fp8_kv_problem("fp8", [1, 1, 1], [5, 40, 16], num_qo_heads=8, num_kv_heads=2, head_dim=64,
                              page_size=16, seed=1)
    assert p.is_fp8_kv and p.k_cache.dtype == torch.uint8 and p.k_cache.shape == (p.num_pages, 16, 2, 64)
    valid = torch.zeros(p.num_pages, 16, dtype=torch.bool)
    for b in range(p.batch):
        for pos in range(int(p.kv_lens[b])):
            valid[int(p.kv_indices[p.kv_indptr[b] + pos // 16]), pos % 16] = True
    assert torch.all(p.k_cache[~valid] == 0) and torch.all(p.v_cache[~valid] == 0x7E)
    codes = p.k_cache[valid]
    assert not torch.any((codes & 0x7F) == 0x7F), "no NaN codes in valid slots"
    for s in (p.meta["k_scale"], p.meta["v_scale"]):
        assert s.shape == (2,) and s.dtype == torch.float32 and torch.all((s >= 0.5) & (s <= 2.0))
    n_keys = int(p.kv_lens.sum())
    fixed = 2 * (2 * 3 * 8 * 64) + 4 * 3 * 8 + 4 * len(p.kv_indices)  # Q and O bf16, LSE, page ids
    assert bench.decode_bytes(p) == 2 * 2 * 64 * n_keys + 8 * 2 + fixed
    pl_like = object()
    with pytest.raises(ValueError):
        pkv.run_fp8_kv(pl_like, p.q, p.k_cache, p.v_cache)  # host tensors are refused before any call


def test_fp8_kv_entry_rejects_unsupported_plans():
    """pkv_run_fp8_kv refuses prefill plans made without the kv_fp8 option and
    HND plans with PKV_EUNSUPPORTED before touching any pointer, and plans that
    were never uploaded with PKV_EINVAL."""
    lib = pkv.load_library()
    args = [None] * 5 + [1, None, None, None]

    def call(pl):
        st = lib.pkv_run_fp8_kv(pl.handle, *args)
        return st, lib.pkv_last_error().decode()

    pre = _plan(W.tiny_prefill())
    assert pre.kind == pkv.KIND_PREFILL
    st, msg = call(pre)
    assert st == 2 and "kv_fp8" in msg
    st, msg = call(_plan(W.tiny_prefill(), kv_fp8=True))
    assert st == 1 and "not uploaded" in msg
    dec = _lengths_problem([1, 1], [300, 40], hq=8, hk=2, d=128, ps=16, causal=False)
    st, msg = call(_plan(dec, kv_layout=1))
    assert st == 2 and "NHD" in msg
    st, msg = call(_plan(dec))
    assert st == 1 and "not uploaded" in msg


def test_fp8_prefill_plan_reserves_page_copy():
    """A prefill plan made with kv_fp8 reserves the bf16 copy of the batch's K and
    V pages ([entries][page_size][Hk][D]) and its identity page table in the
    workspace; a decode plan and an MLA plan reserve nothing for it."""
    def align(x):
        return (x + 255) // 256 * 256

    p = _lengths_problem([30, 0, 70], [100, 17, 70], hq=8, hk=2, d=64, ps=16, causal=True)
    entries = int(p.kv_indptr[-1])
    base, fp8 = _plan(p).workspace_bytes, _plan(p, kv_fp8=True).workspace_bytes
    page = 16 * 2 * 64 * 2
    assert fp8 - base == 2 * align(entries * page) + align(4 * entries)
    dec = _lengths_problem([1, 1], [300, 40], hq=8, hk=2, d=128, ps=16, causal=False)
    assert _plan(dec, kv_fp8=True).workspace_bytes == _plan(dec).workspace_bytes
