"""Seeded synthetic inputs for batched attention over a paged KV cache.

This module only draws random numbers and lays them out in the page-table
format; it holds none of the attention arithmetic. Both the CUDA path (tests,
bench) and the float64 oracle consume what it produces, so it imports nothing
from either of them.

Layouts (FlashInfer 0.7.4 documentation, tutorial "KV-Cache Layout in
FlashInfer": "Layout: NHD/HND", "Ragged Tensor", "Page Table Layout";
flashinfer-trace discussion #15, "Notes on fa3_gqa_prefill_v1"):

* ``q``            ragged, ``[total_q, num_qo_heads, head_dim]``, rows of request
                   ``b`` are ``qo_indptr[b] : qo_indptr[b+1]``.
* ``k_cache``      NHD pages, ``[num_pages, page_size, num_kv_heads, head_dim]``.
* ``v_cache``      NHD pages, ``[num_pages, page_size, num_kv_heads, head_dim_v]``.
* ``kv_indptr``    ``[B+1]`` prefix sum of the number of pages of each request.
* ``kv_indices``   ``[kv_indptr[B]]`` physical page ids, request by request.
* ``kv_last_page_len`` ``[B]`` valid slots in each request's last page
                   (``1..page_size``; 0 only for a request with no page).

MLA (FlashInfer 0.2 release, "Fused MLA decode kernel"; definition
``mla_paged_prefill_causal_h16_ckv512_kpe64_ps1`` in flashinfer-trace
discussion #15): ``q_nope [total_q, H, 512]``, ``q_pe [total_q, H, 64]``,
``ckv_cache [num_pages, page_size, 512]``, ``kpe_cache [num_pages, page_size, 64]``.

Recipe: every value is bf16 drawn as float32 N(0, 1) from a seeded
``torch.Generator`` on the CPU and rounded to bf16. Lengths are integers drawn
uniformly from an inclusive range. ``kv_indices`` is a random permutation of
the pool. Pool slots that hold no valid token (unused pages, and the slots
past ``kv_last_page_len`` in a last page) hold a finite sentinel: 0 in K and
``SENTINEL_V`` in V, so that a kernel that reads one of them without masking
it moves the output by a visible amount.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

SENTINEL_K = 0.0
SENTINEL_V = 1.0e4

SEED_BASE = 1000


@dataclass
class PagedProblem:
    """One batch of paged attention: page table, ragged queries and the page pools."""

    name: str
    qo_indptr: np.ndarray          # int32 [B+1]
    kv_indptr: np.ndarray          # int32 [B+1]
    kv_indices: np.ndarray         # int32 [nnz_pages]
    kv_last_page_len: np.ndarray   # int32 [B]
    page_size: int
    num_qo_heads: int
    num_kv_heads: int
    head_dim: int                  # QK contraction width (512 + 64 split for MLA)
    head_dim_v: int
    causal: bool
    sm_scale: float
    q: Optional[torch.Tensor] = None         # bf16 [total_q, Hq, D]
    k_cache: Optional[torch.Tensor] = None   # bf16 [num_pages, P, Hk, D]
    v_cache: Optional[torch.Tensor] = None   # bf16 [num_pages, P, Hk, Dv]
    # MLA operands (head_dim_pe > 0)
    head_dim_pe: int = 0
    q_nope: Optional[torch.Tensor] = None    # bf16 [total_q, H, Dckv]
    q_pe: Optional[torch.Tensor] = None      # bf16 [total_q, H, Dpe]
    ckv_cache: Optional[torch.Tensor] = None # bf16 [num_pages, P, Dckv]
    kpe_cache: Optional[torch.Tensor] = None # bf16 [num_pages, P, Dpe]
    seed: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return len(self.kv_last_page_len)

    @property
    def qo_lens(self) -> np.ndarray:
        return np.diff(self.qo_indptr).astype(np.int64)

    @property
    def kv_lens(self) -> np.ndarray:
        n = np.diff(self.kv_indptr).astype(np.int64)
        return np.where(n > 0, (n - 1) * self.page_size + self.kv_last_page_len, 0)

    @property
    def num_pages(self) -> int:
        pool = self.k_cache if self.k_cache is not None else self.ckv_cache
        return int(pool.shape[0])

    @property
    def total_q(self) -> int:
        return int(self.qo_indptr[-1])

    @property
    def is_mla(self) -> bool:
        return self.head_dim_pe > 0

    @property
    def is_fp8_kv(self) -> bool:
        return self.k_cache is not None and self.k_cache.dtype == torch.uint8


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def uniform_lengths(batch: int, lo: int, hi: int, gen: torch.Generator) -> np.ndarray:
    """``batch`` integers uniform in ``[lo, hi]`` (both ends included)."""
    return torch.randint(lo, hi + 1, (batch,), generator=gen).numpy().astype(np.int64)


def page_table(kv_lens, page_size: int, gen: torch.Generator, pool_pages: Optional[int] = None):
    """Flat page table for the given KV lengths.

    Request ``b`` owns ``ceil(kv_len_b / page_size)`` pages. Physical ids are the
    first ``nnz`` entries of a seeded random permutation of ``range(pool_pages)``
    (by default the pool is exactly the pages needed).
    Returns ``kv_indptr, kv_indices, kv_last_page_len, pool_pages``.
    """
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    n_pages = (kv_lens + page_size - 1) // page_size
    kv_indptr = np.zeros(len(kv_lens) + 1, dtype=np.int32)
    kv_indptr[1:] = np.cumsum(n_pages)
    nnz = int(kv_indptr[-1])
    if pool_pages is None:
        pool_pages = nnz
    assert pool_pages >= nnz
    perm = torch.randperm(pool_pages, generator=gen).numpy().astype(np.int32)
    kv_indices = perm[:nnz].copy()
    last = np.where(n_pages > 0, kv_lens - (n_pages - 1) * page_size, 0).astype(np.int32)
    return kv_indptr, kv_indices, last, pool_pages


def _valid_slot_mask(kv_indptr, kv_indices, last, page_size, pool_pages) -> torch.Tensor:
    """Bool ``[pool_pages, page_size]``: True where a slot holds a request's token."""
    valid = torch.zeros(pool_pages, page_size, dtype=torch.bool)
    for b in range(len(last)):
        lo, hi = int(kv_indptr[b]), int(kv_indptr[b + 1])
        if hi == lo:
            continue
        pages = torch.from_numpy(kv_indices[lo:hi].astype(np.int64))
        valid[pages[:-1]] = True
        valid[pages[-1], : int(last[b])] = True
    return valid


def make_problem(name: str, qo_lens, kv_lens, *, num_qo_heads: int, num_kv_heads: int,
                 head_dim: int, page_size: int, causal: bool, seed: int,
                 head_dim_v: Optional[int] = None, sm_scale: Optional[float] = None,
                 pool_pages: Optional[int] = None, contiguous: bool = False) -> PagedProblem:
    """A GQA paged problem with the given per-request lengths.

    ``contiguous=True`` lays the pages out in order (``kv_indices = arange``): the
    dense ragged layout of the same problem when ``page_size == 1``.
    """
    head_dim_v = head_dim if head_dim_v is None else head_dim_v
    sm_scale = 1.0 / math.sqrt(head_dim) if sm_scale is None else sm_scale
    gen = _gen(seed)
    qo_lens = np.asarray(qo_lens, dtype=np.int64)
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    kv_indptr, kv_indices, last, pool = page_table(kv_lens, page_size, gen, pool_pages)
    if contiguous:
        kv_indices = np.arange(len(kv_indices), dtype=np.int32)
    qo_indptr = np.zeros(len(qo_lens) + 1, dtype=np.int32)
    qo_indptr[1:] = np.cumsum(qo_lens)
    gen_t = _gen(seed + 100)
    q = _randn_bf16((int(qo_indptr[-1]), num_qo_heads, head_dim), gen_t)
    valid = _valid_slot_mask(kv_indptr, kv_indices, last, page_size, pool)
    vmask_k = valid[:, :, None, None].expand(pool, page_size, num_kv_heads, head_dim)
    vmask_v = valid[:, :, None, None].expand(pool, page_size, num_kv_heads, head_dim_v)
    k = _randn_bf16((pool, page_size, num_kv_heads, head_dim), gen_t)
    v = _randn_bf16((pool, page_size, num_kv_heads, head_dim_v), gen_t)
    k[~vmask_k] = SENTINEL_K
    v[~vmask_v] = SENTINEL_V
    return PagedProblem(name=name, qo_indptr=qo_indptr, kv_indptr=kv_indptr,
                        kv_indices=kv_indices, kv_last_page_len=last, page_size=page_size,
                        num_qo_heads=num_qo_heads, num_kv_heads=num_kv_heads,
                        head_dim=head_dim, head_dim_v=head_dim_v, causal=causal,
                        sm_scale=sm_scale, q=q, k_cache=k, v_cache=v, seed=seed)


def make_fp8_kv_problem(name: str, qo_lens, kv_lens, *, num_qo_heads: int, num_kv_heads: int, head_dim: int,
                        page_size: int, seed: int, causal: bool = False, sm_scale: Optional[float] = None,
                        pool_pages: Optional[int] = None) -> PagedProblem:
    """A GQA paged problem over a per-head-scale FP8 KV cache: ``k_cache`` and
    ``v_cache`` are uint8 ``[num_pages, P, Hk, D]`` pools of E4M3 codes of N(0, 1)
    draws, and ``meta`` holds one fp32 scale per kv head for K and for V
    (``k_scale``, ``v_scale``, uniform in [0.5, 2]). Slots past a request's end
    hold code 0 in K and the code of 448, the largest E4M3 value, in V."""
    sm_scale = 1.0 / math.sqrt(head_dim) if sm_scale is None else sm_scale
    gen = _gen(seed)
    qo_lens = np.asarray(qo_lens, dtype=np.int64)
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    kv_indptr, kv_indices, last, pool = page_table(kv_lens, page_size, gen, pool_pages)
    qo_indptr = np.zeros(len(qo_lens) + 1, dtype=np.int32)
    qo_indptr[1:] = np.cumsum(qo_lens)
    gen_t = _gen(seed + 100)
    q = _randn_bf16((int(qo_indptr[-1]), num_qo_heads, head_dim), gen_t)
    shape = (pool, page_size, num_kv_heads, head_dim)
    k = torch.randn(*shape, generator=gen_t, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
    v = torch.randn(*shape, generator=gen_t, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
    valid = _valid_slot_mask(kv_indptr, kv_indices, last, page_size, pool)
    k[~valid] = 0
    v[~valid] = 0x7E
    k_scale = (0.5 + 1.5 * torch.rand(num_kv_heads, generator=gen_t)).to(torch.float32)
    v_scale = (0.5 + 1.5 * torch.rand(num_kv_heads, generator=gen_t)).to(torch.float32)
    return PagedProblem(name=name, qo_indptr=qo_indptr, kv_indptr=kv_indptr,
                        kv_indices=kv_indices, kv_last_page_len=last, page_size=page_size,
                        num_qo_heads=num_qo_heads, num_kv_heads=num_kv_heads,
                        head_dim=head_dim, head_dim_v=head_dim, causal=causal,
                        sm_scale=sm_scale, q=q, k_cache=k, v_cache=v, seed=seed,
                        meta={"k_scale": k_scale, "v_scale": v_scale})


def make_mla_problem(name: str, qo_lens, kv_lens, *, num_heads: int = 16, head_dim_ckv: int = 512,
                     head_dim_kpe: int = 64, page_size: int = 1, causal: bool = True,
                     seed: int = 0, sm_scale: Optional[float] = None,
                     pool_pages: Optional[int] = None) -> PagedProblem:
    """An absorbed-MLA paged problem: one latent KV (ckv | kpe) shared by all heads."""
    sm_scale = 1.0 / math.sqrt(192.0) if sm_scale is None else sm_scale
    gen = _gen(seed)
    qo_lens = np.asarray(qo_lens, dtype=np.int64)
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    kv_indptr, kv_indices, last, pool = page_table(kv_lens, page_size, gen, pool_pages)
    qo_indptr = np.zeros(len(qo_lens) + 1, dtype=np.int32)
    qo_indptr[1:] = np.cumsum(qo_lens)
    gen_t = _gen(seed + 100)
    tq = int(qo_indptr[-1])
    q_nope = _randn_bf16((tq, num_heads, head_dim_ckv), gen_t)
    q_pe = _randn_bf16((tq, num_heads, head_dim_kpe), gen_t)
    valid = _valid_slot_mask(kv_indptr, kv_indices, last, page_size, pool)
    ckv = _randn_bf16((pool, page_size, head_dim_ckv), gen_t)
    kpe = _randn_bf16((pool, page_size, head_dim_kpe), gen_t)
    ckv[~valid] = SENTINEL_V
    kpe[~valid] = SENTINEL_K
    return PagedProblem(name=name, qo_indptr=qo_indptr, kv_indptr=kv_indptr,
                        kv_indices=kv_indices, kv_last_page_len=last, page_size=page_size,
                        num_qo_heads=num_heads, num_kv_heads=1,
                        head_dim=head_dim_ckv, head_dim_v=head_dim_ckv, causal=causal,
                        sm_scale=sm_scale, head_dim_pe=head_dim_kpe, q_nope=q_nope,
                        q_pe=q_pe, ckv_cache=ckv, kpe_cache=kpe, seed=seed)


# ---------------------------------------------------------------------------
# The five workloads. Seeds: lengths and permutation from SEED_BASE + id,
# tensors from SEED_BASE + id + 100.
# ---------------------------------------------------------------------------

def tiny_prefill() -> PagedProblem:
    """Causal GQA paged prefill, batch 2, qo_len = kv_len = (7, 33), 4 qo / 1 kv head,
    head_dim 64, page_size 16, pages drawn from a permuted 16-page pool."""
    lens = [7, 33]
    return make_problem("tiny_gqa_prefill_b2_h4_kv1_d64_ps16", lens, lens,
                        num_qo_heads=4, num_kv_heads=1, head_dim=64, page_size=16,
                        causal=True, seed=SEED_BASE + 1, pool_pages=16)


def gqa_prefill(batch: int = 8, lo: int = 512, hi: int = 4096, shard: int = 0) -> PagedProblem:
    """Causal GQA paged prefill: qo_len = kv_len ~ U[512, 4096], 16 qo / 1 kv head,
    head_dim 128, page_size 64, permuted pool (h16/kv1/d128/ps64). `shard` draws
    another independent batch of the same shape (one per data-parallel rank)."""
    seed = SEED_BASE + 2 + 10000 * shard
    lens = uniform_lengths(batch, lo, hi, _gen(seed + 7))
    return make_problem("gqa_paged_prefill_causal_h16_kv1_d128_ps64", lens, lens,
                        num_qo_heads=16, num_kv_heads=1, head_dim=128, page_size=64,
                        causal=True, seed=seed)


def gqa_prefill_fp8(batch: int = 8, lo: int = 512, hi: int = 4096, shard: int = 0) -> PagedProblem:
    """The causal GQA prefill batch of ``gqa_prefill`` (same lengths, h16/kv1/d128/ps64)
    over a per-head-scale FP8 E4M3 KV cache."""
    seed = SEED_BASE + 2 + 10000 * shard
    lens = uniform_lengths(batch, lo, hi, _gen(seed + 7))
    return make_fp8_kv_problem("gqa_paged_prefill_fp8kv_h16_kv1_d128_ps64", lens, lens, num_qo_heads=16,
                               num_kv_heads=1, head_dim=128, page_size=64, seed=seed + 900, causal=True)


SPARSE_DENSE_SWEEP = [(1, 512), (1, 2048), (1, 8192), (16, 512), (16, 2048), (16, 8192),
                      (64, 512), (64, 2048)]


def sparse_vs_dense(batch: int, seq_len: int, contiguous: bool) -> PagedProblem:
    """Causal prefill, 32 qo / 8 kv heads, head_dim 128.

    ``contiguous=False``: page_size 1 with the token slots scattered over the
    pool (vector sparsity). ``contiguous=True``: the dense ragged layout of the
    same problem, i.e. every request's K/V rows contiguous and in order; it is
    described to the kernel as 64-slot pages with the identity page table,
    which is the same memory layout ([total_kv, Hk, D] row-major) since every
    length in the sweep is a multiple of 64."""
    seed = SEED_BASE + 3
    lens = [seq_len] * batch
    if contiguous:
        assert seq_len % 64 == 0
        return make_problem(f"dense_prefill_causal_b{batch}_l{seq_len}_h32_kv8_d128", lens, lens,
                            num_qo_heads=32, num_kv_heads=8, head_dim=128, page_size=64,
                            causal=True, seed=seed, contiguous=True)
    return make_problem(f"sparse_prefill_causal_b{batch}_l{seq_len}_h32_kv8_d128_ps1", lens, lens,
                        num_qo_heads=32, num_kv_heads=8, head_dim=128, page_size=1,
                        causal=True, seed=seed)


def paged_decode(batch: int = 128, lo: int = 1024, hi: int = 8192, shard: int = 0) -> PagedProblem:
    """Paged decode: q_len 1, 32 qo / 8 kv heads, head_dim 128, page_size 16,
    kv_len ~ U[1024, 8192]. Non-causal (one query sees every key)."""
    seed = SEED_BASE + 4 + 10000 * shard
    kv = uniform_lengths(batch, lo, hi, _gen(seed + 7))
    return make_problem("paged_decode_b128_h32_kv8_d128_ps16", [1] * batch, kv,
                        num_qo_heads=32, num_kv_heads=8, head_dim=128, page_size=16,
                        causal=False, seed=seed)


def paged_decode_fp8(batch: int = 128, lo: int = 1024, hi: int = 8192, shard: int = 0) -> PagedProblem:
    """The paged decode batch shape (32 qo / 8 kv heads, head_dim 128, page_size
    16, kv_len ~ U[1024, 8192]) over a per-head-scale FP8 E4M3 KV cache."""
    seed = SEED_BASE + 8 + 10000 * shard
    kv = uniform_lengths(batch, lo, hi, _gen(seed + 7))
    return make_fp8_kv_problem("paged_decode_fp8kv_b128_h32_kv8_d128_ps16", [1] * batch, kv, num_qo_heads=32,
                               num_kv_heads=8, head_dim=128, page_size=16, seed=seed)


def mla_decode(batch: int = 64, lo: int = 1024, hi: int = 8192, shard: int = 0) -> PagedProblem:
    """Absorbed MLA decode: one query token per request, 16 heads, ckv 512 + kpe 64,
    page_size 1 (slots scattered over the pool), kv_len ~ U[lo, hi], sm_scale 1/sqrt(192)."""
    seed = SEED_BASE + 6 + 10000 * shard
    kv = uniform_lengths(batch, lo, hi, _gen(seed + 7))
    return make_mla_problem("mla_paged_decode_h16_ckv512_kpe64_ps1", [1] * batch, kv, num_heads=16,
                            causal=False, seed=seed)


def mla_prefill(batch: int = 4, lo: int = 256, hi: int = 2048, shard: int = 0) -> PagedProblem:
    """Absorbed MLA causal paged prefill, 16 heads, ckv 512 + kpe 64, page_size 1,
    sm_scale 1/sqrt(192) (h16/ckv512/kpe64/ps1)."""
    seed = SEED_BASE + 5 + 10000 * shard
    lens = uniform_lengths(batch, lo, hi, _gen(seed + 7))
    return make_mla_problem("mla_paged_prefill_causal_h16_ckv512_kpe64_ps1", lens, lens,
                            num_heads=16, seed=seed)
