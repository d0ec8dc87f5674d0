"""Batched attention over a paged KV cache for B200 (sm_100a).

A thin ctypes binding over the C ABI of ``libpkv.so`` (``include/pkv.h``).
It only marshals arguments: planning runs in the library's C++ planner and
every step of the attention runs in the library's CUDA kernels. PyTorch is
used for device memory and streams. There is no fallback: if the library is
missing, every call raises.

    p = plan(qo_indptr, kv_indptr, kv_indices, kv_last_page_len,
             num_qo_heads, num_kv_heads, head_dim, page_size, causal, sm_scale)
    o, lse = run(p, q, k_cache, v_cache)

Layouts and semantics are those of ``include/pkv.h`` (page table and ragged
queries as in flashinfer-trace discussion #15, "Notes on fa3_gqa_prefill_v1";
base-2 LSE; bottom-right causal mask).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

__all__ = ["plan", "plan_mla", "run", "run_mla", "merge_state", "merge_states", "device_status",
           "Plan", "PkvError", "lib_path", "load_library"]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libpkv.so")

PKV_OK, PKV_EINVAL, PKV_EUNSUPPORTED, PKV_ENOSPACE, PKV_ECUDA, PKV_EDEVICE = range(6)
_STATUS = {0: "OK", 1: "EINVAL", 2: "EUNSUPPORTED", 3: "ENOSPACE", 4: "ECUDA", 5: "EDEVICE"}

KIND_PREFILL, KIND_DECODE, KIND_MLA, KIND_MLA_DECODE = 0, 1, 2, 3


class PkvError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"pkv {_STATUS.get(status, status)}: {msg}")
        self.status = status


class _Options(ctypes.Structure):
    _fields_ = [("num_sms", ctypes.c_int32), ("disable_split_kv", ctypes.c_int32),
                ("kv_chunk", ctypes.c_int32), ("kv_layout", ctypes.c_int32), ("kv_fp8", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 3)]


_lib = None

_P = ctypes.c_void_p
_I32P = ctypes.POINTER(ctypes.c_int32)
_SIGS = {
    "pkv_plan_create": (ctypes.c_int, [_I32P, _I32P, _P, _I32P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                       ctypes.POINTER(_Options), ctypes.POINTER(_P)]),
    "pkv_plan_create_mla": (ctypes.c_int, [_I32P, _I32P, _P, _I32P, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_float, ctypes.POINTER(_Options), ctypes.POINTER(_P)]),
    "pkv_plan_workspace_bytes": (ctypes.c_size_t, [_P]),
    "pkv_plan_upload": (ctypes.c_int, [_P, _P, ctypes.c_size_t, _P]),
    "pkv_run": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int32, _P, _P, _P]),
    "pkv_run_mla": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int32, _P, _P, _P]),
    "pkv_run_fp8_kv": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P, _P]),
    "pkv_merge_state": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_int32, _P]),
    "pkv_merge_states": (ctypes.c_int, [_P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P, _P, _P]),
    "pkv_device_status": (ctypes.c_int, [_P, _P, _I32P]),
    "pkv_plan_info": (ctypes.c_int64, [_P, ctypes.c_int32]),
    "pkv_plan_work_units": (ctypes.c_int32, [_P, _I32P, ctypes.c_int32]),
    "pkv_plan_merge_tasks": (ctypes.c_int32, [_P, _I32P, ctypes.c_int32]),
    "pkv_plan_cta_units": (ctypes.c_int32, [_P, _I32P, ctypes.c_int32]),
    "pkv_merge_state_bf16": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_int32, _P]),
    "pkv_selftest_wait_timeout": (ctypes.c_int, [_P, _P, _P]),
    "pkv_append_kv": (ctypes.c_int, [_P, _P, _P, ctypes.c_int64, _P, _P, _P] + [ctypes.c_int32] * 7 + [_P, _P, _P, _P]),
    "pkv_plan_destroy": (None, [_P]),
    "pkv_last_error": (ctypes.c_char_p, []),
    "pkv_version": (ctypes.c_char_p, []),
}


def load_library():
    """Load libpkv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(f"{lib_path} is missing: build it with "
                               "`python -m paged_kv_attention_38_b200.build`")
        lib = ctypes.CDLL(lib_path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(status: int):
    if status != PKV_OK:
        raise PkvError(status, load_library().pkv_last_error().decode())


def _host_i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        if x.device.type != "cpu":
            raise ValueError("plan takes host (CPU) indptr / last_page_len arrays")
        x = x.detach().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(_I32P)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


class Plan:
    """A planned batch: owns the library plan handle and the device workspace."""

    def __init__(self, handle, kind, meta, kv_indices=None, workspace=None):
        self._h = handle
        self.kind = kind
        self.meta = meta
        self.kv_indices = kv_indices  # keeps the borrowed device array alive
        self.workspace = workspace

    @property
    def handle(self):
        return self._h

    def info(self, key: int) -> int:
        return int(load_library().pkv_plan_info(self._h, key))

    @property
    def num_units(self) -> int:
        return self.info(1)

    @property
    def num_merges(self) -> int:
        return self.info(2)

    @property
    def kv_chunk(self) -> int:
        return self.info(6)

    @property
    def num_ctas(self) -> int:
        return self.info(7)

    @property
    def workspace_bytes(self) -> int:
        return int(load_library().pkv_plan_workspace_bytes(self._h))

    def work_units(self) -> np.ndarray:
        n = self.num_units
        out = np.zeros((max(n, 1), 8), dtype=np.int32)
        got = load_library().pkv_plan_work_units(self._h, _i32p(out), n)
        return out[:got]

    def merge_tasks(self) -> np.ndarray:
        n = self.num_merges
        out = np.zeros((max(n, 1), 8), dtype=np.int32)
        got = load_library().pkv_plan_merge_tasks(self._h, _i32p(out), n)
        return out[:got]

    def cta_units(self) -> np.ndarray:
        """Persistent prefill schedule: CTA b runs work units [out[b], out[b+1]); empty otherwise."""
        n = self.num_ctas + 1
        out = np.zeros(n, dtype=np.int32)
        got = load_library().pkv_plan_cta_units(self._h, _i32p(out), n)
        return out[:got]

    def upload(self, device=None, stream=None):
        """Allocate the device workspace with torch and copy the schedule into it."""
        import torch
        nbytes = self.workspace_bytes
        dev = torch.device("cuda") if device is None else torch.device(device)
        ws = torch.empty(max(nbytes, 256) + 256, dtype=torch.uint8, device=dev)
        base = ws.data_ptr()
        aligned = (base + 255) & ~255
        self.workspace = ws
        _check(load_library().pkv_plan_upload(self._h, aligned, nbytes, _stream_ptr(stream)))
        return self

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h and _lib is not None:
            _lib.pkv_plan_destroy(h)


def _options(num_sms, disable_split_kv, kv_chunk, kv_layout=0, kv_fp8=False):
    o = _Options()
    o.num_sms, o.disable_split_kv, o.kv_chunk = int(num_sms), int(bool(disable_split_kv)), int(kv_chunk)
    o.kv_layout, o.kv_fp8 = int(kv_layout), int(bool(kv_fp8))
    return o


def plan(qo_indptr, kv_indptr, kv_indices, kv_last_page_len, num_qo_heads, num_kv_heads, head_dim,
         page_size, causal, sm_scale, *, num_sms: int = 0, disable_split_kv: bool = False,
         kv_chunk: int = 0, kv_layout: int = 0, kv_fp8: bool = False, upload: bool = True, device=None,
         stream=None) -> Plan:
    """Plan a GQA/MHA paged-attention batch (``pkv_plan_create`` + ``pkv_plan_upload``).

    ``qo_indptr``, ``kv_indptr``, ``kv_last_page_len`` are host int32 arrays;
    ``kv_indices`` is a device int32 tensor (may be None with ``upload=False``
    to inspect the schedule on a machine without a GPU). ``kv_layout``: 0 NHD
    pools ``[num_pages, page_size, Hk, D]``, 1 HND ``[num_pages, Hk, page_size, D]``. ``kv_fp8``: the
    plan will run through ``run_fp8_kv`` (its split-KV chunk is sized for that kernel; results do not
    depend on it).
    """
    lib = load_library()
    qo, kv, last = _host_i32(qo_indptr), _host_i32(kv_indptr), _host_i32(kv_last_page_len)
    h = _P()
    opts = _options(num_sms, disable_split_kv, kv_chunk, kv_layout, kv_fp8)
    _check(lib.pkv_plan_create(_i32p(qo), _i32p(kv), _ptr(kv_indices), _i32p(last), len(last), num_qo_heads,
                               num_kv_heads, head_dim, page_size, int(bool(causal)), float(sm_scale),
                               ctypes.byref(opts), ctypes.byref(h)))
    meta = dict(num_qo_heads=num_qo_heads, num_kv_heads=num_kv_heads, head_dim=head_dim, head_dim_v=head_dim,
                page_size=page_size, causal=bool(causal), sm_scale=float(sm_scale), total_q=int(qo[-1]) if len(qo) else 0)
    p = Plan(h.value, int(lib.pkv_plan_info(h.value, 0)), meta, kv_indices)
    if upload:
        p.upload(device, stream)
    return p


def plan_mla(qo_indptr, kv_indptr, kv_indices, kv_last_page_len, num_heads, head_dim_ckv, head_dim_kpe,
             page_size, causal, sm_scale, *, num_sms: int = 0, disable_split_kv: bool = False,
             kv_chunk: int = 0, upload: bool = True, device=None, stream=None) -> Plan:
    """Plan an absorbed-MLA paged batch (``pkv_plan_create_mla`` + ``pkv_plan_upload``)."""
    lib = load_library()
    qo, kv, last = _host_i32(qo_indptr), _host_i32(kv_indptr), _host_i32(kv_last_page_len)
    h = _P()
    opts = _options(num_sms, disable_split_kv, kv_chunk)
    _check(lib.pkv_plan_create_mla(_i32p(qo), _i32p(kv), _ptr(kv_indices), _i32p(last), len(last), num_heads,
                                   head_dim_ckv, head_dim_kpe, page_size, int(bool(causal)), float(sm_scale),
                                   ctypes.byref(opts), ctypes.byref(h)))
    meta = dict(num_qo_heads=num_heads, num_kv_heads=1, head_dim=head_dim_ckv, head_dim_v=head_dim_ckv,
                head_dim_pe=head_dim_kpe, page_size=page_size, causal=bool(causal), sm_scale=float(sm_scale),
                total_q=int(qo[-1]) if len(qo) else 0)
    p = Plan(h.value, int(lib.pkv_plan_info(h.value, 0)), meta, kv_indices)
    if upload:
        p.upload(device, stream)
    return p


def _check_tensor(t, name, dtype=None):
    import torch
    if t is None or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")


def run(p: Plan, q, k_cache, v_cache, o=None, lse=None, stream=None):
    """``pkv_run``: returns ``(o bf16 [total_q, Hq, D], lse fp32 [total_q, Hq])``."""
    import torch
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check_tensor(t, n, torch.bfloat16)
    total_q, hq = q.shape[0], q.shape[1]
    if o is None:
        o = torch.empty(total_q, hq, v_cache.shape[-1], dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(total_q, hq, dtype=torch.float32, device=q.device)
    _check(load_library().pkv_run(p.handle, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                  k_cache.shape[0], o.data_ptr(), lse.data_ptr(), _stream_ptr(stream)))
    return o, lse


def run_mla(p: Plan, q_nope, q_pe, ckv_cache, kpe_cache, o=None, lse=None, stream=None):
    """``pkv_run_mla``: returns ``(o bf16 [total_q, H, 512], lse fp32 [total_q, H])``."""
    import torch
    for t, n in ((q_nope, "q_nope"), (q_pe, "q_pe"), (ckv_cache, "ckv_cache"), (kpe_cache, "kpe_cache")):
        _check_tensor(t, n, torch.bfloat16)
    total_q, heads = q_nope.shape[0], q_nope.shape[1]
    if o is None:
        o = torch.empty(total_q, heads, ckv_cache.shape[-1], dtype=torch.bfloat16, device=q_nope.device)
    if lse is None:
        lse = torch.empty(total_q, heads, dtype=torch.float32, device=q_nope.device)
    _check(load_library().pkv_run_mla(p.handle, q_nope.data_ptr(), q_pe.data_ptr(), ckv_cache.data_ptr(),
                                      kpe_cache.data_ptr(), ckv_cache.shape[0], o.data_ptr(), lse.data_ptr(),
                                      _stream_ptr(stream)))
    return o, lse


def run_fp8_kv(p: Plan, q, k_codes, v_codes, k_scale=None, v_scale=None, o=None, lse=None, stream=None):
    """``pkv_run_fp8_kv``: attention over FP8 E4M3 K/V pools (``torch.float8_e4m3fn``
    or ``uint8`` codes, NHD) with optional per-kv-head fp32 scales
    ``[num_kv_heads]``, for a decode plan or a prefill plan made with
    ``kv_fp8=True``. Returns ``(o bf16 [total_q, Hq, D], lse fp32 [total_q, Hq])``."""
    import torch
    _check_tensor(q, "q", torch.bfloat16)
    for t, n in ((k_codes, "k_codes"), (v_codes, "v_codes")):
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
            raise ValueError(f"{n} must be uint8 or float8_e4m3fn codes")
        _check_tensor(t, n, t.dtype)
    hk = k_codes.shape[2]
    for t, n in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        if t is not None:
            _check_tensor(t, n, torch.float32)
            if t.numel() != hk:
                raise ValueError(f"{n} must hold one scale per kv head ({hk})")
    total_q, hq = q.shape[0], q.shape[1]
    if o is None:
        o = torch.empty(total_q, hq, v_codes.shape[-1], dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(total_q, hq, dtype=torch.float32, device=q.device)
    ptr = lambda t: t.data_ptr() if t is not None else None  # noqa: E731
    _check(load_library().pkv_run_fp8_kv(p.handle, q.data_ptr(), k_codes.data_ptr(), v_codes.data_ptr(),
                                         ptr(k_scale), ptr(v_scale), k_codes.shape[0], o.data_ptr(),
                                         lse.data_ptr(), _stream_ptr(stream)))
    return o, lse


def merge_state(o_a, lse_a, o_b, lse_b, stream=None, out=None):
    """``pkv_merge_state`` (fp32 O) or ``pkv_merge_state_bf16`` (bf16 O) on states
    ``[rows, dim]`` / ``[rows]`` (fp32 LSE, base 2). ``out``: optional ``(o, lse)``
    to write into (may be the first state)."""
    import torch
    dt = o_a.dtype
    if dt not in (torch.float32, torch.bfloat16):
        raise ValueError("o_a must be float32 or bfloat16")
    for t, n in ((o_a, "o_a"), (o_b, "o_b")):
        _check_tensor(t, n, dt)
    for t, n in ((lse_a, "lse_a"), (lse_b, "lse_b")):
        _check_tensor(t, n, torch.float32)
    dim = o_a.shape[-1]
    rows = o_a.numel() // dim
    o, lse = out if out is not None else (torch.empty_like(o_a), torch.empty_like(lse_a))
    fn = load_library().pkv_merge_state if dt == torch.float32 else load_library().pkv_merge_state_bf16
    _check(fn(o_a.data_ptr(), lse_a.data_ptr(), o_b.data_ptr(), lse_b.data_ptr(), o.data_ptr(), lse.data_ptr(), rows,
              dim, _stream_ptr(stream)))
    return o, lse


def cascade_run(prefix_plan: "Plan", suffix_plan: "Plan", q, k_cache, v_cache, stream=None):
    """Two-level cascade attention (documentation, flashinfer.cascade, "Cascade
    Attention"): ``prefix_plan`` runs every query against the KV prefix the batch
    shares (planned non-causal, typically as one request holding all queries),
    ``suffix_plan`` runs each request against its own pages; the two states are
    merged by their LSE. Returns ``(o bf16, lse fp32)`` as ``run`` does."""
    o, lse = run(prefix_plan, q, k_cache, v_cache, stream=stream)
    o2, lse2 = run(suffix_plan, q, k_cache, v_cache, stream=stream)
    return merge_state(o, lse, o2, lse2, stream=stream, out=(o, lse))


def append_kv(k_new, v_new, append_indptr, kv_indptr, kv_indices, kv_last_page_len, k_cache, v_cache,
              status=None, stream=None, kv_layout: int = 0):
    """``pkv_append_kv``: write new rows ``k_new`` / ``v_new`` ``[nnz, Hk, D]`` into the
    page pools ``[num_pages, page_size, Hk, D]`` in place, at the last positions of
    each request under the page table after the append (all index arrays int32 on
    the device). ``kv_layout`` 1: pools are HND ``[num_pages, Hk, page_size, D]``.
    ``status``: optional int32 device tensor set to 1 on a bad row."""
    import torch
    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check_tensor(t, n)
        if t.element_size() != 2:
            raise ValueError(f"{n} must hold 2-byte elements")
    for t, n in ((append_indptr, "append_indptr"), (kv_indptr, "kv_indptr"), (kv_indices, "kv_indices"),
                 (kv_last_page_len, "kv_last_page_len")):
        _check_tensor(t, n, torch.int32)
    if k_cache.dim() == 3:  # MLA pools [num_pages, page_size, D]: one latent "head"
        k_cache, v_cache = k_cache.unsqueeze(2), v_cache.unsqueeze(2)
        k_new, v_new = k_new.reshape(k_new.shape[0], 1, -1), v_new.reshape(v_new.shape[0], 1, -1)
    num_pages, page_size, hk, d = k_cache.shape
    if kv_layout == 1:
        num_pages, hk, page_size, d = k_cache.shape
    _check(load_library().pkv_append_kv(
        k_new.data_ptr(), v_new.data_ptr(), append_indptr.data_ptr(), int(k_new.shape[0]), kv_indptr.data_ptr(),
        kv_indices.data_ptr(), kv_last_page_len.data_ptr(), int(kv_last_page_len.shape[0]), hk, d,
        int(v_cache.shape[-1]), page_size, num_pages, int(kv_layout), k_cache.data_ptr(), v_cache.data_ptr(),
        status.data_ptr() if status is not None else None, _stream_ptr(stream)))


def merge_states(o_parts, lse_parts, stream=None):
    """``pkv_merge_states``: fp32 ``[num, rows, dim]`` / ``[num, rows]`` -> bf16 O, fp32 LSE."""
    import torch
    _check_tensor(o_parts, "o_parts", torch.float32)
    _check_tensor(lse_parts, "lse_parts", torch.float32)
    num, rows, dim = o_parts.shape
    o = torch.empty(rows, dim, dtype=torch.bfloat16, device=o_parts.device)
    lse = torch.empty(rows, dtype=torch.float32, device=o_parts.device)
    _check(load_library().pkv_merge_states(o_parts.data_ptr(), lse_parts.data_ptr(), num, rows, dim,
                                           o.data_ptr(), lse.data_ptr(), _stream_ptr(stream)))
    return o, lse


def device_status(p: Plan, stream=None) -> int:
    """``pkv_device_status``: 0 if no kernel reported an error (synchronises the stream)."""
    code = ctypes.c_int32(0)
    st = load_library().pkv_device_status(p.handle, _stream_ptr(stream), ctypes.byref(code))
    if st not in (PKV_OK, PKV_EDEVICE):
        _check(st)
    return int(code.value)
