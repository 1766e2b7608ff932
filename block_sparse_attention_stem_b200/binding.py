"""ctypes binding of ``libstem.so`` (the C ABI declared in include/stem.h).

Argument marshalling only: every step of the path runs inside the CUDA
library.  PyTorch supplies device memory and the current stream.  If the
shared library is missing, importing this module raises; there is no fallback.

Entry points mirror the C names: ``stem_plan``, ``stem_score``,
``stem_select``, ``stem_bsa_fwd``, ``stem_prefill``,
``stem_read_device_status``, ``stem_status_string``.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libstem.so")

STEM_OK = 0
STATUS_NAMES = {0: "STEM_OK", 1: "STEM_ERR_INVALID_ARG", 2: "STEM_ERR_UNSUPPORTED",
                3: "STEM_ERR_WORKSPACE_TOO_SMALL", 4: "STEM_ERR_MISALIGNED", 5: "STEM_ERR_CUDA",
                6: "STEM_ERR_TIMEOUT", 7: "STEM_ERR_BAD_BLOCKLIST"}
STEM_BF16, STEM_FP8_E4M3 = 0, 1
EXPORTED = ("stem_plan", "stem_score", "stem_select", "stem_score_select", "stem_bsa_fwd", "stem_bsa_fwd_paged",
            "stem_prefill",
            "stem_prefill_host",
            "stem_prefill_noalloc", "stem_noalloc_read_device_status",
            "stem_selftest_wait_timeout", "stem_read_device_status", "stem_status_string", "stem_version")


class StemParams(ctypes.Structure):
    _fields_ = [("block_size", ctypes.c_int32), ("stride", ctypes.c_int32), ("chunk_size", ctypes.c_int32),
                ("norm", ctypes.c_double), ("beta", ctypes.c_double), ("keep_ratio", ctypes.c_double),
                ("mu", ctypes.c_double), ("sink_blocks", ctypes.c_int32), ("window_blocks", ctypes.c_int32),
                ("softmax_scale", ctypes.c_double), ("budget_mode", ctypes.c_int32), ("bonus_mode", ctypes.c_int32),
                ("list_mode", ctypes.c_int32), ("select_mode", ctypes.c_int32)]


class StemQKV(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
                ("cu_seqlens", ctypes.c_void_p), ("cu_seqlens_host", ctypes.POINTER(ctypes.c_int32)),
                ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("q_scale", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p)]


class StemPagedKV(ctypes.Structure):
    _fields_ = [("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("page_table", ctypes.c_void_p), ("k_pages", ctypes.c_void_p), ("v_pages", ctypes.c_void_p)]


class StemPlan(ctypes.Structure):
    _fields_ = [("nb_total", ctypes.c_int64), ("nb_max", ctypes.c_int64), ("num_rows", ctypes.c_int64),
                ("nnz", ctypes.c_int64), ("nnz_per_head", ctypes.c_int64), ("scores_bytes", ctypes.c_size_t),
                ("vbonus_bytes", ctypes.c_size_t), ("ws_bytes", ctypes.c_size_t),
                ("ws_prefill_bytes", ctypes.c_size_t), ("attn_flops", ctypes.c_double),
                ("dense_attn_flops", ctypes.c_double), ("score_flops", ctypes.c_double),
                ("vwide_bytes", ctypes.c_size_t)]


class StemError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({stem_status_string(code)})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m block_sparse_attention_stem_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    P = ctypes.POINTER
    lib.stem_plan.argtypes = [P(StemQKV), P(StemParams), P(StemPlan)]
    lib.stem_score.argtypes = [P(StemQKV), P(StemParams), vp, vp, vp, sz, vp]
    lib.stem_select.argtypes = [P(StemQKV), P(StemParams), vp, vp, vp, vp, vp, sz, vp]
    lib.stem_score_select.argtypes = [P(StemQKV), P(StemParams), vp, vp, vp, vp, vp, vp, sz, vp]
    lib.stem_bsa_fwd.argtypes = [P(StemQKV), P(StemParams), vp, vp, vp, vp, vp, sz, vp]
    lib.stem_bsa_fwd_paged.argtypes = [P(StemQKV), P(StemPagedKV), P(StemParams), vp, vp, vp, vp, vp, sz, vp]
    lib.stem_prefill.argtypes = [P(StemQKV), P(StemParams), vp, vp, vp, vp, vp, sz, vp]
    lib.stem_prefill_noalloc.argtypes = [P(StemQKV), P(StemParams), vp, vp, vp, vp, vp]
    lib.stem_noalloc_read_device_status.argtypes = [vp, P(ctypes.c_int)]
    lib.stem_prefill_host.argtypes = [P(StemQKV), P(StemParams), vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.stem_selftest_wait_timeout.argtypes = [vp, vp]
    lib.stem_read_device_status.argtypes = [vp, vp, P(ctypes.c_int)]
    lib.stem_status_string.argtypes = [ctypes.c_int]
    lib.stem_status_string.restype = ctypes.c_char_p
    lib.stem_version.restype = ctypes.c_int32
    for name in ("stem_plan", "stem_score", "stem_select", "stem_bsa_fwd", "stem_prefill",
                 "stem_prefill_noalloc", "stem_noalloc_read_device_status", "stem_selftest_wait_timeout",
                 "stem_read_device_status"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


LIB = _load()


def stem_status_string(code: int) -> str:
    return LIB.stem_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != STEM_OK:
        raise StemError(code, where)


def make_params(block_size=128, stride=8, chunk_size=2048, norm=1.0, beta=0.2, keep_ratio=0.25, mu=0.7,
                sink_blocks=4, window_blocks=4, softmax_scale=0.0, budget_mode=0, bonus_mode=0,
                list_mode=0, select_mode=0) -> StemParams:
    return StemParams(block_size, stride, chunk_size, float(norm), float(beta), float(keep_ratio), float(mu),
                      sink_blocks, window_blocks, float(softmax_scale), budget_mode, bonus_mode, list_mode,
                      select_mode)


def _ptr(t):
    return None if t is None else t.data_ptr()


@dataclass
class QKV:
    """Tensors of one call plus the ctypes descriptor that points at them.
    Keeps references so the memory stays alive while the descriptor is used."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    cu_dev: torch.Tensor
    cu_host: torch.Tensor
    q_scale: torch.Tensor | None
    k_scale: torch.Tensor | None
    v_scale: torch.Tensor | None
    desc: StemQKV

    @property
    def total_tokens(self) -> int:
        return int(self.cu_host[-1])


def make_qkv(q, k, v, cu_seqlens, q_scale=None, k_scale=None, v_scale=None, cu_seqlens_dev=None) -> QKV:
    """q [T,Hq,128], k/v [T,Hkv,128]: bf16, or uint8 / float8_e4m3fn bytes with
    fp32 per-head scales.  cu_seqlens: host int32 offsets (list or tensor)."""
    cu_host = torch.as_tensor(cu_seqlens, dtype=torch.int32).cpu().contiguous()
    if cu_seqlens_dev is None:
        cu_seqlens_dev = cu_host.to(q.device)
    if q.dtype == torch.bfloat16:
        dtype = STEM_BF16
    elif q.dtype in (torch.uint8, torch.float8_e4m3fn):
        dtype = STEM_FP8_E4M3
    else:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k and v must be contiguous [T, H, d]")
    desc = StemQKV(dtype, cu_host.numel() - 1, int(cu_host[-1]), _ptr(cu_seqlens_dev),
                   ctypes.cast(cu_host.data_ptr(), ctypes.POINTER(ctypes.c_int32)),
                   q.shape[1], k.shape[1], q.shape[2], _ptr(q), _ptr(k), _ptr(v),
                   _ptr(q_scale), _ptr(k_scale), _ptr(v_scale))
    return QKV(q, k, v, cu_seqlens_dev, cu_host, q_scale, k_scale, v_scale, desc)


def stem_plan(qkv: QKV, params: StemParams) -> StemPlan:
    out = StemPlan()
    _check(LIB.stem_plan(ctypes.byref(qkv.desc), ctypes.byref(params), ctypes.byref(out)), "stem_plan")
    return out


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ws(nbytes: int, device, ws):
    if ws is None:
        ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    return ws


def stem_score(qkv: QKV, params: StemParams, scores=None, vbonus=None, ws=None, stream=None):
    pl = stem_plan(qkv, params)
    dev = qkv.q.device
    hq, hkv = qkv.q.shape[1], qkv.k.shape[1]
    if scores is None:
        scores = torch.empty(hq, pl.nb_total, pl.nb_max, dtype=torch.float32, device=dev)
    if vbonus is None:
        vbonus = torch.empty(hkv, pl.nb_total, dtype=torch.float32, device=dev)
    ws = _ws(pl.ws_bytes, dev, ws)
    _check(LIB.stem_score(ctypes.byref(qkv.desc), ctypes.byref(params), _ptr(scores), _ptr(vbonus),
                          _ptr(ws), ws.numel(), _stream(stream)), "stem_score")
    return scores, vbonus, ws


def stem_select(qkv: QKV, params: StemParams, scores, budgets=None, row_ptr=None, col_idx=None, ws=None,
                stream=None):
    pl = stem_plan(qkv, params)
    dev = scores.device
    if budgets is None:
        budgets = torch.empty(pl.num_rows, dtype=torch.int32, device=dev)
    if row_ptr is None:
        row_ptr = torch.empty(pl.num_rows + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(max(pl.nnz, 1), dtype=torch.int32, device=dev)
    ws = _ws(pl.ws_bytes, dev, ws)
    _check(LIB.stem_select(ctypes.byref(qkv.desc), ctypes.byref(params), _ptr(scores), _ptr(budgets),
                           _ptr(row_ptr), _ptr(col_idx), _ptr(ws), ws.numel(), _stream(stream)), "stem_select")
    return budgets, row_ptr, col_idx[:pl.nnz], ws


def stem_score_select(qkv: QKV, params: StemParams, scores=None, vbonus=None, budgets=None, row_ptr=None,
                      col_idx=None, ws=None, stream=None):
    """stem_score then stem_select in one call (in one pass when params.select_mode is 1)."""
    pl = stem_plan(qkv, params)
    dev = qkv.q.device
    hq, hkv = qkv.q.shape[1], qkv.k.shape[1]
    if scores is None:
        scores = torch.empty(hq, pl.nb_total, pl.nb_max, dtype=torch.float32, device=dev)
    if budgets is None:
        budgets = torch.empty(pl.num_rows, dtype=torch.int32, device=dev)
    if row_ptr is None:
        row_ptr = torch.empty(pl.num_rows + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(max(pl.nnz, 1), dtype=torch.int32, device=dev)
    ws = _ws(pl.ws_bytes, dev, ws)
    _check(LIB.stem_score_select(ctypes.byref(qkv.desc), ctypes.byref(params), _ptr(scores), _ptr(vbonus),
                                 _ptr(budgets), _ptr(row_ptr), _ptr(col_idx), _ptr(ws), ws.numel(),
                                 _stream(stream)), "stem_score_select")
    return scores, budgets, row_ptr, col_idx[:pl.nnz], ws


@dataclass
class PagedKV:
    """A paged K/V pool and the descriptor that points at it; keeps the
    tensors alive while the descriptor is used."""
    k_pages: torch.Tensor
    v_pages: torch.Tensor
    page_table: torch.Tensor
    desc: StemPagedKV


def paged_kv(k_pages, v_pages, page_table, page_size: int) -> PagedKV:
    """k_pages/v_pages [P, page_size, Hkv, d] device tensors, page_table int32
    [num_seqs, max_pages] on the device."""
    if page_table.dtype != torch.int32 or page_table.dim() != 2 or not page_table.is_contiguous():
        raise ValueError("page_table must be a contiguous int32 [num_seqs, max_pages] tensor")
    if k_pages.shape != v_pages.shape or k_pages.shape[1] != page_size:
        raise ValueError("k_pages and v_pages must both be [P, page_size, Hkv, d]")
    desc = StemPagedKV(page_size, k_pages.shape[0], page_table.shape[1], _ptr(page_table), _ptr(k_pages),
                       _ptr(v_pages))
    return PagedKV(k_pages, v_pages, page_table, desc)


def stem_bsa_fwd_paged(qkv: QKV, kv: PagedKV, params: StemParams, row_ptr, col_idx, out=None, lse=None,
                       ws=None, stream=None):
    pl = stem_plan(qkv, params)
    dev = qkv.q.device
    T, hq = qkv.total_tokens, qkv.q.shape[1]
    if out is None:
        out = torch.empty(T, hq, 128, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(hq, T, dtype=torch.float32, device=dev)
    ws = _ws(pl.ws_bytes, dev, ws)
    _check(LIB.stem_bsa_fwd_paged(ctypes.byref(qkv.desc), ctypes.byref(kv.desc), ctypes.byref(params), _ptr(row_ptr),
                                  _ptr(col_idx), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "stem_bsa_fwd_paged")
    return out, lse, ws


def stem_bsa_fwd(qkv: QKV, params: StemParams, row_ptr, col_idx, out=None, lse=None, ws=None, stream=None):
    pl = stem_plan(qkv, params)
    dev = qkv.q.device
    T, hq = qkv.total_tokens, qkv.q.shape[1]
    if out is None:
        out = torch.empty(T, hq, 128, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(hq, T, dtype=torch.float32, device=dev)
    ws = _ws(pl.ws_bytes, dev, ws)
    _check(LIB.stem_bsa_fwd(ctypes.byref(qkv.desc), ctypes.byref(params), _ptr(row_ptr), _ptr(col_idx),
                            _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)), "stem_bsa_fwd")
    return out, lse, ws


def stem_prefill(qkv: QKV, params: StemParams, out=None, lse=None, row_ptr=None, col_idx=None, ws=None,
                 stream=None, return_lists=True):
    pl = stem_plan(qkv, params)
    dev = qkv.q.device
    T, hq = qkv.total_tokens, qkv.q.shape[1]
    if out is None:
        out = torch.empty(T, hq, 128, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(hq, T, dtype=torch.float32, device=dev)
    if return_lists and row_ptr is None:
        row_ptr = torch.empty(pl.num_rows + 1, dtype=torch.int32, device=dev)
    if return_lists and col_idx is None:
        col_idx = torch.empty(max(pl.nnz, 1), dtype=torch.int32, device=dev)
    ws = _ws(pl.ws_prefill_bytes, dev, ws)
    _check(LIB.stem_prefill(ctypes.byref(qkv.desc), ctypes.byref(params), _ptr(out), _ptr(lse), _ptr(row_ptr),
                            _ptr(col_idx), _ptr(ws), ws.numel(), _stream(stream)), "stem_prefill")
    return out, lse, row_ptr, (None if col_idx is None else col_idx[:pl.nnz]), ws


def stem_prefill_host(qkv: QKV, params: StemParams, q_host, k_host, v_host, out_host, lse_host, out=None, lse=None,
                      ws=None, stream=None):
    """stem_prefill with inputs and outputs in (page-locked) host tensors; the
    device tensors of `qkv` are filled by the call, transfers overlap compute.
    Only enqueues: synchronize `stream` before reading out_host / lse_host."""
    pl = stem_plan(qkv, params)
    dev = qkv.q.device
    T, hq = qkv.total_tokens, qkv.q.shape[1]
    for name, t, like in (("q_host", q_host, qkv.q), ("k_host", k_host, qkv.k), ("v_host", v_host, qkv.v)):
        if t.device.type != "cpu" or t.shape != like.shape or t.dtype != like.dtype or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor shaped like the device one")
    if out_host.device.type != "cpu" or tuple(out_host.shape) != (T, hq, 128) or out_host.dtype != torch.bfloat16:
        raise ValueError("out_host must be a host bf16 tensor [T, Hq, 128]")
    if lse_host.device.type != "cpu" or tuple(lse_host.shape) != (hq, T) or lse_host.dtype != torch.float32:
        raise ValueError("lse_host must be a host fp32 tensor [Hq, T]")
    if out is None:
        out = torch.empty(T, hq, 128, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(hq, T, dtype=torch.float32, device=dev)
    ws = _ws(pl.ws_prefill_bytes, dev, ws)
    _check(LIB.stem_prefill_host(ctypes.byref(qkv.desc), ctypes.byref(params), _ptr(q_host), _ptr(k_host),
                                 _ptr(v_host), _ptr(out), _ptr(lse), _ptr(out_host), _ptr(lse_host), _ptr(ws),
                                 ws.numel(), _stream(stream)), "stem_prefill_host")
    return out, lse, ws


def stem_prefill_noalloc(qkv: QKV, params: StemParams, out=None, lse=None, row_ptr=None, col_idx=None,
                         stream=None, return_lists=True):
    """stem_prefill on the library's built-in 32 MiB workspace (for callers that
    cannot allocate one); the outputs are still the caller's."""
    pl = stem_plan(qkv, params)
    dev = qkv.q.device
    T, hq = qkv.total_tokens, qkv.q.shape[1]
    if out is None:
        out = torch.empty(T, hq, 128, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(hq, T, dtype=torch.float32, device=dev)
    if return_lists and row_ptr is None:
        row_ptr = torch.empty(pl.num_rows + 1, dtype=torch.int32, device=dev)
    if return_lists and col_idx is None:
        col_idx = torch.empty(max(pl.nnz, 1), dtype=torch.int32, device=dev)
    _check(LIB.stem_prefill_noalloc(ctypes.byref(qkv.desc), ctypes.byref(params), _ptr(out), _ptr(lse),
                                    _ptr(row_ptr), _ptr(col_idx), _stream(stream)), "stem_prefill_noalloc")
    return out, lse, row_ptr, (None if col_idx is None else col_idx[:pl.nnz])


def stem_noalloc_read_device_status(stream=None) -> int:
    """Status word of stem_prefill_noalloc's built-in workspace on the current
    device (synchronises the stream)."""
    out = ctypes.c_int(0)
    _check(LIB.stem_noalloc_read_device_status(_stream(stream), ctypes.byref(out)),
           "stem_noalloc_read_device_status")
    return out.value


def stem_selftest_wait_timeout(ws, stream=None):
    """Run the bounded-wait self-test; read the result with stem_read_device_status."""
    _check(LIB.stem_selftest_wait_timeout(_ptr(ws), _stream(stream)), "stem_selftest_wait_timeout")


def stem_read_device_status(ws, stream=None) -> int:
    out = ctypes.c_int(0)
    _check(LIB.stem_read_device_status(_ptr(ws), _stream(stream), ctypes.byref(out)), "stem_read_device_status")
    return out.value
