"""Python binding of the s5attn C ABI (``include/s5attn.h``).

Argument marshalling only: every step of the path runs in the CUDA library.
Tensors are torch CUDA tensors (PyTorch provides device memory and streams);
the functions keep the C names and raise ``S5Error`` on a non-OK status.
There is no CPU fallback: importing this module fails if the library is
missing.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libs5attn.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_gqa_indexer_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

ABI_VERSION = 102  # S5_ABI_VERSION of the header this binding follows
N_HEADS, N_KV, HEAD_DIM, PAGE, BLOCK, INDEX_DIM, MAX_TOPK = 64, 4, 192, 64, 8, 256, 512
MAX_LEN = 1 << 21
DEFAULT_SM_SCALE = 1.0 / math.sqrt(HEAD_DIM)

S5_OK, S5_ERR_INVALID_ARG, S5_ERR_UNSUPPORTED, S5_ERR_CUDA, S5_ERR_DEVICE_BOUNDS, S5_ERR_TIMEOUT, \
    S5_ERR_WORKSPACE = range(7)
S5_WS_FIXED_BYTES = 256 + 16384
S5_WS_TEST_STALL_OFFSET = 64  # expired-wait test hook (include/s5attn.h); zero in normal use

# exported symbols (every declaration of include/s5attn.h)
SYMBOLS = ("s5_workspace_size", "s5_index_score_topk", "s5_sparse_gqa_attn", "s5_swa_gqa_attn",
           "s5_index_score_topk_fp8", "s5_sparse_gqa_attn_fp8kv",
           "s5_workspace_size_grouped", "s5_index_score_topk_grouped", "s5_sparse_gqa_attn_grouped",
           "s5_index_score_topk_noalloc", "s5_append_kv", "s5_append_kv_fp8", "s5_reset_device_error", "s5_get_device_error",
           "s5_status_string", "s5_abi_version")


class KvDesc(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p), ("num_pages", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class IndexDesc(ctypes.Structure):
    _fields_ = [("key_pool", ctypes.c_void_p), ("num_pages", ctypes.c_int32), ("index_dim", ctypes.c_int32)]


class BatchDesc(ctypes.Structure):
    _fields_ = [("page_table", ctypes.c_void_p), ("ctx_lens", ctypes.c_void_p), ("cu_q", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("max_pages", ctypes.c_int32), ("total_q", ctypes.c_int32),
                ("max_q", ctypes.c_int32), ("max_len", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_lib.s5_workspace_size.argtypes = [ctypes.POINTER(BatchDesc), _I, ctypes.POINTER(ctypes.c_size_t)]
_lib.s5_index_score_topk.argtypes = [ctypes.POINTER(IndexDesc), ctypes.POINTER(BatchDesc), _P, _I, _P, _P, _P,
                                     ctypes.c_size_t, _P]
_lib.s5_sparse_gqa_attn.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(BatchDesc), _P, _P, _P, _I,
                                    ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]
_lib.s5_swa_gqa_attn.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(BatchDesc), _P, _I, ctypes.c_float, _P,
                                 _P, _P, ctypes.c_size_t, _P]
_lib.s5_index_score_topk_fp8.argtypes = _lib.s5_index_score_topk.argtypes
_lib.s5_sparse_gqa_attn_fp8kv.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(BatchDesc), _P, _P, _P, _I,
                                          ctypes.c_float, ctypes.c_float, ctypes.c_float, _P, _P, _P,
                                          ctypes.c_size_t, _P]
_lib.s5_workspace_size_grouped.argtypes = _lib.s5_workspace_size.argtypes
_lib.s5_index_score_topk_grouped.argtypes = _lib.s5_index_score_topk.argtypes
_lib.s5_sparse_gqa_attn_grouped.argtypes = _lib.s5_sparse_gqa_attn.argtypes
_lib.s5_index_score_topk_noalloc.argtypes = [ctypes.POINTER(IndexDesc), ctypes.POINTER(BatchDesc), _P, _I, _P,
                                             _P, _P]
_lib.s5_append_kv.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(IndexDesc), ctypes.POINTER(BatchDesc), _P, _P,
                              _P, _P, ctypes.c_size_t, _P]
_lib.s5_append_kv_fp8.argtypes = [ctypes.POINTER(KvDesc), ctypes.POINTER(IndexDesc), ctypes.POINTER(BatchDesc), _P,
                                  _P, _P, ctypes.c_float, ctypes.c_float, _P, ctypes.c_size_t, _P]
_lib.s5_reset_device_error.argtypes = [_P, _P]
_lib.s5_get_device_error.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
_lib.s5_status_string.argtypes = [ctypes.c_int]
_lib.s5_status_string.restype = ctypes.c_char_p
_lib.s5_abi_version.restype = ctypes.c_int32
for _name in SYMBOLS:
    if _name not in ("s5_status_string", "s5_abi_version"):
        getattr(_lib, _name).restype = ctypes.c_int
if _lib.s5_abi_version() != ABI_VERSION:
    raise ImportError(f"{LIB_PATH} implements ABI {_lib.s5_abi_version()}, this binding {ABI_VERSION}: rebuild it")


class S5Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {s5_status_string(code)}")


def s5_status_string(code: int) -> str:
    return _lib.s5_status_string(int(code)).decode()


def s5_abi_version() -> int:
    return int(_lib.s5_abi_version())


def _check(code: int, where: str):
    if code != S5_OK:
        raise S5Error(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, dtype, name: str, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


class Batch:
    """Device page table + varlen batch description (``s5_batch_desc``)."""

    def __init__(self, page_table: torch.Tensor, ctx_lens: torch.Tensor, cu_q: torch.Tensor,
                 total_q: int, max_q: int, max_len: int):
        _need(page_table, torch.int32, "page_table")
        _need(ctx_lens, torch.int32, "ctx_lens")
        _need(cu_q, torch.int32, "cu_q")
        assert page_table.dim() == 2 and cu_q.numel() == ctx_lens.numel() + 1
        self.page_table, self.ctx_lens, self.cu_q = page_table, ctx_lens, cu_q
        self.total_q, self.max_q, self.max_len = int(total_q), int(max_q), int(max_len)
        self.desc = BatchDesc(page_table.data_ptr(), ctx_lens.data_ptr(), cu_q.data_ptr(), ctx_lens.numel(),
                              page_table.shape[1], self.total_q, self.max_q, self.max_len)

    @staticmethod
    def from_host(page_table, ctx, nq, device="cuda", max_len: Optional[int] = None):
        """From host data: page table [batch][max_pages] and per-sequence ctx / nq lists."""
        pt = torch.as_tensor(page_table, dtype=torch.int32).to(device).contiguous()
        cu = [0]
        for n in nq:
            cu.append(cu[-1] + int(n))
        lens = [int(c) + int(n) for c, n in zip(ctx, nq)]
        ml = max(lens) if max_len is None else max_len
        return Batch(pt, torch.tensor(list(ctx), dtype=torch.int32, device=device),
                     torch.tensor(cu, dtype=torch.int32, device=device), cu[-1], max(nq) if nq else 0, ml)


def s5_workspace_size(batch: Batch, window: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.s5_workspace_size(ctypes.byref(batch.desc), int(window), ctypes.byref(n)), "s5_workspace_size")
    return int(n.value)


def s5_workspace_size_grouped(batch: Batch, window: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.s5_workspace_size_grouped(ctypes.byref(batch.desc), int(window), ctypes.byref(n)),
           "s5_workspace_size_grouped")
    return int(n.value)


def new_workspace(batch: Batch, window: int = 0, device="cuda", grouped: bool = False) -> torch.Tensor:
    """Allocate (with torch) and zero a workspace sized for ``batch`` (with
    ``grouped``, also for the per-KV-group selection calls)."""
    n = s5_workspace_size_grouped(batch, window) if grouped else s5_workspace_size(batch, window)
    return torch.zeros(max(256, n), dtype=torch.uint8, device=device)


def s5_index_score_topk(key_pool: torch.Tensor, batch: Batch, q_index: torch.Tensor, topk: int,
                        sel: torch.Tensor, sel_count: torch.Tensor, ws: torch.Tensor, stream=None):
    _need(key_pool, torch.bfloat16, "key_pool")
    _need(q_index, torch.bfloat16, "q_index", (batch.total_q, INDEX_DIM))
    _need(sel, torch.int32, "sel", (batch.total_q, topk))
    _need(sel_count, torch.int32, "sel_count", (batch.total_q,))
    _need(ws, torch.uint8, "ws")
    idx = IndexDesc(key_pool.data_ptr(), key_pool.shape[0], key_pool.shape[-1])
    _check(_lib.s5_index_score_topk(ctypes.byref(idx), ctypes.byref(batch.desc), _ptr(q_index), int(topk),
                                    _ptr(sel), _ptr(sel_count), _ptr(ws), ws.numel(), _stream(stream)),
           "s5_index_score_topk")


def s5_index_score_topk_fp8(key_pool: torch.Tensor, batch: Batch, q_index: torch.Tensor, topk: int,
                            sel: torch.Tensor, sel_count: torch.Tensor, ws: torch.Tensor, stream=None):
    """s5_index_score_topk with one-byte E4M3 block keys (key_pool uint8 [num_pages][8][256])."""
    _need(key_pool, torch.uint8, "key_pool")
    _need(q_index, torch.bfloat16, "q_index", (batch.total_q, INDEX_DIM))
    _need(sel, torch.int32, "sel", (batch.total_q, topk))
    _need(sel_count, torch.int32, "sel_count", (batch.total_q,))
    _need(ws, torch.uint8, "ws")
    idx = IndexDesc(key_pool.data_ptr(), key_pool.shape[0], key_pool.shape[-1])
    _check(_lib.s5_index_score_topk_fp8(ctypes.byref(idx), ctypes.byref(batch.desc), _ptr(q_index), int(topk),
                                        _ptr(sel), _ptr(sel_count), _ptr(ws), ws.numel(), _stream(stream)),
           "s5_index_score_topk_fp8")


def s5_index_score_topk_grouped(key_pool: torch.Tensor, batch: Batch, q_index: torch.Tensor, topk: int,
                                sel: torch.Tensor, sel_count: torch.Tensor, ws: torch.Tensor, stream=None):
    """One selection per (token, KV group): q_index [total_q][4][256] ->
    sel [total_q][4][topk], sel_count [total_q][4]."""
    _need(key_pool, torch.bfloat16, "key_pool")
    _need(q_index, torch.bfloat16, "q_index", (batch.total_q, N_KV, INDEX_DIM))
    _need(sel, torch.int32, "sel", (batch.total_q, N_KV, topk))
    _need(sel_count, torch.int32, "sel_count", (batch.total_q, N_KV))
    _need(ws, torch.uint8, "ws")
    idx = IndexDesc(key_pool.data_ptr(), key_pool.shape[0], key_pool.shape[-1])
    _check(_lib.s5_index_score_topk_grouped(ctypes.byref(idx), ctypes.byref(batch.desc), _ptr(q_index), int(topk),
                                            _ptr(sel), _ptr(sel_count), _ptr(ws), ws.numel(), _stream(stream)),
           "s5_index_score_topk_grouped")


def s5_index_score_topk_noalloc(key_pool: torch.Tensor, batch: Batch, q_index: torch.Tensor, topk: int,
                                sel: torch.Tensor, sel_count: torch.Tensor, stream=None):
    """s5_index_score_topk with the library's fixed scratch array instead of a
    workspace: for callers that cannot allocate device memory.  Calls that can
    overlap on the GPU must be serialised by the caller."""
    _need(key_pool, torch.bfloat16, "key_pool")
    _need(q_index, torch.bfloat16, "q_index", (batch.total_q, INDEX_DIM))
    _need(sel, torch.int32, "sel", (batch.total_q, topk))
    _need(sel_count, torch.int32, "sel_count", (batch.total_q,))
    idx = IndexDesc(key_pool.data_ptr(), key_pool.shape[0], key_pool.shape[-1])
    _check(_lib.s5_index_score_topk_noalloc(ctypes.byref(idx), ctypes.byref(batch.desc), _ptr(q_index), int(topk),
                                            _ptr(sel), _ptr(sel_count), _stream(stream)),
           "s5_index_score_topk_noalloc")


def _kv(k_pool, v_pool):
    _need(k_pool, torch.bfloat16, "k_pool")
    _need(v_pool, torch.bfloat16, "v_pool", tuple(k_pool.shape))
    sh = k_pool.shape
    return KvDesc(k_pool.data_ptr(), v_pool.data_ptr(), sh[0], sh[2], sh[1], sh[3])


def s5_sparse_gqa_attn(k_pool, v_pool, batch: Batch, q, sel, sel_count, topk: int, sm_scale: float,
                       out, lse, ws, stream=None):
    kv = _kv(k_pool, v_pool)
    _need(q, torch.bfloat16, "q", (batch.total_q, N_HEADS, HEAD_DIM))
    _need(sel, torch.int32, "sel", (batch.total_q, topk))
    _need(sel_count, torch.int32, "sel_count", (batch.total_q,))
    _need(out, torch.bfloat16, "out", (batch.total_q, N_HEADS, HEAD_DIM))
    if lse is not None:
        _need(lse, torch.float32, "lse", (batch.total_q, N_HEADS))
    _need(ws, torch.uint8, "ws")
    _check(_lib.s5_sparse_gqa_attn(ctypes.byref(kv), ctypes.byref(batch.desc), _ptr(q), _ptr(sel),
                                   _ptr(sel_count), int(topk), float(sm_scale), _ptr(out), _ptr(lse), _ptr(ws),
                                   ws.numel(), _stream(stream)), "s5_sparse_gqa_attn")


def s5_sparse_gqa_attn_fp8kv(k_pool, v_pool, batch: Batch, q, sel, sel_count, topk: int, sm_scale: float,
                             k_scale: float, v_scale: float, out, lse, ws, stream=None):
    """Sparse attention over one-byte KV: k_pool / v_pool uint8 E4M3 codes
    [num_pages][4][64][192]; a K code stands for k_scale times its value, a V
    code for v_scale times its value."""
    _need(k_pool, torch.uint8, "k_pool")
    _need(v_pool, torch.uint8, "v_pool", tuple(k_pool.shape))
    sh = k_pool.shape
    kv = KvDesc(k_pool.data_ptr(), v_pool.data_ptr(), sh[0], sh[2], sh[1], sh[3])
    _need(q, torch.bfloat16, "q", (batch.total_q, N_HEADS, HEAD_DIM))
    _need(sel, torch.int32, "sel", (batch.total_q, topk))
    _need(sel_count, torch.int32, "sel_count", (batch.total_q,))
    _need(out, torch.bfloat16, "out", (batch.total_q, N_HEADS, HEAD_DIM))
    if lse is not None:
        _need(lse, torch.float32, "lse", (batch.total_q, N_HEADS))
    _need(ws, torch.uint8, "ws")
    _check(_lib.s5_sparse_gqa_attn_fp8kv(ctypes.byref(kv), ctypes.byref(batch.desc), _ptr(q), _ptr(sel),
                                         _ptr(sel_count), int(topk), float(sm_scale), float(k_scale),
                                         float(v_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                         _stream(stream)), "s5_sparse_gqa_attn_fp8kv")


def s5_sparse_gqa_attn_grouped(k_pool, v_pool, batch: Batch, q, sel, sel_count, topk: int, sm_scale: float,
                               out, lse, ws, stream=None):
    """Sparse attention with one selection per KV group (sel [total_q][4][topk])."""
    kv = _kv(k_pool, v_pool)
    _need(q, torch.bfloat16, "q", (batch.total_q, N_HEADS, HEAD_DIM))
    _need(sel, torch.int32, "sel", (batch.total_q, N_KV, topk))
    _need(sel_count, torch.int32, "sel_count", (batch.total_q, N_KV))
    _need(out, torch.bfloat16, "out", (batch.total_q, N_HEADS, HEAD_DIM))
    if lse is not None:
        _need(lse, torch.float32, "lse", (batch.total_q, N_HEADS))
    _need(ws, torch.uint8, "ws")
    _check(_lib.s5_sparse_gqa_attn_grouped(ctypes.byref(kv), ctypes.byref(batch.desc), _ptr(q), _ptr(sel),
                                           _ptr(sel_count), int(topk), float(sm_scale), _ptr(out), _ptr(lse),
                                           _ptr(ws), ws.numel(), _stream(stream)), "s5_sparse_gqa_attn_grouped")


def s5_swa_gqa_attn(k_pool, v_pool, batch: Batch, q, window: int, sm_scale: float, out, lse, ws, stream=None):
    kv = _kv(k_pool, v_pool)
    _need(q, torch.bfloat16, "q", (batch.total_q, N_HEADS, HEAD_DIM))
    _need(out, torch.bfloat16, "out", (batch.total_q, N_HEADS, HEAD_DIM))
    if lse is not None:
        _need(lse, torch.float32, "lse", (batch.total_q, N_HEADS))
    _need(ws, torch.uint8, "ws")
    _check(_lib.s5_swa_gqa_attn(ctypes.byref(kv), ctypes.byref(batch.desc), _ptr(q), int(window),
                                float(sm_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "s5_swa_gqa_attn")


def s5_append_kv(k_pool, v_pool, key_pool, batch: Batch, k_new, v_new, key_new, ws, stream=None):
    """Write the new tokens' K/V (and, with a key pool, the keys of the blocks
    they complete) into the paged cache; ``key_pool`` and ``key_new`` may be
    None for a cache without block keys."""
    kv = _kv(k_pool, v_pool)
    _need(k_new, torch.bfloat16, "k_new", (batch.total_q, N_KV, HEAD_DIM))
    _need(v_new, torch.bfloat16, "v_new", (batch.total_q, N_KV, HEAD_DIM))
    idx = None
    if key_pool is not None:
        _need(key_pool, torch.bfloat16, "key_pool")
        _need(key_new, torch.bfloat16, "key_new", (batch.total_q, INDEX_DIM))
        idx = IndexDesc(key_pool.data_ptr(), key_pool.shape[0], key_pool.shape[-1])
    _need(ws, torch.uint8, "ws")
    _check(_lib.s5_append_kv(ctypes.byref(kv), None if idx is None else ctypes.byref(idx), ctypes.byref(batch.desc),
                             _ptr(k_new), _ptr(v_new), None if idx is None else _ptr(key_new), _ptr(ws),
                             ws.numel(), _stream(stream)), "s5_append_kv")


def s5_append_kv_fp8(k_pool, v_pool, key_pool, batch: Batch, k_new, v_new, key_new, k_scale: float, v_scale: float,
                     ws, stream=None):
    """s5_append_kv into one-byte (E4M3) K / V pools (uint8 [num_pages][4][64][192]):
    each bf16 value x is stored as the code nearest to x / scale (an fp32
    product with the reciprocal); block keys as in s5_append_kv."""
    _need(k_pool, torch.uint8, "k_pool")
    _need(v_pool, torch.uint8, "v_pool", tuple(k_pool.shape))
    sh = k_pool.shape
    kv = KvDesc(k_pool.data_ptr(), v_pool.data_ptr(), sh[0], sh[2], sh[1], sh[3])
    _need(k_new, torch.bfloat16, "k_new", (batch.total_q, N_KV, HEAD_DIM))
    _need(v_new, torch.bfloat16, "v_new", (batch.total_q, N_KV, HEAD_DIM))
    idx = None
    if key_pool is not None:
        _need(key_pool, torch.bfloat16, "key_pool")
        _need(key_new, torch.bfloat16, "key_new", (batch.total_q, INDEX_DIM))
        idx = IndexDesc(key_pool.data_ptr(), key_pool.shape[0], key_pool.shape[-1])
    _need(ws, torch.uint8, "ws")
    _check(_lib.s5_append_kv_fp8(ctypes.byref(kv), None if idx is None else ctypes.byref(idx),
                                 ctypes.byref(batch.desc), _ptr(k_new), _ptr(v_new),
                                 None if idx is None else _ptr(key_new), float(k_scale), float(v_scale), _ptr(ws),
                                 ws.numel(), _stream(stream)), "s5_append_kv_fp8")


def s5_reset_device_error(ws: torch.Tensor, stream=None):
    _check(_lib.s5_reset_device_error(_ptr(ws), _stream(stream)), "s5_reset_device_error")


def s5_get_device_error(ws: torch.Tensor, stream=None):
    """(code, info) of the workspace error record; synchronises the stream."""
    code, info = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(_lib.s5_get_device_error(_ptr(ws), _stream(stream), ctypes.byref(code), ctypes.byref(info)),
           "s5_get_device_error")
    return int(code.value), int(info.value)


# ---------------------------------------------------------------- one layer step from host buffers

def sparse_layer_step_host(key_pool, k_pool, v_pool, batch: Batch, q_host, qx_host, out_host, lse_host,
                           sel, sel_count, q_dev, qx_dev, out_dev, lse_dev, ws, topk: int = MAX_TOPK,
                           sm_scale: float = DEFAULT_SM_SCALE, stream=None):
    """One sparse-layer decode step whose per-step inputs (q, q_index) start in
    pinned host memory and whose output (out, lse) ends there; the KV cache and
    block keys stay resident on the device.  Copies are enqueued on ``stream``."""
    st = torch.cuda.current_stream() if stream is None else stream
    with torch.cuda.stream(st):
        q_dev.copy_(q_host, non_blocking=True)
        qx_dev.copy_(qx_host, non_blocking=True)
        s5_index_score_topk(key_pool, batch, qx_dev, topk, sel, sel_count, ws, st)
        s5_sparse_gqa_attn(k_pool, v_pool, batch, q_dev, sel, sel_count, topk, sm_scale, out_dev, lse_dev, ws, st)
        out_host.copy_(out_dev, non_blocking=True)
        lse_host.copy_(lse_dev, non_blocking=True)


class SparseLayerPipeline:
    """Sparse-layer decode steps whose per-step inputs (q, q_index) arrive in
    pinned host memory and whose outputs (out, lse) go back to pinned host
    memory, with the KV cache and block keys resident on the device.

    Two device buffer sets and three streams overlap the host->device copy
    of step i+1 and the device->host copy of step i-1 with the compute of
    step i (s5_index_score_topk + s5_sparse_gqa_attn on the compute stream).
    """

    def __init__(self, key_pool, k_pool, v_pool, batch: Batch, ws, topk: int = MAX_TOPK,
                 sm_scale: float = DEFAULT_SM_SCALE):
        dev = k_pool.device
        self.key_pool, self.k_pool, self.v_pool, self.batch, self.ws = key_pool, k_pool, v_pool, batch, ws
        self.topk, self.sm_scale = topk, sm_scale
        tq = batch.total_q
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.q = [torch.empty((tq, N_HEADS, HEAD_DIM), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.qx = [torch.empty((tq, INDEX_DIM), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.sel = [torch.empty((tq, topk), dtype=torch.int32, device=dev) for _ in range(2)]
        self.cnt = [torch.empty((tq,), dtype=torch.int32, device=dev) for _ in range(2)]
        self.out = [torch.empty((tq, N_HEADS, HEAD_DIM), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.lse = [torch.empty((tq, N_HEADS), dtype=torch.float32, device=dev) for _ in range(2)]
        self.ev_in = [torch.cuda.Event() for _ in range(2)]
        self.ev_comp = [torch.cuda.Event() for _ in range(2)]
        self.ev_out = [torch.cuda.Event() for _ in range(2)]
        self.n = 0

    def step(self, q_host, qx_host, out_host, lse_host):
        b = self.n % 2
        if self.n >= 2:  # buffer set b was last used two steps ago
            self.s_in.wait_event(self.ev_comp[b])
        with torch.cuda.stream(self.s_in):
            self.q[b].copy_(q_host, non_blocking=True)
            self.qx[b].copy_(qx_host, non_blocking=True)
            self.ev_in[b].record(self.s_in)
        self.s_comp.wait_event(self.ev_in[b])
        if self.n >= 2:
            self.s_comp.wait_event(self.ev_out[b])
        s5_index_score_topk(self.key_pool, self.batch, self.qx[b], self.topk, self.sel[b], self.cnt[b], self.ws,
                            self.s_comp)
        s5_sparse_gqa_attn(self.k_pool, self.v_pool, self.batch, self.q[b], self.sel[b], self.cnt[b], self.topk,
                           self.sm_scale, self.out[b], self.lse[b], self.ws, self.s_comp)
        self.ev_comp[b].record(self.s_comp)
        self.s_out.wait_event(self.ev_comp[b])
        with torch.cuda.stream(self.s_out):
            out_host.copy_(self.out[b], non_blocking=True)
            lse_host.copy_(self.lse[b], non_blocking=True)
            self.ev_out[b].record(self.s_out)
        self.n += 1

    def synchronize(self):
        for st in (self.s_in, self.s_comp, self.s_out):
            st.synchronize()
