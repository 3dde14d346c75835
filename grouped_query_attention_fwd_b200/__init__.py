"""Grouped-query attention forward on B200 (sm_100a): Python binding.

Argument marshalling over the C ABI declared in ``include/gqa.h``: tensors go
in as device pointers, sizes and element strides; every step of the attention
runs in the CUDA kernels of ``libgqa_b200.so``.  There is no CPU or PyTorch
fallback: if the library is missing this module raises at import time.

    out = forward(q, k, v, mask=None, causal=False, scale=None)
    kv_append(cache_k, cache_v, k_new, v_new, kv_lens)

q [B, Hq, Sq, D], k and v [B, Hkv, Sk, D] (CUDA tensors, bf16 or fp32, last
dim contiguous), mask bool/uint8 [B, Sq, Sk] (True = attend, shared by all
heads), ``scale`` defaults to 1/sqrt(D).  ``kv_lens`` (int32 CUDA [B]) makes
k and v a cache of capacity Sk whose entry b holds kv_lens[b] keys.
"""
from __future__ import annotations

import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgqa_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libgqa_b200.so is not built (run __graft_entry__.build() or "
        "python -m grouped_query_attention_fwd_b200._build); there is no fallback path")

_lib = ctypes.CDLL(LIB_PATH)

GQA_OK = 0
GQA_ERR_NULL, GQA_ERR_SHAPE, GQA_ERR_LAYOUT, GQA_ERR_UNSUPPORTED = 1, 2, 3, 4
GQA_ERR_WORKSPACE, GQA_ERR_CUDA, GQA_ERR_TIMEOUT, GQA_ERR_ARG, GQA_ERR_DEVICE = 5, 6, 7, 8, 9
GQA_ERR_SCRATCH_LIMIT, GQA_ERR_KV_LENGTH, GQA_ERR_PAGE = 10, 11, 12
STATIC_SCRATCH_BYTES = 8 * 1024 * 1024
GQA_DTYPE_BF16, GQA_DTYPE_F32, GQA_DTYPE_F16 = 0, 1, 2
KERNEL_NAMES = {0: "none", 1: "decode", 2: "prefill", 3: "f32", 4: "zero", 5: "nan"}

EXPORTS = ("gqa_query", "gqa_forward", "gqa_device_status", "gqa_status_string", "gqa_version",
           "gqa_forward_decode_noalloc", "gqa_kv_append", "gqa_debug_decode_trace",
           "gqa_debug_decode_withhold")


class Problem(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32), ("causal", ctypes.c_int32), ("has_mask", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("batch", ctypes.c_int64), ("heads_q", ctypes.c_int64), ("heads_kv", ctypes.c_int64),
        ("seq_q", ctypes.c_int64), ("seq_k", ctypes.c_int64), ("head_dim", ctypes.c_int64),
        ("q_stride", ctypes.c_int64 * 4), ("k_stride", ctypes.c_int64 * 4),
        ("v_stride", ctypes.c_int64 * 4), ("o_stride", ctypes.c_int64 * 4),
        ("mask_stride", ctypes.c_int64 * 3),
        ("causal_offset", ctypes.c_int64), ("window", ctypes.c_int64),
        ("kv_lens", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("block_table_stride", ctypes.c_int64),
        ("page_size", ctypes.c_int64), ("num_pages", ctypes.c_int64),
    ]


class AppendDesc(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("batch", ctypes.c_int64), ("heads_kv", ctypes.c_int64), ("capacity", ctypes.c_int64),
        ("head_dim", ctypes.c_int64), ("n_new", ctypes.c_int64),
        ("cache_k_stride", ctypes.c_int64 * 4), ("cache_v_stride", ctypes.c_int64 * 4),
        ("k_new_stride", ctypes.c_int64 * 4), ("v_new_stride", ctypes.c_int64 * 4),
        ("block_table", ctypes.c_void_p), ("block_table_stride", ctypes.c_int64),
        ("page_size", ctypes.c_int64), ("num_pages", ctypes.c_int64),
    ]


class Plan(ctypes.Structure):
    _fields_ = [
        ("kernel", ctypes.c_int32), ("grid", ctypes.c_int32), ("block", ctypes.c_int32),
        ("smem_bytes", ctypes.c_int32), ("launches", ctypes.c_int32),
        ("work_units", ctypes.c_int32), ("workspace_bytes", ctypes.c_int64),
        ("algorithmic_bytes", ctypes.c_int64), ("algorithmic_flops", ctypes.c_double),
    ]

    def as_dict(self):
        d = {f: getattr(self, f) for f, _ in self._fields_}
        d["kernel_name"] = KERNEL_NAMES.get(self.kernel, "?")
        return d


_vp = ctypes.c_void_p
_lib.gqa_query.argtypes = [ctypes.POINTER(Problem), ctypes.c_int, ctypes.POINTER(Plan)]
_lib.gqa_query.restype = ctypes.c_int
_lib.gqa_forward.argtypes = [ctypes.POINTER(Problem), _vp, _vp, _vp, _vp, _vp, _vp,
                             ctypes.c_size_t, _vp]
_lib.gqa_forward.restype = ctypes.c_int
_lib.gqa_device_status.argtypes = [_vp, ctypes.c_size_t, _vp]
_lib.gqa_device_status.restype = ctypes.c_int
_lib.gqa_status_string.argtypes = [ctypes.c_int]
_lib.gqa_status_string.restype = ctypes.c_char_p
_lib.gqa_version.argtypes = []
_lib.gqa_version.restype = ctypes.c_int
_lib.gqa_forward_decode_noalloc.argtypes = [ctypes.POINTER(Problem), _vp, _vp, _vp, _vp, _vp,
                                            _vp]
_lib.gqa_forward_decode_noalloc.restype = ctypes.c_int
_lib.gqa_kv_append.argtypes = [ctypes.POINTER(AppendDesc), _vp, _vp, _vp, _vp, _vp, _vp,
                               ctypes.c_size_t, _vp]
_lib.gqa_kv_append.restype = ctypes.c_int
_lib.gqa_debug_decode_trace.argtypes = [_vp, ctypes.c_int64]
_lib.gqa_debug_decode_trace.restype = ctypes.c_int
_lib.gqa_debug_decode_withhold.argtypes = [ctypes.c_int64, ctypes.c_int64]
_lib.gqa_debug_decode_withhold.restype = ctypes.c_int


class GQAError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where or "gqa", status_string(status), status))


def status_string(status: int) -> str:
    return _lib.gqa_status_string(status).decode()


def version() -> int:
    return _lib.gqa_version()


def make_problem(dtype: int, B: int, Hq: int, Hkv: int, Sq: int, Sk: int, D: int,
                 q_stride, k_stride, v_stride, o_stride, mask_stride=None,
                 causal: bool = False, scale: float | None = None, causal_offset: int = 0,
                 window: int = 0, kv_lens_ptr: int | None = None) -> Problem:
    """Build the C problem descriptor from plain sizes and element strides
    (``kv_lens_ptr``: device address of int32 [B] cache lengths, or None)."""
    p = Problem()
    p.kv_lens = kv_lens_ptr
    p.dtype = dtype
    p.causal = int(bool(causal))
    p.causal_offset = int(causal_offset)
    p.window = int(window)
    p.has_mask = int(mask_stride is not None)
    p.scale = float((1.0 / math.sqrt(D) if D > 0 else 1.0) if scale is None else scale)
    p.batch, p.heads_q, p.heads_kv, p.seq_q, p.seq_k, p.head_dim = B, Hq, Hkv, Sq, Sk, D
    for i in range(4):
        p.q_stride[i], p.k_stride[i] = int(q_stride[i]), int(k_stride[i])
        p.v_stride[i], p.o_stride[i] = int(v_stride[i]), int(o_stride[i])
    if mask_stride is not None:
        for i in range(3):
            p.mask_stride[i] = int(mask_stride[i])
    return p


def query_problem(p: Problem, sm_count: int = 0) -> Plan:
    plan = Plan()
    rc = _lib.gqa_query(ctypes.byref(p), int(sm_count), ctypes.byref(plan))
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_query")
    return plan


def forward_ptrs(p: Problem, q: int, k: int, v: int, mask: int | None, out: int,
                 workspace: int, workspace_bytes: int, stream: int) -> None:
    """Raw pointer form of gqa_forward (all device pointers)."""
    rc = _lib.gqa_forward(ctypes.byref(p), q, k, v, mask, out, workspace,
                          workspace_bytes, stream)
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_forward")


# --------------------------------------------------------------- torch glue
# torch is used only to own device memory and to name the current stream.

def _torch():
    import torch
    return torch


_workspaces = {}


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return GQA_DTYPE_BF16
    if t.dtype == torch.float32:
        return GQA_DTYPE_F32
    if t.dtype == torch.float16:
        return GQA_DTYPE_F16
    raise TypeError("q/k/v must be bfloat16, float16 or float32, got %s" % t.dtype)


def _offset(causal, causal_offset, Sq, Sk) -> int:
    """Causal diagonal: j <= i + offset.  With Sq == Sk the pages' causal
    attention is offset 0; otherwise the caller must say which alignment it
    wants ("bottom_right" = Sk - Sq, "top_left" = 0, or an integer)."""
    if not causal:
        return 0
    if causal_offset is None:
        if Sq != Sk:
            raise ValueError("causal with seq_q != seq_k needs causal_offset "
                             "('bottom_right', 'top_left' or an integer)")
        return 0
    if causal_offset == "bottom_right":
        return Sk - Sq
    if causal_offset == "top_left":
        return 0
    return int(causal_offset)


def _lens_ptr(kv_lens, B):
    if kv_lens is None:
        return None
    torch = _torch()
    if not kv_lens.is_cuda or kv_lens.dtype != torch.int32 or tuple(kv_lens.shape) != (B,) or \
            not kv_lens.is_contiguous():
        raise ValueError("kv_lens must be a contiguous int32 CUDA tensor of shape [B]")
    return kv_lens.data_ptr()


def _table(block_table, B):
    torch = _torch()
    if not block_table.is_cuda or block_table.dtype != torch.int32 or block_table.dim() != 2 or \
            block_table.shape[0] != B or block_table.stride(1) != 1:
        raise ValueError("block_table must be an int32 CUDA tensor [B, pages per sequence] "
                         "with unit stride along the pages")
    return block_table.data_ptr(), block_table.stride(0), block_table.shape[1]


def problem_for(q, k, v, mask=None, causal=False, scale=None, out=None, causal_offset=None,
                window=0, kv_lens=None, block_table=None) -> Problem:
    """With block_table, k and v are page pools [num_pages, Hkv, page_size, D]
    and a sequence holds up to block_table.shape[1] * page_size keys."""
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, S, D]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share a dtype")
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Sk, Dk = k.shape
    paged = block_table is not None
    if paged:
        num_pages, page_size = Bk, Sk
        bt_ptr, bt_stride, per_seq = _table(block_table, B)
        Sk = per_seq * page_size
        if tuple(v.shape) != tuple(k.shape) or Dk != D:
            raise ValueError("paged k and v must be [num_pages, Hkv, page_size, D] with q's D")
    elif tuple(v.shape) != tuple(k.shape) or Bk != B or Dk != D:
        raise ValueError("k and v must be [B, Hkv, Sk, D] with q's B and D")
    ost = out.stride() if out is not None else (Hq * Sq * D, Sq * D, D, 1)
    mst = None
    if mask is not None:
        if tuple(mask.shape) != (B, Sq, Sk):
            raise ValueError("mask must be [B, Sq, Sk]")
        mst = mask.stride()
    p = make_problem(_dtype_code(q), B, Hq, Hkv, Sq, Sk, D, q.stride(), k.stride(),
                     v.stride(), ost, mst, causal=causal, scale=scale,
                     causal_offset=_offset(causal, causal_offset, Sq, Sk), window=window,
                     kv_lens_ptr=_lens_ptr(kv_lens, B))
    if paged:
        p.block_table, p.block_table_stride = bt_ptr, bt_stride
        p.page_size, p.num_pages = page_size, num_pages
    return p


def query(q, k, v, mask=None, causal=False, scale=None, sm_count: int = 0, causal_offset=None,
          window=0, kv_lens=None, block_table=None) -> dict:
    return query_problem(problem_for(q, k, v, mask, causal, scale, causal_offset=causal_offset,
                                     window=window, kv_lens=kv_lens, block_table=block_table),
                         sm_count).as_dict()


def _stream_object(idx: int, stream):
    """torch stream object for a raw cudaStream_t handle on device ``idx``."""
    torch = _torch()
    cur = torch.cuda.current_stream(idx)
    if stream is None or int(stream) == cur.cuda_stream:
        return cur
    dflt = torch.cuda.default_stream(idx)
    if int(stream) == dflt.cuda_stream:
        return dflt
    return torch.cuda.ExternalStream(int(stream), device=torch.device("cuda", idx))


def workspace_for(device, nbytes: int, stream=None):
    """A zeroed, cached device workspace of at least ``nbytes`` for ``device``
    and ``stream`` (a cudaStream_t handle; None = the current stream).

    One workspace per (device, stream): calls sharing a workspace must be
    ordered on one stream, since the split-merge counters it holds are not
    safe for calls that overlap on the GPU.  A new workspace is allocated and
    zero-filled on that stream, so the caching allocator orders its reuse
    after the stream's earlier work."""
    torch = _torch()
    dev = torch.device(device)
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    st = _stream_object(idx, stream)
    key = (idx, int(st.cuda_stream))
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        with torch.cuda.device(idx), torch.cuda.stream(st):
            ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=torch.device("cuda", idx))
        _workspaces[key] = ws
    return ws


def forward(q, k, v, mask=None, causal=False, scale=None, out=None, workspace=None,
            stream=None, causal_offset=None, window=0, kv_lens=None, block_table=None):
    """out = softmax(mask(q k_{h/g}^T * scale)) v_{h/g} on the GPU.

    causal: key j visible to query i iff j <= i + offset (offset 0 for
    Sq == Sk; pass causal_offset="bottom_right" for a query block at the end
    of the keys).  window > 0 keeps only the last `window` keys up to the
    diagonal (sliding-window attention).  kv_lens (int32 CUDA [B]): entry b
    holds kv_lens[b] keys of the Sk-long cache; the offset is given for a
    full cache and moves by kv_lens[b] - Sk.  block_table (int32 CUDA
    [B, pages per sequence]): k and v are page pools [num_pages, Hkv,
    page_size, D] (page_size a multiple of 64) and Sk = pages per sequence *
    page_size."""
    torch = _torch()
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors (there is no CPU path)")
    if mask is not None:
        if not mask.is_cuda:
            raise ValueError("mask must be a CUDA tensor")
        if mask.dtype == torch.bool:
            mask = mask.view(torch.uint8)
        elif mask.dtype != torch.uint8:
            raise TypeError("mask must be bool or uint8")
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    p = problem_for(q, k, v, mask, causal, scale, out, causal_offset=causal_offset, window=window,
                    kv_lens=kv_lens, block_table=block_table)
    plan = query_problem(p)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    if workspace is None:
        workspace = workspace_for(q.device, plan.workspace_bytes, stream)
    forward_ptrs(p, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                 mask.data_ptr() if mask is not None else None, out.data_ptr(),
                 workspace.data_ptr(), workspace.numel(), stream)
    return out


def append_desc(dtype: int, B: int, Hkv: int, capacity: int, D: int, n_new: int,
                cache_k_stride, cache_v_stride, k_new_stride, v_new_stride) -> AppendDesc:
    d = AppendDesc()
    d.dtype, d.reserved = dtype, 0
    d.batch, d.heads_kv, d.capacity, d.head_dim, d.n_new = B, Hkv, capacity, D, n_new
    for i in range(4):
        d.cache_k_stride[i], d.cache_v_stride[i] = int(cache_k_stride[i]), int(cache_v_stride[i])
        d.k_new_stride[i], d.v_new_stride[i] = int(k_new_stride[i]), int(v_new_stride[i])
    return d


def kv_append_ptrs(d: AppendDesc, cache_k: int, cache_v: int, k_new: int, v_new: int,
                   kv_lens: int, workspace: int, workspace_bytes: int, stream: int) -> None:
    """Raw pointer form of gqa_kv_append (all device pointers)."""
    rc = _lib.gqa_kv_append(ctypes.byref(d), cache_k, cache_v, k_new, v_new, kv_lens, workspace,
                            workspace_bytes, stream)
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_kv_append")


def kv_append(cache_k, cache_v, k_new, v_new, kv_lens, workspace=None, stream=None,
              block_table=None):
    """Write k_new / v_new [B, Hkv, n_new, D] into rows kv_lens[b] .. kv_lens[b] + n_new
    of cache_k / cache_v [B, Hkv, capacity, D], then advance kv_lens (int32 CUDA [B])
    in place.  An entry that does not fit is left as it was and device_status()
    reports GQA_ERR_KV_LENGTH.  With block_table the caches are page pools
    [num_pages, Hkv, page_size, D] and capacity = pages per sequence * page_size."""
    torch = _torch()
    for t in (cache_k, cache_v, k_new, v_new, kv_lens):
        if not t.is_cuda:
            raise ValueError("kv_append takes CUDA tensors only")
    if cache_k.dim() != 4 or tuple(cache_v.shape) != tuple(cache_k.shape):
        raise ValueError("cache_k and cache_v must be [B, Hkv, capacity, D]")
    B, Hkv, cap, D = cache_k.shape
    if block_table is not None:
        num_pages, page_size = B, cap
        B = k_new.shape[0]
        bt_ptr, bt_stride, per_seq = _table(block_table, B)
        cap = per_seq * page_size
    if k_new.dim() != 4 or tuple(v_new.shape) != tuple(k_new.shape) or \
            k_new.shape[0] != B or k_new.shape[1] != Hkv or k_new.shape[3] != D:
        raise ValueError("k_new and v_new must be [B, Hkv, n_new, D]")
    if not (cache_k.dtype == cache_v.dtype == k_new.dtype == v_new.dtype):
        raise TypeError("cache and new rows must share a dtype")
    d = append_desc(_dtype_code(cache_k), B, Hkv, cap, D, k_new.shape[2], cache_k.stride(),
                    cache_v.stride(), k_new.stride(), v_new.stride())
    if block_table is not None:
        d.block_table, d.block_table_stride = bt_ptr, bt_stride
        d.page_size, d.num_pages = page_size, num_pages
    lp = _lens_ptr(kv_lens, B)
    if stream is None:
        stream = torch.cuda.current_stream(cache_k.device).cuda_stream
    if workspace is None:
        workspace = workspace_for(cache_k.device, 256, stream)
    kv_append_ptrs(d, cache_k.data_ptr(), cache_v.data_ptr(), k_new.data_ptr(),
                   v_new.data_ptr(), lp, workspace.data_ptr(), workspace.numel(), stream)


def device_status(workspace=None, stream=None) -> int:
    """Synchronise and read/clear the workspace error word (GQA_OK or an error);
    the default workspace is the one of (current device, ``stream``)."""
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    if workspace is None:
        workspace = workspace_for(torch.cuda.current_device(), 256, stream)
    return _lib.gqa_device_status(workspace.data_ptr(), workspace.numel(), stream)


def debug_decode_trace(buf=None) -> None:
    """Diagnostics: record per-CTA phase timestamps of every following decode
    launch into ``buf`` (an int64 CUDA tensor; None stops recording).  See
    gqa_debug_decode_trace in include/gqa.h for the record layout."""
    if buf is None:
        rc = _lib.gqa_debug_decode_trace(None, 0)
    else:
        rc = _lib.gqa_debug_decode_trace(buf.data_ptr(), buf.numel() * buf.element_size())
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_debug_decode_trace")


def debug_decode_withhold(unit: int, wait_limit_ns: int) -> None:
    """Test of the bounded waits: the next decode launch withholds the copies
    of `unit` and gives up its waits after `wait_limit_ns`; device_status()
    then reports GQA_ERR_TIMEOUT.  See gqa_debug_decode_withhold in
    include/gqa.h."""
    rc = _lib.gqa_debug_decode_withhold(int(unit), int(wait_limit_ns))
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_debug_decode_withhold")
