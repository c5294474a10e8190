"""Python binding of libpagedkv, the C ABI declared in ``include/pagedkv.h``.

Argument marshalling only: every function forwards to the C function of the
same name, passing raw pointers (``tensor.data_ptr()``) and the current torch
CUDA stream.  PyTorch serves for device memory and streams; all of the decode
step runs in the library's CUDA kernels and its host C++ block manager.

The shared library must have been built (``python
pagedattention_decode_02_b200/build.py``); importing this package without it
raises ImportError - there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing; build it with `python pagedattention_decode_02_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

# ---------------------------------------------------------------------------
# enums and structs (mirror include/pagedkv.h)
# ---------------------------------------------------------------------------
PKV_OK, PKV_ERR_INVALID_ARG, PKV_ERR_NO_BLOCKS, PKV_ERR_UNKNOWN_SEQ, PKV_ERR_SEQ_EXISTS, \
    PKV_ERR_CUDA, PKV_ERR_DEVICE, PKV_ERR_SCRATCH_LIMIT = range(8)
PKV_F32, PKV_F16, PKV_BF16, PKV_FP8_E4M3 = range(4)
PKV_DEVERR_CONTEXT_LEN, PKV_DEVERR_BLOCK_ID, PKV_DEVERR_SLOT, PKV_DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8
PKV_POOL_HOST_ONLY = 0x1
PKV_KERNEL_AUTO, PKV_KERNEL_SIMT, PKV_KERNEL_TENSOR, PKV_KERNEL_SIMT_BULK, PKV_KERNEL_SIMT_TMA = 0, 1, 2, 3, 4
PKV_KERNEL_LEAN = 5
PKV_PREFILL_AUTO, PKV_PREFILL_TCGEN05, PKV_PREFILL_MMA_SYNC = 0, 1, 2

DTYPE_NAMES = {"f32": PKV_F32, "f16": PKV_F16, "bf16": PKV_BF16, "fp8": PKV_FP8_E4M3}
ELEM_BYTES = {PKV_F32: 4, PKV_F16: 2, PKV_BF16: 2, PKV_FP8_E4M3: 1}


class pkv_stats(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("free_blocks", ctypes.c_int32), ("used_blocks", ctypes.c_int32),
                ("num_seqs", ctypes.c_int32), ("pad_", ctypes.c_int32),
                ("stored_slots", ctypes.c_int64), ("logical_tokens", ctypes.c_int64),
                ("table_slots", ctypes.c_int64), ("cow_count", ctypes.c_int64),
                ("prefix_hit_tokens", ctypes.c_int64), ("cached_blocks", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_ if f != "pad_"}


class pkv_pool_info(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("host_only", ctypes.c_int32),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float),
                ("k_buf", ctypes.c_void_p), ("v_buf", ctypes.c_void_p),
                ("bytes_per_buffer", ctypes.c_size_t), ("error_word", ctypes.c_void_p)]


class pkv_sim_request(ctypes.Structure):
    _fields_ = [("arrival", ctypes.c_int32), ("prompt", ctypes.c_int32), ("output", ctypes.c_int32)]


class pkv_sim_result(ctypes.Structure):
    _fields_ = [("rounds", ctypes.c_int32), ("peak_running", ctypes.c_int32),
                ("preemptions", ctypes.c_int32), ("admitted", ctypes.c_int32),
                ("stored_token_rounds", ctypes.c_int64), ("reserved_slot_rounds", ctypes.c_int64),
                ("future_slot_rounds", ctypes.c_int64), ("internal_frag_slot_rounds", ctypes.c_int64),
                ("mean_utilisation", ctypes.c_double)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


_P = ctypes.c_void_p
_I32P = ctypes.POINTER(ctypes.c_int32)
_I64P = ctypes.POINTER(ctypes.c_int64)
_st = ctypes.c_int


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("kv_pool_create", _st, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
     ctypes.c_float, ctypes.c_float, _P, _P, ctypes.c_uint, ctypes.POINTER(ctypes.c_size_t),
     ctypes.POINTER(_P))
_sig("kv_pool_destroy", None, _P)
_sig("kv_pool_get_info", _st, _P, ctypes.POINTER(pkv_pool_info))
_sig("kv_pool_check_guards", _st, _P, ctypes.POINTER(ctypes.c_int))
_sig("bt_reset", _st, _P, _I32P)
_sig("bt_alloc", _st, _P, ctypes.c_int64, ctypes.c_int, _I32P)
_sig("bt_append", _st, _P, ctypes.c_int64, _I32P, _I32P, _I32P)
_sig("bt_append_batch", _st, _P, _I64P, ctypes.c_int, _I32P, _I32P, _I32P, ctypes.POINTER(ctypes.c_int))
_sig("bt_fork", _st, _P, ctypes.c_int64, ctypes.c_int64)
_sig("bt_set_prefix_caching", _st, _P, ctypes.c_int)
_sig("pkv_simulate", _st, ctypes.POINTER(pkv_sim_request), ctypes.c_int, ctypes.c_int, ctypes.c_int,
     ctypes.c_int, ctypes.c_int, ctypes.POINTER(pkv_sim_result), _I32P)
_sig("bt_alloc_prefix", _st, _P, ctypes.c_int64, _I32P, ctypes.c_int, _I32P, _I32P)
_sig("bt_free", _st, _P, ctypes.c_int64)
_sig("bt_export", _st, _P, _I64P, ctypes.c_int, ctypes.c_int, _I32P, _I32P, _I32P)
_sig("bt_num_blocks", _st, _P, ctypes.c_int64, _I32P)
_sig("bt_refcount", _st, _P, ctypes.c_int32, _I32P)
_sig("bt_free_queue", _st, _P, _I32P, ctypes.c_int, ctypes.POINTER(ctypes.c_int))
_sig("bt_stats", _st, _P, ctypes.POINTER(pkv_stats))
_sig("kv_append", _st, _P, _P, ctypes.c_int, _P, _P, ctypes.c_int, _P)
_sig("block_copy", _st, _P, _P, _P, ctypes.c_int, _P)
_sig("paged_decode_attention", _st, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, ctypes.c_int,
     ctypes.c_int, ctypes.c_float, _P, _P, ctypes.c_size_t, _P)
_sig("paged_decode_attention_ex", _st, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, ctypes.c_int,
     ctypes.c_int, ctypes.c_float, _P, _P, ctypes.c_size_t, ctypes.c_int, ctypes.c_int, _P)
_sig("paged_decode_workspace_bytes", ctypes.c_size_t, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int)
_sig("paged_decode_workspace_bytes_ex", ctypes.c_size_t, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
     ctypes.c_int)
_sig("pkv_device_error", _st, _P, _P, ctypes.POINTER(ctypes.c_uint32))
_sig("paged_prefill_attention", _st, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, ctypes.c_int, _P,
     ctypes.c_int, ctypes.c_int, ctypes.c_float, _P, _P)
_sig("paged_prefill_attention_ex", _st, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, ctypes.c_int, _P,
     ctypes.c_int, ctypes.c_int, ctypes.c_float, _P, ctypes.c_int, _P)
_sig("pkv_status_str", ctypes.c_char_p, ctypes.c_int)
_sig("pkv_set_wait_budget", _st, _P, ctypes.c_uint64)
_sig("pkv_wait_probe", _st, _P, _P)
_sig("pkv_step_create", _st, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
     ctypes.c_int, ctypes.c_int, ctypes.POINTER(_P))
_sig("pkv_step_destroy", None, _P)
_sig("pkv_decode_step", _st, _P, _I64P, ctypes.c_int, _P, _P, _P, ctypes.c_float, _P, _P)
_sig("pkv_decode_step_host", _st, _P, _I64P, ctypes.c_int, _P, _P, _P, ctypes.c_float, _P, _P)
_sig("pkv_step_last_launches", ctypes.c_int, _P)
_sig("pkv_step_last_kernel", ctypes.c_int, _P)
_sig("pkv_step_profile", _st, _P, ctypes.c_int, ctypes.c_int)
_sig("paged_decode_attention_static", _st, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, ctypes.c_int,
     ctypes.c_int, ctypes.c_float, _P, ctypes.c_int, _P)
_sig("paged_decode_static_scratch_bytes", ctypes.c_size_t)
_sig("kv_swap_out", _st, _P, ctypes.c_int64, _P, _P, ctypes.c_size_t, _I32P, _I64P, _P)
_sig("kv_swap_in", _st, _P, ctypes.c_int64, _P, _P, ctypes.c_size_t, ctypes.c_int64, _P)
_sig("pkv_step_profile_read", _st, _P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float),
     ctypes.POINTER(ctypes.c_float), ctypes.c_int, ctypes.POINTER(ctypes.c_int))

EXPORTED = [
    "kv_pool_create", "kv_pool_destroy", "kv_pool_get_info", "kv_pool_check_guards", "bt_reset", "bt_alloc", "bt_append",
    "bt_append_batch", "bt_fork", "bt_free", "bt_export", "bt_num_blocks", "bt_refcount",
    "bt_free_queue", "bt_stats", "kv_append", "block_copy", "paged_decode_attention",
    "paged_decode_attention_ex", "paged_decode_workspace_bytes", "paged_decode_workspace_bytes_ex",
    "pkv_device_error", "pkv_status_str", "pkv_step_create", "pkv_step_destroy", "pkv_decode_step",
    "pkv_decode_step_host",
    "pkv_step_last_launches", "pkv_step_last_kernel", "pkv_step_profile", "pkv_step_profile_read",
    "paged_decode_attention_static", "paged_decode_static_scratch_bytes", "kv_swap_out", "kv_swap_in",
    "paged_prefill_attention", "paged_prefill_attention_ex",
    "pkv_set_wait_budget", "pkv_wait_probe",
    "bt_set_prefix_caching", "bt_alloc_prefix", "pkv_simulate",
]


class PagedKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = pkv_status_str(status)
        super().__init__(f"{where}: {self.name}")


def pkv_status_str(status: int) -> str:
    return _lib.pkv_status_str(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != PKV_OK:
        raise PagedKVError(status, where)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr32(a: np.ndarray):
    return a.ctypes.data_as(_I32P)


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _dev_ptr(t) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def torch_dtype_code(dt) -> int:
    import torch
    m = {torch.float32: PKV_F32, torch.float16: PKV_F16, torch.bfloat16: PKV_BF16}
    if dt not in m:
        raise ValueError(f"unsupported dtype {dt}")
    return m[dt]


# ---------------------------------------------------------------------------
# pool
# ---------------------------------------------------------------------------
class Pool:
    """Owns a ``pkv_pool*``; destroyed with the object (or ``close()``)."""

    def __init__(self, handle: int, keepalive=None):
        self.handle = ctypes.c_void_p(handle)
        self._keepalive = keepalive
        info = pkv_pool_info()
        _check(_lib.kv_pool_get_info(self.handle, ctypes.byref(info)), "kv_pool_get_info")
        self.info = info
        self.num_blocks = info.num_blocks
        self.block_size = info.block_size
        self.n_kv_heads = info.n_kv_heads
        self.head_dim = info.head_dim
        self.dtype = info.dtype
        self.k_scale = info.k_scale
        self.v_scale = info.v_scale

    def close(self) -> None:
        if self.handle:
            _lib.kv_pool_destroy(self.handle)
            self.handle = ctypes.c_void_p(0)
            self._keepalive = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def _as_parameter_(self):
        return self.handle

    def device_buffers(self):
        """torch uint8 views [num_blocks][H_kv][bs][d * elem] of the K and V pools."""
        import torch
        if self.info.host_only:
            raise ValueError("host-only pool")
        shape = (self.num_blocks, self.n_kv_heads, self.block_size,
                 self.head_dim * ELEM_BYTES[self.dtype])
        out = []
        for ptr in (self.info.k_buf, self.info.v_buf):
            holder = _CudaArray(ptr, shape)
            out.append(torch.as_tensor(holder, device="cuda"))
        return out


class _CudaArray:
    def __init__(self, ptr: int, shape):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": "|u1",
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def kv_pool_create(num_blocks: int, block_size: int, n_kv_heads: int, head_dim: int, dtype,
                   k_scale: float = 1.0, v_scale: float = 1.0, k_buf=None, v_buf=None,
                   host_only: bool = False) -> Pool:
    """Create a pool.  ``dtype``: "f32" | "f16" | "bf16" | "fp8" or a PKV_* code.
    ``k_buf``/``v_buf``: optional caller-owned torch uint8 CUDA tensors (kept
    alive by the returned Pool)."""
    dt = DTYPE_NAMES[dtype] if isinstance(dtype, str) else int(dtype)
    out = ctypes.c_void_p()
    need = ctypes.c_size_t()
    kp = _dev_ptr(k_buf) if k_buf is not None else None
    vp = _dev_ptr(v_buf) if v_buf is not None else None
    _check(_lib.kv_pool_create(num_blocks, block_size, n_kv_heads, head_dim, dt, k_scale, v_scale,
                               kp, vp, PKV_POOL_HOST_ONLY if host_only else 0,
                               ctypes.byref(need), ctypes.byref(out)), "kv_pool_create")
    return Pool(out.value, keepalive=(k_buf, v_buf))


def kv_pool_bytes(num_blocks: int, block_size: int, n_kv_heads: int, head_dim: int, dtype) -> int:
    dt = DTYPE_NAMES[dtype] if isinstance(dtype, str) else int(dtype)
    need = ctypes.c_size_t()
    _check(_lib.kv_pool_create(num_blocks, block_size, n_kv_heads, head_dim, dt, 1.0, 1.0, None,
                               None, 0, ctypes.byref(need), None), "kv_pool_create")
    return need.value


def kv_pool_destroy(pool: Pool) -> None:
    pool.close()


# ---------------------------------------------------------------------------
# block tables (host)
# ---------------------------------------------------------------------------
def bt_reset(pool: Pool, free_order: Optional[Sequence[int]] = None) -> None:
    if free_order is None:
        _check(_lib.bt_reset(pool.handle, None), "bt_reset")
        return
    o = _i32(free_order)
    if o.size != pool.num_blocks:
        raise PagedKVError(PKV_ERR_INVALID_ARG, "bt_reset")
    _check(_lib.bt_reset(pool.handle, _ptr32(o)), "bt_reset")


def bt_alloc(pool: Pool, seq_id: int, n_tokens: int) -> np.ndarray:
    slots = np.empty(max(n_tokens, 0), dtype=np.int32)
    _check(_lib.bt_alloc(pool.handle, int(seq_id), int(n_tokens),
                         _ptr32(slots) if n_tokens > 0 else None), "bt_alloc")
    return slots


def bt_append(pool: Pool, seq_id: int):
    """-> (slot, cow_src, cow_dst); -1 for no copy."""
    s, a, b = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.bt_append(pool.handle, int(seq_id), ctypes.byref(s), ctypes.byref(a),
                          ctypes.byref(b)), "bt_append")
    return s.value, a.value, b.value


def bt_append_batch(pool: Pool, seq_ids):
    """-> (slots [n] int32, cow_src [n_cow], cow_dst [n_cow])."""
    ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
    n = ids.size
    slots = np.empty(n, np.int32)
    src = np.empty(max(n, 1), np.int32)
    dst = np.empty(max(n, 1), np.int32)
    ncow = ctypes.c_int()
    _check(_lib.bt_append_batch(pool.handle, ids.ctypes.data_as(_I64P), n, _ptr32(slots),
                                _ptr32(src), _ptr32(dst), ctypes.byref(ncow)), "bt_append_batch")
    return slots, src[: ncow.value].copy(), dst[: ncow.value].copy()


def bt_set_prefix_caching(pool: Pool, enable: bool) -> None:
    _check(_lib.bt_set_prefix_caching(pool.handle, 1 if enable else 0), "bt_set_prefix_caching")


def bt_alloc_prefix(pool: Pool, seq_id: int, token_ids):
    """-> (slots [n] int32, n_cached_tokens)."""
    toks = _i32(token_ids)
    n = toks.size
    slots = np.empty(max(n, 1), np.int32)
    nc = ctypes.c_int32()
    _check(_lib.bt_alloc_prefix(pool.handle, int(seq_id), _ptr32(toks) if n else None, int(n),
                                _ptr32(slots) if n else None, ctypes.byref(nc)), "bt_alloc_prefix")
    return slots[:n].copy(), nc.value


def bt_fork(pool: Pool, parent_id: int, child_id: int) -> None:
    _check(_lib.bt_fork(pool.handle, int(parent_id), int(child_id)), "bt_fork")


def bt_free(pool: Pool, seq_id: int) -> None:
    _check(_lib.bt_free(pool.handle, int(seq_id)), "bt_free")


def bt_export(pool: Pool, seq_ids, max_blocks: int):
    """-> (block_tables [n][max_blocks], context_lens [n], fill_of_last [n]) int32."""
    ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
    n = ids.size
    tables = np.empty((n, max_blocks), np.int32)
    lens = np.empty(n, np.int32)
    fills = np.empty(n, np.int32)
    _check(_lib.bt_export(pool.handle, ids.ctypes.data_as(_I64P), n, int(max_blocks),
                          _ptr32(tables), _ptr32(lens), _ptr32(fills)), "bt_export")
    return tables, lens, fills


def bt_num_blocks(pool: Pool, seq_id: int) -> int:
    n = ctypes.c_int32()
    _check(_lib.bt_num_blocks(pool.handle, int(seq_id), ctypes.byref(n)), "bt_num_blocks")
    return n.value


def bt_refcount(pool: Pool, block_id: int) -> int:
    n = ctypes.c_int32()
    _check(_lib.bt_refcount(pool.handle, int(block_id), ctypes.byref(n)), "bt_refcount")
    return n.value


def bt_free_queue(pool: Pool) -> np.ndarray:
    out = np.empty(pool.num_blocks, np.int32)
    n = ctypes.c_int()
    _check(_lib.bt_free_queue(pool.handle, _ptr32(out), pool.num_blocks, ctypes.byref(n)),
           "bt_free_queue")
    return out[: n.value].copy()


def bt_stats(pool: Pool) -> dict:
    st = pkv_stats()
    _check(_lib.bt_stats(pool.handle, ctypes.byref(st)), "bt_stats")
    return st.as_dict()


# ---------------------------------------------------------------------------
# device calls
# ---------------------------------------------------------------------------
def kv_append(pool: Pool, slot_mapping, k, v, stream=None) -> None:
    """slot_mapping: int32 CUDA [T]; k, v: CUDA [T][H_kv][d] (pool dtype, or
    f32/f16/bf16 for FP8 pools)."""
    n = int(slot_mapping.numel())
    _check(_lib.kv_append(pool.handle, _dev_ptr(slot_mapping), n, _dev_ptr(k), _dev_ptr(v),
                          torch_dtype_code(k.dtype), _stream_ptr(stream)), "kv_append")


def block_copy(pool: Pool, src, dst, stream=None) -> None:
    """src, dst: int32 CUDA [n_pairs]."""
    _check(_lib.block_copy(pool.handle, _dev_ptr(src), _dev_ptr(dst), int(src.numel()),
                           _stream_ptr(stream)), "block_copy")


def paged_decode_workspace_bytes(pool: Pool, B: int, n_q_heads: int, max_blocks: int,
                                 partition_tokens: int = 0) -> int:
    return int(_lib.paged_decode_workspace_bytes_ex(pool.handle, B, n_q_heads, max_blocks,
                                                    partition_tokens))


def paged_decode_attention(pool: Pool, q, block_tables, context_lens, scale: float, out=None,
                           workspace=None, partition_tokens: int = 0,
                           kernel: int = PKV_KERNEL_AUTO, stream=None):
    """q: CUDA [B][H_q][d]; block_tables: int32 CUDA [B][max_blocks];
    context_lens: int32 CUDA [B].  Returns out (allocated if None)."""
    import torch
    B, H_q, _ = q.shape
    max_blocks = int(block_tables.shape[1])
    if out is None:
        out = torch.empty_like(q)
    need = paged_decode_workspace_bytes(pool, B, H_q, max_blocks, partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.paged_decode_attention_ex(
        pool.handle, _dev_ptr(q), torch_dtype_code(q.dtype), _dev_ptr(block_tables), max_blocks,
        _dev_ptr(context_lens), B, H_q, float(scale), _dev_ptr(out),
        _dev_ptr(workspace) if workspace is not None else None, ws_bytes, int(partition_tokens),
        int(kernel), _stream_ptr(stream)), "paged_decode_attention")
    return out


def paged_prefill_attention(pool: Pool, q, q_starts, block_tables, context_lens, scale: float,
                            max_q_len: Optional[int] = None, out=None, stream=None,
                            kernel: int = 0):
    """Prompt-phase attention.  q: CUDA [rows][H_q][d]; q_starts: int32 CUDA [B+1]
    (row offsets per sequence); block_tables: int32 CUDA [B][max_blocks];
    context_lens: int32 CUDA [B] (cached tokens, the prompt's included).
    max_q_len: the longest prompt (read from q_starts when None); kernel:
    PKV_PREFILL_* (0 = automatic).  Returns out."""
    import torch
    B = int(context_lens.shape[0])
    H_q = int(q.shape[1])
    if out is None:
        out = torch.empty_like(q)
    if max_q_len is None:
        max_q_len = int((q_starts[1:] - q_starts[:-1]).max().item()) if B else 0
    _check(_lib.paged_prefill_attention_ex(
        pool.handle, _dev_ptr(q), torch_dtype_code(q.dtype), _dev_ptr(q_starts), int(max_q_len),
        _dev_ptr(block_tables), int(block_tables.shape[1]), _dev_ptr(context_lens), B, H_q,
        float(scale), _dev_ptr(out), int(kernel), _stream_ptr(stream)),
        "paged_prefill_attention")
    return out


def pkv_set_wait_budget(pool: Pool, budget_ns: int) -> None:
    """Budget of the pool's kernels' main-loop waits in ns (0 = the default 2 s)."""
    _check(_lib.pkv_set_wait_budget(pool.handle, int(budget_ns)), "pkv_set_wait_budget")


def pkv_wait_probe(pool: Pool, stream=None) -> None:
    """Queue the probe kernel: a wait that nothing completes, with the pool's budget."""
    _check(_lib.pkv_wait_probe(pool.handle, _stream_ptr(stream)), "pkv_wait_probe")


def kv_pool_check_guards(pool: Pool) -> bool:
    """Wait for the device; True when the guard blocks around the pool's own
    K/V buffers still hold their fixed byte (always True without guards)."""
    ok = ctypes.c_int(0)
    _check(_lib.kv_pool_check_guards(pool.handle, ctypes.byref(ok)), "kv_pool_check_guards")
    return bool(ok.value)


def pkv_device_error(pool: Pool, stream=None) -> int:
    """Synchronise, return and clear the device error bits (0 = none)."""
    bits = ctypes.c_uint32()
    st = _lib.pkv_device_error(pool.handle, _stream_ptr(stream), ctypes.byref(bits))
    if st not in (PKV_OK, PKV_ERR_DEVICE):
        raise PagedKVError(st, "pkv_device_error")
    return bits.value


# ---------------------------------------------------------------------------
# decode-step runtime
# ---------------------------------------------------------------------------
class Step:
    """Owns a ``pkv_step*`` (staging, device tables, workspace for one batch shape)."""

    def __init__(self, pool: Pool, max_batch: int, max_blocks: int, n_q_heads: int, q_dtype,
                 partition_tokens: int = 0, kernel: int = PKV_KERNEL_AUTO,
                 max_seqs: Optional[int] = None):
        qd = DTYPE_NAMES[q_dtype] if isinstance(q_dtype, str) else int(q_dtype)
        h = ctypes.c_void_p()
        ms = max_batch if max_seqs is None else max_seqs
        _check(_lib.pkv_step_create(pool.handle, max_batch, ms, max_blocks, n_q_heads, qd,
                                    partition_tokens, kernel, ctypes.byref(h)), "pkv_step_create")
        self.handle = h
        self.pool = pool
        self.max_batch = max_batch
        self._ids = None

    def close(self) -> None:
        if self.handle:
            _lib.pkv_step_destroy(self.handle)
            self.handle = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def last_launches(self) -> int:
        return int(_lib.pkv_step_last_launches(self.handle))

    @property
    def last_kernel(self) -> int:
        return int(_lib.pkv_step_last_kernel(self.handle))

    def run_raw(self, ids: np.ndarray, q_ptr: int, k_ptr: int, v_ptr: int, scale: float,
                out_ptr: int, stream_ptr: int) -> None:
        """pkv_decode_step with pre-resolved device pointers (int64 ``ids``):
        the same C call without per-call tensor checks, for tight loops."""
        st = _lib.pkv_decode_step(self.handle, ids.ctypes.data_as(_I64P), int(ids.size), q_ptr,
                                  k_ptr, v_ptr, scale, out_ptr, stream_ptr)
        if st != PKV_OK:
            raise PagedKVError(st, "pkv_decode_step")

    def run_host_raw(self, ids: np.ndarray, q_ptr: int, k_ptr: int, v_ptr: int, scale: float,
                     out_ptr: int, stream_ptr: int) -> None:
        """pkv_decode_step_host with pre-resolved HOST pointers: returns with the
        round's output in the host buffer at ``out_ptr``."""
        st = _lib.pkv_decode_step_host(self.handle, ids.ctypes.data_as(_I64P), int(ids.size),
                                       q_ptr, k_ptr, v_ptr, scale, out_ptr, stream_ptr)
        if st != PKV_OK:
            raise PagedKVError(st, "pkv_decode_step_host")


def pkv_step_create(pool: Pool, max_batch: int, max_blocks: int, n_q_heads: int, q_dtype,
                    partition_tokens: int = 0, kernel: int = PKV_KERNEL_AUTO,
                    max_seqs: Optional[int] = None) -> Step:
    return Step(pool, max_batch, max_blocks, n_q_heads, q_dtype, partition_tokens, kernel, max_seqs)


def pkv_step_destroy(step: Step) -> None:
    step.close()


def pkv_decode_step(step: Step, seq_ids, q, k_new, v_new, scale: float, out, stream=None) -> None:
    """One decode round (host bookkeeping, table upload, copy-on-write, append,
    attention) for the sequences in ``seq_ids`` (int64 numpy array, kept by the
    caller between calls to avoid re-marshalling)."""
    ids = seq_ids if isinstance(seq_ids, np.ndarray) and seq_ids.dtype == np.int64 \
        else np.ascontiguousarray(seq_ids, dtype=np.int64)
    _check(_lib.pkv_decode_step(step.handle, ids.ctypes.data_as(_I64P), int(ids.size),
                                _dev_ptr(q), _dev_ptr(k_new), _dev_ptr(v_new), float(scale),
                                _dev_ptr(out), _stream_ptr(stream)), "pkv_decode_step")


def _host_ptr(t) -> int:
    """Address of a contiguous host buffer: a CPU torch tensor (pinned or not)
    or a numpy array."""
    if isinstance(t, np.ndarray):
        if not t.flags["C_CONTIGUOUS"]:
            raise ValueError("expected a contiguous array")
        return t.ctypes.data
    if t.is_cuda:
        raise ValueError("expected a host tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def pkv_decode_step_host(step: Step, seq_ids, q, k_new, v_new, scale: float, out,
                         stream=None) -> None:
    """pkv_decode_step with q, k_new, v_new and out in host memory (CPU torch
    tensors, pinned for speed, or numpy arrays of the q dtype's bits); returns
    with the round's attention output in ``out``."""
    ids = seq_ids if isinstance(seq_ids, np.ndarray) and seq_ids.dtype == np.int64 \
        else np.ascontiguousarray(seq_ids, dtype=np.int64)
    _check(_lib.pkv_decode_step_host(step.handle, ids.ctypes.data_as(_I64P), int(ids.size),
                                     _host_ptr(q), _host_ptr(k_new), _host_ptr(v_new),
                                     float(scale), _host_ptr(out), _stream_ptr(stream)),
           "pkv_decode_step_host")


def pkv_step_last_launches(step: Step) -> int:
    return step.last_launches


def pkv_step_last_kernel(step: Step) -> int:
    return step.last_kernel


KERNEL_NAMES = {PKV_KERNEL_LEAN: "decode_lean_kernel", PKV_KERNEL_TENSOR: "decode_tc_kernel",
                PKV_KERNEL_SIMT_TMA: "decode_simt2_kernel", PKV_KERNEL_SIMT_BULK: "decode_simt_kernel"}


def pkv_step_profile(step: Step, n: int, every: int = 1) -> None:
    _check(_lib.pkv_step_profile(step.handle, int(n), int(every)), "pkv_step_profile")


def pkv_step_profile_read(step: Step, cap: int):
    """-> (prologue_ms [n], decode_ms [n], merge_ms [n]) numpy float32, oldest first."""
    bufs = [np.zeros(max(cap, 1), np.float32) for _ in range(3)]
    n = ctypes.c_int()
    fp = ctypes.POINTER(ctypes.c_float)
    _check(_lib.pkv_step_profile_read(step.handle, *(b.ctypes.data_as(fp) for b in bufs), int(cap),
                                      ctypes.byref(n)), "pkv_step_profile_read")
    return tuple(b[: n.value].copy() for b in bufs)


def paged_decode_static_scratch_bytes() -> int:
    return int(_lib.paged_decode_static_scratch_bytes())


def paged_decode_attention_static(pool: Pool, q, block_tables, context_lens, scale: float,
                                  out=None, partition_tokens: int = 0, stream=None):
    """paged_decode_attention without a workspace: for callers that cannot
    allocate device memory (the split scratch is the library's static device
    array).  ``out`` should be preallocated by such callers; if None it is
    allocated here for convenience."""
    import torch
    B, H_q, _ = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(_lib.paged_decode_attention_static(
        pool.handle, _dev_ptr(q), torch_dtype_code(q.dtype), _dev_ptr(block_tables),
        int(block_tables.shape[1]), _dev_ptr(context_lens), B, H_q, float(scale), _dev_ptr(out),
        int(partition_tokens), _stream_ptr(stream)), "paged_decode_attention_static")
    return out


# ---------------------------------------------------------------------------
# swap to host memory
# ---------------------------------------------------------------------------
def block_bytes(pool: Pool) -> int:
    return pool.n_kv_heads * pool.block_size * pool.head_dim * ELEM_BYTES[pool.dtype]


def kv_swap_out(pool: Pool, seq_id: int, h_k, h_v, stream=None):
    """Copy seq_id's blocks into pinned host uint8 tensors h_k/h_v and release
    the sequence.  -> (n_blocks, n_tokens)."""
    nb = ctypes.c_int32()
    nt = ctypes.c_int64()
    cap = min(h_k.numel() * h_k.element_size(), h_v.numel() * h_v.element_size())
    _check(_lib.kv_swap_out(pool.handle, int(seq_id), h_k.data_ptr(), h_v.data_ptr(), cap,
                            ctypes.byref(nb), ctypes.byref(nt), _stream_ptr(stream)), "kv_swap_out")
    return nb.value, nt.value


def kv_swap_in(pool: Pool, seq_id: int, h_k, h_v, n_tokens: int, stream=None) -> None:
    cap = min(h_k.numel() * h_k.element_size(), h_v.numel() * h_v.element_size())
    _check(_lib.kv_swap_in(pool.handle, int(seq_id), h_k.data_ptr(), h_v.data_ptr(), cap,
                           int(n_tokens), _stream_ptr(stream)), "kv_swap_in")


# ---------------------------------------------------------------------------
# the exhibit's allocation bench (host only)
# ---------------------------------------------------------------------------
SIM_MAX, SIM_POW2, SIM_ORACLE = 0, -1, -2


def pkv_simulate(requests, num_slots: int, block_size: int, max_len: int, max_rounds: int = 10000):
    """requests: sequence of (arrival, prompt, output).  block_size > 0 pages
    the memory; SIM_MAX (0), SIM_POW2 (-1) or SIM_ORACLE (-2) reserve one
    contiguous run per request of max_len slots, the next power of two of its
    final length, or exactly that length.  -> (result dict, running count per
    round)."""
    n = len(requests)
    arr = (pkv_sim_request * max(n, 1))()
    for i, (a, p, o) in enumerate(requests):
        arr[i].arrival, arr[i].prompt, arr[i].output = int(a), int(p), int(o)
    res = pkv_sim_result()
    per = np.zeros(max_rounds, np.int32)
    _check(_lib.pkv_simulate(arr, n, num_slots, block_size, max_len, max_rounds, ctypes.byref(res),
                             _ptr32(per)), "pkv_simulate")
    return res.as_dict(), per[: res.rounds].copy()
