"""Python binding of libpagedattn.so (paged decode attention for B200).

Argument marshalling only: each function checks tensor dtypes, devices and
shapes, then calls the C entry point of the same name with raw pointers and
the current CUDA stream.  Every step of the computation runs in the
library's kernels; there is no fallback.  The library is loaded from this
package's directory and must have been built with

    python -m paged_kv_cache_478_b200.build

Layouts (see include/pagedattn.h): pools [num_blocks, heads, 16, head_dim];
q, out, k_new, v_new [tokens or seqs, heads, head_dim]; block_tables int32
[num_seqs, max_blocks]; context_lens int32 [num_seqs]; slot_mapping int32
[num_tokens]; pairs int32 [num_pairs, 2].
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_F32, PA_F16, PA_BF16 = 0, 1, 2
PA_OK = 0
PA_ERR_NO_FREE_BLOCKS = 5
PA_DEVERR_BLOCK_ID = 0x1
PA_DEVERR_SLOT = 0x2
PA_DEVERR_CONTEXT_LEN = 0x4
PA_DEVERR_PAIR = 0x8
PA_DEVERR_TIMEOUT = 0x10
PA_DEVERR_PLAN = 0x20


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_status_name(status)}: {message}")
        self.status = status


class pa_pool(ctypes.Structure):
    _fields_ = [
        ("num_blocks", ctypes.c_int64),
        ("block_size", ctypes.c_int32),
        ("heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("elem_bytes", ctypes.c_int32),
        ("q_per_kv", ctypes.c_int32),
        ("token_stride", ctypes.c_int64),
        ("head_stride", ctypes.c_int64),
        ("block_stride", ctypes.c_int64),
        ("bytes_per_pool", ctypes.c_int64),
    ]


_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_478_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i32, i64, vp, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
        P = ctypes.POINTER
        sigs = {
            "pa_pool_create": [i64, i32, i32, i32, i32, P(pa_pool)],
            "pa_pool_set_query_heads": [P(pa_pool), i32],
            "pa_reshape_and_cache": [P(pa_pool), vp, vp, vp, i32, vp, vp, vp],
            "pa_decode_workspace_bytes": [P(pa_pool), i32, i32, i32, i32, P(sz)],
            "pa_decode_attention": [P(pa_pool), vp, vp, vp, vp, i32, vp, i32, i32, ctypes.c_float,
                                    vp, vp, sz, i32, vp],
            "pa_decode_plan": [P(pa_pool), vp, i32, i32, i32, i32, vp, sz, vp],
            "pa_decode_attention_planned": [P(pa_pool), vp, vp, vp, vp, i32, i32, i32,
                                            ctypes.c_float, vp, vp, sz, i32, vp],
            "pa_decode_append_attention": [P(pa_pool), vp, vp, vp, vp, vp, vp, i32, vp, i32, i32,
                                           ctypes.c_float, vp, vp, sz, i32, vp],
            "pa_decode_append_attention_planned": [P(pa_pool), vp, vp, vp, vp, vp, vp, i32, i32,
                                                   i32, ctypes.c_float, vp, vp, sz, i32, vp],
            "pa_decode_attention_static": [P(pa_pool), vp, vp, vp, vp, i32, vp, i32, i32,
                                           ctypes.c_float, vp, i32, vp],
            "pa_decode_shared_prefix_workspace_bytes": [P(pa_pool), i32, i32, i32, i32, i32, P(sz)],
            "pa_decode_attention_shared_prefix": [P(pa_pool), vp, vp, vp, vp, i32, vp, i32, vp, vp,
                                                  i32, vp, i32, i32, i32, i32, ctypes.c_float, vp,
                                                  vp, sz, i32, vp],
            "pa_find_shared_prefixes": [vp, i32, vp, i32, i32, i32, vp, vp, vp, P(i32), P(i32),
                                        P(i32)],
            "pa_prefill_attention": [P(pa_pool), vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32,
                                     ctypes.c_float, vp, vp],
            "pa_copy_blocks": [P(pa_pool), vp, vp, vp, i32, vp],
            "pa_device_errors": [vp, P(ctypes.c_uint32)],
            "pa_selftest_wait_timeout": [vp],
            "pa_alloc_create": [i64, P(vp)],
            "pa_alloc_block": [vp, P(i32)],
            "pa_share_block": [vp, i32],
            "pa_free_block": [vp, i32],
            "pa_cow_block": [vp, i32, P(i32)],
            "pa_refcount": [vp, i32, P(i32)],
            "pa_append_tokens": [vp, i32, vp, i32, P(i32), i32, vp, vp, P(i32)],
            "pa_fork_table": [vp, vp, i32, vp],
            "pa_release_table": [vp, vp, i32],
            "pa_decode_slots": [vp, i32, vp, i32, i32, vp],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.pa_alloc_destroy.argtypes = [vp]
        L.pa_alloc_destroy.restype = None
        L.pa_num_free.argtypes = [vp]
        L.pa_num_free.restype = i64
        L.pa_last_error.argtypes = []
        L.pa_last_error.restype = ctypes.c_char_p
        L.pa_status_string.argtypes = [i32]
        L.pa_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _status_name(status: int) -> str:
    try:
        return lib().pa_status_string(status).decode()
    except Exception:  # pragma: no cover
        return f"status {status}"


def _check(status: int):
    if status != PA_OK:
        raise PagedAttnError(status, lib().pa_last_error().decode())


# ---- torch marshalling -------------------------------------------------------------

def _torch():
    import torch

    return torch


def _dtype_code(t):
    torch = _torch()
    return {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}[t]


def _dev_ptr(t, name, dtype=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def pa_pool_create(num_blocks: int, block_size: int, heads: int, head_dim: int, dtype) -> pa_pool:
    """Describe a pool; dtype is a torch dtype or a PA_* code."""
    code = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    p = pa_pool()
    _check(lib().pa_pool_create(num_blocks, block_size, heads, head_dim, code, ctypes.byref(p)))
    return p


def pa_pool_set_query_heads(pool: pa_pool, num_q_heads: int) -> pa_pool:
    """GQA/MQA: q and out carry num_q_heads (1, 2, 4 or 8 per KV head)."""
    _check(lib().pa_pool_set_query_heads(ctypes.byref(pool), num_q_heads))
    return pool


def _q_heads(pool: pa_pool) -> int:
    return pool.heads * pool.q_per_kv


def _pool_torch_dtype(pool: pa_pool):
    torch = _torch()
    return {PA_F32: torch.float32, PA_F16: torch.float16, PA_BF16: torch.bfloat16}[pool.dtype]


def _check_pool_tensor(pool, t, name):
    shape = (pool.num_blocks, pool.heads, pool.block_size, pool.head_dim)
    if tuple(t.shape) != shape:
        raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
    return _dev_ptr(t, name, _pool_torch_dtype(pool))


def pa_reshape_and_cache(pool, k_new, v_new, slot_mapping, k_pool, v_pool, stream=None):
    torch = _torch()
    T = slot_mapping.shape[0]
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if tuple(t.shape) != (T, pool.heads, pool.head_dim):
            raise ValueError(f"{name} must have shape {(T, pool.heads, pool.head_dim)}")
    _check(lib().pa_reshape_and_cache(
        ctypes.byref(pool), _dev_ptr(k_new, "k_new", _pool_torch_dtype(pool)),
        _dev_ptr(v_new, "v_new", _pool_torch_dtype(pool)),
        _dev_ptr(slot_mapping, "slot_mapping", torch.int32), T,
        _check_pool_tensor(pool, k_pool, "k_pool"), _check_pool_tensor(pool, v_pool, "v_pool"),
        _stream(stream)))


def pa_decode_workspace_bytes(pool, num_seqs, max_blocks_per_seq, max_context_len=0,
                              partition_size=0) -> int:
    n = ctypes.c_size_t()
    _check(lib().pa_decode_workspace_bytes(ctypes.byref(pool), num_seqs, max_blocks_per_seq,
                                           max_context_len, partition_size, ctypes.byref(n)))
    return n.value


def pa_decode_attention(pool, q, k_pool, v_pool, block_tables, context_lens, scale, out,
                        workspace, max_context_len=0, partition_size=0, stream=None):
    torch = _torch()
    S = q.shape[0]
    if tuple(q.shape) != (S, _q_heads(pool), pool.head_dim) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [num_seqs, query heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [num_seqs, max_blocks], context_lens [num_seqs]")
    dt = _pool_torch_dtype(pool)
    _check(lib().pa_decode_attention(
        ctypes.byref(pool), _dev_ptr(q, "q", dt), _check_pool_tensor(pool, k_pool, "k_pool"),
        _check_pool_tensor(pool, v_pool, "v_pool"),
        _dev_ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev_ptr(context_lens, "context_lens", torch.int32), S, max_context_len, float(scale),
        _dev_ptr(out, "out", dt), _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), partition_size, _stream(stream)))


def pa_decode_plan(pool, context_lens, max_blocks_per_seq, workspace, max_context_len=0,
                   partition_size=0, stream=None):
    torch = _torch()
    _check(lib().pa_decode_plan(
        ctypes.byref(pool), _dev_ptr(context_lens, "context_lens", torch.int32),
        context_lens.shape[0], max_blocks_per_seq, max_context_len, partition_size,
        _dev_ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def pa_decode_attention_planned(pool, q, k_pool, v_pool, block_tables, scale, out, workspace,
                                max_context_len=0, partition_size=0, stream=None):
    torch = _torch()
    S = q.shape[0]
    if tuple(q.shape) != (S, _q_heads(pool), pool.head_dim) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [num_seqs, query heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S:
        raise ValueError("block_tables must be [num_seqs, max_blocks]")
    dt = _pool_torch_dtype(pool)
    _check(lib().pa_decode_attention_planned(
        ctypes.byref(pool), _dev_ptr(q, "q", dt), _check_pool_tensor(pool, k_pool, "k_pool"),
        _check_pool_tensor(pool, v_pool, "v_pool"),
        _dev_ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1], S,
        max_context_len, float(scale), _dev_ptr(out, "out", dt), _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), partition_size, _stream(stream)))


def pa_decode_append_attention(pool, q, k_new, v_new, k_pool, v_pool, block_tables, context_lens,
                               scale, out, workspace, max_context_len=0, partition_size=0,
                               stream=None):
    """reshape_and_cache of each sequence's new token (at position L-1) and
    decode attention in one launch; k_new/v_new are [num_seqs, heads, head_dim]."""
    torch = _torch()
    S = q.shape[0]
    if tuple(q.shape) != (S, _q_heads(pool), pool.head_dim) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [num_seqs, query heads, head_dim]")
    kv_shape = (S, pool.heads, pool.head_dim)
    if tuple(k_new.shape) != kv_shape or tuple(v_new.shape) != kv_shape:
        raise ValueError("k_new and v_new must be [num_seqs, KV heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [num_seqs, max_blocks], context_lens [num_seqs]")
    dt = _pool_torch_dtype(pool)
    _check(lib().pa_decode_append_attention(
        ctypes.byref(pool), _dev_ptr(q, "q", dt), _dev_ptr(k_new, "k_new", dt),
        _dev_ptr(v_new, "v_new", dt), _check_pool_tensor(pool, k_pool, "k_pool"),
        _check_pool_tensor(pool, v_pool, "v_pool"),
        _dev_ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev_ptr(context_lens, "context_lens", torch.int32), S, max_context_len, float(scale),
        _dev_ptr(out, "out", dt), _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), partition_size, _stream(stream)))


def pa_decode_append_attention_planned(pool, q, k_new, v_new, k_pool, v_pool, block_tables, scale,
                                       out, workspace, max_context_len=0, partition_size=0,
                                       stream=None):
    torch = _torch()
    S = q.shape[0]
    if tuple(q.shape) != (S, _q_heads(pool), pool.head_dim) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [num_seqs, query heads, head_dim]")
    kv_shape = (S, pool.heads, pool.head_dim)
    if tuple(k_new.shape) != kv_shape or tuple(v_new.shape) != kv_shape:
        raise ValueError("k_new and v_new must be [num_seqs, KV heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S:
        raise ValueError("block_tables must be [num_seqs, max_blocks]")
    dt = _pool_torch_dtype(pool)
    _check(lib().pa_decode_append_attention_planned(
        ctypes.byref(pool), _dev_ptr(q, "q", dt), _dev_ptr(k_new, "k_new", dt),
        _dev_ptr(v_new, "v_new", dt), _check_pool_tensor(pool, k_pool, "k_pool"),
        _check_pool_tensor(pool, v_pool, "v_pool"),
        _dev_ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1], S,
        max_context_len, float(scale), _dev_ptr(out, "out", dt), _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), partition_size, _stream(stream)))


def pa_find_shared_prefixes(block_tables, context_lens, min_shared_blocks=1, block_size=16):
    """Host helper: shared-prefix groups from host block tables.  Returns a
    dict of numpy arrays (offsets, members, blocks) and the launch bounds."""
    import numpy as np

    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S = cl.shape[0]
    offs = np.zeros(S + 1, dtype=np.int32)
    mem = np.zeros(max(S, 1), dtype=np.int32)
    blk = np.zeros(max(S, 1), dtype=np.int32)
    ng, mg, mb = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib().pa_find_shared_prefixes(bt.ctypes.data, bt.shape[1], cl.ctypes.data, S, block_size,
                                         min_shared_blocks, offs.ctypes.data, mem.ctypes.data,
                                         blk.ctypes.data, ctypes.byref(ng), ctypes.byref(mg),
                                         ctypes.byref(mb)))
    n = ng.value
    return dict(offsets=offs[:n + 1].copy(), members=mem[:offs[n]].copy(), blocks=blk[:n].copy(),
                num_groups=n, max_group_size=mg.value, max_shared_blocks=mb.value)


def pa_decode_shared_prefix_workspace_bytes(pool, num_seqs, max_blocks_per_seq, max_shared_blocks,
                                            max_context_len=0, partition_size=0) -> int:
    n = ctypes.c_size_t()
    _check(lib().pa_decode_shared_prefix_workspace_bytes(
        ctypes.byref(pool), num_seqs, max_blocks_per_seq, max_context_len, partition_size,
        max_shared_blocks, ctypes.byref(n)))
    return n.value


def pa_decode_attention_shared_prefix(pool, q, k_pool, v_pool, block_tables, context_lens, groups,
                                      scale, out, workspace, max_context_len=0, partition_size=0,
                                      stream=None):
    """groups: dict with device int32 tensors offsets, members, blocks and
    ints num_groups, max_group_size, max_shared_blocks (see
    pa_find_shared_prefixes for the host-side arrays)."""
    torch = _torch()
    S = q.shape[0]
    if tuple(q.shape) != (S, _q_heads(pool), pool.head_dim) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [num_seqs, query heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [num_seqs, max_blocks], context_lens [num_seqs]")
    dt = _pool_torch_dtype(pool)
    ng = groups["num_groups"]
    gp = [_dev_ptr(groups[k], k, torch.int32) if ng > 0 else None
          for k in ("offsets", "members", "blocks")]
    nm = groups["members"].numel() if ng > 0 else 0
    if ng > 0 and (groups["offsets"].numel() != ng + 1 or groups["blocks"].numel() != ng):
        raise ValueError("groups: offsets must have num_groups + 1 entries, blocks num_groups")
    _check(lib().pa_decode_attention_shared_prefix(
        ctypes.byref(pool), _dev_ptr(q, "q", dt), _check_pool_tensor(pool, k_pool, "k_pool"),
        _check_pool_tensor(pool, v_pool, "v_pool"),
        _dev_ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev_ptr(context_lens, "context_lens", torch.int32), S, gp[0], gp[1], nm, gp[2], ng,
        groups["max_group_size"], groups["max_shared_blocks"], max_context_len, float(scale),
        _dev_ptr(out, "out", dt), _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), partition_size, _stream(stream)))


def pa_prefill_attention(pool, q, k_pool, v_pool, block_tables, context_lens, query_start, scale,
                         out, max_new_tokens, max_context_len=0, stream=None):
    """Causal attention of many new tokens per sequence over the paged cache
    (tcgen05).  q, out: [T, query heads, head_dim]; query_start: int32 [S+1]."""
    torch = _torch()
    S = context_lens.shape[0]
    T = q.shape[0]
    if tuple(q.shape) != (T, _q_heads(pool), pool.head_dim) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [tokens, query heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(query_start.shape) != (S + 1,):
        raise ValueError("block_tables [S, max_blocks], context_lens [S], query_start [S+1]")
    dt = _pool_torch_dtype(pool)
    _check(lib().pa_prefill_attention(
        ctypes.byref(pool), _dev_ptr(q, "q", dt), _check_pool_tensor(pool, k_pool, "k_pool"),
        _check_pool_tensor(pool, v_pool, "v_pool"),
        _dev_ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev_ptr(context_lens, "context_lens", torch.int32),
        _dev_ptr(query_start, "query_start", torch.int32), S, T, max_new_tokens, max_context_len,
        float(scale), _dev_ptr(out, "out", dt), _stream(stream)))


STATIC_SCRATCH_BYTES = 32 << 20


def pa_decode_attention_static(pool, q, k_pool, v_pool, block_tables, context_lens, scale, out,
                               max_context_len=0, partition_size=0, stream=None):
    """pa_decode_attention without a workspace: the library's static scratch
    buffer (STATIC_SCRATCH_BYTES per GPU) holds the plan and the partials, so
    neither the caller nor the library allocates.  Calls must not overlap on
    the GPU; the first call on a device must come before any stream capture."""
    torch = _torch()
    S = q.shape[0]
    if tuple(q.shape) != (S, _q_heads(pool), pool.head_dim) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [num_seqs, query heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [num_seqs, max_blocks], context_lens [num_seqs]")
    dt = _pool_torch_dtype(pool)
    _check(lib().pa_decode_attention_static(
        ctypes.byref(pool), _dev_ptr(q, "q", dt), _check_pool_tensor(pool, k_pool, "k_pool"),
        _check_pool_tensor(pool, v_pool, "v_pool"),
        _dev_ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev_ptr(context_lens, "context_lens", torch.int32), S, max_context_len, float(scale),
        _dev_ptr(out, "out", dt), partition_size, _stream(stream)))


def pa_copy_blocks(pool, k_pool, v_pool, pairs, stream=None):
    torch = _torch()
    n = pairs.shape[0] if pairs.dim() == 2 else pairs.numel() // 2
    _check(lib().pa_copy_blocks(
        ctypes.byref(pool), _check_pool_tensor(pool, k_pool, "k_pool"),
        _check_pool_tensor(pool, v_pool, "v_pool"), _dev_ptr(pairs, "pairs", torch.int32), n,
        _stream(stream)))


def pa_device_errors(stream=None) -> int:
    """Synchronise the stream; return and clear the device error bits."""
    flags = ctypes.c_uint32()
    lib().pa_device_errors(_stream(stream), ctypes.byref(flags))
    return flags.value


def pa_selftest_wait_timeout(stream=None):
    """Launch the wait-limit self-test kernel (see include/pagedattn.h)."""
    _check(lib().pa_selftest_wait_timeout(_stream(stream)))


def pa_decode_slots(block_tables, context_lens, block_size=16):
    """Host numpy helper: slot of each sequence's last token."""
    import numpy as np

    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    out = np.empty(cl.shape[0], dtype=np.int32)
    _check(lib().pa_decode_slots(bt.ctypes.data, bt.shape[1], cl.ctypes.data, cl.shape[0],
                                 block_size, out.ctypes.data))
    return out


class BlockManager:
    """Host block manager (pa_alloc_*): free list and reference counts."""

    def __init__(self, num_blocks: int):
        h = ctypes.c_void_p()
        _check(lib().pa_alloc_create(num_blocks, ctypes.byref(h)))
        self._h = h

    def close(self):
        if self._h:
            lib().pa_alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def alloc(self) -> int:
        i = ctypes.c_int32()
        _check(lib().pa_alloc_block(self._h, ctypes.byref(i)))
        return i.value

    def share(self, block: int):
        _check(lib().pa_share_block(self._h, block))

    def free(self, block: int):
        _check(lib().pa_free_block(self._h, block))

    def cow(self, block: int) -> int:
        i = ctypes.c_int32()
        _check(lib().pa_cow_block(self._h, block, ctypes.byref(i)))
        return i.value

    def refcount(self, block: int) -> int:
        i = ctypes.c_int32()
        _check(lib().pa_refcount(self._h, block, ctypes.byref(i)))
        return i.value

    def num_free(self) -> int:
        return lib().pa_num_free(self._h)

    def append_tokens(self, table, context_len: int, num_new: int, block_size: int = 16):
        """table: int32 numpy row (modified in place).  Returns
        (new_context_len, slots[num_new], cow_pairs[k, 2])."""
        import numpy as np

        assert table.dtype == np.int32 and table.flags.c_contiguous
        slots = np.empty(num_new, dtype=np.int32)
        pairs = np.empty((max(num_new, 1), 2), dtype=np.int32)
        cl = ctypes.c_int32(context_len)
        nc = ctypes.c_int32(0)
        _check(lib().pa_append_tokens(self._h, block_size, table.ctypes.data, table.shape[0],
                                      ctypes.byref(cl), num_new, slots.ctypes.data,
                                      pairs.ctypes.data, ctypes.byref(nc)))
        return cl.value, slots, pairs[:nc.value].copy()

    def fork_table(self, src_table, num_blocks: int, dst_table):
        _check(lib().pa_fork_table(self._h, src_table.ctypes.data, num_blocks, dst_table.ctypes.data))

    def release_table(self, table, num_blocks: int):
        _check(lib().pa_release_table(self._h, table.ctypes.data, num_blocks))
