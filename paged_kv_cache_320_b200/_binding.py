"""ctypes binding of libpagedkv.so: argument marshalling only.

Every function here reads pointers, sizes and the current CUDA stream from torch
tensors and calls the C entry point of the same name; all device work runs in the
library's kernels. There is no fallback: if the library is missing, the first call
raises. Before a call, every tensor whose address the library will dereference is checked
to be a contiguous CUDA tensor on the query's device, of the element type and with at
least the rows the C declaration reads (ValueError / TypeError otherwise), so that a host
tensor or a short index array never reaches a kernel.
"""
from __future__ import annotations

import ctypes
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# PAGEDKV_LIB may name a library built elsewhere (e.g. with other compile options)
LIB_PATH = os.environ.get("PAGEDKV_LIB") or os.path.join(HERE, "libpagedkv.so")

PKV_OK = 0
PKV_ERR_INVALID_ARG = -1
PKV_ERR_OUT_OF_BLOCKS = -2
PKV_ERR_UNKNOWN_SEQ = -3
PKV_ERR_SEQ_EXISTS = -4
PKV_ERR_TABLE_FULL = -5
PKV_ERR_BAD_INDEX = -6
PKV_ERR_TIMEOUT = -7
PKV_ERR_CUDA = -8
PKV_ERR_WORKSPACE = -9
PKV_ERR_HOST_MEMORY = -10

PKV_F16 = 0
PKV_BF16 = 1

STATUS_BAD_SLOT = 1 << 0
STATUS_BAD_PAIR = 1 << 1
STATUS_BAD_BLOCK = 1 << 2
STATUS_BAD_LEN = 1 << 3
STATUS_WAIT_TIMEOUT = 1 << 4
STATUS_NO_BLOCKS = 1 << 5
STATUS_WORKSPACE = 1 << 6
STATUS_SHARED_BLOCK = 1 << 7

_lib = None


class PagedKVError(RuntimeError):
    def __init__(self, code, what=""):
        self.code = code
        msg = lib().pkv_status_string(code).decode() if _lib is not None else str(code)
        super().__init__(f"{what}: {msg} ({code})")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_320_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.pkv_status_string.argtypes = [I]
        L.pkv_status_string.restype = ctypes.c_char_p
        L.pkv_paged_attention_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I,
                                                 ctypes.c_float, I, I, P, SZ, P]
        L.pkv_paged_attention_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I,
                                                         I, I, ctypes.c_float, I, I, P]
        L.pkv_paged_attention_decode_partitions.argtypes = L.pkv_paged_attention_decode.argtypes
        L.pkv_paged_attention_merge.argtypes = [P, P, I, I, I, I, I, I, I, I, P, SZ, P]
        L.pkv_decode_workspace_size.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(SZ)]
        L.pkv_paged_attention_decode_shared_prefix.argtypes = [
            P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, ctypes.c_float, I, I, P, SZ, P]
        L.pkv_decode_shared_prefix_workspace_size.argtypes = [I, I, I, I, I, I, I,
                                                              ctypes.POINTER(SZ)]
        L.pkv_decode_partition_size.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(I)]
        L.pkv_decode_shared_prefix_partition_size.argtypes = [I, I, I, I, I, I, I,
                                                               ctypes.POINTER(I)]
        L.pkv_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P]
        L.pkv_copy_blocks.argtypes = [P, P, I, P, I, I, I, I, I, I, P]
        L.pkv_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), I, P]
        L.pkv_swap_blocks.argtypes = [P, P, I, P, I, P, SZ, I, I, I, I, I, I, P]
        L.pkv_swap_blocks_staged.argtypes = [P, P, I, P, I, P, SZ, I, I, I, I, I, I, P, SZ, P]
        L.pkv_alloc_create.argtypes = [ctypes.POINTER(P), I, I, I, P]
        L.pkv_alloc_destroy.argtypes = [P]
        L.pkv_seq_append.argtypes = [P, I64, I, P, P, ctypes.POINTER(I)]
        L.pkv_seq_append_batch.argtypes = [P, P, I, I, P, P, ctypes.POINTER(I),
                                           ctypes.POINTER(I)]
        L.pkv_seq_append_tables.argtypes = [P, P, I, I, P, P, ctypes.POINTER(I),
                                            ctypes.POINTER(I), P, P]
        L.pkv_prefix_groups.argtypes = [P, P, I, P, P, P, ctypes.POINTER(I)]
        L.pkv_seq_fork.argtypes = [P, I64, I64]
        L.pkv_seq_free.argtypes = [P, I64]
        L.pkv_block_tables.argtypes = [P, P, I, P, P]
        L.pkv_stats.argtypes = [P, ctypes.POINTER(I), ctypes.POINTER(I),
                                ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_double)]
        L.pkv_paged_decode_step.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I,
                                            ctypes.c_float, I, I, P, SZ, P]
        L.pkv_paged_decode_step_partitions.argtypes = L.pkv_paged_decode_step.argtypes
        L.pkv_decode_step_workspace_size.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(SZ)]
        L.pkv_device_append.argtypes = [P, P, P, I, P, P, P, I, I, I, I, I, P]
        L.pkv_alloc_refcounts.argtypes = [P, P, I]
        L.pkv_decode_step_launches.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(I)]
        L.pkv_alloc_free_list.argtypes = [P, P, I, ctypes.POINTER(I)]
        L.pkv_shared_prefix_plan.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, I, P, SZ, P]
        L.pkv_paged_attention_decode_shared_prefix_planned.argtypes = [
            P, P, P, P, P, P, I, I, I, I, I, I, I, I, ctypes.c_float, I, I, P, SZ, P]
        L.pkv_seq_fork_batch.argtypes = [P, P, P, I, ctypes.POINTER(I)]
        L.pkv_seq_free_batch.argtypes = [P, P, I, ctypes.POINTER(I)]
        L.pkv_alloc_set_prefix_cache.argtypes = [P, I]
        L.pkv_seq_append_tokens.argtypes = [P, I64, P, I, P, P, ctypes.POINTER(I)]
        L.pkv_seq_share_prefix.argtypes = [P, I64, P, I, ctypes.POINTER(I)]
        L.pkv_prefix_cache_stats.argtypes = [P, ctypes.POINTER(I), ctypes.POINTER(I),
                                             ctypes.POINTER(ctypes.c_int64),
                                             ctypes.POINTER(ctypes.c_int64)]
        for name in ("pkv_paged_attention_decode", "pkv_paged_attention_decode_noalloc",
                     "pkv_paged_attention_decode_partitions", "pkv_paged_attention_merge",
                     "pkv_paged_decode_step_partitions",
                     "pkv_paged_attention_decode_shared_prefix",
                     "pkv_decode_shared_prefix_workspace_size", "pkv_decode_workspace_size",
                     "pkv_decode_partition_size", "pkv_decode_shared_prefix_partition_size",
                     "pkv_reshape_and_cache", "pkv_copy_blocks",
                     "pkv_swap_blocks",
                     "pkv_get_device_status", "pkv_alloc_create", "pkv_alloc_destroy",
                     "pkv_seq_append", "pkv_seq_append_batch", "pkv_seq_fork", "pkv_seq_free",
                     "pkv_block_tables", "pkv_stats", "pkv_alloc_set_prefix_cache",
                     "pkv_paged_decode_step", "pkv_decode_step_workspace_size", "pkv_device_append",
                     "pkv_alloc_free_list", "pkv_alloc_refcounts", "pkv_decode_step_launches",
                     "pkv_seq_fork_batch",
                     "pkv_seq_free_batch", "pkv_shared_prefix_plan",
                     "pkv_paged_attention_decode_shared_prefix_planned",
                     "pkv_seq_append_tokens", "pkv_seq_share_prefix", "pkv_prefix_cache_stats",
                     "pkv_seq_append_tables", "pkv_swap_blocks_staged", "pkv_prefix_groups"):
            getattr(L, name).restype = I
        _lib = L
    return _lib


def _check(rc, what):
    if rc != PKV_OK:
        raise PagedKVError(rc, what)


# ---------------------------------------------------------------------------
# tensor marshalling helpers
# ---------------------------------------------------------------------------
def _dtype_code(t):
    import torch
    if t.dtype == torch.float16:
        return PKV_F16
    if t.dtype == torch.bfloat16:
        return PKV_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libpagedkv must be contiguous")
    return t.data_ptr()


def _nbytes(t):
    return t.numel() * t.element_size()


def _need(t, name, device=None, dtype=None, min_numel=0):
    """Raise unless ``t`` is a contiguous CUDA tensor (on ``device`` when given, of
    ``dtype`` when given) holding at least ``min_numel`` elements."""
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call runs on {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, not {t.dtype}")
    if t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, the call reads {min_numel}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _tables(block_tables, context_lens, B, device):
    """block_tables int32 [>= B, MB] and context_lens int32 [>= B] on ``device``."""
    import torch
    if block_tables.dim() != 2 or block_tables.shape[0] < B:
        raise ValueError(f"block_tables must be [num_seqs >= {B}, max_blocks_per_seq], "
                         f"not {tuple(block_tables.shape)}")
    _need(block_tables, "block_tables", device, torch.int32)
    _need(context_lens, "context_lens", device, torch.int32, B)


def _decode_shapes(out, q, k_cache, v_cache, block_tables, context_lens, k_new=None,
                   v_new=None):
    """Checks the decode family's tensors; returns (B, Hq, D, NB, Hkv, BS)."""
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [B, Hq, D] and k_cache [NB, Hkv, BS, D]")
    B, Hq, D = q.shape
    NB, Hkv, BS, D2 = k_cache.shape
    if D2 != D or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    _dtype_code(q)
    dev = q.device
    for name, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("k_new", k_new), ("v_new", v_new)):
        if t is not None:
            _need(t, name, dev, q.dtype)
    _tables(block_tables, context_lens, B, dev)
    return B, Hq, D, NB, Hkv, BS


def _groups(group_start, prefix_lens, device):
    """group_start int32 [num_groups + 1] and prefix_lens int32 [num_groups]."""
    import torch
    _need(prefix_lens, "prefix_lens", device, torch.int32)
    _need(group_start, "group_start", device, torch.int32, prefix_lens.numel() + 1)


def _cache_ptrs(k_cache_ptrs, v_cache_ptrs):
    """Per-layer cache address arrays: int64 device tensors of one length."""
    import torch
    _need(k_cache_ptrs, "k_cache_ptrs", None, torch.int64)
    _need(v_cache_ptrs, "v_cache_ptrs", k_cache_ptrs.device, torch.int64,
          k_cache_ptrs.numel())


# ---------------------------------------------------------------------------
# device entry points
# ---------------------------------------------------------------------------
def pkv_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                              max_context_len, partition_size=0) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().pkv_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                           block_size, max_context_len, partition_size,
                                           ctypes.byref(out)), "pkv_decode_workspace_size")
    return out.value


def pkv_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                              max_context_len, partition_size=0) -> int:
    out = ctypes.c_int(0)
    _check(lib().pkv_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                           block_size, max_context_len, partition_size,
                                           ctypes.byref(out)), "pkv_decode_partition_size")
    return out.value


def pkv_decode_shared_prefix_partition_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                            block_size, max_context_len, partition_size=0) -> int:
    out = ctypes.c_int(0)
    _check(lib().pkv_decode_shared_prefix_partition_size(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
        partition_size, ctypes.byref(out)), "pkv_decode_shared_prefix_partition_size")
    return out.value


def pkv_paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens,
                               max_context_len, scale=None, partition_size=0, workspace=None,
                               stream=None):
    """out/q [B, Hq, D]; k_cache/v_cache [NB, Hkv, BS, D]; block_tables int32 [B, MB];
    context_lens int32 [B]; workspace: uint8 tensor of pkv_decode_workspace_size bytes
    (allocated here when None and needed)."""
    return _decode("pkv_paged_attention_decode", out, q, k_cache, v_cache, block_tables,
                   context_lens, max_context_len, scale, partition_size, workspace, stream)


def pkv_paged_attention_decode_partitions(out, q, k_cache, v_cache, block_tables, context_lens,
                                          max_context_len, workspace, scale=None,
                                          partition_size=0, stream=None):
    """The decode kernel of pkv_paged_attention_decode alone: one-partition sequences'
    outputs, the others' partials left in workspace for pkv_paged_attention_merge."""
    return _decode("pkv_paged_attention_decode_partitions", out, q, k_cache, v_cache,
                   block_tables, context_lens, max_context_len, scale, partition_size, workspace,
                   stream)


def pkv_paged_attention_merge(out, context_lens, num_kv_heads, block_size, max_context_len,
                              workspace, partition_size=0, stream=None):
    """Merge of the partials a partitions call left in workspace into out [B, Hq, D]."""
    import torch
    _need(out, "out")
    _need(context_lens, "context_lens", out.device, torch.int32, out.shape[0])
    _need(workspace, "workspace", out.device)
    B, Hq, D = out.shape
    _check(lib().pkv_paged_attention_merge(
        _ptr(out), _ptr(context_lens), B, Hq, int(num_kv_heads), D, int(block_size),
        int(max_context_len), int(partition_size), _dtype_code(out), _ptr(workspace),
        _nbytes(workspace), _stream(stream)), "pkv_paged_attention_merge")
    return out


def _decode(name, out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
            partition_size, workspace, stream):
    B, Hq, D, NB, Hkv, BS = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                           context_lens)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if workspace is None:
        need = pkv_decode_workspace_size(B, Hq, Hkv, D, BS, max_context_len, partition_size)
        if need:
            import torch
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None:
        _need(workspace, "workspace", q.device)
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_bytes = _nbytes(workspace) if workspace is not None else 0
    _check(getattr(lib(), name)(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        B, Hq, Hkv, D, BS, block_tables.shape[1], NB, int(max_context_len), float(scale),
        _dtype_code(q), int(partition_size), ws_ptr, ws_bytes, _stream(stream)), name)
    return out


def pkv_paged_attention_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens,
                                       max_context_len, scale=None, partition_size=0,
                                       stream=None):
    """pkv_paged_attention_decode without a workspace: the library's fixed scratch
    array is used instead (see pagedkv.h); raises PagedKVError(PKV_ERR_WORKSPACE)
    when the sizes need more scratch than it holds."""
    B, Hq, D, NB, Hkv, BS = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                           context_lens)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _check(lib().pkv_paged_attention_decode_noalloc(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        B, Hq, Hkv, D, BS, block_tables.shape[1], NB, int(max_context_len), float(scale),
        _dtype_code(q), int(partition_size), _stream(stream)),
        "pkv_paged_attention_decode_noalloc")
    return out


def pkv_decode_shared_prefix_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                            block_size, max_context_len, partition_size=0):
    out = ctypes.c_size_t(0)
    _check(lib().pkv_decode_shared_prefix_workspace_size(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len, partition_size,
        ctypes.byref(out)), "pkv_decode_shared_prefix_workspace_size")
    return out.value


def pkv_paged_attention_decode_shared_prefix(out, q, k_cache, v_cache, block_tables,
                                             context_lens, group_start, prefix_lens,
                                             max_context_len, scale=None, partition_size=0,
                                             workspace=None, stream=None):
    """As pkv_paged_attention_decode, with group_start int32 [num_groups + 1] and
    prefix_lens int32 [num_groups] device tensors describing shared prefixes."""
    B, Hq, D, NB, Hkv, BS = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                           context_lens)
    _groups(group_start, prefix_lens, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if workspace is None:
        import torch
        need = pkv_decode_shared_prefix_workspace_size(B, Hq, Hkv, D, BS, max_context_len,
                                                       partition_size)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", q.device)
    _check(lib().pkv_paged_attention_decode_shared_prefix(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        _ptr(group_start), _ptr(prefix_lens), prefix_lens.numel(), B, Hq, Hkv, D, BS,
        block_tables.shape[1], NB, int(max_context_len), float(scale), _dtype_code(q),
        int(partition_size), _ptr(workspace), _nbytes(workspace), _stream(stream)),
        "pkv_paged_attention_decode_shared_prefix")
    return out


def pkv_decode_step_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                   max_context_len, partition_size=0) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().pkv_decode_step_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                                block_size, max_context_len, partition_size,
                                                ctypes.byref(out)),
           "pkv_decode_step_workspace_size")
    return out.value


def pkv_decode_step_launches(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                             max_context_len, partition_size=0) -> int:
    out = ctypes.c_int(0)
    _check(lib().pkv_decode_step_launches(num_seqs, num_heads, num_kv_heads, head_dim,
                                          block_size, max_context_len, partition_size,
                                          ctypes.byref(out)), "pkv_decode_step_launches")
    return out.value


def pkv_paged_decode_step(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens,
                          max_context_len, workspace, scale=None, partition_size=0, stream=None):
    """Cache write of each sequence's newest token + decode attention in one launch.
    k_new/v_new [B, Hkv, D]; workspace: uint8 device tensor of
    pkv_decode_step_workspace_size bytes, zero-filled before its first use (torch.zeros)."""
    return _step("pkv_paged_decode_step", out, q, k_new, v_new, k_cache, v_cache, block_tables,
                 context_lens, max_context_len, workspace, scale, partition_size, stream)


def pkv_paged_decode_step_partitions(out, q, k_new, v_new, k_cache, v_cache, block_tables,
                                     context_lens, max_context_len, workspace, scale=None,
                                     partition_size=0, stream=None):
    """The write-and-decode launch of pkv_paged_decode_step alone (merge with
    pkv_paged_attention_merge on the same workspace)."""
    return _step("pkv_paged_decode_step_partitions", out, q, k_new, v_new, k_cache, v_cache,
                 block_tables, context_lens, max_context_len, workspace, scale, partition_size,
                 stream)


def _step(name, out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens,
          max_context_len, workspace, scale, partition_size, stream):
    B, Hq, D, NB, Hkv, BS = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                           context_lens, k_new, v_new)
    if tuple(k_new.shape) != (B, Hkv, D) or v_new.shape != k_new.shape:
        raise ValueError("k_new / v_new must be [B, Hkv, D]")
    _need(workspace, "workspace", q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _check(getattr(lib(), name)(
        _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv, D, BS, block_tables.shape[1], NB,
        int(max_context_len), float(scale), _dtype_code(q), int(partition_size), _ptr(workspace),
        _nbytes(workspace), _stream(stream)), name)
    return out


def pkv_device_append(block_tables, context_lens, free_blocks, free_used, num_blocks,
                      max_context_len, block_size, slots_out=None, block_refcounts=None,
                      stream=None):
    """One token appended to every sequence on the device (see pagedkv.h): block_tables
    int32 [B, MB] and context_lens int32 [B] updated in place; free_blocks int32 [F] in pop
    order; free_used int32 [1] advanced by the blocks taken; slots_out int64 [B] or None;
    block_refcounts int32 [num_blocks] (the host manager's pkv_alloc_refcounts) or None:
    with it, a write into a shared partly filled block refuses the step."""
    import torch
    _need(context_lens, "context_lens", None, torch.int32)
    B = context_lens.numel()
    dev = context_lens.device
    _tables(block_tables, context_lens, B, dev)
    _need(free_blocks, "free_blocks", dev, torch.int32)
    _need(free_used, "free_used", dev, torch.int32, 1)
    if slots_out is not None:
        _need(slots_out, "slots_out", dev, torch.int64, B)
    if block_refcounts is not None:
        _need(block_refcounts, "block_refcounts", dev, torch.int32, int(num_blocks))
    _check(lib().pkv_device_append(
        _ptr(block_tables), _ptr(context_lens), _ptr(free_blocks), free_blocks.numel(),
        _ptr(free_used), _ptr(block_refcounts), _ptr(slots_out), B, block_tables.shape[1],
        int(block_size), int(num_blocks), int(max_context_len), _stream(stream)),
        "pkv_device_append")


def pkv_shared_prefix_plan(block_tables, context_lens, group_start, prefix_lens, num_heads,
                           num_kv_heads, head_dim, block_size, max_context_len, workspace,
                           partition_size=0, stream=None):
    """Build the shared-prefix item list in workspace (uint8 device tensor of
    pkv_decode_shared_prefix_workspace_size bytes) for every layer of a step."""
    import torch
    _need(context_lens, "context_lens", None, torch.int32)
    B = context_lens.numel()
    dev = context_lens.device
    _tables(block_tables, context_lens, B, dev)
    _groups(group_start, prefix_lens, dev)
    _need(workspace, "workspace", dev)
    _check(lib().pkv_shared_prefix_plan(
        _ptr(block_tables), _ptr(context_lens), _ptr(group_start), _ptr(prefix_lens),
        prefix_lens.numel(), B, int(num_heads), int(num_kv_heads), int(head_dim),
        int(block_size), block_tables.shape[1], int(max_context_len), int(partition_size),
        _ptr(workspace), _nbytes(workspace), _stream(stream)), "pkv_shared_prefix_plan")


def pkv_paged_attention_decode_shared_prefix_planned(out, q, k_cache, v_cache, block_tables,
                                                     context_lens, max_context_len, workspace,
                                                     scale=None, partition_size=0,
                                                     stream=None):
    """Decode over the plan pkv_shared_prefix_plan left in workspace."""
    B, Hq, D, NB, Hkv, BS = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                           context_lens)
    _need(workspace, "workspace", q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _check(lib().pkv_paged_attention_decode_shared_prefix_planned(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        B, Hq, Hkv, D, BS, block_tables.shape[1], NB, int(max_context_len), float(scale),
        _dtype_code(q), int(partition_size), _ptr(workspace), _nbytes(workspace),
        _stream(stream)), "pkv_paged_attention_decode_shared_prefix_planned")
    return out


def pkv_reshape_and_cache(k_new, v_new, k_cache, v_cache, slot_mapping, stream=None):
    """k_new/v_new [T, Hkv, D]; caches [NB, Hkv, BS, D]; slot_mapping int64 [T]."""
    import torch
    if k_new.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("k_new must be [T, Hkv, D] and k_cache [NB, Hkv, BS, D]")
    T, Hkv, D = k_new.shape
    NB, Hkv2, BS, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or v_new.shape != k_new.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    dev = k_cache.device
    for name, t in (("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache),
                    ("v_cache", v_cache)):
        _need(t, name, dev, k_cache.dtype)
    _need(slot_mapping, "slot_mapping", dev, torch.int64, T)
    _check(lib().pkv_reshape_and_cache(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(slot_mapping), T, Hkv, D, BS, NB,
                                       _dtype_code(k_cache), _stream(stream)),
           "pkv_reshape_and_cache")


def pkv_copy_blocks(k_cache_ptrs, v_cache_ptrs, block_pairs, num_kv_heads, head_dim, block_size,
                    num_blocks, dtype, stream=None):
    """k_cache_ptrs / v_cache_ptrs: int64 device tensors [L] of cache addresses;
    block_pairs: int32 device tensor [n, 2]."""
    import torch
    n = block_pairs.shape[0] if block_pairs.numel() else 0
    if n and (block_pairs.dim() != 2 or block_pairs.shape[1] != 2):
        raise ValueError("block_pairs must be [n, 2]")
    _cache_ptrs(k_cache_ptrs, v_cache_ptrs)
    _need(block_pairs, "block_pairs", k_cache_ptrs.device, torch.int32)
    _check(lib().pkv_copy_blocks(_ptr(k_cache_ptrs), _ptr(v_cache_ptrs), k_cache_ptrs.numel(),
                                 _ptr(block_pairs), n, num_kv_heads, head_dim, block_size,
                                 num_blocks, dtype, _stream(stream)), "pkv_copy_blocks")


def pkv_swap_blocks(k_cache_ptrs, v_cache_ptrs, block_ids, host_buffer, to_host, num_kv_heads,
                    head_dim, block_size, num_blocks, dtype, stream=None):
    """Moves whole blocks between the caches and a pinned host tensor (see pagedkv.h).
    k_cache_ptrs / v_cache_ptrs: int64 device tensors of cache addresses; block_ids:
    int32 device tensor; host_buffer: pinned CPU tensor (checked by the library)."""
    import torch
    n = block_ids.numel()
    _cache_ptrs(k_cache_ptrs, v_cache_ptrs)
    _need(block_ids, "block_ids", k_cache_ptrs.device, torch.int32)
    _check(lib().pkv_swap_blocks(_ptr(k_cache_ptrs), _ptr(v_cache_ptrs), k_cache_ptrs.numel(),
                                 _ptr(block_ids), n, _ptr(host_buffer),
                                 _nbytes(host_buffer), int(to_host),
                                 num_kv_heads, head_dim, block_size, num_blocks, dtype,
                                 _stream(stream)), "pkv_swap_blocks")


def pkv_swap_blocks_staged(k_cache_ptrs, v_cache_ptrs, block_ids, host_buffer, to_host,
                           num_kv_heads, head_dim, block_size, num_blocks, dtype, staging,
                           stream=None):
    """pkv_swap_blocks through a device staging tensor (uint8, CUDA) and large copies (see
    pagedkv.h)."""
    import torch
    n = block_ids.numel()
    _cache_ptrs(k_cache_ptrs, v_cache_ptrs)
    _need(block_ids, "block_ids", k_cache_ptrs.device, torch.int32)
    _need(staging, "staging", k_cache_ptrs.device, torch.uint8)
    _check(lib().pkv_swap_blocks_staged(_ptr(k_cache_ptrs), _ptr(v_cache_ptrs),
                                        k_cache_ptrs.numel(), _ptr(block_ids), n,
                                        _ptr(host_buffer), _nbytes(host_buffer), int(to_host),
                                        num_kv_heads, head_dim, block_size, num_blocks, dtype,
                                        _ptr(staging), _nbytes(staging), _stream(stream)),
           "pkv_swap_blocks_staged")


def pkv_get_device_status(clear=True, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(lib().pkv_get_device_status(ctypes.byref(v), int(bool(clear)), _stream(stream)),
           "pkv_get_device_status")
    return v.value


# ---------------------------------------------------------------------------
# host block manager
# ---------------------------------------------------------------------------
class BlockManager:
    """Owner of a pkv_alloc handle (host-only; no CUDA call)."""

    def __init__(self, num_blocks, block_size, max_blocks_per_seq, initial_order=None):
        import numpy as np
        self.num_blocks, self.block_size, self.max_blocks_per_seq = (
            num_blocks, block_size, max_blocks_per_seq)
        h = ctypes.c_void_p()
        order = None
        if initial_order is not None:
            order = np.ascontiguousarray(initial_order, dtype=np.int32)
        _check(lib().pkv_alloc_create(ctypes.byref(h), num_blocks, block_size, max_blocks_per_seq,
                                      order.ctypes.data if order is not None else None),
               "pkv_alloc_create")
        self._h = h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().pkv_alloc_destroy(self._h)
            self._h = None

    __del__ = close

    def pkv_seq_append(self, seq_id, n_tokens):
        """Returns (status, slots int64 array, cow pairs int32 [k, 2])."""
        import numpy as np
        slots = np.zeros(max(n_tokens, 1), dtype=np.int64)
        cows = np.zeros((max(n_tokens, 1), 2), dtype=np.int32)
        n_cow = ctypes.c_int(0)
        rc = lib().pkv_seq_append(self._h, int(seq_id), int(n_tokens), slots.ctypes.data,
                                  cows.ctypes.data, ctypes.byref(n_cow))
        if rc != PKV_OK:
            return rc, slots[:0], cows[:0]
        return rc, slots[:n_tokens], cows[:n_cow.value]

    def pkv_seq_append_batch(self, seq_ids, n_tokens):
        """Returns (status, n_done, slots int64 [n, n_tokens], cow pairs int32 [k, 2])."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.shape[0]
        slots = np.zeros((max(n, 1), max(n_tokens, 1)), dtype=np.int64)
        cows = np.zeros((max(n * n_tokens, 1), 2), dtype=np.int32)
        n_cow, n_done = ctypes.c_int(0), ctypes.c_int(0)
        rc = lib().pkv_seq_append_batch(self._h, ids.ctypes.data, n, int(n_tokens),
                                        slots.ctypes.data, cows.ctypes.data,
                                        ctypes.byref(n_cow), ctypes.byref(n_done))
        return rc, n_done.value, slots[:n, :n_tokens], cows[:n_cow.value]

    def pkv_seq_append_tables(self, seq_ids, n_tokens, slots_out=None, cows_out=None,
                              tables_out=None, lens_out=None):
        """pkv_seq_append_batch then, if it succeeded, pkv_block_tables of the same sequences,
        in one call. Returns (status, n_done, slots [n, n_tokens], cow pairs [k, 2], tables
        [n, max_blocks_per_seq], lens [n]). Each output may be given as a writable C-contiguous
        array of the right dtype and shape (e.g. a view of a pinned host buffer; cows_out with
        room for n * n_tokens pairs): the library then writes into it."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.shape[0]
        mb = self.max_blocks_per_seq

        def out(arr, shape, dtype, what):
            if arr is None:
                return np.zeros(shape, dtype=dtype)
            if (not isinstance(arr, np.ndarray) or arr.dtype != dtype or tuple(arr.shape) != shape
                    or not arr.flags.c_contiguous or not arr.flags.writeable):
                raise ValueError(f"{what} must be a writable C-contiguous {np.dtype(dtype)} "
                                 f"array of shape {shape}")
            return arr

        slots = out(slots_out, (n, int(n_tokens)), np.int64, "slots_out")
        cows = out(cows_out, (n * int(n_tokens), 2), np.int32, "cows_out")
        tables = out(tables_out, (n, mb), np.int32, "tables_out")
        lens = out(lens_out, (n,), np.int32, "lens_out")
        n_cow, n_done = ctypes.c_int(0), ctypes.c_int(0)
        rc = lib().pkv_seq_append_tables(self._h, ids.ctypes.data, n, int(n_tokens),
                                         slots.ctypes.data, cows.ctypes.data,
                                         ctypes.byref(n_cow), ctypes.byref(n_done),
                                         tables.ctypes.data, lens.ctypes.data)
        return rc, n_done.value, slots, cows[:n_cow.value], tables, lens

    def pkv_prefix_groups(self, seq_ids):
        """Groups of sequences sharing their first pages, for the shared-prefix decode.
        Returns (status, order int64 [n], group_start int32 [groups + 1], prefix_lens int32
        [groups])."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.shape[0]
        order = np.zeros(max(n, 1), dtype=np.int64)
        starts = np.zeros(n + 1, dtype=np.int32)
        prefixes = np.zeros(max(n, 1), dtype=np.int32)
        ng = ctypes.c_int(0)
        rc = lib().pkv_prefix_groups(self._h, ids.ctypes.data, n, order.ctypes.data,
                                     starts.ctypes.data, prefixes.ctypes.data, ctypes.byref(ng))
        g = ng.value
        return rc, order[:n], starts[:g + 1], prefixes[:g]

    def pkv_alloc_free_list(self, max_out=None):
        """Blocks the next allocations would take, in order (int32 array)."""
        import numpy as np
        m = self.num_blocks if max_out is None else int(max_out)
        buf = np.zeros(max(m, 1), dtype=np.int32)
        n = ctypes.c_int(0)
        _check(lib().pkv_alloc_free_list(self._h, buf.ctypes.data, m, ctypes.byref(n)),
               "pkv_alloc_free_list")
        return buf[:n.value].copy()

    def pkv_alloc_refcounts(self):
        """Reference count of every block (int32 array of num_blocks)."""
        import numpy as np
        buf = np.zeros(self.num_blocks, dtype=np.int32)
        _check(lib().pkv_alloc_refcounts(self._h, buf.ctypes.data, self.num_blocks),
               "pkv_alloc_refcounts")
        return buf

    def pkv_alloc_set_prefix_cache(self, enable):
        return lib().pkv_alloc_set_prefix_cache(self._h, int(bool(enable)))

    def pkv_seq_append_tokens(self, seq_id, tokens):
        """Append with token ids (int32); returns (status, slots, cow pairs [k, 2])."""
        import numpy as np
        tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1)
        n = tok.shape[0]
        slots = np.zeros(max(n, 1), dtype=np.int64)
        cows = np.zeros((max(n, 1), 2), dtype=np.int32)
        n_cow = ctypes.c_int(0)
        rc = lib().pkv_seq_append_tokens(self._h, int(seq_id), tok.ctypes.data if n else None,
                                         n, slots.ctypes.data, cows.ctypes.data,
                                         ctypes.byref(n_cow))
        if rc != PKV_OK:
            return rc, slots[:0], cows[:0]
        return rc, slots[:n], cows[:n_cow.value]

    def pkv_seq_share_prefix(self, seq_id, tokens):
        """Create seq_id on the longest cached prefix of tokens; returns (status,
        tokens covered)."""
        import numpy as np
        tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1)
        got = ctypes.c_int(0)
        rc = lib().pkv_seq_share_prefix(self._h, int(seq_id),
                                        tok.ctypes.data if tok.shape[0] else None,
                                        tok.shape[0], ctypes.byref(got))
        return rc, got.value

    def pkv_prefix_cache_stats(self):
        """Returns (cached blocks, evictable blocks, queried tokens, hit tokens)."""
        c, e = ctypes.c_int(), ctypes.c_int()
        q, h = ctypes.c_int64(), ctypes.c_int64()
        _check(lib().pkv_prefix_cache_stats(self._h, ctypes.byref(c), ctypes.byref(e),
                                            ctypes.byref(q), ctypes.byref(h)),
               "pkv_prefix_cache_stats")
        return c.value, e.value, q.value, h.value

    def pkv_seq_fork(self, parent, child):
        return lib().pkv_seq_fork(self._h, int(parent), int(child))

    def pkv_seq_free(self, seq_id):
        return lib().pkv_seq_free(self._h, int(seq_id))

    def pkv_seq_fork_batch(self, parents, children):
        """Returns (status, forks done)."""
        import numpy as np
        pa = np.ascontiguousarray(parents, dtype=np.int64)
        ch = np.ascontiguousarray(children, dtype=np.int64)
        if pa.shape != ch.shape:
            raise ValueError("parents and children differ in length")
        done = ctypes.c_int(0)
        rc = lib().pkv_seq_fork_batch(self._h, pa.ctypes.data, ch.ctypes.data, pa.shape[0],
                                      ctypes.byref(done))
        return rc, done.value

    def pkv_seq_free_batch(self, seq_ids):
        """Returns (status, frees done)."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        done = ctypes.c_int(0)
        rc = lib().pkv_seq_free_batch(self._h, ids.ctypes.data, ids.shape[0], ctypes.byref(done))
        return rc, done.value

    def pkv_block_tables(self, seq_ids):
        """Returns (status, tables int32 [n, MB], lens int32 [n])."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.shape[0]
        tables = np.zeros((n, self.max_blocks_per_seq), dtype=np.int32)
        lens = np.zeros(n, dtype=np.int32)
        rc = lib().pkv_block_tables(self._h, ids.ctypes.data, n, tables.ctypes.data,
                                    lens.ctypes.data)
        return rc, tables, lens

    def pkv_stats(self):
        """Returns (free, held, logical_tokens, utilisation)."""
        f, h = ctypes.c_int(), ctypes.c_int()
        t, u = ctypes.c_int64(), ctypes.c_double()
        _check(lib().pkv_stats(self._h, ctypes.byref(f), ctypes.byref(h), ctypes.byref(t),
                               ctypes.byref(u)), "pkv_stats")
        return f.value, h.value, t.value, u.value
