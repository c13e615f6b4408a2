"""Python binding of libkvq (quantized-KV decode attention for B200).

Argument marshalling only: every entry point forwards to the C ABI declared in
``include/kvq.h`` under the same name, passing raw device pointers and a CUDA
stream handle.  All work runs in the library's CUDA kernels; there is no
Python or CPU implementation behind these functions.  Importing fails loudly
when the compiled library is missing.

Pointers may be given as ``torch.Tensor`` (its ``data_ptr()``), as ``None``
(NULL) or as a plain integer address; streams as ``torch.cuda.Stream``, an
integer handle, or ``None`` for the current torch stream.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libkvq.so not found at {LIB_PATH}; build it with "
        "`python decode_attention_q8_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

KVQ_F16, KVQ_Q8_0, KVQ_Q4_0, KVQ_TURBO3, KVQ_TURBO2, KVQ_TURBO4, KVQ_Q5_0, KVQ_TURBO3_QJL = 0, 1, 2, 3, 4, 5, 6, 7
TYPES = {"f16": KVQ_F16, "q8_0": KVQ_Q8_0, "q4_0": KVQ_Q4_0, "turbo3": KVQ_TURBO3, "turbo2": KVQ_TURBO2,
         "turbo4": KVQ_TURBO4, "q5_0": KVQ_Q5_0, "turbo3_qjl": KVQ_TURBO3_QJL}

KVQ_OK, KVQ_ERR_INVALID, KVQ_ERR_UNSUPPORTED, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA = 0, 1, 2, 3, 4

EXPORTED = (
    "kvq_status_string", "kvq_last_cuda_error", "kvq_row_bytes", "kvq_check_desc",
    "kvq_cache_layout", "kvq_cache_bytes", "kvq_auto_splits", "kvq_workspace_bytes",
    "kvq_turbo3_codebook", "kvq_turbo_codebook", "kvq_turbo3_signs", "kvq_append_quantize",
    "kvq_decode_attention", "kvq_combine", "kvq_decode_attention_noalloc", "kvq_decode_step",
    "kvq_decode_attention_varlen", "kvq_decode_step_varlen", "kvq_append_quantize_varlen",
    "kvq_paged_layout", "kvq_paged_cache_bytes", "kvq_append_quantize_paged", "kvq_decode_attention_paged",
    "kvq_decode_step_paged", "kvq_partials_region", "kvq_combine_ranks", "kvq_workspace_status_offset",
)


class kvq_cache_desc(ctypes.Structure):
    _fields_ = [
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("k_type", ctypes.c_int32),
        ("v_type", ctypes.c_int32),
        ("flags", ctypes.c_int32),
        ("max_ctx", ctypes.c_int64),
        ("turbo_seed", ctypes.c_uint64),
        ("qjl_proj", ctypes.c_void_p),
    ]


class kvq_plane_layout(ctypes.Structure):
    _fields_ = [
        ("rows_per_plane", ctypes.c_int64),
        ("code_bytes", ctypes.c_int64),
        ("n_scales", ctypes.c_int64),
        ("scale_offset", ctypes.c_int64),
        ("total_bytes", ctypes.c_int64),
    ]


class kvq_paged(ctypes.Structure):
    _fields_ = [
        ("block_table", ctypes.c_void_p),
        ("max_pages", ctypes.c_int32),
        ("page_rows", ctypes.c_int32),
        ("n_pages", ctypes.c_int64),
    ]


_P = ctypes.c_void_p
_D = ctypes.POINTER(kvq_cache_desc)
_PG = ctypes.POINTER(kvq_paged)
_sigs = {
    "kvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kvq_last_cuda_error": (ctypes.c_char_p, []),
    "kvq_row_bytes": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int32]),
    "kvq_check_desc": (ctypes.c_int, [_D]),
    "kvq_cache_layout": (ctypes.c_int, [_D, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(kvq_plane_layout)]),
    "kvq_cache_bytes": (ctypes.c_size_t, [_D, ctypes.c_int32, ctypes.c_int32]),
    "kvq_auto_splits": (ctypes.c_int32, [_D, ctypes.c_int32, ctypes.c_int64]),
    "kvq_workspace_bytes": (ctypes.c_size_t, [_D, ctypes.c_int32, ctypes.c_int32]),
    "kvq_turbo3_codebook": (ctypes.c_int, [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]),
    "kvq_turbo3_signs": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int32, ctypes.POINTER(ctypes.c_float)]),
    "kvq_turbo_codebook": (ctypes.c_int, [ctypes.c_int32, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]),
    "kvq_append_quantize": (ctypes.c_int, [_D, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_int64,
                                           ctypes.c_int32, _P]),
    "kvq_decode_attention": (ctypes.c_int, [_D, _P, _P, _P, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                            ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "kvq_combine": (ctypes.c_int, [_D, _P, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                   _P, _P]),
    "kvq_decode_attention_noalloc": (ctypes.c_int, [_D, _P, _P, _P, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                                    ctypes.c_int32, _P, _P]),
    "kvq_decode_step": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                       ctypes.c_int32, _P, ctypes.c_size_t, _P, _P]),
    "kvq_decode_attention_varlen": (ctypes.c_int, [_D, _P, _P, _P, ctypes.c_int32, _P, ctypes.c_int64,
                                                   ctypes.c_float, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "kvq_decode_step_varlen": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, ctypes.c_int32, _P, ctypes.c_int64,
                                              ctypes.c_float, ctypes.c_int32, _P, ctypes.c_size_t, _P, _P]),
    "kvq_append_quantize_varlen": (ctypes.c_int, [_D, _P, _P, _P, _P, ctypes.c_int32, _P, ctypes.c_int32, _P]),
    "kvq_paged_layout": (ctypes.c_int, [_D, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                        ctypes.POINTER(kvq_plane_layout)]),
    "kvq_paged_cache_bytes": (ctypes.c_size_t, [_D, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32]),
    "kvq_append_quantize_paged": (ctypes.c_int, [_D, _P, _P, _P, _P, ctypes.c_int32, _PG, _P, ctypes.c_int32,
                                                 _P]),
    "kvq_decode_attention_paged": (ctypes.c_int, [_D, _P, _P, _P, ctypes.c_int32, _PG, _P, ctypes.c_int64,
                                                  ctypes.c_float, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "kvq_decode_step_paged": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, ctypes.c_int32, _PG, _P, ctypes.c_int64,
                                             ctypes.c_float, ctypes.c_int32, _P, ctypes.c_size_t, _P, _P]),
    "kvq_partials_region": (ctypes.c_int, [_D, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t),
                                           ctypes.POINTER(ctypes.c_size_t)]),
    "kvq_combine_ranks": (ctypes.c_int, [_D, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P, _P]),
    "kvq_workspace_status_offset": (ctypes.c_int, [_D, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]),
}
for _name, (_res, _args) in _sigs.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class KvqError(RuntimeError):
    def __init__(self, status, where):
        msg = _lib.kvq_status_string(status).decode()
        if status == KVQ_ERR_CUDA:
            msg += ": " + _lib.kvq_last_cuda_error().decode()
        super().__init__(f"{where}: {msg}")
        self.status = status


def _check(status, where):
    if status != KVQ_OK:
        raise KvqError(status, where)
    return status


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _type(t):
    return TYPES[t] if isinstance(t, str) else int(t)


KVQ_FLAG_OVERLAP_PREVIOUS = 1


def make_desc(n_q_heads, n_kv_heads, head_dim, k_type, v_type, max_ctx, turbo_seed=0, qjl_proj=None, flags=0):
    """A kvq_cache_desc.  qjl_proj: the turbo3_qjl projection (device fp32
    [head_dim][head_dim]); the descriptor keeps a reference to it.  flags:
    KVQ_FLAG_* bits (see include/kvq.h)."""
    d = kvq_cache_desc(n_q_heads, n_kv_heads, head_dim, _type(k_type), _type(v_type), flags,
                       max_ctx, turbo_seed, _ptr(qjl_proj))
    d.qjl_tensor = qjl_proj
    return d


# ----------------------------------------------------------------- queries

def kvq_status_string(status):
    return _lib.kvq_status_string(status).decode()


def kvq_row_bytes(type_, head_dim):
    return _lib.kvq_row_bytes(_type(type_), head_dim)


def kvq_check_desc(desc):
    return _lib.kvq_check_desc(ctypes.byref(desc))


def kvq_cache_layout(desc, batch, which):
    out = kvq_plane_layout()
    _check(_lib.kvq_cache_layout(ctypes.byref(desc), batch, which, ctypes.byref(out)), "kvq_cache_layout")
    return out


def kvq_cache_bytes(desc, batch, which):
    return _lib.kvq_cache_bytes(ctypes.byref(desc), batch, which)


def kvq_auto_splits(desc, batch, ctx_len):
    return _lib.kvq_auto_splits(ctypes.byref(desc), batch, ctx_len)


def kvq_workspace_bytes(desc, batch, n_splits=0):
    return _lib.kvq_workspace_bytes(ctypes.byref(desc), batch, n_splits)


def kvq_workspace_status_offset(desc, batch):
    """Byte offset of the workspace's status word (bits: 1 a tile wait gave up,
    2 a combine wait gave up, 4 a block-table entry outside the pool)."""
    off = ctypes.c_size_t()
    _check(_lib.kvq_workspace_status_offset(ctypes.byref(desc), batch, ctypes.byref(off)),
           "kvq_workspace_status_offset")
    return off.value


STATUS_TILE_WAIT, STATUS_COMBINE_WAIT, STATUS_BAD_PAGE = 1, 2, 4


def kvq_turbo3_codebook():
    lv = (ctypes.c_float * 8)()
    th = (ctypes.c_float * 7)()
    _check(_lib.kvq_turbo3_codebook(lv, th), "kvq_turbo3_codebook")
    return list(lv), list(th)


def kvq_turbo_codebook(type_):
    """(levels[2^b], thresholds[2^b - 1]) of a turbo type ("turbo2", "turbo3", "turbo4";
    "turbo3_qjl": the 4-level codebook of its 2-bit codes)."""
    t = _type(type_)
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 15)()
    _check(_lib.kvq_turbo_codebook(t, lv, th), "kvq_turbo_codebook")
    n = {KVQ_TURBO2: 4, KVQ_TURBO3: 8, KVQ_TURBO4: 16, KVQ_TURBO3_QJL: 4}[t]
    return list(lv)[:n], list(th)[:n - 1]


def kvq_turbo3_signs(seed, head_dim):
    out = (ctypes.c_float * head_dim)()
    _check(_lib.kvq_turbo3_signs(seed, head_dim, out), "kvq_turbo3_signs")
    return list(out)


# ----------------------------------------------------------------- kernels

def kvq_append_quantize(desc, k_cache, v_cache, k_new, v_new, batch, pos, n_tok, stream=None):
    return _check(_lib.kvq_append_quantize(ctypes.byref(desc), _ptr(k_cache), _ptr(v_cache), _ptr(k_new),
                                           _ptr(v_new), batch, pos, n_tok, _stream(stream)),
                  "kvq_append_quantize")


def kvq_decode_attention(desc, k_cache, v_cache, q, batch, ctx_len, softmax_scale, n_splits, workspace,
                         workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return _check(_lib.kvq_decode_attention(ctypes.byref(desc), _ptr(k_cache), _ptr(v_cache), _ptr(q), batch,
                                            ctx_len, softmax_scale, n_splits, _ptr(workspace), workspace_bytes,
                                            _stream(stream)),
                  "kvq_decode_attention")


def kvq_combine(desc, workspace, batch, ctx_len, n_splits, out, workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return _check(_lib.kvq_combine(ctypes.byref(desc), _ptr(workspace), workspace_bytes, batch, ctx_len,
                                   n_splits, _ptr(out), _stream(stream)),
                  "kvq_combine")


def kvq_decode_attention_noalloc(desc, k_cache, v_cache, q, batch, ctx_len, softmax_scale, n_splits, out,
                                 stream=None):
    """Decode + combine into ``out`` using the library's own 8 MiB per-GPU
    scratch array instead of a caller workspace (see include/kvq.h)."""
    return _check(_lib.kvq_decode_attention_noalloc(ctypes.byref(desc), _ptr(k_cache), _ptr(v_cache), _ptr(q),
                                                    batch, ctx_len, softmax_scale, n_splits, _ptr(out),
                                                    _stream(stream)),
                  "kvq_decode_attention_noalloc")


def kvq_decode_step(desc, k_cache, v_cache, q, k_new, v_new, batch, ctx_len, softmax_scale, n_splits, workspace,
                    out, workspace_bytes=None, stream=None):
    """Append one row per batch entry at row ctx_len - 1, decode over rows
    0 .. ctx_len-1 and combine into ``out``, in one launch (see include/kvq.h;
    the workspace's counter words must be zero before its first use)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return _check(_lib.kvq_decode_step(ctypes.byref(desc), _ptr(k_cache), _ptr(v_cache), _ptr(q), _ptr(k_new),
                                       _ptr(v_new), batch, ctx_len, softmax_scale, n_splits, _ptr(workspace),
                                       workspace_bytes, _ptr(out), _stream(stream)),
                  "kvq_decode_step")


def kvq_append_quantize_varlen(desc, k_cache, v_cache, k_new, v_new, batch, lens, n_tok, stream=None):
    """Append n_tok rows per batch entry at rows lens[b] - n_tok .. lens[b] - 1
    (``lens``: device int32 [batch], each sequence's length after the append)."""
    return _check(_lib.kvq_append_quantize_varlen(ctypes.byref(desc), _ptr(k_cache), _ptr(v_cache), _ptr(k_new),
                                                  _ptr(v_new), batch, _ptr(lens), n_tok, _stream(stream)),
                  "kvq_append_quantize_varlen")


def kvq_decode_attention_varlen(desc, k_cache, v_cache, q, batch, ctx_lens, max_ctx_len, softmax_scale, n_splits,
                                workspace, workspace_bytes=None, stream=None):
    """Split-KV decode where batch row b attends rows 0 .. ctx_lens[b]-1
    (``ctx_lens``: device int32 [batch]; ``max_ctx_len`` bounds them)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return _check(_lib.kvq_decode_attention_varlen(ctypes.byref(desc), _ptr(k_cache), _ptr(v_cache), _ptr(q), batch,
                                                   _ptr(ctx_lens), max_ctx_len, softmax_scale, n_splits,
                                                   _ptr(workspace), workspace_bytes, _stream(stream)),
                  "kvq_decode_attention_varlen")


def kvq_decode_step_varlen(desc, k_cache, v_cache, q, k_new, v_new, batch, ctx_lens, max_ctx_len, softmax_scale,
                           n_splits, workspace, out, workspace_bytes=None, stream=None):
    """kvq_decode_step with per-sequence lengths: row b's new K/V row lands at
    ctx_lens[b] - 1 and rows 0 .. ctx_lens[b]-1 are attended."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return _check(_lib.kvq_decode_step_varlen(ctypes.byref(desc), _ptr(k_cache), _ptr(v_cache), _ptr(q),
                                              _ptr(k_new), _ptr(v_new), batch, _ptr(ctx_lens), max_ctx_len,
                                              softmax_scale, n_splits, _ptr(workspace), workspace_bytes, _ptr(out),
                                              _stream(stream)),
                  "kvq_decode_step_varlen")


def make_paged(block_table, page_rows, n_pages):
    """kvq_paged for a device int32 block table [batch][max_pages] (the caller
    keeps the tensor alive while the description is in use)."""
    assert block_table.dtype.itemsize == 4 and block_table.dim() == 2 and block_table.is_contiguous()
    return kvq_paged(block_table.data_ptr(), block_table.shape[1], page_rows, n_pages)


def kvq_paged_layout(desc, page_rows, n_pages, which):
    out = kvq_plane_layout()
    _check(_lib.kvq_paged_layout(ctypes.byref(desc), page_rows, n_pages, which, ctypes.byref(out)),
           "kvq_paged_layout")
    return out


def kvq_paged_cache_bytes(desc, page_rows, n_pages, which):
    return _lib.kvq_paged_cache_bytes(ctypes.byref(desc), page_rows, n_pages, which)


def kvq_append_quantize_paged(desc, k_pool, v_pool, k_new, v_new, batch, pages, lens, n_tok, stream=None):
    """Append n_tok rows per sequence at logical rows lens[b] - n_tok .. lens[b] - 1
    of a paged pool (``pages``: kvq_paged)."""
    return _check(_lib.kvq_append_quantize_paged(ctypes.byref(desc), _ptr(k_pool), _ptr(v_pool), _ptr(k_new),
                                                 _ptr(v_new), batch, ctypes.byref(pages), _ptr(lens), n_tok,
                                                 _stream(stream)),
                  "kvq_append_quantize_paged")


def kvq_decode_attention_paged(desc, k_pool, v_pool, q, batch, pages, ctx_lens, max_ctx_len, softmax_scale,
                               n_splits, workspace, workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return _check(_lib.kvq_decode_attention_paged(ctypes.byref(desc), _ptr(k_pool), _ptr(v_pool), _ptr(q), batch,
                                                  ctypes.byref(pages), _ptr(ctx_lens), max_ctx_len, softmax_scale,
                                                  n_splits, _ptr(workspace), workspace_bytes, _stream(stream)),
                  "kvq_decode_attention_paged")


def kvq_decode_step_paged(desc, k_pool, v_pool, q, k_new, v_new, batch, pages, ctx_lens, max_ctx_len, softmax_scale,
                          n_splits, workspace, out, workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return _check(_lib.kvq_decode_step_paged(ctypes.byref(desc), _ptr(k_pool), _ptr(v_pool), _ptr(q), _ptr(k_new),
                                             _ptr(v_new), batch, ctypes.byref(pages), _ptr(ctx_lens), max_ctx_len,
                                             softmax_scale, n_splits, _ptr(workspace), workspace_bytes, _ptr(out),
                                             _stream(stream)),
                  "kvq_decode_step_paged")


def kvq_partials_region(desc, batch, n_splits):
    """(byte offset, bytes) of the split partials inside a workspace."""
    off, n = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.kvq_partials_region(ctypes.byref(desc), batch, n_splits, ctypes.byref(off), ctypes.byref(n)),
           "kvq_partials_region")
    return off.value, n.value


def kvq_combine_ranks(desc, partials, n_ranks, batch, n_splits, out, stream=None):
    """Merge n_ranks ranks' gathered partial regions (rank after rank) into ``out``."""
    return _check(_lib.kvq_combine_ranks(ctypes.byref(desc), _ptr(partials), n_ranks, batch, n_splits, _ptr(out),
                                         _stream(stream)),
                  "kvq_combine_ranks")


def gather_partials(region, group=None):
    """All-gather every rank's partial region (a 1-D uint8 tensor) into one
    buffer, rank after rank: the exchange step of a context split across GPUs."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty(world * region.numel(), dtype=region.dtype, device=region.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, region, group=group)
    else:
        dist.all_gather(list(out.chunk(world)), region, group=group)
    return out


def decode_context_parallel(desc, k_cache, v_cache, q, batch, ctx_len, softmax_scale, n_splits, workspace, out,
                            group=None):
    """Context split across GPUs: this rank decodes its own ctx_len rows
    (kvq_decode_attention), the ranks' partials are all-gathered, and every
    rank combines all of them into ``out`` (kvq_combine_ranks).  Everything
    runs on torch's current stream, which the collective also orders on."""
    import torch.distributed as dist
    kvq_decode_attention(desc, k_cache, v_cache, q, batch, ctx_len, softmax_scale, n_splits, workspace)
    off, n = kvq_partials_region(desc, batch, n_splits)
    gathered = gather_partials(workspace[off:off + n], group)
    return kvq_combine_ranks(desc, gathered, dist.get_world_size(group), batch, n_splits, out)


def raw_status(name, *args):
    """Calls a C entry point with already-marshalled arguments and returns its
    raw status (for tests of the error paths)."""
    return getattr(_lib, name)(*args)
