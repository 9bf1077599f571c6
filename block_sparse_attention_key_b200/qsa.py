"""Thin ctypes binding of libqsa.so (the C ABI in include/qsa.h).

Argument marshalling only: every step runs in the CUDA library.  Tensors are
torch CUDA tensors (device memory and streams come from PyTorch); their
data_ptr() values and the current stream's handle are passed straight through.
There is no CPU fallback: if the library or a GPU is missing, calls raise.
"""

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqsa.so")

QSA_SEL_CAP = 512

QSA_OK = 0
QSA_ERR_INVALID_ARG = -1
QSA_ERR_WORKSPACE_TOO_SMALL = -2
QSA_ERR_UNSUPPORTED = -3
QSA_ERR_CUDA = -4

QSA_DEV_BAD_SEQ = 0x1
QSA_DEV_BAD_POS = 0x2
QSA_DEV_BLOCKS_OVER = 0x4
QSA_DEV_BAD_LEN = 0x8
QSA_DEV_BAD_SEL = 0x10
QSA_DEV_TOO_MANY_NEW = 0x20
QSA_DEV_TIMEOUT = 0x40
QSA_DEV_BAD_PAGE = 0x80

QSA_MODE_DECODE = 0
QSA_MODE_PREFILL = 1
QSA_MODE_MIXED = 2

EXPORTED = (
    "qsa_workspace_bytes", "qsa_workspace_init", "qsa_read_device_status", "qsa_status_string",
    "qsa_pool_block_keys", "qsa_index_scores", "qsa_topk_blocks", "qsa_sparse_attn", "qsa_forward",
    "qsa_sparse_attn_noalloc", "qsa_sparse_attn_ex", "qsa_select_blocks",
    "qsa_cp_workspace_bytes", "qsa_cp_select_keys", "qsa_cp_merge_keys", "qsa_cp_attn_partial", "qsa_cp_combine",
    "qsa_attn_plan",
)

CP_PART_ROW = 132  # floats per (query, head) partial of a context shard


class QsaError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn} failed: {msg} ({code})")
        self.code = code


class qsa_dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("n_idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32), ("top_k", ctypes.c_int32), ("kv_capacity", ctypes.c_int64),
        ("softmax_scale", ctypes.c_float),
    ]


class qsa_forward_args(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("idx_k", ctypes.c_void_p), ("pooled", ctypes.c_void_p), ("q_idx", ctypes.c_void_p),
        ("w", ctypes.c_void_p), ("len_before", ctypes.c_void_p), ("len_after", ctypes.c_void_p),
        ("q_seq", ctypes.c_void_p), ("q_pos", ctypes.c_void_p), ("n_q", ctypes.c_int32),
        ("max_new_tokens", ctypes.c_int32), ("max_blocks", ctypes.c_int64), ("mode", ctypes.c_int32),
        ("sel_idx", ctypes.c_void_p), ("sel_cnt", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("group_q", ctypes.c_int32), ("page_table", ctypes.c_void_p), ("page_tokens", ctypes.c_int32),
        ("n_pages", ctypes.c_int64), ("n_decode", ctypes.c_int32),
    ]


class qsa_attn_args(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("q_seq", ctypes.c_void_p), ("q_pos", ctypes.c_void_p), ("sel_idx", ctypes.c_void_p),
        ("sel_cnt", ctypes.c_void_p), ("n_q", ctypes.c_int32), ("group_q", ctypes.c_int32),
        ("page_table", ctypes.c_void_p), ("page_tokens", ctypes.c_int32), ("n_pages", ctypes.c_int64),
        ("out", ctypes.c_void_p),
    ]


class qsa_attn_plan_info(ctypes.Structure):
    _fields_ = [
        ("n_split", ctypes.c_int32), ("n_stages", ctypes.c_int32), ("threads", ctypes.c_int32),
        ("smem_bytes", ctypes.c_int32), ("ctas", ctypes.c_int64), ("cluster_merge", ctypes.c_int32),
        ("rows", ctypes.c_int32),
    ]


_lib = None


def load(path=LIB_PATH):
    """Load libqsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libqsa.so not built at {path}: run `python -m block_sparse_attention_key_b200.build`")
    L = ctypes.CDLL(path)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    D = ctypes.POINTER(qsa_dims)
    L.qsa_workspace_bytes.argtypes = [D, I32, I64, I32]
    L.qsa_workspace_bytes.restype = SZ
    L.qsa_workspace_init.argtypes = [P, SZ, P]
    L.qsa_read_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32), P]
    L.qsa_status_string.argtypes = [ctypes.c_int]
    L.qsa_status_string.restype = ctypes.c_char_p
    L.qsa_pool_block_keys.argtypes = [D, P, P, P, P, I32, P, P]
    L.qsa_index_scores.argtypes = [D, P, P, P, P, P, I32, I64, P, I64, P, P]
    L.qsa_topk_blocks.argtypes = [D, P, I64, P, I32, I64, P, P, P, SZ, P]
    L.qsa_sparse_attn.argtypes = [D, P, P, P, P, P, P, P, I32, P, P, SZ, P]
    L.qsa_forward.argtypes = [D, ctypes.POINTER(qsa_forward_args), P, SZ, P]
    L.qsa_sparse_attn_noalloc.argtypes = [D, P, P, P, P, P, P, P, I32, P, P]
    L.qsa_sparse_attn_ex.argtypes = [D, ctypes.POINTER(qsa_attn_args), P, SZ, P]
    L.qsa_select_blocks.argtypes = [D, P, P, P, P, P, I32, I64, I32, P, P, P, SZ, P]
    L.qsa_cp_workspace_bytes.argtypes = [D, I32]
    L.qsa_cp_workspace_bytes.restype = SZ
    L.qsa_cp_select_keys.argtypes = [D, P, P, P, P, P, I32, I64, P, P, P, SZ, P]
    L.qsa_cp_merge_keys.argtypes = [D, I32, P, P, I32, I64, P, P, P, P, P]
    L.qsa_cp_attn_partial.argtypes = [D, P, P, P, P, P, I32, I64, P, P, P, P, SZ, P]
    L.qsa_cp_combine.argtypes = [D, I32, P, I32, P, P]
    L.qsa_attn_plan.argtypes = [D, I32, I32, ctypes.POINTER(qsa_attn_plan_info)]
    for name in EXPORTED:
        if name not in ("qsa_workspace_bytes", "qsa_status_string", "qsa_cp_workspace_bytes"):
            getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def make_dims(batch, n_q_heads, n_kv_heads, kv_capacity, head_dim=128, n_idx_heads=4, idx_dim=64,
              block_size=4, top_k=512, softmax_scale=0.0):
    return qsa_dims(batch, n_q_heads, n_kv_heads, head_dim, n_idx_heads, idx_dim, block_size, top_k,
                    kv_capacity, softmax_scale)


def status_string(code):
    return load().qsa_status_string(code).decode()


def _check(fn, rc):
    if rc != QSA_OK:
        raise QsaError(fn, rc, status_string(rc))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libqsa takes CUDA tensors only (no CPU path)")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


# ---------------------------------------------------------------- entry points (same names as the C ABI)

def qsa_workspace_bytes(dims, n_q, max_blocks, mode):
    return int(load().qsa_workspace_bytes(ctypes.byref(dims), n_q, max_blocks, mode))


def qsa_workspace_init(workspace, stream=None):
    _check("qsa_workspace_init", load().qsa_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                                           _stream(stream)))


def qsa_read_device_status(workspace, stream=None):
    flags = ctypes.c_uint32(0)
    _check("qsa_read_device_status", load().qsa_read_device_status(_ptr(workspace), ctypes.byref(flags),
                                                                   _stream(stream)))
    return flags.value


def qsa_pool_block_keys(dims, idx_k, pooled, len_before, len_after, max_new_tokens, workspace=None, stream=None):
    _check("qsa_pool_block_keys", load().qsa_pool_block_keys(
        ctypes.byref(dims), _ptr(idx_k), _ptr(pooled), _ptr(len_before), _ptr(len_after), max_new_tokens,
        _ptr(workspace), _stream(stream)))


def qsa_index_scores(dims, q_idx, w, pooled, q_seq, q_pos, n_q, max_blocks, scores, ld_scores,
                     workspace=None, stream=None):
    _check("qsa_index_scores", load().qsa_index_scores(
        ctypes.byref(dims), _ptr(q_idx), _ptr(w), _ptr(pooled), _ptr(q_seq), _ptr(q_pos), n_q, max_blocks,
        _ptr(scores), ld_scores, _ptr(workspace), _stream(stream)))


def qsa_topk_blocks(dims, scores, ld_scores, q_pos, n_q, max_blocks, sel_idx, sel_cnt, workspace, stream=None):
    _check("qsa_topk_blocks", load().qsa_topk_blocks(
        ctypes.byref(dims), _ptr(scores), ld_scores, _ptr(q_pos), n_q, max_blocks, _ptr(sel_idx), _ptr(sel_cnt),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def qsa_select_blocks(dims, q_idx, w, pooled, q_seq, q_pos, n_q, max_blocks, mode, sel_idx, sel_cnt, workspace,
                      stream=None):
    _check("qsa_select_blocks", load().qsa_select_blocks(
        ctypes.byref(dims), _ptr(q_idx), _ptr(w), _ptr(pooled), _ptr(q_seq), _ptr(q_pos), n_q, max_blocks, mode,
        _ptr(sel_idx), _ptr(sel_cnt), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def qsa_sparse_attn(dims, q, k_cache, v_cache, q_seq, q_pos, sel_idx, sel_cnt, n_q, out, workspace, stream=None):
    _check("qsa_sparse_attn", load().qsa_sparse_attn(
        ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(q_seq), _ptr(q_pos), _ptr(sel_idx),
        _ptr(sel_cnt), n_q, _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def qsa_sparse_attn_noalloc(dims, q, k_cache, v_cache, q_seq, q_pos, sel_idx, sel_cnt, n_q, out, stream=None):
    """qsa_sparse_attn for callers that cannot allocate: scratch comes from a fixed
    16 MiB array inside the library (see include/qsa.h)."""
    _check("qsa_sparse_attn_noalloc", load().qsa_sparse_attn_noalloc(
        ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(q_seq), _ptr(q_pos), _ptr(sel_idx),
        _ptr(sel_cnt), n_q, _ptr(out), _stream(stream)))


def qsa_sparse_attn_ex(dims, *, q, k_cache, v_cache, q_seq, q_pos, sel_idx, sel_cnt, n_q, out, workspace,
                       group_q=1, page_table=None, page_tokens=0, n_pages=0, stream=None):
    args = qsa_attn_args(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(q_seq), _ptr(q_pos), _ptr(sel_idx),
                         _ptr(sel_cnt), n_q, group_q, _ptr(page_table), page_tokens, n_pages, _ptr(out))
    _check("qsa_sparse_attn_ex", load().qsa_sparse_attn_ex(ctypes.byref(dims), ctypes.byref(args), _ptr(workspace),
                                                           workspace.numel() * workspace.element_size(),
                                                           _stream(stream)))


def qsa_attn_plan(dims, n_q, group_q=1):
    """The attention launch for n_q queries in groups of group_q (host arithmetic only):
    a dict of splits, stages, threads, shared memory, CTAs, cluster merge and rows."""
    info = qsa_attn_plan_info()
    _check("qsa_attn_plan", load().qsa_attn_plan(ctypes.byref(dims), n_q, group_q, ctypes.byref(info)))
    return {name: getattr(info, name) for name, _ in qsa_attn_plan_info._fields_}


def qsa_forward(dims, *, q, k_cache, v_cache, idx_k, pooled, q_idx, w, len_before, len_after, q_seq, q_pos,
                n_q, max_new_tokens, max_blocks, mode, out, workspace, sel_idx=None, sel_cnt=None, group_q=0,
                page_table=None, page_tokens=0, n_pages=0, n_decode=0, stream=None):
    args = qsa_forward_args(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx_k), _ptr(pooled), _ptr(q_idx),
                            _ptr(w), _ptr(len_before), _ptr(len_after), _ptr(q_seq), _ptr(q_pos), n_q,
                            max_new_tokens, max_blocks, mode, _ptr(sel_idx), _ptr(sel_cnt), _ptr(out), group_q,
                            _ptr(page_table), page_tokens, n_pages, n_decode)
    _check("qsa_forward", load().qsa_forward(ctypes.byref(dims), ctypes.byref(args), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(), _stream(stream)))


# ---------------------------------------------------------------- context parallelism (see include/qsa.h)

def qsa_cp_workspace_bytes(shard_dims, n_q):
    return int(load().qsa_cp_workspace_bytes(ctypes.byref(shard_dims), n_q))


def qsa_cp_select_keys(shard_dims, q_idx, w, pooled_shard, q_seq, q_pos, n_q, blk_lo, keys, key_cnt, workspace,
                       stream=None):
    _check("qsa_cp_select_keys", load().qsa_cp_select_keys(
        ctypes.byref(shard_dims), _ptr(q_idx), _ptr(w), _ptr(pooled_shard), _ptr(q_seq), _ptr(q_pos), n_q, blk_lo,
        _ptr(keys), _ptr(key_cnt), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def qsa_cp_merge_keys(shard_dims, n_ranks, keys_all, cnt_all, n_q, blk_lo, sel_local, cnt_local, sel_global=None,
                      cnt_global=None, stream=None):
    _check("qsa_cp_merge_keys", load().qsa_cp_merge_keys(
        ctypes.byref(shard_dims), n_ranks, _ptr(keys_all), _ptr(cnt_all), n_q, blk_lo, _ptr(sel_local),
        _ptr(cnt_local), _ptr(sel_global), _ptr(cnt_global), _stream(stream)))


def qsa_cp_attn_partial(shard_dims, q, k_shard, v_shard, q_seq, q_pos, n_q, blk_lo, sel_local, cnt_local, part,
                        workspace, stream=None):
    _check("qsa_cp_attn_partial", load().qsa_cp_attn_partial(
        ctypes.byref(shard_dims), _ptr(q), _ptr(k_shard), _ptr(v_shard), _ptr(q_seq), _ptr(q_pos), n_q, blk_lo,
        _ptr(sel_local), _ptr(cnt_local), _ptr(part), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def qsa_cp_combine(dims, n_ranks, parts_all, n_q, out, stream=None):
    _check("qsa_cp_combine", load().qsa_cp_combine(ctypes.byref(dims), n_ranks, _ptr(parts_all), n_q, _ptr(out),
                                                   _stream(stream)))
