"""Python face of the CPU oracle (ctypes over liboracle_qsa.so).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The CUDA library never imports this.

``query_forward`` runs the method's steps in order for one query (pool, score,
select, attended tokens, attention), each step a call into the C oracle.
Inputs come from ``qsa_synth`` (the shared seeded generator), never from the GPU.
"""

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_qsa.so")

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")


def build(force=False):
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "qsa_oracle.h"))):
        return _LIB
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-fno-fast-math", "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.qo_bf16_value.argtypes = [ctypes.c_uint16]
        L.qo_bf16_value.restype = ctypes.c_double
        L.qo_round_bf16.argtypes = [ctypes.c_double]
        L.qo_round_bf16.restype = ctypes.c_uint16
        L.qo_pool_blocks.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _u16p]
        L.qo_pool_blocks.restype = None
        L.qo_block_scores.argtypes = [_u16p, _f32p, _u16p, ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_int32, _f64p]
        L.qo_block_scores.restype = None
        L.qo_select_top_blocks.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int32, _i32p]
        L.qo_select_top_blocks.restype = ctypes.c_int32
        L.qo_attended_tokens.argtypes = [_i32p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, _i64p]
        L.qo_attended_tokens.restype = ctypes.c_int64
        L.qo_attended_tokens_shared.argtypes = [_i32p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int64,
                                                ctypes.c_int32, _i64p]
        L.qo_attended_tokens_shared.restype = ctypes.c_int64
        L.qo_gqa_attention.argtypes = [_u16p, _u16p, _u16p, ctypes.c_int64, ctypes.c_int32,
                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_double, _f64p]
        L.qo_gqa_attention.restype = None
        _lib = L
    return _lib


# ---------------------------------------------------------------- step wrappers

def bf16_value(bits):
    return lib().qo_bf16_value(int(bits))


def round_bf16(x):
    return lib().qo_round_bf16(float(x))


def pool_blocks(idx_k_bits, block_size=4):
    """Step 1: bf16 mean of every complete block of ``idx_k_bits`` [n_tok][idx_dim]."""
    idx_k_bits = np.ascontiguousarray(idx_k_bits, dtype=np.uint16)
    n_tok, idx_dim = idx_k_bits.shape
    n_blocks = n_tok // block_size
    out = np.zeros((n_blocks, idx_dim), dtype=np.uint16)
    if n_blocks:
        lib().qo_pool_blocks(idx_k_bits, n_blocks, idx_dim, block_size, out)
    return out


def block_scores(q_idx_bits, w, pooled_bits):
    """Step 2: scores of the candidate blocks ``pooled_bits`` [n_cand][idx_dim]."""
    q_idx_bits = np.ascontiguousarray(q_idx_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.float32)
    pooled_bits = np.ascontiguousarray(pooled_bits, dtype=np.uint16)
    n_heads, idx_dim = q_idx_bits.shape
    n_cand = pooled_bits.shape[0]
    out = np.zeros(max(n_cand, 1), dtype=np.float64)
    if n_cand:
        lib().qo_block_scores(q_idx_bits, w, pooled_bits if pooled_bits.size else
                              np.zeros(1, np.uint16), n_cand, n_heads, idx_dim, out)
    return out[:n_cand]


def select_top_blocks(scores, top_k=512):
    """Step 3: ascending list of the selected block indices."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    sel = np.zeros(max(top_k, 1), dtype=np.int32)
    cnt = lib().qo_select_top_blocks(scores if scores.size else np.zeros(1), scores.size, top_k, sel)
    if cnt < 0:
        raise MemoryError("oracle select: allocation failed")
    return sel[:cnt].copy()


def attended_tokens(sel, t, block_size=4):
    """Step 4: token positions the query attends (selected blocks + own partial block)."""
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    buf = np.zeros(sel.size * block_size + block_size, dtype=np.int64)
    n = lib().qo_attended_tokens(sel if sel.size else np.zeros(1, np.int32), sel.size, int(t),
                                 block_size, buf)
    return buf[:n].copy()


def attended_tokens_shared(sel, t_sel, t, block_size=4):
    """Step 4 for a draft query at ``t`` reusing the selection made at ``t_sel``:
    the selected blocks' tokens, then every token from the selection query's first
    incomplete block up to ``t``."""
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    tail = int(t) + 1 - ((int(t_sel) + 1) // block_size) * block_size
    buf = np.zeros(sel.size * block_size + max(tail, 0) + 1, dtype=np.int64)
    n = lib().qo_attended_tokens_shared(sel if sel.size else np.zeros(1, np.int32), sel.size, int(t_sel), int(t),
                                        block_size, buf)
    return buf[:n].copy()


def gqa_attention(q_bits, k_rows_bits, v_rows_bits, scale=None):
    """Step 5: fp64 attention output [n_q_heads][head_dim] over the given rows."""
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_rows_bits = np.ascontiguousarray(k_rows_bits, dtype=np.uint16)
    v_rows_bits = np.ascontiguousarray(v_rows_bits, dtype=np.uint16)
    n_q_heads, head_dim = q_bits.shape
    n_tok, n_kv_heads, _ = k_rows_bits.shape
    if scale is None:
        scale = 1.0 / np.sqrt(head_dim)
    out = np.zeros((n_q_heads, head_dim), dtype=np.float64)
    lib().qo_gqa_attention(q_bits, k_rows_bits, v_rows_bits, n_tok, n_q_heads, n_kv_heads,
                           head_dim, float(scale), out)
    return out


# ---------------------------------------------------------------- one query

def query_forward(pooled_seq_bits, q_idx_bits, w, t, q_bits, fetch_kv, top_k=512, block_size=4,
                  scale=None):
    """The whole layer for one query at position ``t``.

    ``pooled_seq_bits`` holds (at least) the sequence's complete blocks below
    the query; ``fetch_kv(tokens)`` returns (k_rows, v_rows) bf16 bits
    [len(tokens)][n_kv_heads][head_dim].  Returns (selected blocks, fp64 output).
    """
    n_c = (int(t) + 1) // block_size
    scores = block_scores(q_idx_bits, w, pooled_seq_bits[:n_c])
    sel = select_top_blocks(scores, top_k)
    tokens = attended_tokens(sel, t, block_size)
    k_rows, v_rows = fetch_kv(tokens)
    out = gqa_attention(q_bits, k_rows, v_rows, scale)
    return sel, out


# ---------------------------------------------------------------- workloads

class WorkloadOracle:
    """Expected outputs for queries of one ``qsa_synth.workloads.Workload``.

    Pooled blocks are recomputed from the generated indexer keys (the
    definition), once per sequence and cached.
    """

    def __init__(self, wl):
        import qsa_synth as syn
        self.wl = wl
        self.syn = syn
        self._pooled = {}

    def pooled(self, seq, n_blocks):
        have = self._pooled.get(seq)
        if have is None or have.shape[0] < n_blocks:
            idx_k = self.syn.gen_idx_k(self.wl.seed, seq, 0, n_blocks * self.wl.block_size,
                                       self.wl.idx_dim)
            self._pooled[seq] = pool_blocks(idx_k, self.wl.block_size)
        return self._pooled[seq][:n_blocks]

    def query(self, step, qi):
        wl, syn = self.wl, self.syn
        st = wl.steps[step]
        s, t, qid = st.q_seq[qi], st.q_pos[qi], st.query_ids[qi]
        n_c = (t + 1) // wl.block_size
        pooled = self.pooled(s, n_c)
        q_idx = syn.gen_q_idx(wl.seed, [qid], wl.n_idx_heads, wl.idx_dim)[0]
        w = syn.gen_w(wl.seed, [qid], wl.n_idx_heads)[0]
        q = syn.gen_q(wl.seed, [qid], wl.n_q_heads, wl.head_dim)[0]

        def fetch(tokens):
            k = syn.gen_kv_rows(wl.seed, "k", s, tokens, wl.n_kv_heads, wl.head_dim)
            v = syn.gen_kv_rows(wl.seed, "v", s, tokens, wl.n_kv_heads, wl.head_dim)
            return k, v

        return query_forward(pooled, q_idx, w, t, q, fetch, wl.top_k, wl.block_size)
