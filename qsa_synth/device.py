"""Device-side synthetic inputs: fills torch CUDA tensors with the same values the
host generator (gen.py) produces, via the small CUDA library built from gen_cuda.cu.

``DeviceWorkload`` allocates the caches of a ``workloads.Workload`` in HBM, fills
every position of them, and hands out per-step query tensors.  Input setup only.
"""

import ctypes
import os
import subprocess

import numpy as np

from . import gen

HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(HERE, "gen_cuda.cu")
_LIB = os.path.join(HERE, "libqsa_synth.so")


def build(force=False):
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    subprocess.check_call([nvcc, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-Xcompiler", "-fPIC", "-shared", "-o", _LIB, _SRC])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB):
            raise ImportError(f"{_LIB} not built: run qsa_synth.device.build()")
        L = ctypes.CDLL(_LIB)
        P, I64, U64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int
        L.synth_fill_kv.argtypes = [P, I64, I64, I64, I64, U64, P]
        L.synth_fill_idxk.argtypes = [P, I64, I64, I64, U64, I, I, P]
        L.synth_fill_query.argtypes = [P, I64, I64, I64, I64, U64, I, I, I, P]
        L.synth_fill_weights.argtypes = [P, I64, I64, I64, U64, I, I, P]
        _lib = L
    return _lib


def _key(seed, tid):
    return int(gen.stream_key(seed, tid))


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _ok(rc):
    if rc != 0:
        raise RuntimeError(f"synthetic input fill failed: cuda error {rc}")


def fill_kv(t, seed, which):
    B, H, T, D = t.shape
    _ok(lib().synth_fill_kv(t.data_ptr(), B, H, T, D, _key(seed, gen.T_K if which == "k" else gen.T_V), _stream()))


def fill_idx_k(t, seed, lo=-4, hi=4):
    B, T, Di = t.shape
    _ok(lib().synth_fill_idxk(t.data_ptr(), B, T, Di, _key(seed, gen.T_IDXK), lo, hi, _stream()))


def fill_q(t, seed, qid0):
    n, H, D = t.shape
    _ok(lib().synth_fill_query(t.data_ptr(), n, H, D, qid0, _key(seed, gen.T_Q), 0, 0, 0, _stream()))


def fill_q_idx(t, seed, qid0, lo=-4, hi=4):
    n, H, D = t.shape
    _ok(lib().synth_fill_query(t.data_ptr(), n, H, D, qid0, _key(seed, gen.T_QIDX), 1, lo, hi, _stream()))


def fill_w(t, seed, qid0, lo=1, hi=3):
    n, H = t.shape
    _ok(lib().synth_fill_weights(t.data_ptr(), n, H, qid0, _key(seed, gen.T_W), lo, hi, _stream()))


class DeviceWorkload:
    """Caches and per-step inputs of one workload, resident in HBM.

    k_cache, v_cache: bf16 [B][Hkv][T][128]; idx_k: bf16 [B][T][64];
    pooled: bf16 [B][T/4][64] (zero until pooled).
    """

    def __init__(self, wl, device="cuda"):
        import torch
        self.wl = wl
        self.device = device
        B, H, T = wl.batch, wl.n_kv_heads, wl.kv_capacity
        self.k_cache = torch.empty((B, H, T, wl.head_dim), dtype=torch.bfloat16, device=device)
        self.v_cache = torch.empty_like(self.k_cache)
        self.idx_k = torch.empty((B, T, wl.idx_dim), dtype=torch.bfloat16, device=device)
        self.pooled = torch.zeros((B, T // wl.block_size, wl.idx_dim), dtype=torch.bfloat16, device=device)
        fill_kv(self.k_cache, wl.seed, "k")
        fill_kv(self.v_cache, wl.seed, "v")
        fill_idx_k(self.idx_k, wl.seed)

    def step_tensors(self, step):
        """Device tensors of step `step`: queries, indexer inputs and position arrays."""
        import torch
        wl, st = self.wl, self.wl.steps[step]
        n = len(st.q_pos)
        qid0 = st.query_ids[0]
        assert st.query_ids == list(range(qid0, qid0 + n)), "query ids of a step are consecutive"
        dev = self.device
        q = torch.empty((n, wl.n_q_heads, wl.head_dim), dtype=torch.bfloat16, device=dev)
        q_idx = torch.empty((n, wl.n_idx_heads, wl.idx_dim), dtype=torch.bfloat16, device=dev)
        w = torch.empty((n, wl.n_idx_heads), dtype=torch.float32, device=dev)
        fill_q(q, wl.seed, qid0)
        fill_q_idx(q_idx, wl.seed, qid0)
        fill_w(w, wl.seed, qid0)
        i32 = lambda v: torch.tensor(np.asarray(v, dtype=np.int32), device=dev)
        return dict(q=q, q_idx=q_idx, w=w, len_before=i32(st.len_before), len_after=i32(st.len_after),
                    q_seq=i32(st.q_seq), q_pos=i32(st.q_pos), n_q=n,
                    max_new_tokens=max(a - b for a, b in zip(st.len_after, st.len_before)),
                    max_blocks=max((p + 1) // wl.block_size for p in st.q_pos))
