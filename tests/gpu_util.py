"""Helpers of the GPU parity tests: run the CUDA library on a synthetic workload
and compare it with the CPU oracle."""

import numpy as np
import torch

import block_sparse_attention_key_b200 as qsa
from block_sparse_attention_key_b200 import build as qbuild
from qsa_synth import device as sdev
from qsa_synth import gen as sgen

# tolerance on bf16 attention outputs against the fp64 oracle
ATOL_MAX = 1e-2
REL_L2 = 5e-3


def ensure_built():
    qbuild.build()
    sdev.build()


def to_bits(t):
    """bf16 CUDA tensor -> numpy uint16 bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(t):
    return sgen.bf16_bits_to_f32(to_bits(t)).astype(np.float64)


def from_bits(bits, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def dims_of(wl):
    return qsa.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.kv_capacity, wl.head_dim, wl.n_idx_heads,
                         wl.idx_dim, wl.block_size, wl.top_k)


def new_workspace(nbytes):
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device="cuda")
    qsa.qsa_workspace_init(ws)
    return ws


def pool_history(dw, step):
    """Pool every block completed before the step (the state a previous call left)."""
    wl, st = dw.wl, dw.wl.steps[step]
    lb = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    la = torch.tensor(st.len_before, dtype=torch.int32, device="cuda")
    if max(st.len_before) > 0:
        qsa.qsa_pool_block_keys(dims_of(wl), dw.idx_k, dw.pooled, lb, la, max(st.len_before))


def run_forward(dw, step, mode=None, ws=None):
    """qsa_forward on one step; returns (out, sel_idx, sel_cnt, status flags)."""
    wl = dw.wl
    mode = (qsa.QSA_MODE_PREFILL if wl.mode == "prefill" else qsa.QSA_MODE_DECODE) if mode is None else mode
    T = dw.step_tensors(step)
    dims = dims_of(wl)
    need = qsa.qsa_workspace_bytes(dims, T["n_q"], T["max_blocks"], mode)
    assert need > 0
    if ws is None or ws.numel() < need:
        ws = new_workspace(need)
    out = torch.empty((T["n_q"], wl.n_q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    sel_idx = torch.empty((T["n_q"], qsa.QSA_SEL_CAP), dtype=torch.int32, device="cuda")
    sel_cnt = torch.empty((T["n_q"],), dtype=torch.int32, device="cuda")
    qsa.qsa_forward(dims, q=T["q"], k_cache=dw.k_cache, v_cache=dw.v_cache, idx_k=dw.idx_k, pooled=dw.pooled,
                    q_idx=T["q_idx"], w=T["w"], len_before=T["len_before"], len_after=T["len_after"],
                    q_seq=T["q_seq"], q_pos=T["q_pos"], n_q=T["n_q"], max_new_tokens=T["max_new_tokens"],
                    max_blocks=T["max_blocks"], mode=mode, out=out, workspace=ws, sel_idx=sel_idx,
                    sel_cnt=sel_cnt)
    flags = qsa.qsa_read_device_status(ws)
    return out, sel_idx, sel_cnt, flags


def check_selection_properties(wl, step, sel_idx, sel_cnt):
    """Properties every row must satisfy whatever the scores: count, range, order."""
    st = wl.steps[step]
    n_c = (np.asarray(st.q_pos, dtype=np.int64) + 1) // wl.block_size
    cnt = sel_cnt.cpu().numpy()
    idx = sel_idx.cpu().numpy()
    np.testing.assert_array_equal(cnt, np.minimum(n_c, wl.top_k))
    for r in range(idx.shape[0]):
        live, pad = idx[r, :cnt[r]], idx[r, cnt[r]:]
        assert (pad == -1).all(), f"row {r}: padding must be -1"
        assert (live >= 0).all() and (live < n_c[r]).all(), f"row {r}: block outside [0, n_c)"
        assert (np.diff(live) > 0).all(), f"row {r}: selected blocks must be strictly ascending"


def compare_outputs(got, want):
    """got: GPU bf16 output rows as float64; want: oracle fp64 rows."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.isfinite(got).all()
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err.max() <= ATOL_MAX, f"max abs error {err.max():.3e}"
    assert rel <= REL_L2, f"relative L2 error {rel:.3e}"
    return err.max(), rel
