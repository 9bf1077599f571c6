"""The allocation-free attention entry point (qsa_sparse_attn_noalloc).

It serves callers that cannot allocate device memory (an engine whose allocator
already gave all of HBM to its KV cache, a frozen CUDA-graph memory plan, a C host
that only owns the tensors it passes) and so cannot hand qsa_sparse_attn a
workspace.  It must give the oracle's results, the same as qsa_sparse_attn on the
same inputs, call after call, since every call reuses the library's one built-in
scratch array; and it must not allocate.  Shapes are chosen so that a (query, KV
head) pair's block list is split over 1, 2, 4 and 7 CTAs, whose partials meet in
the scratch array.  This file is collected last and builds its own inputs, so it
passes alone in a fresh process as well as after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

import gpu_util as gu
from oracle import oracle as O
from qsa_synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gu.ensure_built()
    O.lib()
    import block_sparse_attention_key_b200 as qsa
    return qsa


def _case(n_q, hkv, seed):
    """n_q sequences at ragged positions near 16K tokens, one query each, with
    random (valid, ascending) selections of 512 blocks."""
    from qsa_synth import device as sdev
    cap = 16384
    pos = [cap - 1 - 7 * i for i in range(n_q)]
    wl = W.Workload(f"noalloc_{n_q}x{hkv}", seed, "decode", n_q, 8 * hkv, hkv, cap,
                    [W.Step([cap] * n_q, [cap] * n_q, list(range(n_q)), pos, list(range(n_q)))])
    dw = sdev.DeviceWorkload(wl)
    T = dw.step_tensors(0)
    rng = np.random.default_rng(seed)
    sel = np.full((n_q, 512), -1, dtype=np.int32)
    for r, t in enumerate(pos):
        sel[r] = np.sort(rng.choice((t + 1) // 4, size=512, replace=False))
    cnt = np.full(n_q, 512, dtype=np.int32)
    return wl, dw, T, sel, cnt


def _oracle_rows(wl, sel, cnt, rows):
    """Oracle attention of the given rows over the given selections (host generator inputs)."""
    import qsa_synth as syn
    st = wl.steps[0]
    want = []
    for r in rows:
        s, t, qid = st.q_seq[r], st.q_pos[r], st.query_ids[r]
        toks = O.attended_tokens(sel[r, :cnt[r]], t, wl.block_size)
        k = syn.gen_kv_rows(wl.seed, "k", s, toks, wl.n_kv_heads, wl.head_dim)
        v = syn.gen_kv_rows(wl.seed, "v", s, toks, wl.n_kv_heads, wl.head_dim)
        q = syn.gen_q(wl.seed, [qid], wl.n_q_heads, wl.head_dim)[0]
        want.append(O.gqa_attention(q, k, v))
    return np.stack(want)


# (queries, KV heads): 160 pairs -> 1 split per pair, 128 -> 2, 64 -> 4, 16 -> 7
@pytest.mark.parametrize("n_q,hkv", [(40, 4), (32, 4), (16, 4), (4, 4)])
def test_noalloc_matches_oracle_twice_without_allocating(lib, n_q, hkv):
    qsa = lib
    wl, dw, T, sel_h, cnt_h = _case(n_q, hkv, 70 + n_q)
    sel, cnt = torch.tensor(sel_h, device="cuda"), torch.tensor(cnt_h, device="cuda")
    dims = gu.dims_of(wl)
    rows = list(range(n_q)) if n_q <= 16 else list(range(0, n_q, 3))
    want = _oracle_rows(wl, sel_h, cnt_h, rows)

    # the workspace entry point on the same inputs
    ws = gu.new_workspace(qsa.qsa_workspace_bytes(dims, n_q, 0, qsa.QSA_MODE_DECODE))
    with_ws = torch.empty((n_q, wl.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    qsa.qsa_sparse_attn(dims, T["q"], dw.k_cache, dw.v_cache, T["q_seq"], T["q_pos"], sel, cnt, n_q, with_ws, ws)

    outs = [torch.full_like(with_ws, float("nan")) for _ in range(3)]
    # a first call outside the measurement: it looks up the scratch address and may
    # load the library's module on this device
    qsa.qsa_sparse_attn_noalloc(dims, T["q"], dw.k_cache, dw.v_cache, T["q_seq"], T["q_pos"], sel, cnt, n_q,
                                outs[0])
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for out in outs[1:]:  # the second call starts from the first call's leftover scratch
        qsa.qsa_sparse_attn_noalloc(dims, T["q"], dw.k_cache, dw.v_cache, T["q_seq"], T["q_pos"], sel, cnt, n_q,
                                    out)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0, "device memory changed across the calls"
    gu.compare_outputs(gu.bf16_to_f64(with_ws[rows]), want)
    for out in outs:
        gu.compare_outputs(gu.bf16_to_f64(out[rows]), want)
        gu.compare_outputs(gu.bf16_to_f64(out), gu.bf16_to_f64(with_ws))
        assert torch.equal(out, outs[0]), "repeated calls on the same inputs differ"


def test_noalloc_rejects_calls_beyond_its_scratch(lib):
    qsa = lib
    L = qsa.load()
    # 32,769 queries x 128 KV heads need just over 16 MiB of completion counters (4
    # bytes per query and KV head): refused on the host before any launch.  Every
    # buffer is real and sized for the call, and every query would attend one token,
    # so even a launch could not read or write outside them.
    n_q, hkv, cap = 32769, 128, 16
    dims = qsa.make_dims(batch=1, n_q_heads=hkv, n_kv_heads=hkv, kv_capacity=cap)
    q = torch.zeros((n_q, hkv, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    kc = torch.zeros((1, hkv, cap, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    q_seq = torch.zeros(n_q, dtype=torch.int32, device="cuda")
    q_pos = torch.zeros(n_q, dtype=torch.int32, device="cuda")
    sel = torch.full((n_q, 512), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(n_q, dtype=torch.int32, device="cuda")
    ptrs = [t.data_ptr() for t in (q, kc, vc, q_seq, q_pos, sel, cnt)]
    rc = L.qsa_sparse_attn_noalloc(ctypes.byref(dims), *ptrs, n_q, out.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == qsa.QSA_ERR_WORKSPACE_TOO_SMALL
    # null pointers are refused before anything else is looked at
    assert L.qsa_sparse_attn_noalloc(ctypes.byref(dims), *([None] * 7), 16, None, None) == qsa.QSA_ERR_INVALID_ARG
