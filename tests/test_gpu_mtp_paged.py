"""Serving shapes through the C ABI against the oracle: multi-token decode with one
shared selection per group of draft queries, paged K/V caches, and one call mixing
decode queries with a prefill chunk.

keieiax.jp glossary "Qwen Sparse Attention", FAQ on multi-token prediction: the
top index is reused between speculative steps.  A group of k draft queries of a
sequence is scored and selected once, at its first query t_0; draft j at t_j
attends the shared blocks plus every token from t_0's first incomplete block to
t_j (oracle: attended_tokens_shared).  Paged caches hold the same K/V values in
pages of a pool, addressed through a per-sequence page table.
"""

import numpy as np
import pytest
import torch

import qsa_synth as syn
from oracle import oracle as O
from qsa_synth import workloads as W

import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gu.ensure_built()
    O.lib()


def _mtp_workload(k, hq, hkv, cap, t0s, seed):
    """One group of k consecutive draft queries per sequence, the drafts' tokens
    appended in this step."""
    q_seq, q_pos = [], []
    for s, t0 in enumerate(t0s):
        q_seq += [s] * k
        q_pos += [t0 + j for j in range(k)]
    n = len(q_pos)
    b = len(t0s)
    return W.Workload(f"mtp{k}_{hq}_{hkv}", seed, "decode", b, hq, hkv, cap,
                      [W.Step(list(t0s), [t0 + k for t0 in t0s], q_seq, q_pos, list(range(n)))])


def _run_mtp(wl, k, page=None):
    """qsa_forward with group_q = k (and optionally a page table); returns outputs,
    selections, counts and the status flags."""
    import block_sparse_attention_key_b200 as qsa
    from qsa_synth import device as sdev
    dw = sdev.DeviceWorkload(wl)
    gu.pool_history(dw, 0)
    T = dw.step_tensors(0)
    n = T["n_q"]
    groups = n // k
    dims = gu.dims_of(wl)
    kc, vc, table, page_tokens, n_pages = dw.k_cache, dw.v_cache, None, 0, 0
    if page is not None:
        kc, vc, table, page_tokens, n_pages = page(dw)
    ws = gu.new_workspace(qsa.qsa_workspace_bytes(dims, n, T["max_blocks"], qsa.QSA_MODE_DECODE))
    out = torch.empty((n, wl.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((groups, 512), dtype=torch.int32, device="cuda")
    cnt = torch.empty((groups,), dtype=torch.int32, device="cuda")
    qsa.qsa_forward(dims, q=T["q"], k_cache=kc, v_cache=vc, idx_k=dw.idx_k, pooled=dw.pooled,
                    q_idx=T["q_idx"][::k].contiguous(), w=T["w"][::k].contiguous(), len_before=T["len_before"],
                    len_after=T["len_after"], q_seq=T["q_seq"], q_pos=T["q_pos"], n_q=n,
                    max_new_tokens=T["max_new_tokens"], max_blocks=T["max_blocks"], mode=qsa.QSA_MODE_DECODE,
                    out=out, workspace=ws, sel_idx=sel, sel_cnt=cnt, group_q=k, page_table=table,
                    page_tokens=page_tokens, n_pages=n_pages)
    flags = qsa.qsa_read_device_status(ws)
    return out, sel.cpu().numpy(), cnt.cpu().numpy(), flags


def _oracle_mtp(wl, k):
    """Per group: the oracle's selection at the group's first query; per draft query:
    attention over the shared blocks and its tail."""
    st = wl.steps[0]
    wo = O.WorkloadOracle(wl)
    sels, outs = [], []
    for g0 in range(0, len(st.q_pos), k):
        s, t0, qid0 = st.q_seq[g0], st.q_pos[g0], st.query_ids[g0]
        n_c = (t0 + 1) // wl.block_size
        q_idx = syn.gen_q_idx(wl.seed, [qid0], wl.n_idx_heads, wl.idx_dim)[0]
        w = syn.gen_w(wl.seed, [qid0], wl.n_idx_heads)[0]
        sel = O.select_top_blocks(O.block_scores(q_idx, w, wo.pooled(s, n_c)), wl.top_k)
        sels.append(sel)
        for j in range(k):
            t, qid = st.q_pos[g0 + j], st.query_ids[g0 + j]
            toks = O.attended_tokens_shared(sel, t0, t, wl.block_size)
            kr = syn.gen_kv_rows(wl.seed, "k", s, toks, wl.n_kv_heads, wl.head_dim)
            vr = syn.gen_kv_rows(wl.seed, "v", s, toks, wl.n_kv_heads, wl.head_dim)
            q = syn.gen_q(wl.seed, [qid], wl.n_q_heads, wl.head_dim)[0]
            outs.append(O.gqa_attention(q, kr, vr))
    return sels, np.stack(outs)


# the selection query at every offset within its block; long rows (up to 4,096 blocks) and a
# row below the 512-block budget
T0S = [16380, 16381, 16382, 16383 - 4 * 7, 9001, 1500]


@pytest.mark.parametrize("k,hq,hkv", [(2, 32, 4), (3, 32, 4), (4, 32, 4), (4, 16, 4), (1, 32, 4), (5, 8, 2)])
def test_forward_mtp_groups_share_one_selection(k, hq, hkv):
    wl = _mtp_workload(k, hq, hkv, 16384 + 8, T0S, 40 + k * 10 + hq)
    out, sel, cnt, flags = _run_mtp(wl, k)
    assert flags == 0
    want_sel, want_out = _oracle_mtp(wl, k)
    for g, ws_ in enumerate(want_sel):
        assert cnt[g] == len(ws_)
        np.testing.assert_array_equal(sel[g, : cnt[g]], ws_, err_msg=f"group {g}")
    gu.compare_outputs(gu.bf16_to_f64(out), want_out)


def _paged(seed, page_tokens, spare=3):
    """Page pools holding the dense caches' values at a random page permutation."""
    def build(dw):
        wl = dw.wl
        B, H, T, D = dw.k_cache.shape
        per_seq = T // page_tokens
        n_pages = B * per_seq + spare
        rng = np.random.default_rng(seed)
        perm = rng.permutation(n_pages)[: B * per_seq].reshape(B, per_seq).astype(np.int32)
        kp = torch.zeros((n_pages, H, page_tokens, D), dtype=torch.bfloat16, device="cuda")
        vp = torch.zeros_like(kp)
        src_k = dw.k_cache.view(B, H, per_seq, page_tokens, D).permute(0, 2, 1, 3, 4)
        src_v = dw.v_cache.view(B, H, per_seq, page_tokens, D).permute(0, 2, 1, 3, 4)
        idx = torch.tensor(perm, device="cuda").long()
        kp[idx.reshape(-1)] = src_k.reshape(-1, H, page_tokens, D)
        vp[idx.reshape(-1)] = src_v.reshape(-1, H, page_tokens, D)
        return kp, vp, torch.tensor(perm, device="cuda"), page_tokens, n_pages
    return build


@pytest.mark.parametrize("page_tokens", [16, 256])
def test_forward_decode_paged_kv_matches_oracle(page_tokens):
    k = 1
    wl = _mtp_workload(k, 32, 4, 16384, [16383, 16001, 9002, 700], 60 + page_tokens)
    out, sel, cnt, flags = _run_mtp(wl, k, page=_paged(7, page_tokens))
    assert flags == 0
    want_sel, want_out = _oracle_mtp(wl, k)
    for g, ws_ in enumerate(want_sel):
        np.testing.assert_array_equal(sel[g, : cnt[g]], ws_)
    gu.compare_outputs(gu.bf16_to_f64(out), want_out)


def test_forward_mtp_paged_kv_matches_oracle():
    k = 3
    wl = _mtp_workload(k, 32, 4, 16384 + 64, T0S, 61)
    out, sel, cnt, flags = _run_mtp(wl, k, page=_paged(8, 64))
    assert flags == 0
    want_sel, want_out = _oracle_mtp(wl, k)
    for g, ws_ in enumerate(want_sel):
        np.testing.assert_array_equal(sel[g, : cnt[g]], ws_)
    gu.compare_outputs(gu.bf16_to_f64(out), want_out)


def test_forward_prefill_paged_kv_matches_oracle():
    """A prefill chunk whose K/V live in pages: same selections and outputs as the oracle."""
    import block_sparse_attention_key_b200 as qsa
    from qsa_synth import device as sdev
    wl = W.Workload("pf_paged", 62, "prefill", 1, 32, 4, 8192, [W._prefill_step(6000, 200)])
    dw = sdev.DeviceWorkload(wl)
    gu.pool_history(dw, 0)
    T = dw.step_tensors(0)
    n = T["n_q"]
    dims = gu.dims_of(wl)
    kp, vp, table, pt, n_pages = _paged(9, 32)(dw)
    ws = gu.new_workspace(qsa.qsa_workspace_bytes(dims, n, T["max_blocks"], qsa.QSA_MODE_PREFILL))
    out = torch.empty((n, 32, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((n, 512), dtype=torch.int32, device="cuda")
    cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    qsa.qsa_forward(dims, q=T["q"], k_cache=kp, v_cache=vp, idx_k=dw.idx_k, pooled=dw.pooled, q_idx=T["q_idx"],
                    w=T["w"], len_before=T["len_before"], len_after=T["len_after"], q_seq=T["q_seq"],
                    q_pos=T["q_pos"], n_q=n, max_new_tokens=T["max_new_tokens"], max_blocks=T["max_blocks"],
                    mode=qsa.QSA_MODE_PREFILL, out=out, workspace=ws, sel_idx=sel, sel_cnt=cnt, page_table=table,
                    page_tokens=pt, n_pages=n_pages)
    assert qsa.qsa_read_device_status(ws) == 0
    wo = O.WorkloadOracle(wl)
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    rows = [0, 1, 2, 3, 99, 127, 128, 199]
    got = gu.bf16_to_f64(out[rows])
    want = np.zeros_like(got)
    for j, r in enumerate(rows):
        s_want, o_want = wo.query(0, r)
        np.testing.assert_array_equal(sel[r, : cnt[r]], s_want)
        want[j] = o_want
    gu.compare_outputs(got, want)


def test_bad_page_entry_is_reported_and_skipped():
    """A page-table entry outside the pool: its blocks are skipped, QSA_DEV_BAD_PAGE set."""
    import block_sparse_attention_key_b200 as qsa

    def bad(dw):
        kp, vp, table, pt, n_pages = _paged(10, 64)(dw)
        table[0, :] = n_pages + 5  # sequence 0: every page out of range
        return kp, vp, table, pt, n_pages
    wl = _mtp_workload(1, 32, 4, 8192, [8191, 5000], 63)
    out, sel, cnt, flags = _run_mtp(wl, 1, page=bad)
    assert flags & qsa.QSA_DEV_BAD_PAGE
    assert torch.isfinite(out.float()).all()


def _mixed_workload(n_pf):
    """Three decode queries of three sequences, then an n_pf-query prefill chunk of a
    fourth sequence (16K capacity, 32 / 4 heads)."""
    dec = [(0, 16383), (1, 12001), (2, 702)]
    t0 = 9000
    q_seq = [s for s, _ in dec] + [3] * n_pf
    q_pos = [t for _, t in dec] + list(range(t0, t0 + n_pf))
    lb = [t for _, t in dec] + [t0]
    la = [t + 1 for _, t in dec] + [t0 + n_pf]
    return len(dec), W.Workload("mixed", 64, "prefill", 4, 32, 4, 16384,
                                [W.Step(lb, la, q_seq, q_pos, list(range(len(q_pos))))])


def _forward_mixed(dw, T, m, n_dec, ws, q_idx=None):
    """qsa_forward in QSA_MODE_MIXED over the step's first m rows."""
    import block_sparse_attention_key_b200 as qsa
    wl = dw.wl
    out = torch.empty((m, wl.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((m, 512), dtype=torch.int32, device="cuda")
    cnt = torch.empty((m,), dtype=torch.int32, device="cuda")
    qi = T["q_idx"] if q_idx is None else q_idx
    qsa.qsa_forward(gu.dims_of(wl), q=T["q"][:m], k_cache=dw.k_cache, v_cache=dw.v_cache, idx_k=dw.idx_k,
                    pooled=dw.pooled, q_idx=qi[:m], w=T["w"][:m], len_before=T["len_before"],
                    len_after=T["len_after"], q_seq=T["q_seq"][:m], q_pos=T["q_pos"][:m], n_q=m,
                    max_new_tokens=T["max_new_tokens"], max_blocks=T["max_blocks"], mode=qsa.QSA_MODE_MIXED,
                    out=out, workspace=ws, sel_idx=sel, sel_cnt=cnt, n_decode=n_dec)
    return out, sel, cnt


def test_forward_mixed_calls_with_fallback_rows_share_a_workspace():
    """One workspace, two mixed calls.  In the first every prefill row's indexer query
    is zero, so all its scores tie, which sends the prefill rows to the fallback select
    (each keeps blocks 0..511); the second has fewer prefill rows and ordinary inputs
    and must match the oracle (the fallback's worklist starts empty in every call)."""
    import block_sparse_attention_key_b200 as qsa
    from qsa_synth import device as sdev
    n_dec, wl = _mixed_workload(150)
    dw = sdev.DeviceWorkload(wl)
    gu.pool_history(dw, 0)
    T = dw.step_tensors(0)
    n = T["n_q"]
    ws = gu.new_workspace(qsa.qsa_workspace_bytes(gu.dims_of(wl), n, T["max_blocks"], qsa.QSA_MODE_MIXED))
    wo = O.WorkloadOracle(wl)
    q_tie = T["q_idx"].clone()
    q_tie[n_dec:] = 0
    _, sel, cnt = _forward_mixed(dw, T, n, n_dec, ws, q_idx=q_tie)
    assert qsa.qsa_read_device_status(ws) == 0
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for r in range(n):
        if r < n_dec:
            np.testing.assert_array_equal(sel[r, : cnt[r]], wo.query(0, r)[0], err_msg=f"row {r}")
        else:
            n_c = (wl.steps[0].q_pos[r] + 1) // 4
            assert cnt[r] == min(512, n_c)
            np.testing.assert_array_equal(sel[r, : cnt[r]], np.arange(cnt[r]), err_msg=f"row {r}")
    m = n_dec + 100
    out, sel, cnt = _forward_mixed(dw, T, m, n_dec, ws)
    assert qsa.qsa_read_device_status(ws) == 0
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    rows = [0, 2, 3, 50, m - 1]
    want = np.zeros((len(rows), 32, 128))
    for r in range(m):
        s_want, o_want = wo.query(0, r) if (r in rows or r % 7 == 0) else (None, None)
        if s_want is None:
            continue
        np.testing.assert_array_equal(sel[r, : cnt[r]], s_want, err_msg=f"row {r}")
        if r in rows:
            want[rows.index(r)] = o_want
    gu.compare_outputs(gu.bf16_to_f64(out[rows]), want)


def test_forward_mixed_decode_and_prefill_rows():
    """A serving batch in one call: three decode queries of three sequences, then a
    150-query prefill chunk of a fourth; every row against the oracle."""
    import block_sparse_attention_key_b200 as qsa
    from qsa_synth import device as sdev
    dec = [(0, 16383), (1, 12001), (2, 702)]
    t0, n_pf = 9000, 150
    q_seq = [s for s, _ in dec] + [3] * n_pf
    q_pos = [t for _, t in dec] + list(range(t0, t0 + n_pf))
    lb = [t for _, t in dec] + [t0]
    la = [t + 1 for _, t in dec] + [t0 + n_pf]
    wl = W.Workload("mixed", 64, "prefill", 4, 32, 4, 16384, [W.Step(lb, la, q_seq, q_pos, list(range(len(q_pos))))])
    dw = sdev.DeviceWorkload(wl)
    gu.pool_history(dw, 0)
    T = dw.step_tensors(0)
    n = T["n_q"]
    dims = gu.dims_of(wl)
    ws = gu.new_workspace(qsa.qsa_workspace_bytes(dims, n, T["max_blocks"], qsa.QSA_MODE_MIXED))
    out = torch.empty((n, 32, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((n, 512), dtype=torch.int32, device="cuda")
    cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    qsa.qsa_forward(dims, q=T["q"], k_cache=dw.k_cache, v_cache=dw.v_cache, idx_k=dw.idx_k, pooled=dw.pooled,
                    q_idx=T["q_idx"], w=T["w"], len_before=T["len_before"], len_after=T["len_after"],
                    q_seq=T["q_seq"], q_pos=T["q_pos"], n_q=n, max_new_tokens=T["max_new_tokens"],
                    max_blocks=T["max_blocks"], mode=qsa.QSA_MODE_MIXED, out=out, workspace=ws, sel_idx=sel,
                    sel_cnt=cnt, n_decode=len(dec))
    assert qsa.qsa_read_device_status(ws) == 0
    gu.check_selection_properties(wl, 0, sel, cnt)
    wo = O.WorkloadOracle(wl)
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    rows = [0, 1, 2, 3, 4, 64, 130, 131, 152]
    got = gu.bf16_to_f64(out[rows])
    want = np.zeros_like(got)
    for j, r in enumerate(rows):
        s_want, o_want = wo.query(0, r)
        np.testing.assert_array_equal(sel[r, : cnt[r]], s_want, err_msg=f"row {r}")
        want[j] = o_want
    gu.compare_outputs(got, want)
    for r in range(5, n, 10):  # more rows' selections
        s_want, _ = wo.query(0, r)
        np.testing.assert_array_equal(sel[r, : cnt[r]], s_want, err_msg=f"row {r}")
