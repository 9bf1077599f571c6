"""Context-parallel decode through the C ABI against the oracle.

One GPU holds every shard here: the ranks' steps run one after another on their own
slices of the caches, and stacking their outputs stands in for the all-gathers (no
rank waits on another).  The orchestrating module runs once more over a one-rank
NCCL group, with real collectives.
"""

import numpy as np
import pytest
import torch

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


def _setup(bs=4, k=512):
    from qsa_synth import device as sdev
    cap = 65536
    # queries whose complete blocks end in different shards, one below the budget
    pos = [65535, 40001, 20002, 1503]
    n = len(pos)
    wl = W.Workload(f"cp_bs{bs}", 170 + bs, "decode", n, 32, 4, cap,
                    [W.Step(list(pos), [p + 1 for p in pos], list(range(n)), pos, list(range(n)))],
                    block_size=bs, top_k=k)
    dw = sdev.DeviceWorkload(wl)
    T = dw.step_tensors(0)
    # every block complete after the step is pooled (the forward's pooling step)
    import block_sparse_attention_key_b200 as qsa
    zeros = torch.zeros(n, dtype=torch.int32, device="cuda")
    qsa.qsa_pool_block_keys(gu.dims_of(wl), dw.idx_k, dw.pooled, zeros, T["len_after"], max(wl.steps[0].len_after))
    return wl, dw, T


def _shard_tensors(wl, dw, lo, nb):
    bs = wl.block_size
    return (dw.k_cache[:, :, lo * bs:(lo + nb) * bs].contiguous(), dw.v_cache[:, :, lo * bs:(lo + nb) * bs].contiguous(),
            dw.pooled[:, lo:lo + nb].contiguous())


@pytest.mark.parametrize("R,bs", [(2, 4), (3, 4), (4, 4), (8, 4), (3, 1)])
def test_cp_shards_reproduce_the_layer(R, bs):
    import block_sparse_attention_key_b200 as qsa
    from block_sparse_attention_key_b200 import cp
    wl, dw, T = _setup(bs)
    n = T["n_q"]
    full = gu.dims_of(wl)
    n_blocks = wl.kv_capacity // bs
    shards = [cp.shard_range(n_blocks, R, r) for r in range(R)]
    keys_all = torch.zeros((R, n, qsa.QSA_SEL_CAP), dtype=torch.int64, device="cuda")
    cnt_all = torch.zeros((R, n), dtype=torch.int32, device="cuda")
    state = []
    for r, (lo, nb) in enumerate(shards):
        sd = qsa.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, nb * bs, block_size=bs, top_k=wl.top_k)
        ks, vs, ps = _shard_tensors(wl, dw, lo, nb)
        ws = gu.new_workspace(qsa.qsa_cp_workspace_bytes(sd, n))
        qsa.qsa_cp_select_keys(sd, T["q_idx"], T["w"], ps, T["q_seq"], T["q_pos"], n, lo, keys_all[r], cnt_all[r], ws)
        state.append((sd, ks, vs, ws, lo))
    parts = torch.zeros((R, n, wl.n_q_heads, qsa.CP_PART_ROW), dtype=torch.float32, device="cuda")
    globals_ = []
    for r, (sd, ks, vs, ws, lo) in enumerate(state):
        sel_l = torch.empty((n, qsa.QSA_SEL_CAP), dtype=torch.int32, device="cuda")
        cnt_l = torch.empty((n,), dtype=torch.int32, device="cuda")
        sel_g = torch.empty_like(sel_l)
        cnt_g = torch.empty_like(cnt_l)
        qsa.qsa_cp_merge_keys(sd, R, keys_all, cnt_all, n, lo, sel_l, cnt_l, sel_g, cnt_g)
        qsa.qsa_cp_attn_partial(sd, T["q"], ks, vs, T["q_seq"], T["q_pos"], n, lo, sel_l, cnt_l, parts[r], ws)
        globals_.append((sel_g.cpu().numpy(), cnt_g.cpu().numpy()))
        # this rank's blocks are exactly the global selection's blocks inside its shard
        sg, cg, sl, cl = globals_[-1][0], globals_[-1][1], sel_l.cpu().numpy(), cnt_l.cpu().numpy()
        for i in range(n):
            g = sg[i, : cg[i]]
            mine = g[(g >= lo) & (g < lo + shards[r][1])] - lo
            np.testing.assert_array_equal(sl[i, : cl[i]], mine)
    out = torch.empty((n, wl.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    qsa.qsa_cp_combine(full, R, parts, n, out)
    torch.cuda.synchronize()
    wo = O.WorkloadOracle(wl)
    want = np.zeros((n, wl.n_q_heads, 128))
    for i in range(n):
        s_want, want[i] = wo.query(0, i)
        for sg, cg in globals_:  # every rank reaches the same global selection, the oracle's
            np.testing.assert_array_equal(sg[i, : cg[i]], s_want, err_msg=f"query {i}")
    gu.compare_outputs(gu.bf16_to_f64(out), want)


def test_cp_merge_breaks_score_ties_by_block():
    """Every score equal (zero indexer queries): each of 4 shards keeps 512 tied keys,
    the merge cuts 2,048 tied keys and must keep the 512 lowest blocks."""
    import block_sparse_attention_key_b200 as qsa
    import qsa_synth as syn
    from block_sparse_attention_key_b200 import cp
    wl, dw, T = _setup()
    n, R, bs = T["n_q"], 4, wl.block_size
    q_idx0 = torch.zeros_like(T["q_idx"])
    shards = [cp.shard_range(wl.kv_capacity // bs, R, r) for r in range(R)]
    keys_all = torch.zeros((R, n, qsa.QSA_SEL_CAP), dtype=torch.int64, device="cuda")
    cnt_all = torch.zeros((R, n), dtype=torch.int32, device="cuda")
    state = []
    for r, (lo, nb) in enumerate(shards):
        sd = qsa.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, nb * bs, block_size=bs, top_k=wl.top_k)
        ks, vs, ps = _shard_tensors(wl, dw, lo, nb)
        ws = gu.new_workspace(qsa.qsa_cp_workspace_bytes(sd, n))
        qsa.qsa_cp_select_keys(sd, q_idx0, T["w"], ps, T["q_seq"], T["q_pos"], n, lo, keys_all[r], cnt_all[r], ws)
        state.append((sd, ks, vs, ws, lo))
    parts = torch.zeros((R, n, wl.n_q_heads, qsa.CP_PART_ROW), dtype=torch.float32, device="cuda")
    for r, (sd, ks, vs, ws, lo) in enumerate(state):
        sel_l = torch.empty((n, qsa.QSA_SEL_CAP), dtype=torch.int32, device="cuda")
        cnt_l = torch.empty((n,), dtype=torch.int32, device="cuda")
        sel_g = torch.empty_like(sel_l)
        cnt_g = torch.empty_like(cnt_l)
        qsa.qsa_cp_merge_keys(sd, R, keys_all, cnt_all, n, lo, sel_l, cnt_l, sel_g, cnt_g)
        qsa.qsa_cp_attn_partial(sd, T["q"], ks, vs, T["q_seq"], T["q_pos"], n, lo, sel_l, cnt_l, parts[r], ws)
        sg, cg = sel_g.cpu().numpy(), cnt_g.cpu().numpy()
        for i in range(n):
            n_c = (wl.steps[0].q_pos[i] + 1) // bs
            np.testing.assert_array_equal(sg[i, : cg[i]], np.arange(min(n_c, wl.top_k)), err_msg=f"query {i}")
    out = torch.empty((n, wl.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    qsa.qsa_cp_combine(gu.dims_of(wl), R, parts, n, out)
    torch.cuda.synchronize()
    # the oracle with the same (zero) indexer queries
    wo = O.WorkloadOracle(wl)
    st = wl.steps[0]
    zero_bits = gu.to_bits(torch.zeros((wl.n_idx_heads, wl.idx_dim), dtype=torch.bfloat16))
    want = np.zeros((n, wl.n_q_heads, 128))
    for i in range(n):
        s_, t, qid = st.q_seq[i], st.q_pos[i], st.query_ids[i]
        pooled = wo.pooled(s_, (t + 1) // bs)
        w_ = syn.gen_w(wl.seed, [qid], wl.n_idx_heads)[0]
        q_ = syn.gen_q(wl.seed, [qid], wl.n_q_heads, wl.head_dim)[0]
        fetch = lambda toks, s_=s_: (syn.gen_kv_rows(wl.seed, "k", s_, toks, wl.n_kv_heads, wl.head_dim),
                                     syn.gen_kv_rows(wl.seed, "v", s_, toks, wl.n_kv_heads, wl.head_dim))
        sel, want[i] = O.query_forward(pooled, zero_bits, w_, t, q_, fetch, wl.top_k, bs)
        np.testing.assert_array_equal(sel, np.arange(min((t + 1) // bs, wl.top_k)))
    gu.compare_outputs(gu.bf16_to_f64(out), want)


def test_cp_decode_over_a_process_group():
    """The orchestrating module end to end with real NCCL collectives (one rank)."""
    import os
    import torch.distributed as dist
    import block_sparse_attention_key_b200 as qsa
    from block_sparse_attention_key_b200 import cp
    wl, dw, T = _setup()
    n = T["n_q"]
    port = 29500 + os.getpid() % 1000
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        full = gu.dims_of(wl)
        ws = gu.new_workspace(qsa.qsa_cp_workspace_bytes(full, n))
        out = torch.empty((n, wl.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
        cp.cp_decode(full, full, q=T["q"], k_shard=dw.k_cache, v_shard=dw.v_cache, q_idx=T["q_idx"], w=T["w"],
                     pooled_shard=dw.pooled, q_seq=T["q_seq"], q_pos=T["q_pos"], n_q=n, blk_lo=0, out=out,
                     workspace=ws)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    wo = O.WorkloadOracle(wl)
    want = np.stack([wo.query(0, i)[1] for i in range(n)])
    gu.compare_outputs(gu.bf16_to_f64(out), want)
