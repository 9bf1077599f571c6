"""Context parallelism on CPU ranks: two gloo processes hold halves of a sequence's
blocks and exchange what the GPU path exchanges (each rank's top-k as (score,
block) keys, then per-(query, head) attention partials).  The per-rank steps use
the oracle; the tests check that the exchange and the two merges reproduce the
oracle's whole-sequence selection and attention exactly (selection) and to fp64
rounding (attention), and the host logic that cuts the shards.  The last test runs
the orchestrating module (cp.cp_decode) itself over the two ranks, with the
library's per-rank steps stood in for on CPU.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_key_b200.cp import shard_range

BS, TOP_K, T_CAP, HQ, HKV, D = 4, 48, 2400, 8, 2, 32
POSITIONS = [2399, 1700, 1201, 300, 93, 2]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(5)
    import torch as T
    to_bits = lambda x: T.tensor(np.asarray(x, dtype=np.float32)).to(T.bfloat16).view(T.int16).numpy().view(np.uint16)
    idx_k = to_bits(rng.integers(-4, 5, (T_CAP, 64)))
    q_idx = [to_bits(rng.integers(-4, 5, (4, 64))) for _ in POSITIONS]
    w = [rng.integers(1, 4, 4).astype(np.float32) for _ in POSITIONS]
    q = [to_bits(rng.normal(size=(HQ, D))) for _ in POSITIONS]
    k = to_bits(rng.normal(size=(T_CAP, HKV, D)))
    v = to_bits(rng.normal(size=(T_CAP, HKV, D)))
    return idx_k, q_idx, w, q, k, v


def _val(bits):
    import qsa_synth as syn
    return syn.bf16_bits_to_f32(bits).astype(np.float64)


def _rank(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle as O
        idx_k, q_idx, w, q, k, v = _inputs()
        pooled = O.pool_blocks(idx_k, BS)
        lo, nb = shard_range(T_CAP // BS, world, rank)
        keys_s = torch.full((len(POSITIONS), TOP_K), -np.inf, dtype=torch.float64)
        keys_b = torch.full((len(POSITIONS), TOP_K), -1, dtype=torch.int64)
        for i, t in enumerate(POSITIONS):
            n_c = (t + 1) // BS
            hi = min(lo + nb, n_c)
            if hi <= lo:
                continue
            sc = O.block_scores(q_idx[i], w[i], pooled[lo:hi])   # this rank's candidate blocks
            loc = O.select_top_blocks(sc, TOP_K)                 # its local top-k
            keys_s[i, : len(loc)] = torch.tensor(sc[loc])
            keys_b[i, : len(loc)] = torch.tensor(loc + lo)
        all_s = [torch.empty_like(keys_s) for _ in range(world)]
        all_b = [torch.empty_like(keys_b) for _ in range(world)]
        dist.all_gather(all_s, keys_s)
        dist.all_gather(all_b, keys_b)
        # merge: score descending, lower block first, the first TOP_K
        sels = []
        for i in range(len(POSITIONS)):
            s = torch.cat([a[i] for a in all_s]).numpy()
            b = torch.cat([a[i] for a in all_b]).numpy()
            ok = b >= 0
            order = np.lexsort((b[ok], -s[ok]))[:TOP_K]
            sels.append(np.sort(b[ok][order]).astype(np.int32))
        # partials over this rank's selected blocks (and the partial block if it is here)
        parts = torch.zeros((len(POSITIONS), HQ, 2 + D), dtype=torch.float64)
        G = HQ // HKV
        for i, t in enumerate(POSITIONS):
            toks = O.attended_tokens(sels[i], t, BS)
            toks = toks[(toks >= lo * BS) & (toks < (lo + nb) * BS)]
            if len(toks) == 0:
                parts[i, :, 0] = -np.inf
                continue
            qv, kv, vv = _val(q[i]), _val(k[toks]), _val(v[toks])
            for h in range(HQ):
                x = kv[:, h // G, :] @ qv[h] / np.sqrt(D)
                m = x.max()
                p = np.exp(x - m)
                parts[i, h, 0] = m
                parts[i, h, 1] = p.sum()
                parts[i, h, 2:] = torch.tensor(p @ vv[:, h // G, :])
        all_p = [torch.empty_like(parts) for _ in range(world)]
        dist.all_gather(all_p, parts)
        outs = []
        for i in range(len(POSITIONS)):
            o = np.zeros((HQ, D))
            for h in range(HQ):
                ms = np.array([float(a[i, h, 0]) for a in all_p])
                M = ms.max()
                f = np.where(np.isfinite(ms), np.exp(ms - M), 0.0)
                L = sum(f[r] * float(all_p[r][i, h, 1]) for r in range(world))
                o[h] = sum(f[r] * all_p[r][i, h, 2:].numpy() for r in range(world)) / L
            outs.append(o)
        results[rank] = ([s.tolist() for s in sels], [o.tolist() for o in outs])
    finally:
        dist.destroy_process_group()


def test_shard_range_covers_every_block_once():
    for n in (0, 1, 7, 600, 262144):
        for world in (1, 2, 3, 4, 8):
            parts = [shard_range(n, world, r) for r in range(world)]
            assert parts[0][0] == 0
            assert sum(nb for _, nb in parts) == n
            for (lo, nb), (lo2, _) in zip(parts, parts[1:]):
                assert lo + nb == lo2
            assert max(nb for _, nb in parts) - min(nb for _, nb in parts) <= 1
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def test_two_gloo_ranks_reproduce_selection_and_attention():
    from oracle import oracle as O
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
            assert p.exitcode == 0
        res = dict(results)
    idx_k, q_idx, w, q, k, v = _inputs()
    pooled = O.pool_blocks(idx_k, BS)
    for i, t in enumerate(POSITIONS):
        fetch = lambda toks: (k[toks], v[toks])
        sel, out = O.query_forward(pooled, q_idx[i], w[i], t, q[i], fetch, top_k=TOP_K, block_size=BS)
        for r in range(2):
            sels, outs = res[r]
            assert sels[i] == sel.tolist(), f"rank {r} query {i}"
            np.testing.assert_allclose(np.array(outs[i]), out, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- the orchestrating module itself
#
# cp.cp_decode over two gloo ranks, with the library's four context-parallel steps
# replaced by CPU stand-ins written from their header contracts and the oracle: the
# test covers the module's exchange (buffer shapes, all-gathers, argument order) on
# CPU.  Keys follow the documented encoding (order-preserving fp32 score << 32 |
# ~global block); partials here use the natural-exponential domain in both stand-ins.

D128, HQ4, HKV2 = 128, 4, 2
MASK32 = 0xFFFFFFFF


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _orderable(f32):
    u = int(np.asarray(f32, dtype=np.float32).view(np.uint32))
    if u == 0x80000000:  # -0 orders as +0
        u = 0
    return (~u & MASK32) if u & 0x80000000 else (u | 0x80000000)


def _stand_in_select_keys(shard_dims, q_idx, w, pooled_shard, q_seq, q_pos, n_q, blk_lo, keys, key_cnt, workspace,
                          stream=None):
    from oracle import oracle as O
    bs, n_local = shard_dims.block_size, shard_dims.kv_capacity // shard_dims.block_size
    keys.zero_()
    key_cnt.zero_()
    for i in range(n_q):
        s, t = int(q_seq[i]), int(q_pos[i])
        n_loc = min(max((t + 1) // bs - blk_lo, 0), n_local)
        if n_loc == 0:
            continue
        sc = O.block_scores(_bits(q_idx[i]), w[i].double().numpy(), _bits(pooled_shard[s, :n_loc]))
        loc = O.select_top_blocks(sc, shard_dims.top_k)
        for j, b in enumerate(loc):
            u = (_orderable(np.float32(sc[b])) << 32) | (~(blk_lo + int(b)) & MASK32)
            keys[i, j] = u - (1 << 64) if u >= 1 << 63 else u
        key_cnt[i] = len(loc)


def _stand_in_merge_keys(shard_dims, n_ranks, keys_all, cnt_all, n_q, blk_lo, sel_local, cnt_local, sel_global=None,
                         cnt_global=None, stream=None):
    n_local = shard_dims.kv_capacity // shard_dims.block_size
    ka = keys_all.view(n_ranks, n_q, -1)
    ca = cnt_all.view(n_ranks, n_q)
    sel_local.fill_(-1)
    for i in range(n_q):
        union = [int(ka[r, i, j]) & ((1 << 64) - 1) for r in range(n_ranks) for j in range(int(ca[r, i]))]
        blocks = sorted(~u & MASK32 for u in sorted(union, reverse=True)[: shard_dims.top_k])
        mine = [b - blk_lo for b in blocks if blk_lo <= b < blk_lo + n_local]
        sel_local[i, : len(mine)] = torch.tensor(mine, dtype=torch.int32)
        cnt_local[i] = len(mine)


def _stand_in_attn_partial(shard_dims, q, k_shard, v_shard, q_seq, q_pos, n_q, blk_lo, sel_local, cnt_local, part,
                           workspace, stream=None):
    from oracle import oracle as O
    bs = shard_dims.block_size
    tok_lo, tok_hi = blk_lo * bs, blk_lo * bs + shard_dims.kv_capacity
    G = shard_dims.n_q_heads // shard_dims.n_kv_heads
    part.zero_()
    for i in range(n_q):
        s, t = int(q_seq[i]), int(q_pos[i])
        own = sel_local[i, : int(cnt_local[i])].numpy().astype(np.int64) + blk_lo
        toks = O.attended_tokens(own, t, bs)
        toks = toks[(toks >= tok_lo) & (toks < tok_hi)] - tok_lo
        qv = q[i].double().numpy()
        for h in range(shard_dims.n_q_heads):
            if len(toks) == 0:
                part[i, h, 0] = -np.inf
                continue
            kv = k_shard[s, h // G, toks].double().numpy()
            vv = v_shard[s, h // G, toks].double().numpy()
            x = kv @ qv[h] / np.sqrt(D128)
            m = x.max()
            p = np.exp(x - m)
            part[i, h, 0] = m
            part[i, h, 1] = p.sum()
            part[i, h, 4:] = torch.from_numpy(p @ vv)


def _stand_in_combine(dims, n_ranks, parts_all, n_q, out, stream=None):
    P = parts_all.view(n_ranks, n_q, dims.n_q_heads, -1).double().numpy()
    for i in range(n_q):
        for h in range(dims.n_q_heads):
            ms = P[:, i, h, 0]
            M = ms.max()
            f = np.where(np.isfinite(ms), np.exp(ms - M), 0.0)
            out[i, h] = torch.from_numpy((f[:, None] * P[:, i, h, 4:]).sum(0) / (f * P[:, i, h, 1]).sum())


def _module_inputs():
    rng = np.random.default_rng(11)
    to_bits = lambda x: _bits(torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16))
    n = len(POSITIONS)
    return (to_bits(rng.integers(-4, 5, (T_CAP, 64))), to_bits(rng.integers(-4, 5, (n, 4, 64))),
            rng.integers(1, 4, (n, 4)).astype(np.float32), to_bits(rng.normal(size=(n, HQ4, D128))),
            to_bits(rng.normal(size=(HKV2, T_CAP, D128))), to_bits(rng.normal(size=(HKV2, T_CAP, D128))))


def _rank_module(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import block_sparse_attention_key_b200 as qsa
        from block_sparse_attention_key_b200 import cp
        from block_sparse_attention_key_b200 import qsa as binding
        from oracle import oracle as O
        binding.qsa_cp_select_keys = _stand_in_select_keys
        binding.qsa_cp_merge_keys = _stand_in_merge_keys
        binding.qsa_cp_attn_partial = _stand_in_attn_partial
        binding.qsa_cp_combine = _stand_in_combine
        idx_k, q_idx, w, q, k, v = _module_inputs()
        n = len(POSITIONS)
        lo, nb = shard_range(T_CAP // BS, world, rank)
        tl, th = lo * BS, (lo + nb) * BS
        pooled = O.pool_blocks(idx_k, BS)
        shard = qsa.make_dims(1, HQ4, HKV2, nb * BS, block_size=BS, top_k=TOP_K)
        full = qsa.make_dims(1, HQ4, HKV2, T_CAP, block_size=BS, top_k=TOP_K)
        out = torch.zeros((n, HQ4, D128), dtype=torch.float64)
        sel, cnt = cp.cp_decode(shard, full, q=_bf16(q), k_shard=_bf16(k[None, :, tl:th]),
                                v_shard=_bf16(v[None, :, tl:th]), q_idx=_bf16(q_idx), w=torch.from_numpy(w),
                                pooled_shard=_bf16(pooled[None, lo:lo + nb]), q_seq=torch.zeros(n, dtype=torch.int32),
                                q_pos=torch.tensor(POSITIONS, dtype=torch.int32), n_q=n, blk_lo=lo, out=out,
                                workspace=None)
        results[rank] = ([(sel[i, : int(cnt[i])].numpy() + lo).tolist() for i in range(n)], out.tolist())
    finally:
        dist.destroy_process_group()


def test_cp_decode_module_over_two_gloo_ranks():
    from oracle import oracle as O
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_module, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
            assert p.exitcode == 0
        res = dict(results)
    idx_k, q_idx, w, q, k, v = _module_inputs()
    pooled = O.pool_blocks(idx_k, BS)
    for i, t in enumerate(POSITIONS):
        fetch = lambda toks: (k[:, toks].transpose(1, 0, 2), v[:, toks].transpose(1, 0, 2))
        sel, want = O.query_forward(pooled, q_idx[i], w[i], t, q[i], fetch, top_k=TOP_K, block_size=BS)
        # the ranks' own blocks partition the whole-sequence selection
        assert sorted(res[0][0][i] + res[1][0][i]) == sel.tolist(), f"query {i}"
        for r in range(2):
            np.testing.assert_allclose(np.array(res[r][1][i]), want, rtol=0, atol=1e-6)
