"""Context parallelism on CPU ranks: two gloo processes hold halves of a sequence's
blocks and exchange what the GPU path exchanges (each rank's top-k as (score,
block) keys, then per-(query, head) attention partials).  The per-rank steps use
the oracle; the test checks that the exchange and the two merges reproduce the
oracle's whole-sequence selection and attention exactly (selection) and to fp64
rounding (attention), and the host logic that cuts the shards.
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
