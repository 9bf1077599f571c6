"""Oracle selections for many query rows at once, spread over the host's cores.

Test infrastructure: every row is one single-threaded call chain of the CPU
oracle (block scores of the row's complete causal blocks, then the top 512),
exactly as the per-row parity checks make it; only the rows are shared out
between worker processes.  The pool starts with ``spawn``, so it is safe to
create after the CUDA context exists.  Inputs come from the seeded host
generator; nothing is read back from the GPU.
"""

import multiprocessing as mp
import os
import tempfile
import time

import numpy as np

_POOLED = None  # per worker: {seq: memmapped pooled keys}


def _init(paths):
    global _POOLED
    _POOLED = {s: np.load(p, mmap_mode="r") for s, p in paths.items()}


def _rows(job):
    from oracle import oracle as O
    import qsa_synth as syn
    seed, n_idx_heads, idx_dim, block_size, top_k, rows = job
    out = []
    for r, s, t, qid in rows:
        n_c = (t + 1) // block_size
        q_idx = syn.gen_q_idx(seed, [qid], n_idx_heads, idx_dim)[0]
        w = syn.gen_w(seed, [qid], n_idx_heads)[0]
        scores = O.block_scores(q_idx, w, np.ascontiguousarray(_POOLED[s][:n_c]))
        out.append((r, O.select_top_blocks(scores, top_k)))
    return out


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_selections(wl, step, rows=None, processes=None, chunk=16):
    """{row: ascending selected blocks} for the given rows of ``wl.steps[step]``
    (every row by default), plus (wall seconds, processes used)."""
    from oracle import oracle as O
    st = wl.steps[step]
    rows = list(range(len(st.q_pos))) if rows is None else list(rows)
    procs = processes or cores()
    t0 = time.perf_counter()
    wo = O.WorkloadOracle(wl)
    tmp = tempfile.mkdtemp(prefix="qsa_oracle_")
    paths = {}
    try:
        for s in sorted({st.q_seq[r] for r in rows}):
            n_blocks = max((st.q_pos[r] + 1) // wl.block_size for r in rows if st.q_seq[r] == s)
            paths[s] = os.path.join(tmp, f"pooled_{s}.npy")
            np.save(paths[s], wo.pooled(s, n_blocks))
        # long rows first, so the pool's tail is short
        order = sorted(rows, key=lambda r: -st.q_pos[r])
        jobs = [(wl.seed, wl.n_idx_heads, wl.idx_dim, wl.block_size, wl.top_k,
                 [(r, st.q_seq[r], st.q_pos[r], st.query_ids[r]) for r in order[k:k + chunk]])
                for k in range(0, len(order), chunk)]
        want = {}
        with mp.get_context("spawn").Pool(procs, initializer=_init, initargs=(paths,)) as pool:
            for part in pool.imap_unordered(_rows, jobs):
                for r, sel in part:
                    want[r] = sel
    finally:
        for p in paths.values():
            if os.path.exists(p):
                os.remove(p)
        os.rmdir(tmp)
    return want, time.perf_counter() - t0, procs
