#!/usr/bin/env python3
"""Benchmark of the QSA layer forward on B200: tokens/s of one decode step of
16 sequences at 65,536 tokens of context (32 query / 4 KV heads, top-512 blocks).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One process per GPU (torchrun for N > 1).  Every rank owns its own batch of
sequences (independent problems: weak scaling, no data-path collective).  A step
is the whole layer through the C ABI (qsa_forward): pool the appended token's
block, score every complete causal block, select the top 512, gathered attention.
Inputs sit in HBM when the timed region starts; L2 is flushed (a 512 MiB write,
then a 512 MiB read) before every timed step, outside the timed events.  Rank 0 prints
one JSON line.  After the headline (unless --no-workload-map) the line also carries
every other configuration (`workloads`) and two serving shapes on the headline's
geometry (`serving_modes`: 4 draft queries per sequence sharing one selection, and
K/V in 256-token pages).  `--impl reference` times the CPU oracle on the same workload.
"""

import argparse
import json
import os
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QSA layer tokens/s at 64K–1M ctx (decode, prefill); % HBM / tensor roofline"
L2_FLUSH_BYTES = 512 << 20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="decode_64k_b16",
                   help="headline configuration (the others are measured after it unless --no-workload-map)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-workload-map", dest="workload_map", action="store_false",
                   help="skip the other configurations' measurements")
    return p.parse_args()


def workload_by_name(name):
    from qsa_synth import workloads as W
    for f in W.ALL:
        wl = f()
        if wl.name == name:
            return wl
    raise SystemExit(f"unknown workload {name}")


def workload_config(wl):
    st = wl.steps[0]
    return {"workload": wl.name, "mode": wl.mode, "batch": wl.batch, "queries_per_step": len(st.q_pos),
            "context": max(st.len_after), "q_heads": wl.n_q_heads, "kv_heads": wl.n_kv_heads,
            "head_dim": wl.head_dim, "indexer": f"{wl.n_idx_heads}x{wl.idx_dim}", "block": wl.block_size,
            "top_k_blocks": wl.top_k, "steps_per_unit": len(wl.steps),
            "l2": "flushed before every timed step (512 MiB write, then 512 MiB read; outside the timed events)"}


# ------------------------------------------------------------------ CPU oracle timing

def time_oracle(wl, budget_s=20.0, max_queries=None):
    """Time the oracle as it stands (pool + score + select + attention per query)
    on a bounded sample of the workload's queries.  Input generation is untimed."""
    import qsa_synth as syn
    from oracle import oracle as O
    O.lib()
    t_oracle = 0.0
    done = 0
    pooled_cache = {}
    queries = [(si, r) for si, st in enumerate(wl.steps) for r in range(len(st.q_pos))]
    if max_queries:
        queries = queries[:max_queries]
    for si, r in queries:
        st = wl.steps[si]
        s, t, qid = st.q_seq[r], st.q_pos[r], st.query_ids[r]
        n_c = (t + 1) // wl.block_size
        key = (s, n_c)
        if key not in pooled_cache:
            pooled_cache[key] = syn.gen_idx_k(wl.seed, s, 0, n_c * wl.block_size, wl.idx_dim)
        idx_k = pooled_cache[key]
        q_idx = syn.gen_q_idx(wl.seed, [qid], wl.n_idx_heads, wl.idx_dim)[0]
        w = syn.gen_w(wl.seed, [qid], wl.n_idx_heads)[0]
        q = syn.gen_q(wl.seed, [qid], wl.n_q_heads, wl.head_dim)[0]
        t0 = time.perf_counter()
        pooled = O.pool_blocks(idx_k, wl.block_size)
        scores = O.block_scores(q_idx, w, pooled[:n_c])
        sel = O.select_top_blocks(scores, wl.top_k)
        toks = O.attended_tokens(sel, t, wl.block_size)
        t_oracle += time.perf_counter() - t0
        k = syn.gen_kv_rows(wl.seed, "k", s, toks, wl.n_kv_heads, wl.head_dim)
        v = syn.gen_kv_rows(wl.seed, "v", s, toks, wl.n_kv_heads, wl.head_dim)
        t0 = time.perf_counter()
        O.gqa_attention(q, k, v)
        t_oracle += time.perf_counter() - t0
        done += 1
        if t_oracle >= budget_s:
            break
    return done, t_oracle


def cpu_baseline(wl, budget_s=20.0):
    done, secs = time_oracle(wl, budget_s)
    return {"value": done / secs, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} of {wl.n_queries()} queries of {wl.name} (pool + score + select + attention "
                      f"per query, fp64, single thread; input generation untimed): {secs:.2f} s"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = []
    n_step_queries = len(wl.steps[0].q_pos)
    for _ in range(args.warmup):
        time_oracle(wl, budget_s=1e9, max_queries=1)
    total_q = 0
    for _ in range(args.steps):
        done, secs = time_oracle(wl, budget_s=6.0, max_queries=n_step_queries)
        per_step.append(secs)
        total_q += done
    secs = sum(per_step)
    value = total_q / secs
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"{total_q} queries of {wl.name} over {args.steps} steps (each step a "
                                       f"bounded sample of up to {n_step_queries} queries, ~6 s cap)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

class Clocks:
    """nvidia-smi samples during the timed region."""

    def __init__(self, index):
        out_dir = os.environ.get("QSA_BENCH_OUT") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_bench_{os.getpid()}.csv")
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons), "samples": len(sm)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def load_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu capture, if it still matches the kernel source."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(f"{kernel}@{workload}")
    if not rec:
        return None
    src = os.path.join(ROOT, "block_sparse_attention_key_b200", "csrc", rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != rec["sha"]:
        return None
    return rec["bytes_per_launch"]


def forward_launches(wl, prefill, T):
    """Kernels one qsa_forward call launches (the library's launch plan):
    decode: pool + control-block clearing, scoring (rows of up to 16,384 blocks are
    also selected there), the two-pass select for longer rows, attention;
    prefill: pool when tokens are appended, the sampling launch (when the capacity is
    a multiple of 64 tokens and rows exceed 1,024 blocks), scoring, finishing select,
    fallback, attention."""
    mb = T["max_blocks"]
    if mb == 0:
        return (1 if T["max_new_tokens"] > 0 else 0) + 1
    if not prefill:
        return 1 + 1 + (1 if mb > 16384 else 0) + 1
    sampled = wl.kv_capacity % 64 == 0 and mb > 1024
    return (1 if T["max_new_tokens"] > 0 else 0) + (1 if sampled else 0) + 4


def max_over_ranks(x, world, device):
    """Largest value of x over the job's ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, tokens_per_rank, ms_per_step):
    """Whole-job throughput: every rank processes its own tokens_per_rank in each step."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def attended_tokens_of(wl, step, cnt):
    """Tokens each query attends: 4 per selected block plus its partial block."""
    part = (np.asarray(wl.steps[step].q_pos, dtype=np.int64) + 1) % wl.block_size
    return np.asarray(cnt, dtype=np.int64) * wl.block_size + part


def attn_bytes_of(wl, toks):
    """Algorithmic bytes of gathered attention: K+V rows of every attended token for
    every KV head, q read and out written."""
    n_q = len(toks)
    return int(toks.sum() * wl.n_kv_heads * wl.head_dim * 2 * 2 + 2 * n_q * wl.n_q_heads * wl.head_dim * 2)


def select_work_of(wl, step):
    """(flops, bytes) of indexer scoring for one step: 4 heads x 64 dims x 2 flops per
    (query, complete causal block), 128 B of pooled key per (query, block) read."""
    n_c = (np.asarray(wl.steps[step].q_pos, dtype=np.int64) + 1) // wl.block_size
    return int(n_c.sum() * wl.n_idx_heads * wl.idx_dim * 2), int(n_c.sum() * wl.idx_dim * 2)


class Env:
    """Per-rank GPU state shared by the workload measurements."""

    def __init__(self, args):
        import torch
        import torch.distributed as dist
        import block_sparse_attention_key_b200 as qsa
        from block_sparse_attention_key_b200 import build as qbuild
        from qsa_synth import device as sdev
        self.torch, self.dist, self.qsa, self.sdev = torch, dist, qsa, sdev
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world != args.gpus:
            raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={self.world}")
        torch.cuda.set_device(self.local)
        if self.world > 1:
            import datetime
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", self.local))
        if self.rank == 0:
            qbuild.build()
            sdev.build()
        self.barrier()
        qsa.load()
        # L2 flush: write one buffer larger than L2, then read another, so L2 ends up
        # full of clean lines that belong to neither the inputs nor the outputs
        self.flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
        self.flush_sink = torch.empty((), dtype=torch.float32, device="cuda")

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_ms(self, x):
        return max_over_ranks(x, self.world, "cuda")

    def flush(self):
        self.flush_w.fill_(1)
        self.torch.sum(self.flush_r, dim=0, out=self.flush_sink)

    def timed(self, fn, k):
        """k timed calls of fn, each after an L2 flush, CUDA events on the current stream."""
        torch = self.torch
        stream = torch.cuda.current_stream()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        for a, b in evs:
            self.flush()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]


class Bench:
    """One workload resident in HBM: its caches, step inputs, workspace and outputs."""

    def __init__(self, env, wl):
        torch, qsa, sdev = env.torch, env.qsa, env.sdev
        self.env, self.wl = env, wl
        self.mode = qsa.QSA_MODE_PREFILL if wl.mode == "prefill" else qsa.QSA_MODE_DECODE
        self.dims = qsa.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.kv_capacity)
        self.dw = sdev.DeviceWorkload(wl)
        st0 = wl.steps[0]
        zeros = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
        # history: every block completed before the first step is already pooled
        qsa.qsa_pool_block_keys(self.dims, self.dw.idx_k, self.dw.pooled, zeros,
                                torch.tensor(st0.len_before, dtype=torch.int32, device="cuda"), max(st0.len_before))
        self.steps = [self.dw.step_tensors(i) for i in range(len(wl.steps))]
        self.n_q_unit = sum(T["n_q"] for T in self.steps)
        ws_bytes = max(qsa.qsa_workspace_bytes(self.dims, T["n_q"], T["max_blocks"], self.mode) for T in self.steps)
        self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        qsa.qsa_workspace_init(self.ws)
        self.outs = [torch.empty((T["n_q"], wl.n_q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
                     for T in self.steps]
        self.sels = [torch.empty((T["n_q"], qsa.QSA_SEL_CAP), dtype=torch.int32, device="cuda") for T in self.steps]
        self.cnts = [torch.empty((T["n_q"],), dtype=torch.int32, device="cuda") for T in self.steps]

    def forward(self, T, out, sel, cnt, src=None):
        src = src or T
        dw = self.dw
        self.env.qsa.qsa_forward(
            self.dims, q=src["q"], k_cache=dw.k_cache, v_cache=dw.v_cache, idx_k=dw.idx_k, pooled=dw.pooled,
            q_idx=src["q_idx"], w=src["w"], len_before=src["len_before"], len_after=src["len_after"],
            q_seq=src["q_seq"], q_pos=src["q_pos"], n_q=T["n_q"], max_new_tokens=T["max_new_tokens"],
            max_blocks=T["max_blocks"], mode=self.mode, out=out, workspace=self.ws, sel_idx=sel, sel_cnt=cnt)

    def unit(self):
        """One unit of work: every step of the workload (one step for most workloads)."""
        for T, out, sel, cnt in zip(self.steps, self.outs, self.sels, self.cnts):
            self.forward(T, out, sel, cnt)

    def step_timing(self, args):
        """The unit as a CUDA graph (all lengths and positions are device-side), K timed
        replays with L2 flushed before each; returns (ms per unit, eager ms, graph)."""
        env, torch, qsa = self.env, self.env.torch, self.env.qsa
        for _ in range(max(args.warmup, 3)):
            self.unit()
        torch.cuda.synchronize()
        flags = qsa.qsa_read_device_status(self.ws)
        if flags:
            raise SystemExit(f"{self.wl.name}: device status flags {flags:#x} after warm-up")
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.unit()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        ms = env.max_ms(float(np.mean(env.timed(graph.replay, args.steps))))
        ms_eager = env.max_ms(float(np.mean(env.timed(self.unit, args.steps))))
        return ms, ms_eager, graph

    def kernels(self, args, hbm_peak, tc_peak, peak_kind, attn_sets):
        """Standalone timing of the two hot steps of the last step's inputs:
        selection (qsa_select_blocks: scores + top-512) and gathered attention
        (qsa_sparse_attn, the kernel the forward runs for this shape).  Decode
        attention is timed as `attn_sets` back-to-back launches on distinct query
        sets (distinct selections, so no launch finds another's rows in L2) in one
        CUDA graph, L2 flushed before each replay; per-launch time = replay / sets."""
        env, torch, qsa, sdev, wl = self.env, self.env.torch, self.env.qsa, self.env.sdev, self.wl
        si = len(self.steps) - 1
        T = self.steps[si]
        n_q, mb = T["n_q"], T["max_blocks"]
        res = {}
        sel = torch.empty((n_q, qsa.QSA_SEL_CAP), dtype=torch.int32, device="cuda")
        cnt = torch.empty((n_q,), dtype=torch.int32, device="cuda")
        run_sel = lambda: qsa.qsa_select_blocks(self.dims, T["q_idx"], T["w"], self.dw.pooled, T["q_seq"],
                                                 T["q_pos"], n_q, mb, self.mode, sel, cnt, self.ws)
        run_sel()
        sel_ms = env.max_ms(float(np.mean(env.timed(run_sel, args.steps))))
        assert torch.equal(sel, self.sels[si]) and torch.equal(cnt, self.cnts[si])
        flops, pbytes = select_work_of(wl, si)
        res["select_us"] = 1e3 * sel_ms
        if self.mode == qsa.QSA_MODE_PREFILL:
            ach = flops / (sel_ms / 1e3) / 1e12
            res["roofline_select"] = {"kernels": "k_prefill_scores_tc (sampling + main), k_prefill_finish, "
                                                 "k_prefill_fallback", "bound": "tensor",
                                      "achieved": round(ach, 1), "peak": tc_peak, "unit": "TFLOP/s",
                                      "frac": round(ach / tc_peak, 4),
                                      "peak_source": f"{peak_kind} bf16_tflops (burst)", "flops_per_call": flops}
        else:
            ach = pbytes / (sel_ms / 1e3) / 1e9
            res["roofline_select"] = {"kernels": "k_score_decode (+ k_topk_collect beyond 16,384 blocks)",
                                      "bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                                      "frac": round(ach / hbm_peak, 4),
                                      "peak_source": f"{peak_kind} hbm_gbs (burst copy)",
                                      "algorithmic_bytes_per_call": pbytes}

        # attention: `sets` query sets with their own selections
        sets = attn_sets if self.mode == qsa.QSA_MODE_DECODE else 1
        qs, sels, cnts, nbytes = [T["q"]], [self.sels[si]], [self.cnts[si]], 0
        toks = attended_tokens_of(wl, si, self.cnts[si].cpu().numpy())
        nbytes += attn_bytes_of(wl, toks)
        for r in range(1, sets):
            q = torch.empty_like(T["q"])
            q_idx = torch.empty_like(T["q_idx"])
            w = torch.empty_like(T["w"])
            qid0 = 1_000_000 * r
            sdev.fill_q(q, wl.seed, qid0)
            sdev.fill_q_idx(q_idx, wl.seed, qid0)
            sdev.fill_w(w, wl.seed, qid0)
            s_r = torch.empty_like(sel)
            c_r = torch.empty_like(cnt)
            qsa.qsa_select_blocks(self.dims, q_idx, w, self.dw.pooled, T["q_seq"], T["q_pos"], n_q, mb, self.mode,
                                  s_r, c_r, self.ws)
            qs.append(q)
            sels.append(s_r)
            cnts.append(c_r)
            nbytes += attn_bytes_of(wl, attended_tokens_of(wl, si, c_r.cpu().numpy()))
        out_k = torch.empty_like(self.outs[si])

        def attn_all():
            for q, s_r, c_r in zip(qs, sels, cnts):
                qsa.qsa_sparse_attn(self.dims, q, self.dw.k_cache, self.dw.v_cache, T["q_seq"], T["q_pos"], s_r,
                                    c_r, n_q, out_k, self.ws)
        attn_all()
        torch.cuda.synchronize()
        # the first set is the forward's own query set: same output
        qsa.qsa_sparse_attn(self.dims, qs[0], self.dw.k_cache, self.dw.v_cache, T["q_seq"], T["q_pos"], sels[0],
                            cnts[0], n_q, out_k, self.ws)
        res["attn_matches_forward"] = bool(torch.equal(out_k, self.outs[si]))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            attn_all()
        g.replay()
        torch.cuda.synchronize()
        attn_ms = env.max_ms(float(np.mean(env.timed(g.replay, args.steps)))) / sets
        del g
        res["attn_us"] = 1e3 * attn_ms
        res["attn_sets_per_graph"] = sets
        ach = (nbytes / sets) / (attn_ms / 1e3) / 1e9
        res["roofline_attention"] = {
            "kernel": "k_sparse_attn", "bound": "hbm",
            "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s", "frac": round(ach / hbm_peak, 4),
            "peak_source": f"{peak_kind} hbm_gbs (burst copy)", "algorithmic_bytes_per_launch": int(nbytes / sets)}
        if self.mode == qsa.QSA_MODE_PREFILL:
            # a block chosen by several queries of the chunk is gathered once per query
            blocks = torch.cat([s_r[s_r >= 0] for s_r in sels]).unique().numel()
            res["roofline_attention"]["unique_bytes"] = int(blocks * wl.block_size * wl.n_kv_heads * wl.head_dim * 4)
        return res

    def e2e(self, args):
        """End to end: host buffers in, host buffer out, copies inside the timed region.
        Every step's inputs travel in one pinned host buffer: queries, indexer inputs,
        positions, and the appended tokens' K/V rows and indexer keys, which are
        scattered into the caches on the device."""
        env, torch, dw = self.env, self.env.torch, self.dw
        e2e_steps = []
        for si, T in enumerate(self.steps):
            st = self.wl.steps[si]
            parts = {k: T[k] for k in ("q", "q_idx", "w", "len_before", "len_after", "q_seq", "q_pos")}
            new = [(s, a, b) for s, (a, b) in enumerate(zip(st.len_before, st.len_after)) if b > a]
            seq_i = torch.tensor([s for s, a, b in new for _ in range(a, b)], dtype=torch.int64, device="cuda")
            pos_i = torch.tensor([p for s, a, b in new for p in range(a, b)], dtype=torch.int64, device="cuda")
            parts["k_new"] = dw.k_cache[seq_i, :, pos_i].contiguous()
            parts["v_new"] = dw.v_cache[seq_i, :, pos_i].contiguous()
            parts["ik_new"] = dw.idx_k[seq_i, pos_i].contiguous()
            layout, off = {}, 0
            for k, v in parts.items():
                nb = v.numel() * v.element_size()
                layout[k] = (off, nb, v.dtype, tuple(v.shape))
                off += (nb + 255) // 256 * 256
            h_in = torch.empty(off, dtype=torch.uint8).pin_memory()
            for k, v in parts.items():
                o, nb, _, _ = layout[k]
                h_in[o:o + nb].copy_(v.reshape(-1).view(torch.uint8).cpu())
            d_in = torch.empty(off, dtype=torch.uint8, device="cuda")
            view = {k: d_in[o:o + nb].view(dt).view(shape) for k, (o, nb, dt, shape) in layout.items()}
            h_out = torch.empty(tuple(self.outs[si].shape), dtype=self.outs[si].dtype).pin_memory()
            e2e_steps.append((T, h_in, d_in, view, seq_i, pos_i, h_out))

        def unit_e2e():
            for (T, h_in, d_in, view, seq_i, pos_i, h_out), out, sel, cnt in zip(e2e_steps, self.outs, self.sels,
                                                                                  self.cnts):
                d_in.copy_(h_in, non_blocking=True)
                dw.k_cache[seq_i, :, pos_i] = view["k_new"]
                dw.v_cache[seq_i, :, pos_i] = view["v_new"]
                dw.idx_k[seq_i, pos_i] = view["ik_new"]
                self.forward(T, out, sel, cnt, src=view)
                h_out.copy_(out, non_blocking=True)

        for _ in range(3):
            unit_e2e()
        torch.cuda.synchronize()
        graph_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_e2e):
            unit_e2e()
        e2e_ms = []
        for _ in range(args.steps):
            env.flush()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            graph_e2e.replay()
            torch.cuda.current_stream().synchronize()
            e2e_ms.append(1e3 * (time.perf_counter() - t0))
        del graph_e2e
        e2e_ms = env.max_ms(float(np.mean(e2e_ms)))
        h2d = sum(x[1].numel() for x in e2e_steps)
        d2h = sum(x[6].numel() * x[6].element_size() for x in e2e_steps)
        return {"value": job_tokens_per_s(env.world, self.n_q_unit, e2e_ms), "unit": "tokens/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "timing": "host wall clock around one CUDA-graph replay of: one H2D copy of the step's inputs from "
                          "pinned memory, scatter of the appended K/V/indexer rows, qsa_forward, D2H copy of the "
                          "output, stream sync"}


def serving_modes(env, args):
    """Serving shapes on the headline's geometry (16 sequences at 64K context, 32 / 4
    heads), each timed like the headline (CUDA-graph replays of qsa_forward, L2
    flushed before each): 4 draft queries per sequence sharing one selection
    (multi-token prediction), and the K/V caches held in 256-token pages at a random
    page order."""
    torch, qsa, sdev = env.torch, env.qsa, env.sdev
    from qsa_synth import workloads as W
    out = {}
    for name, k, page_tokens in (("mtp4_decode_64k_b16", 4, 0), ("paged256_decode_64k_b16", 1, 256)):
        cap, batch = 65536, 16
        t0 = cap - k
        q_seq = [s for s in range(batch) for _ in range(k)]
        q_pos = [t0 + j for _ in range(batch) for j in range(k)]
        wl = W.Workload(name, 201 + k, "decode", batch, 32, 4, cap,
                        [W.Step([t0] * batch, [cap] * batch, q_seq, q_pos, list(range(len(q_pos))))])
        dw = sdev.DeviceWorkload(wl)
        zeros = torch.zeros(batch, dtype=torch.int32, device="cuda")
        dims = qsa.make_dims(batch, 32, 4, cap, block_size=wl.block_size, top_k=wl.top_k)
        qsa.qsa_pool_block_keys(dims, dw.idx_k, dw.pooled, zeros,
                                torch.tensor([t0] * batch, dtype=torch.int32, device="cuda"), t0)
        T = dw.step_tensors(0)
        n = T["n_q"]
        kc, vc, table, n_pages = dw.k_cache, dw.v_cache, None, 0
        if page_tokens:
            B, H, Tt, D = dw.k_cache.shape
            per_seq = Tt // page_tokens
            n_pages = B * per_seq
            perm = torch.tensor(np.random.default_rng(7).permutation(n_pages).reshape(B, per_seq).astype(np.int32),
                                device="cuda")
            kc = torch.empty((n_pages, H, page_tokens, D), dtype=torch.bfloat16, device="cuda")
            vc = torch.empty_like(kc)
            kc[perm.long().reshape(-1)] = dw.k_cache.view(B, H, per_seq, page_tokens, D).permute(0, 2, 1, 3, 4).reshape(-1, H, page_tokens, D)
            vc[perm.long().reshape(-1)] = dw.v_cache.view(B, H, per_seq, page_tokens, D).permute(0, 2, 1, 3, 4).reshape(-1, H, page_tokens, D)
            table = perm
            del dw.k_cache, dw.v_cache
            torch.cuda.empty_cache()
        ws = torch.empty(qsa.qsa_workspace_bytes(dims, n, T["max_blocks"], qsa.QSA_MODE_DECODE), dtype=torch.uint8,
                         device="cuda")
        qsa.qsa_workspace_init(ws)
        o = torch.empty((n, 32, 128), dtype=torch.bfloat16, device="cuda")
        sel = torch.empty((n // k, qsa.QSA_SEL_CAP), dtype=torch.int32, device="cuda")
        cnt = torch.empty((n // k,), dtype=torch.int32, device="cuda")
        q_idx, w = T["q_idx"][::k].contiguous(), T["w"][::k].contiguous()

        def fwd():
            qsa.qsa_forward(dims, q=T["q"], k_cache=kc, v_cache=vc, idx_k=dw.idx_k, pooled=dw.pooled, q_idx=q_idx,
                            w=w, len_before=T["len_before"], len_after=T["len_after"], q_seq=T["q_seq"],
                            q_pos=T["q_pos"], n_q=n, max_new_tokens=T["max_new_tokens"], max_blocks=T["max_blocks"],
                            mode=qsa.QSA_MODE_DECODE, out=o, workspace=ws, sel_idx=sel, sel_cnt=cnt, group_q=k,
                            page_table=table, page_tokens=page_tokens, n_pages=n_pages)
        for _ in range(max(args.warmup, 3)):
            fwd()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fwd()
        g.replay()
        torch.cuda.synchronize()
        ms = env.max_ms(float(np.mean(env.timed(g.replay, args.steps))))
        del g
        out[name] = {"tokens_per_s": job_tokens_per_s(1, n, ms), "ms_per_unit": ms, "queries_per_unit": n,
                     "selections_per_unit": n // k, "draft_queries_per_selection": k, "page_tokens": page_tokens,
                     "device_status": qsa.qsa_read_device_status(ws)}
        del dw, kc, vc, ws
        torch.cuda.empty_cache()
    return out


ATTN_SETS = {"decode_8k_b1": 16, "decode_64k_b16": 8, "decode_1m_b4": 8}


def run_ours(args, wl):
    env = Env(args)
    torch, qsa = env.torch, env.qsa
    hbm_peak, tc_peak, peak_kind = load_peaks()

    B = Bench(env, wl)
    clocks = Clocks(env.local) if env.rank == 0 else None
    time.sleep(0.3)
    env.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    ms_per_step, ms_eager, graph = B.step_timing(args)
    torch.cuda.synchronize()
    env.barrier()
    wall = time.perf_counter() - wall0
    clk = clocks.stop() if clocks else None
    value = job_tokens_per_s(env.world, B.n_q_unit, ms_per_step)
    del graph
    kern = B.kernels(args, hbm_peak, tc_peak, peak_kind, ATTN_SETS.get(wl.name, 4))
    kern["step_eager_us"] = 1e3 * ms_eager
    e2e = B.e2e(args)
    flags = qsa.qsa_read_device_status(B.ws)
    roofline = dict(kern["roofline_attention"])
    roofline["traffic"] = load_traffic(roofline["kernel"], wl.name)
    launches_per_step = sum(forward_launches(wl, B.mode == qsa.QSA_MODE_PREFILL, T) for T in B.steps)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": env.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded SplitMix64 inputs, integer indexer inputs, approx. N(0,1) Q/K/V)",
            "config": dict(workload_config(wl), parallelism=f"replicas x{env.world} (independent sequences per GPU)",
                           execution="CUDA graph of the unit's qsa_forward calls"),
            "roofline": roofline, "roofline_select": kern["roofline_select"],
            "kernels": {k: v for k, v in kern.items() if not k.startswith("roofline")}, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps, "clocks": clk,
            "wall_s_timed_region": round(wall, 4), "device_status": flags}
    if env.rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    del B
    torch.cuda.empty_cache()

    # every other synthetic configuration: its own step time, throughput and rooflines
    if args.workload_map and env.world == 1:
        from qsa_synth import workloads as W
        wmap = {}
        for f in W.ALL:
            other = f()
            if other.name == wl.name:
                continue
            Bo = Bench(env, other)
            steps = max(3, min(args.steps, 5)) if other.mode == "prefill" else args.steps
            a2 = argparse.Namespace(**dict(vars(args), steps=steps))
            ms, _, g = Bo.step_timing(a2)
            del g
            k2 = Bo.kernels(a2, hbm_peak, tc_peak, peak_kind, ATTN_SETS.get(other.name, 4))
            wmap[other.name] = {"tokens_per_s": job_tokens_per_s(1, Bo.n_q_unit, ms), "ms_per_unit": ms,
                                "queries_per_unit": Bo.n_q_unit, "steps_timed": steps,
                                "select_us": k2["select_us"], "attn_us": k2["attn_us"],
                                "roofline_select": k2["roofline_select"],
                                "roofline_attention": k2["roofline_attention"],
                                "device_status": qsa.qsa_read_device_status(Bo.ws)}
            del Bo
            torch.cuda.empty_cache()
        line["workloads"] = wmap
        line["serving_modes"] = serving_modes(env, args)
        line["workloads_note"] = ("each configuration measured alone on this GPU after the headline: CUDA-graph "
                                  "replays of its whole unit with L2 flushed before each; selection and attention "
                                  "timed through their standalone entry points")
    if env.rank == 0:
        print(json.dumps(line), flush=True)
    if env.world > 1:
        env.dist.destroy_process_group()


def main():
    args = parse()
    wl = workload_by_name(args.workload)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
