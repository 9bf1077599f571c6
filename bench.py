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
one JSON line.  `--impl reference` times the CPU oracle on the same workload.
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
    p.add_argument("--workload", default="decode_64k_b16")
    p.add_argument("--no-cpu-baseline", action="store_true")
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


def run_ours(args, wl):
    import torch
    import torch.distributed as dist
    import block_sparse_attention_key_b200 as qsa
    from block_sparse_attention_key_b200 import build as qbuild
    from qsa_synth import device as sdev

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_ms(x):
        return max_over_ranks(x, world, "cuda")

    if rank == 0:
        qbuild.build()
        sdev.build()
    barrier()
    qsa.load()

    mode = qsa.QSA_MODE_PREFILL if wl.mode == "prefill" else qsa.QSA_MODE_DECODE
    dims = qsa.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.kv_capacity)
    dw = sdev.DeviceWorkload(wl)
    # history: every block completed before the first step is already pooled
    st0 = wl.steps[0]
    zeros = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    qsa.qsa_pool_block_keys(dims, dw.idx_k, dw.pooled, zeros,
                            torch.tensor(st0.len_before, dtype=torch.int32, device="cuda"), max(st0.len_before))
    steps = [dw.step_tensors(i) for i in range(len(wl.steps))]
    n_q_unit = sum(T["n_q"] for T in steps)
    ws_bytes = max(qsa.qsa_workspace_bytes(dims, T["n_q"], T["max_blocks"], mode) for T in steps)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    qsa.qsa_workspace_init(ws)
    outs = [torch.empty((T["n_q"], wl.n_q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda") for T in steps]
    sels = [torch.empty((T["n_q"], wl.top_k), dtype=torch.int32, device="cuda") for T in steps]
    cnts = [torch.empty((T["n_q"],), dtype=torch.int32, device="cuda") for T in steps]
    # L2 flush: write one buffer larger than L2, then read another, so L2 ends up
    # full of clean lines that belong to neither the inputs nor the outputs
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_sink = torch.empty((), dtype=torch.float32, device="cuda")

    def flush():
        flush_w.fill_(1)
        torch.sum(flush_r, dim=0, out=flush_sink)

    def forward(T, out, sel, cnt, src=None):
        src = src or T
        qsa.qsa_forward(dims, q=src["q"], k_cache=dw.k_cache, v_cache=dw.v_cache, idx_k=dw.idx_k, pooled=dw.pooled,
                        q_idx=src["q_idx"], w=src["w"], len_before=src["len_before"], len_after=src["len_after"],
                        q_seq=src["q_seq"], q_pos=src["q_pos"], n_q=T["n_q"], max_new_tokens=T["max_new_tokens"],
                        max_blocks=T["max_blocks"], mode=mode, out=out, workspace=ws, sel_idx=sel, sel_cnt=cnt)

    def unit():
        """One unit of work: every step of the workload (one step for most workloads)."""
        for T, out, sel, cnt in zip(steps, outs, sels, cnts):
            forward(T, out, sel, cnt)

    def timed(fn, k):
        stream = torch.cuda.current_stream()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        for a, b in evs:
            flush()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    for _ in range(max(args.warmup, 3)):
        unit()
    torch.cuda.synchronize()
    flags = qsa.qsa_read_device_status(ws)
    if flags:
        raise SystemExit(f"device status flags {flags:#x} after warm-up")
    # the step as a CUDA graph: all lengths and positions are device-side, so it replays as is
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        unit()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()

    clocks = Clocks(local) if rank == 0 else None
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    ms = timed(graph.replay, args.steps)
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - wall0
    clk = clocks.stop() if clocks else None
    ms_per_step = max_ms(sum(ms) / len(ms))
    value = job_tokens_per_s(world, n_q_unit, ms_per_step)
    ms_eager = max_ms(float(np.mean(timed(unit, args.steps))))

    # ---- per-kernel breakdown through the standalone entry points (same inputs) ----
    T = steps[-1]
    n_q, mb = T["n_q"], T["max_blocks"]
    ld = (mb + 3) // 4 * 4
    scores = torch.empty((n_q, ld), dtype=torch.float32, device="cuda")
    out_k = torch.empty_like(outs[-1])
    sel_k, cnt_k = sels[-1].clone(), cnts[-1].clone()
    ws_k = torch.empty(qsa.qsa_workspace_bytes(dims, n_q, mb, 0), dtype=torch.uint8, device="cuda")
    qsa.qsa_workspace_init(ws_k)
    kernels = {}
    if mode == qsa.QSA_MODE_DECODE:
        run_score = lambda: qsa.qsa_index_scores(dims, T["q_idx"], T["w"], dw.pooled, T["q_seq"], T["q_pos"], n_q,
                                                  mb, scores, ld, ws_k)
        run_score()
        run_topk = lambda: qsa.qsa_topk_blocks(dims, scores, ld, T["q_pos"], n_q, mb, sel_k, cnt_k, ws_k)
        run_topk()  # first launch of its kernels outside the timing (module loading)
        kernels["index_scores_us"] = 1e3 * float(np.mean(timed(run_score, args.steps)))
        kernels["topk_us"] = 1e3 * float(np.mean(timed(run_topk, args.steps)))
    run_attn = lambda: qsa.qsa_sparse_attn(dims, T["q"], dw.k_cache, dw.v_cache, T["q_seq"], T["q_pos"], sel_k,
                                            cnt_k, n_q, out_k, ws_k)
    run_attn()
    attn_ms = float(np.mean(timed(run_attn, args.steps)))
    kernels["sparse_attn_us"] = 1e3 * attn_ms
    kernels["attn_matches_forward"] = bool(torch.equal(out_k, outs[-1]))
    kernels["step_eager_us"] = 1e3 * ms_eager

    # algorithmic bytes of the gathered attention: K+V rows of every attended token
    # (4 per selected block plus the partial block) for every KV head, q in, out written
    cnt_h = cnt_k.cpu().numpy().astype(np.int64)
    part = (np.asarray(wl.steps[-1].q_pos, dtype=np.int64) + 1) % wl.block_size
    toks = cnt_h * wl.block_size + part
    attn_bytes = int(toks.sum() * wl.n_kv_heads * wl.head_dim * 2 * 2 + 2 * n_q * wl.n_q_heads * wl.head_dim * 2)
    hbm_peak, tc_peak, peak_kind = load_peaks()
    achieved = attn_bytes / (attn_ms / 1e3) / 1e9
    roofline = {"kernel": "k_sparse_attn", "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                "peak_source": f"{peak_kind} hbm_gbs (burst copy)",
                "algorithmic_bytes_per_launch": attn_bytes, "traffic": load_traffic("k_sparse_attn", wl.name)}

    # ---- end to end: host buffers in, host buffer out, copies inside the timed region ----
    # Every step's inputs travel in one pinned host buffer: queries, indexer inputs,
    # positions, and the appended tokens' K/V rows and indexer keys, which are
    # scattered into the caches on the device.
    e2e_steps = []
    for si, T in enumerate(steps):
        st = wl.steps[si]
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
        h_out = torch.empty(tuple(outs[si].shape), dtype=outs[si].dtype).pin_memory()
        e2e_steps.append((T, h_in, d_in, view, seq_i, pos_i, h_out))

    def unit_e2e():
        for (T, h_in, d_in, view, seq_i, pos_i, h_out), out, sel, cnt in zip(e2e_steps, outs, sels, cnts):
            d_in.copy_(h_in, non_blocking=True)
            dw.k_cache[seq_i, :, pos_i] = view["k_new"]
            dw.v_cache[seq_i, :, pos_i] = view["v_new"]
            dw.idx_k[seq_i, pos_i] = view["ik_new"]
            forward(T, out, sel, cnt, src=view)
            h_out.copy_(out, non_blocking=True)

    for _ in range(3):
        unit_e2e()
    torch.cuda.synchronize()
    graph_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_e2e):
        unit_e2e()
    e2e_ms = []
    for _ in range(args.steps):
        flush()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        graph_e2e.replay()
        torch.cuda.current_stream().synchronize()
        e2e_ms.append(1e3 * (time.perf_counter() - t0))
    e2e_ms = max_ms(float(np.mean(e2e_ms)))
    h2d = sum(x[1].numel() for x in e2e_steps)
    d2h = sum(x[6].numel() * x[6].element_size() for x in e2e_steps)
    e2e = {"value": job_tokens_per_s(world, n_q_unit, e2e_ms), "unit": "tokens/s", "ms_per_step": e2e_ms,
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "timing": "host wall clock around one CUDA-graph replay of: one H2D copy of the step's inputs from "
                     "pinned memory, scatter of the appended K/V/indexer rows, qsa_forward, D2H copy of the "
                     "output, stream sync"}

    flags = qsa.qsa_read_device_status(ws)
    launches_per_step = sum(forward_launches(wl, mode == qsa.QSA_MODE_PREFILL, T) for T in steps)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded SplitMix64 inputs, integer indexer inputs, approx. N(0,1) Q/K/V)",
            "config": dict(workload_config(wl), parallelism=f"replicas x{world} (independent sequences per GPU)",
                           execution="CUDA graph of the unit's qsa_forward calls"),
            "roofline": roofline, "kernels": kernels, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps, "clocks": clk,
            "wall_s_timed_region": round(wall, 4), "device_status": flags}
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, graph_e2e
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    wl = workload_by_name(args.workload)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
