"""Benchmark of one sparse-layer decode step (indexer + top-512 + gathered GQA).

Workload: batch 64, 131,072 cached tokens per sequence, one query token each
(64 query heads sharing 4 KV groups of dimension 192, bf16 KV in 64-token
pages, an integer-valued 256-wide bf16 key for each 8-token block), seeded
synthetic data.
A step is s5_index_score_topk followed by s5_sparse_gqa_attn on resident
inputs.  Metric: algorithmic bytes of the step (selected KV + scored block
keys + queries / outputs) per second, with queries/s beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own replica (weak scaling; no collective
on the data path); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_gqa_indexer_b200 import roofline as R  # noqa: E402
from block_sparse_gqa_indexer_b200 import synth as S  # noqa: E402

METRIC = "sparse-layer decode selected-KV GB/s (% HBM peak) & queries/s, B=64, 128K ctx"
UNIT = "GB/s"
N_ROT = 4  # rotating query sets: each step selects different blocks
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _workload(rank: int = 0, batch: int = 64, world: int = 1) -> S.Workload:
    """This rank's shard of a global batch of batch * world sequences (every
    sequence has 131,072 cached tokens and one query token)."""
    (w,) = S.config_workloads(0)
    w.ctx, w.nq = [w.ctx[0]] * (batch * world), [1] * (batch * world)
    return S.shard(w, rank, world)


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _step_bytes(w: S.Workload) -> dict:
    sp = R.sparse_decode_bytes(w.ctx, w.nq)
    # split into the two calls of the step
    keys = sp["keys"] + w.total_q * (R.index_key_bytes() + 4 * (R.TOPK + 1))  # keys + q_index + sel
    attn = sp["kv"] + w.total_q * (R.q_bytes() + R.out_bytes() + 4 * (R.TOPK + 1))
    return {"total": sp["total"], "index": keys, "attn": attn, "kv": sp["kv"], "keys": sp["keys"]}


# ---------------------------------------------------------------- clocks

CLOCK_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons during the timed
    loop, written to S5_CLOCKS_DIR (default: _clocks/ in the repository)."""

    def __init__(self, gpu_index: int):
        self.proc = None
        out_dir = os.environ.get("S5_CLOCKS_DIR") or os.path.join(ROOT, "_clocks")
        self.path = os.path.join(out_dir, f"clocks_rank{gpu_index}.csv")
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- CPU oracle leg

def _oracle_sample(w: S.Workload, rows):
    """Inputs of the oracle for `rows` of the workload, drawn on the host."""
    from oracle import s5_oracle as O
    seqs, pos = w.query_seq_pos()
    rt = torch.as_tensor(rows, dtype=torch.int64)
    qx = w.qx_rows(rt).double().numpy()
    q = w.q_rows(rt).double().numpy()
    items = []
    for i, r in enumerate(rows):
        s, t = seqs[r], pos[r]
        c = t // S.BLOCK
        kx = w.kx_blocks(s, torch.arange(c)).double().numpy()
        sel = O.index_topk_query(qx[i], kx, t)  # only to know which K/V rows to draw
        T = O.sparse_token_set(sel, t)
        kv_pos = torch.as_tensor(T)
        K = w.k_tokens(s, kv_pos).double().numpy()
        V = w.v_tokens(s, kv_pos).double().numpy()
        items.append((qx[i], kx, t, q[i], {int(p): j for j, p in enumerate(T)}, K, V))
    return items


class _RowsByPos:
    def __init__(self, table, rows):
        self.table, self.rows = table, rows

    def __getitem__(self, pos):
        return self.rows[[self.table[int(p)] for p in pos]]


def _oracle_time(items) -> float:
    """Wall time of the oracle (selection + sparse attention) over the sample."""
    from oracle import s5_oracle as O
    t0 = time.perf_counter()
    for qx, kx, t, q, table, K, V in items:
        sel = O.index_topk_query(qx, kx, t)
        O.sparse_attention_query(q, sel, t, _RowsByPos(table, K), _RowsByPos(table, V))
    return time.perf_counter() - t0


def _oracle_worker(batch, rows, repeats, barrier, results):
    """One process of the parallel oracle leg: draw the inputs of `rows`, wait
    for every worker, then run the oracle over them `repeats` times on one
    thread (BLAS limited to 1)."""
    import threadpoolctl
    with threadpoolctl.threadpool_limits(1):
        torch.set_num_threads(1)
        items = _oracle_sample(_workload(0, batch), rows)
        barrier.wait(timeout=600)
        t0 = time.time()
        for _ in range(repeats):
            _oracle_time(items)
        results.put((t0, time.time(), len(rows) * repeats))


def parallel_oracle(batch: int, rows: list, workers: int, repeats: int):
    """Run the oracle over `rows` of the bench workload in `workers` spawned
    processes (one thread each; rows dealt round-robin), all starting together.
    Returns (query rows processed, wall seconds from first start to last end)."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    barrier = ctx.Barrier(workers)
    results = ctx.Queue()
    procs = [ctx.Process(target=_oracle_worker, args=(batch, rows[k::workers], repeats, barrier, results))
             for k in range(workers)]
    for p in procs:
        p.start()
    got = [results.get(timeout=900) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    t0 = min(g[0] for g in got)
    t1 = max(g[1] for g in got)
    return sum(g[2] for g in got), t1 - t0


def cpu_baseline(w: S.Workload, repeats: int = 2) -> dict:
    """The oracle on the host cores: every query row of the workload, spread
    over one single-threaded process per core (at most one per row), each row
    evaluated `repeats` times (about 20 s of CPU work in all)."""
    rows = list(range(w.total_q))
    workers = max(1, min(os.cpu_count() or 1, len(rows)))
    n, dt = parallel_oracle(w.batch, rows, workers, repeats)
    b = R.sparse_decode_bytes([w.ctx[0]] * n, [1] * n)["total"]
    return {"value": b / dt / 1e9, "unit": UNIT, "cores": workers, "kind": "oracle",
            "sample": f"all {len(rows)} query rows x {repeats} (float64 numpy oracle: full-sort top-512 over 16,384 "
                      f"block scores + sparse attention) in {workers} single-threaded processes; {dt:.2f} s wall; "
                      "inputs drawn before timing",
            "queries_per_s": n / dt}


def bench_config(batch: int, n: int) -> dict:
    """The workload description both arms report."""
    return {"workload": f"sparse-layer decode: B={batch} per GPU, 131,072 cached tokens each, 1 query "
                        "token; 64 q heads / 4 KV groups / head dim 192; top-512 of 16,384 blocks + current "
                        "block",
            "batch": batch, "ctx": 131072, "topk": 512, "page": 64, "parallelism": f"replicas x{n}",
            "l2": "inputs larger than L2: each step reads 1.35 GB (806 MB selected KV + 537 MB block "
                  "keys) and rotates 4 query sets so consecutive steps select different blocks"}


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = _workload(0)
    per_step = 4
    n = (args.warmup + args.steps) * per_step
    rows = [(i * 7) % w.total_q for i in range(n)]
    items = _oracle_sample(w, rows)
    import threadpoolctl
    with threadpoolctl.threadpool_limits(1):  # the oracle as it stands, on one core
        for i in range(args.warmup):
            _oracle_time(items[i * per_step:(i + 1) * per_step])
        times = []
        for i in range(args.warmup, args.warmup + args.steps):
            times.append(_oracle_time(items[i * per_step:(i + 1) * per_step]))
    total = sum(times)
    b = R.sparse_decode_bytes([w.ctx[0]] * per_step, [1] * per_step)["total"]
    value = b * args.steps / total / 1e9
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(w.batch, args.gpus),
            "queries_per_s": per_step * args.steps / total,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{per_step} of the 64 query rows per step (float64 numpy oracle: full-sort "
                                       f"top-512 over 16,384 block scores + sparse attention) on one thread "
                                       f"(BLAS limited to 1), {args.steps} steps"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU leg

KERNEL_SOURCES = {
    "gqa_decode_kernel": ("attn_decode.cu", "s5_common.cuh", "s5_kernels.h"),
    "index_score_kernel": ("index_topk.cu", "s5_common.cuh", "s5_kernels.h"),
}


def src_hash(kernel: str) -> str:
    """Hash of the source files that define `kernel`."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_gqa_indexer_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def _ncu_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    sources have not changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel)
    if not e or e.get("src_hash") != src_hash(kernel):
        return None
    return e.get("bytes_per_launch")


def run_ours(args) -> None:
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)

    from block_sparse_gqa_indexer_b200 import s5
    w = _workload(rank, args.batch, world)
    pt = w.page_table()
    k_pool, v_pool = w.kv_pools(dev, pt)
    key_pool = w.index_pool(dev, pt)
    batch = s5.Batch.from_host(pt, w.ctx, w.nq, dev)
    ws = s5.new_workspace(batch, device=dev)
    tq = w.total_q
    qs, qxs = [], []
    for i in range(N_ROT):
        rows = torch.arange(tq, dtype=torch.int64) + i * tq * world  # a fresh query set per rotation
        qs.append(w.q_rows(rows, dev))
        qxs.append(w.qx_rows(rows, dev))
    sel = torch.empty((tq, S.TOPK), dtype=torch.int32, device=dev)
    cnt = torch.empty((tq,), dtype=torch.int32, device=dev)
    out = torch.empty((tq, 64, 192), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((tq, 64), dtype=torch.float32, device=dev)
    scale = 1.0 / (192 ** 0.5)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        if ev is not None:
            ev[0].record(stream)
        s5.s5_index_score_topk(key_pool, batch, qxs[i % N_ROT], S.TOPK, sel, cnt, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        s5.s5_sparse_gqa_attn(k_pool, v_pool, batch, qs[i % N_ROT], sel, cnt, S.TOPK, scale, out, lse, ws, stream)
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    code, info = s5.s5_get_device_error(ws)
    if code != 0:
        raise RuntimeError(f"device error after warm-up: {s5.s5_status_string(code)} row {info}")

    # ---- device-timed region: K steps back to back, nothing between the calls ----
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    time.sleep(0.3)
    t_start.record(stream)
    for i in range(args.steps):
        step(i)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if dist is not None:
        dist.barrier()
    ms = max_over_ranks(t_start.elapsed_time(t_end), dist, dev)

    # ---- per-call durations: the same steps again with an event around each call ----
    # (events between the calls stop the attention kernel from launching under the
    # select kernel's tail, so these durations include each call's launch latency)
    n_ev = min(args.steps, 1000)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_ev)]
    for i in range(n_ev):
        step(i, evs[i])
    torch.cuda.synchronize(dev)
    idx_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)

    # ---- end to end through the public API: per-step inputs from pinned host memory ----
    q_host = [x.cpu().pin_memory() for x in qs]
    qx_host = [x.cpu().pin_memory() for x in qxs]
    out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    lse_host = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    pipe = s5.SparseLayerPipeline(key_pool, k_pool, v_pool, batch, ws)
    e2e_steps = max(10, args.steps // 4)
    for i in range(3):
        pipe.step(q_host[i % N_ROT], qx_host[i % N_ROT], out_host, lse_host)
    pipe.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    for i in range(e2e_steps):
        pipe.step(q_host[i % N_ROT], qx_host[i % N_ROT], out_host, lse_host)
    pipe.s_out.wait_stream(pipe.s_comp)
    e1.record(pipe.s_out)
    pipe.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    code, info = s5.s5_get_device_error(ws)
    if code != 0:
        raise RuntimeError(f"device error: {s5.s5_status_string(code)} row {info}")

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return

    by = _step_bytes(w)
    n = world
    step_ms = ms / args.steps
    value = n * by["total"] * args.steps / (ms * 1e-3) / 1e9
    peak, peak_kind = _peaks()
    # dominant call of the step: the longer of the two, per launch of its main kernel
    if attn_ms >= idx_ms:
        dom, dom_ms, dom_bytes = "gqa_decode_kernel", attn_ms, by["attn"]
    else:
        dom, dom_ms, dom_bytes = "index_score_kernel", idx_ms, by["index"]
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    cpu = cpu_baseline(w) if (n == 1 and not args.no_cpu) else None
    launches_per_step = 3  # key scoring, select, attention (partitions merge inside the attention kernel)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": n, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": bench_config(w.batch, n),
        "queries_per_s": n * w.total_q * args.steps / (ms * 1e-3),
        "pct_hbm_peak": 100.0 * (by["total"] / (step_ms * 1e-3) / 1e9) / peak,
        "kernels_ms": {"s5_index_score_topk": idx_ms, "s5_sparse_gqa_attn": attn_ms,
                       "timing": f"CUDA events around each call over {n_ev} steps after the timed loop"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": f"{peak_kind} hbm_gbs (copy)",
                     "traffic": _ncu_traffic(dom), "algorithmic_bytes_per_launch": dom_bytes},
        "cpu_baseline": cpu,
        "e2e": {"value": n * by["total"] * e2e_steps / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
                "h2d_bytes_per_step": int(qs[0].numel() * 2 + qxs[0].numel() * 2),
                "d2h_bytes_per_step": int(out.numel() * 2 + lse.numel() * 4), "ms_per_step": e2e_ms / e2e_steps,
                "how": "s5.SparseLayerPipeline: per-step q / q_index copied in from pinned host memory and "
                       "out / lse copied back, overlapped with the previous step's compute"},
        "clocks": clk,
        "gpu_launches": launches_per_step * args.steps,  # timed loop only
    }
    print(json.dumps(line), flush=True)


def run_config(args) -> None:
    """Time one step of numbered configuration `args.config` (0..6) on this GPU and
    print a JSON line with its own bytes / FLOPs (a measurement aid; the bench
    line is the default mode).  The step and each call are captured in CUDA
    graphs and replayed, so small batches are timed on the device rather than
    by the host's launch rate.  Each step is timed twice: with a 512 MiB
    write between replays, which leaves none of the step's inputs in the
    126 MB L2 (``ms_per_step``, the HBM figure), and replayed back to back
    (``ms_per_step_warm``; inputs smaller than L2 then stay resident)."""
    from block_sparse_gqa_indexer_b200 import s5
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    layers = [S.shard(w, 0, args.shard) for w in S.config_workloads(args.config)]
    if args.ctx is not None:  # the same batch with another cached length (e.g. a smaller profiling case)
        for w in layers:
            w.ctx = [args.ctx] * w.batch
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / (192 ** 0.5)
    calls, kinds, bytes_total, flops_total = [], [], 0, 0
    for li, w in enumerate(layers):
        swa = (args.config == 2) or (args.config == 5 and li < 3)
        pt = w.page_table()
        kv8 = args.fp8_kv and not swa  # one-byte KV: sparse (full-attention) layers only
        if args.index_only and swa:
            continue
        if args.index_only:  # the indexer alone: no KV pools
            k_pool = v_pool = None
        else:
            k_pool, v_pool = w.kv_pools(dev, pt, window_only=S.WINDOW if swa else None, fp8=kv8)
        batch = s5.Batch.from_host(pt, w.ctx, w.nq, dev)
        ws = s5.new_workspace(batch, window=S.WINDOW, device=dev)
        q, qx = w.queries(dev)
        out = torch.empty((w.total_q, 64, 192), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.total_q, 64), dtype=torch.float32, device=dev)
        key_pool = None if swa else w.index_pool(dev, pt, fp8=args.fp8_keys)
        if args.append:
            # the step starts by storing its new tokens (and completed block
            # keys); the pools already hold these values, so every replay
            # writes the same bytes
            kn, vn, xn = w.new_tokens(dev)
            calls.append(lambda k=k_pool, v=v_pool, kp=key_pool, b=batch, kn=kn, vn=vn, xn=xn, ws=ws:
                         s5.s5_append_kv(k, v, kp, b, kn, vn, None if kp is None else xn, ws))
            kinds.append("append")
            bytes_total += R.append_bytes(w.ctx, w.nq, with_keys=not swa)["total"]
        # calls take the current stream, so the same lambdas run eagerly or under capture
        if swa:
            calls.append(lambda k=k_pool, v=v_pool, b=batch, q=q, o=out, l=lse, ws=ws:
                         s5.s5_swa_gqa_attn(k, v, b, q, S.WINDOW, scale, o, l, ws))
            kinds.append("swa")
            bytes_total += R.swa_decode_bytes(w.ctx, w.nq)["total"]
            flops_total += sum(R.attn_flops(R.swa_tokens(c + j)) for c, n in zip(w.ctx, w.nq) for j in range(n))
        elif args.grouped:
            # one indexer query and one selection per KV group
            ws = s5.new_workspace(batch, window=S.WINDOW, device=dev, grouped=True)
            qxg = w.qx_group_rows(torch.arange(w.total_q), dev).contiguous()
            sel = torch.empty((w.total_q, S.N_KV, S.TOPK), dtype=torch.int32, device=dev)
            cnt = torch.empty((w.total_q, S.N_KV), dtype=torch.int32, device=dev)
            calls.append(lambda kp=key_pool, b=batch, qx=qxg, sel=sel, cnt=cnt, ws=ws:
                         s5.s5_index_score_topk_grouped(kp, b, qx, S.TOPK, sel, cnt, ws))
            kinds.append("index_grouped")
            calls.append(lambda k=k_pool, v=v_pool, b=batch, q=q, sel=sel, cnt=cnt, o=out, l=lse, ws=ws:
                         s5.s5_sparse_gqa_attn_grouped(k, v, b, q, sel, cnt, S.TOPK, scale, o, l, ws))
            kinds.append("sparse_grouped")
            # the same KV and key bytes; 4 indexer queries and selections per token
            extra = w.total_q * (S.N_KV - 1) * (R.index_key_bytes() + 4 * (S.TOPK + 1))
            bytes_total += R.sparse_decode_bytes(w.ctx, w.nq)["total"] + extra
            flops_total += R.sparse_flops(w.ctx, w.nq)["attn"] + S.N_KV * R.sparse_flops(w.ctx, w.nq)["index"]
        else:
            sel = torch.empty((w.total_q, S.TOPK), dtype=torch.int32, device=dev)
            cnt = torch.empty((w.total_q,), dtype=torch.int32, device=dev)
            index_fn = s5.s5_index_score_topk_fp8 if args.fp8_keys else s5.s5_index_score_topk
            calls.append(lambda kp=key_pool, b=batch, qx=qx, sel=sel, cnt=cnt, ws=ws, f=index_fn:
                         f(kp, b, qx, S.TOPK, sel, cnt, ws))
            kinds.append("index_fp8keys" if args.fp8_keys else "index")
            sp = R.sparse_decode_bytes(w.ctx, w.nq)
            if args.index_only:
                # keys (at one or two bytes per value) + indexer queries + selections
                bytes_total += (sp["keys"] // 2 if args.fp8_keys else sp["keys"]) + w.total_q * (
                    R.index_key_bytes() + 4 * (R.TOPK + 1))
                flops_total += R.sparse_flops(w.ctx, w.nq)["index"]
                continue
            if kv8:
                calls.append(lambda k=k_pool, v=v_pool, b=batch, q=q, sel=sel, cnt=cnt, o=out, l=lse, ws=ws:
                             s5.s5_sparse_gqa_attn_fp8kv(k, v, b, q, sel, cnt, S.TOPK, scale, 1.0, 1.0, o, l, ws))
                kinds.append("sparse_fp8kv")
            else:
                calls.append(lambda k=k_pool, v=v_pool, b=batch, q=q, sel=sel, cnt=cnt, o=out, l=lse, ws=ws:
                             s5.s5_sparse_gqa_attn(k, v, b, q, sel, cnt, S.TOPK, scale, o, l, ws))
                kinds.append("sparse")
            # one-byte keys: the indexer reads half the key bytes; one-byte KV: half the KV bytes
            bytes_total += sp["total"] - (sp["keys"] // 2 if args.fp8_keys else 0) - (sp["kv"] // 2 if kv8 else 0)
            flops_total += R.sparse_flops(w.ctx, w.nq)["total"]
    for _ in range(args.warmup):
        for c in calls:
            c()
    torch.cuda.synchronize(dev)

    def capture(fns):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for f in fns:
                f()
        return g

    step_graph = capture(calls)
    call_graphs = [capture([c]) for c in calls]
    scratch = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush_graph = capture([lambda: scratch.fill_(1)])
    torch.cuda.synchronize(dev)

    def replay_ms(g, n):
        g.replay()  # warm
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(n):
            g.replay()
        t1.record(stream)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1) / n

    def replay_cold_ms(g, n):
        # the flush runs before each replay's start event, so the event pair
        # brackets the step alone, enqueued behind the flush
        n = min(n, 500)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for e0, e1 in evs:
            flush_graph.replay()
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)

    ms_warm = replay_ms(step_graph, args.steps)
    ms = replay_cold_ms(step_graph, args.steps)
    per_call = [replay_cold_ms(g, args.steps) for g in call_graphs]
    peak, kind = _peaks()
    line = {"config": args.config, "ms_per_step": ms, "calls_ms": dict(zip([f"{k}{i}" for i, k in enumerate(kinds)],
                                                                           per_call)),
            "ms_per_step_warm": ms_warm,
            "timing": "CUDA-graph replay of the step (and of each call), CUDA events; ms_per_step and calls_ms: "
                      "median over replays each preceded by a 512 MiB write (L2 flushed); ms_per_step_warm: "
                      "back-to-back replays",
            "algorithmic_bytes": bytes_total, "useful_flops": flops_total,
            "gbs": bytes_total / (ms * 1e-3) / 1e9, "pct_hbm_peak": 100 * bytes_total / (ms * 1e-3) / 1e9 / peak,
            "useful_tflops": flops_total / (ms * 1e-3) / 1e12, "steps": args.steps, "warmup": args.warmup,
            "gbs_warm": bytes_total / (ms_warm * 1e-3) / 1e9,
            "append": bool(args.append), "grouped": bool(args.grouped), "fp8_keys": bool(args.fp8_keys),
            "fp8_kv": bool(args.fp8_kv), "ctx_override": args.ctx, "index_only": bool(args.index_only)}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batch", type=int, default=64, help="sequences per GPU (64 = the stated workload)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle leg")
    ap.add_argument("--config", type=int, default=None,
                    help="time numbered configuration 0..6 (0: the bench workload) per call instead")
    ap.add_argument("--shard", type=int, default=1, help="with --config: run the first of this many batch shards")
    ap.add_argument("--append", action="store_true",
                    help="with --config: each layer step first appends its new tokens to the cache")
    ap.add_argument("--grouped", action="store_true",
                    help="with --config: sparse layers select per KV group (4 indexer queries per token)")
    ap.add_argument("--fp8-keys", action="store_true",
                    help="with --config: block keys stored as one-byte E4M3 codes")
    ap.add_argument("--index-only", action="store_true",
                    help="with --config: time the sparse layers' indexer call alone (no KV pools)")
    ap.add_argument("--ctx", type=int, default=None,
                    help="with --config: every sequence's cached tokens (default: the configuration's)")
    ap.add_argument("--fp8-kv", action="store_true",
                    help="with --config: the sparse layers' K/V stored as one-byte E4M3 codes")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.grouped and args.fp8_keys:
        ap.error("--grouped selection runs on bf16 block keys only")
    if args.append and args.fp8_keys:
        ap.error("the cache append writes bf16 block keys")
    if args.index_only and (args.grouped or args.append or args.fp8_kv):
        ap.error("--index-only times the shared indexer call alone")
    if args.fp8_kv and (args.grouped or args.append):
        ap.error("--fp8-kv runs the shared-selection sparse layer on a resident cache")
    if args.impl == "reference":
        args.steps = min(args.steps, 20)
        run_reference(args)
    elif args.config is not None:
        run_config(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
