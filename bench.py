"""Benchmark of the fused PISA forward (pyramid -> selection -> sparse attention).

Workload: GQA prefill, B=1, 32 query heads / 8 KV heads, N=131072, D=128,
block 64, factor 4, K=64, causal, iid N(0,1) inputs with 16 planted needle
blocks per KV head (bf16). One step = one pass of the whole path: key pyramid
(pisa_build_pyramid), query summaries + pyramid descent (pisa_select_blocks),
fused block-sparse attention (pisa_sparse_attention), on one stream, exactly
the kernel sequence pisa_forward enqueues, with CUDA events between the stages.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun each rank runs its own sequence (weak scaling, no data-path
collective); rank 0 prints one JSON line.

--impl reference times the CPU oracle (numpy) on a bounded sample of the same
workload and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

WORKLOAD = "gqa128k"
METRIC = "fused sparse-attn tokens/s at N=128K (PISA pyramid block-sparse attention forward)"
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # FFMA peak at the max SM clock (no measured figure)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_source_hash(sources) -> str:
    import hashlib
    h = hashlib.sha256()
    for src in sources:
        h.update(open(os.path.join(ROOT, src), "rb").read())
    return h.hexdigest()[:16]


ATTN_SOURCES = ("block_sparse_long_pisa_b200/csrc/attn_prefill.cu", "block_sparse_long_pisa_b200/csrc/pisa_device.cuh")


def attention_kernel_name(shape) -> str:
    """The prefill attention kernel the library launches for this shape: a CTA takes the largest
    divisor of the group whose rows fit two 128-row tiles (one for 128-key blocks; one head under
    per-query-head selection); units of at most 128 rows run two per CTA."""
    g = 1 if shape.select_per_qhead else shape.heads_q // shape.heads_kv
    max_rows = 128 if shape.block == 128 else 256
    gh = max(d for d in range(1, g + 1) if g % d == 0 and d * shape.block <= max_rows)
    nm = 2 if gh * shape.block > 128 else 1
    if nm == 1 and shape.n_qblocks >= 2:
        return f"attn_prefill_dual_kernel<{shape.head_dim},{shape.block}>"
    return f"attn_prefill_kernel<{shape.head_dim},{shape.block},{nm}>"


def profiled_traffic(kernel_file: str, sources) -> float | None:
    """dram bytes per full-size launch recorded from an ncu capture (profiles/<file>, JSON), or None
    when absent or when the kernel sources have changed since the capture (sha256 prefix recorded
    there)."""
    p = os.path.join(ROOT, "profiles", kernel_file)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("source_sha256_16") != kernel_source_hash(sources):
        return None
    v = rec.get("dram_bytes_per_launch_full_size")
    return float(v) if v is not None else None


# ----------------------------------------------------------------------------- ranks

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_workload(w, rank: int):
    """Weak scaling: rank r processes its own sequence (same shape, its own seed)."""
    return w.replace(seed=w.seed + 1000 * rank)


def max_over_ranks(value: float, world: int) -> float:
    """Slowest rank's time: every rank contributes its own CUDA-event measurement."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    on_gpu = dist.get_backend() == "nccl"
    t = torch.tensor([value], dtype=torch.float64, device="cuda" if on_gpu else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(tokens_per_rank: int, world: int, ms_step_max: float) -> float:
    """Weak scaling: every rank processes its own sequence; the job rate uses the slowest rank."""
    return tokens_per_rank * world / (ms_step_max / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.file.flush()
        rows = [r.split(",") for r in open(self.file.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if len(r) >= 9 and r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows if len(r) >= 9 for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- oracle timing

_PLANES = {}


def _oracle_planes(w):
    """Seeded input planes of KV head 0 and its query heads (generated once, not timed)."""
    key = (w.name, w.seed)
    if key not in _PLANES:
        k = workloads.plane_f32(w, "k", 0, 0)
        v = workloads.plane_f32(w, "v", 0, 0)
        q_heads = np.stack([workloads.plane_f32(w, "q", 0, h) for h in range(w.group)])
        _PLANES[key] = (k, v, q_heads)
    return _PLANES[key]


def oracle_sample(w, budget_s: float = 15.0) -> dict:
    """Time the CPU oracle on a bounded sample of the workload; extrapolate to tokens/s.

    Sample: the pyramid of one KV head (1/8 of the keys) and its query heads'
    summaries, then the pyramid descent and the attention (all query heads of the
    group) of seeded query blocks of that KV head, taken in a random order until
    the time budget is spent (a third of it for the descent, the rest for the
    attention). Whole-problem time = per-unit times x unit counts.
    """
    import oracle
    k, v, q_heads = _oracle_planes(w)
    t0 = time.perf_counter()
    levels = oracle.build_pyramid(k, w.block, w.factor)
    qbar = oracle.query_summary(q_heads, w.block)
    t_pool = time.perf_counter() - t0          # one KV head's keys + its group's queries
    nqb = w.seq_q // w.block
    rng = np.random.Generator(np.random.PCG64(0))
    order = [nqb - 1] + [int(x) for x in rng.permutation(nqb - 1)]
    sel, margin = {}, {}
    t0 = time.perf_counter()
    for i in order:
        r = oracle.select_blocks(qbar[i], levels, w.factor, w.topk, i if w.causal else nqb - 1)
        sel[i], margin[i] = r["idx"], r["margin"]
        if time.perf_counter() - t0 > budget_s / 3:
            break
    t_sel = (time.perf_counter() - t0) / len(sel)
    t0 = time.perf_counter()
    n_att = 0
    for i in sel:
        rows = np.arange(i * w.block, (i + 1) * w.block)
        for hh in range(w.group):
            oracle.attend(q_heads[hh, rows], rows, k, v, sel[i], w.block, bool(w.causal), 1 / np.sqrt(w.head_dim))
        n_att += 1
        if time.perf_counter() - t0 > budget_s * 2 / 3:
            break
    t_att = (time.perf_counter() - t0) / n_att
    units = w.batch * w.heads_kv
    total = units * t_pool + units * nqb * (t_sel + t_att)
    tokens = w.batch * w.seq_q
    try:
        import threadpoolctl
        cores = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()) or os.cpu_count()
    except Exception:
        cores = os.cpu_count()
    return {"value": tokens / total, "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
            "sample": (f"pyramid+summaries of 1/{units} of the keys ({t_pool:.2f}s), descent of {len(sel)} random "
                       f"query blocks ({t_sel * 1e3:.1f} ms each), attention of {n_att} of them x {w.group} heads "
                       f"({t_att * 1e3:.1f} ms each); extrapolated to {units} KV heads x {nqb} query blocks"),
            "seconds": round(t_pool + t_sel * len(sel) + t_att * n_att, 1),
            "estimated_full_seconds": round(total, 1),
            "_sample": {"levels": levels, "qbar": qbar, "sel": sel, "margin": margin}}


def check_sampled_selection(w, sample: dict, gpu_rows) -> dict:
    """The oracle rows the CPU-baseline sample computed (KV head 0 of batch 0) against the GPU's
    rows for the same query blocks: near-ties (oracle margin below 1e-3), rows that differ, and
    whether each differing row is one the descent reaches with its near-ties resolved the other
    way (checked by the oracle, outside every timed region)."""
    import oracle
    nqb = w.seq_q // w.block
    near = differ = admissible = 0
    for i, want in sample["sel"].items():
        near += sample["margin"][i] < oracle.NEAR_TIE_REL
        row = [int(x) for x in gpu_rows[i]]
        if row == list(want) + [-1] * (w.topk - len(want)):
            continue
        differ += 1
        ok, _ = oracle.selection_is_admissible(sample["qbar"][i], sample["levels"], w.factor, w.topk,
                                               i if w.causal else nqb - 1, row)
        admissible += ok
    return {"rows": len(sample["sel"]), "near_ties": int(near), "differ": differ, "differ_admissible": admissible,
            "sample": "the CPU baseline's descents (KV head 0, random query blocks) vs the GPU's rows"}


def needle_recall(w, idx_h) -> dict | None:
    """Planted needle blocks (16 per KV head) found in their target query block's selection."""
    if w.keys != "needle":
        return None
    found = planted = 0
    for b in range(w.batch):
        for kvh in range(w.heads_kv):
            for (i, j) in workloads.needles(w, b, kvh):
                planted += 1
                found += int(j in idx_h[b, kvh, i])
    return {"planted": planted, "selected": found, "recall": found / planted}


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = workloads.WORKLOADS[WORKLOAD]
    _oracle_planes(w)
    for _ in range(args.warmup):
        oracle_sample(w, budget_s=1.0)
    t0 = time.perf_counter()
    vals = [oracle_sample(w, budget_s=4.0) for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    for x in vals:
        x.pop("_sample")
    v = statistics.median([x["value"] for x in vals])
    base = dict(vals[-1])
    base["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall / max(args.steps, 1) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config_dict(w, args.gpus),
            "cpu_baseline": base, "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                          "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(w, n_gpus):
    return {"workload": f"{w.name}: GQA prefill B={w.batch} Hq={w.heads_q} Hkv={w.heads_kv} N={w.seq_kv} "
                        f"D={w.head_dim} block={w.block} factor={w.factor} K={w.topk} causal, iid N(0,1) bf16 "
                        f"+ 16 needles/KV head",
            "global_batch": w.batch * n_gpus, "seq_len": w.seq_kv, "parallelism": f"replicas x{n_gpus}",
            "l2": "inputs larger than L2 (Q 1.07 GB, K/V 268 MB each)"}


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(args, world, rank, local):
    import torch
    import block_sparse_long_pisa_b200 as pisa
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = rank_workload(bench_workload(args), rank)
    shape = pisa.Shape.of(w, select_per_qhead=int(args.per_qhead))
    q, k, v = (workloads.device_tensor(w, t, dev) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, dev)
    pyr = torch.empty(pisa.pyramid_size(shape) // 4, dtype=torch.float32, device=dev)
    idx = torch.empty((w.batch, shape.hsel, shape.n_qblocks, w.topk), dtype=torch.int32, device=dev)
    O = torch.empty_like(q)
    lse = torch.empty((w.batch, w.heads_q, w.seq_q), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches = [0]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        pisa.build_pyramid(shape, k, pyr)
        launches[0] += pisa.last_launch_count()
        if ev is not None:
            ev[1].record(stream)
        pisa.select_blocks(shape, q, pyr, ws, idx=idx)
        launches[0] += pisa.last_launch_count()
        if ev is not None:
            ev[2].record(stream)
        pisa.sparse_attention(shape, q, k, v, idx, ws, O=O, lse=lse)
        launches[0] += pisa.last_launch_count()
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws, "warmup")
    launches[0] = 0
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clock = ClockSampler(local)
    if rank == 0:
        clock.start()
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        step(events[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = clock.stop() if rank == 0 else None
    gpu_launches = launches[0]
    st, detail = pisa.check_status(ws)
    if st != pisa.OK:
        raise pisa.PisaError(st, "timed region", detail)
    ms_total = t_start.elapsed_time(t_end)
    ms_step = max_over_ranks(ms_total / args.steps, world)
    stage_ms = [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in events) for i in range(3)]

    # algorithmic work of this launch configuration
    idx_h = idx.cpu().numpy()
    attn_flops = pisa.attention_flops(idx_h, shape)
    sizes, _ = pisa.level_layout(shape)
    pool_bytes = (k.numel() * 2 + pisa.pyramid_size(shape))
    sel_bytes = (q.numel() * 2 + w.batch * shape.hsel * shape.n_qblocks * (w.head_dim * 4 + w.topk * 4))
    n_top_scored = scored_candidates(shape, sizes)
    sel_flops = 2.0 * w.head_dim * n_top_scored
    pk, how = peaks()
    hbm = pk["hbm_gbs"] * 1e9
    bf16 = pk["bf16_tflops"] * 1e12
    roof_s = pool_bytes / hbm + max(sel_bytes / hbm, sel_flops / (FP32_ALU_TFLOPS * 1e12)) + attn_flops / bf16
    attn_s = stage_ms[2] / 1e3
    achieved = attn_flops / attn_s / 1e12
    value = whole_job_tokens_per_s(w.batch * w.seq_q, world, ms_step)

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e = None
    if rank == 0 and not args.no_e2e:
        sess = pisa.Session(shape, dev)
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        hout = torch.empty(tuple(q.shape), dtype=torch.bfloat16).pin_memory()
        sess.forward(hq, hk, hv, out=hout)
        torch.cuda.synchronize()
        n_e2e = max(2, min(args.steps, 5))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            sess.forward(hq, hk, hv, out=hout)
        e1.record(stream)
        torch.cuda.synchronize()
        pisa.raise_on_device_error(sess.ws, "e2e")
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        e2e = {"value": w.batch * w.seq_q / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": (hq.numel() + hk.numel() + hv.numel()) * 2,
               "d2h_bytes_per_step": hout.numel() * 2, "ms_per_step": e2e_ms,
               "path": "Session.forward: pinned host Q/K/V -> device, pisa_forward, O -> pinned host"}

    # near-ties over every row from the library's own margins (outside the timed region)
    _, marg = pisa.select_blocks(shape, q, pyr, ws, margin=True)
    near_gpu = int((marg < 1e-3).sum().item())
    pisa.raise_on_device_error(ws, "margins")
    if rank != 0:
        return
    cpu = (oracle_sample(bench_workload(args))
           if world == 1 and not args.no_cpu_baseline and not args.per_qhead else None)
    near_ties = {"rows": int(marg.numel()), "gpu_margin_below_1e-3": near_gpu}
    if cpu is not None:
        near_ties["oracle_sample"] = check_sampled_selection(w, cpu.pop("_sample"), idx_h[0, 0])
    # the recorded ncu traffic belongs to the group-shared launch of the full-length 128K workload
    headline = args.workload == WORKLOAD and not args.seq and not args.per_qhead
    traffic = profiled_traffic("attn_prefill_gqa128k.json", ATTN_SOURCES) if headline else None
    config = config_dict(w, world)
    if args.per_qhead:
        config["workload"] += ", per-query-head selection"
    line = {
        "metric": METRIC + (" [per-query-head selection]" if args.per_qhead else ""), "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded numpy, bf16 RNE)",
        "config": config,
        "effective_tflops": attn_flops * world / (ms_step / 1e3) / 1e12,
        "fused_roofline_frac": roof_s / (ms_step / 1e3),
        "stages_ms": {"pyramid": stage_ms[0], "select": stage_ms[1], "attention": stage_ms[2]},
        "stage_roofline": {
            "pyramid_gbs": pool_bytes / (stage_ms[0] / 1e3) / 1e9,
            "select_gbs_qread": sel_bytes / (stage_ms[1] / 1e3) / 1e9,
            "attention_tflops": achieved,
        },
        "roofline": {"bound": "tensor",
                     "kernel": attention_kernel_name(shape), "achieved": achieved,
                     "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                     "peak_source": f"{how} bf16 dense (burst)", "traffic": traffic,
                     "flops_per_launch": attn_flops},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": gpu_launches, "clocks": clocks,
        "near_ties": near_ties, "needle_recall": None if args.per_qhead else needle_recall(w, idx_h),
    }
    print(json.dumps(line), flush=True)


def bench_workload(args):
    w = workloads.WORKLOADS[args.workload]
    if args.seq:  # decode keeps its single query token
        w = w.replace(seq_q=1 if w.decode else args.seq, seq_kv=args.seq, name=f"{w.name}@N={args.seq}")
    return w


def run_decode(args, world, rank, local):
    """Decode step: query summaries + pyramid descent + split-KV attention (pyramid prebuilt).

    Reported separately from the prefill line. The pyramid of the KV cache is built once
    before timing (a prefill-side cost). Roofline: HBM bytes of the selected K/V blocks
    plus the pyramid nodes the descent scores, plus q, o and the index rows.
    """
    import torch
    import block_sparse_long_pisa_b200 as pisa
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = rank_workload(bench_workload(args), rank)
    shape = pisa.Shape.of(w)
    q, k, v = (workloads.device_tensor(w, t, dev) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, dev)
    pyr = pisa.build_pyramid(shape, k)
    idx = torch.empty((w.batch, shape.hsel, 1, w.topk), dtype=torch.int32, device=dev)
    O = torch.empty_like(q)
    lse = torch.empty((w.batch, w.heads_q, 1), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches = [0]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        pisa.select_blocks(shape, q, pyr, ws, idx=idx)
        launches[0] += pisa.last_launch_count()
        if ev is not None:
            ev[1].record(stream)
        pisa.sparse_attention(shape, q, k, v, idx, ws, O=O, lse=lse)
        launches[0] += pisa.last_launch_count()
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    launches[0] = 0
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clock = ClockSampler(local)
    if rank == 0:
        clock.start()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s_ in range(args.steps):
        step(events[s_])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = clock.stop() if rank == 0 else None
    pisa.raise_on_device_error(ws, "decode")
    ms_step = max_over_ranks(t0.elapsed_time(t1) / args.steps, world)
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in events)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in events)
    n_sel = int((idx >= 0).sum().item())
    kv_bytes = n_sel * w.block * w.head_dim * 2 * 2
    sizes, _ = pisa.level_layout(shape)
    node_bytes = scored_candidates(shape, sizes) * w.head_dim * 4  # pyramid node vectors the descent reads
    small = q.numel() * 2 * 2 + idx.numel() * 4 + lse.numel() * 4
    pk, how = peaks()
    total_bytes = kv_bytes + node_bytes + small
    if rank != 0:
        return
    line = {
        "metric": "decode tokens/s (one query token per sequence, KV 131072)",
        "value": whole_job_tokens_per_s(w.batch, world, ms_step),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy, bf16 RNE)",
        "config": {"workload": f"{w.name}: {w.batch} sequences x 1 query token, KV {w.seq_kv}, Hq={w.heads_q} "
                               f"Hkv={w.heads_kv} D={w.head_dim} block={w.block} factor={w.factor} K={w.topk}, "
                               f"pyramid prebuilt", "global_batch": w.batch * world, "seq_len": w.seq_kv,
                   "parallelism": f"replicas x{world}"},
        "stages_ms": {"select": sel_ms, "attention": att_ms},
        "roofline": {"bound": "hbm", "achieved": total_bytes / (ms_step / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": total_bytes / (ms_step / 1e3) / 1e9 / pk["hbm_gbs"],
                     "bytes_per_step": total_bytes, "peak_source": f"{how} HBM copy", "traffic": None},
        "gpu_launches": launches[0], "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_backward(args, world, rank, local):
    """Backward step of the sparse attention (dQ, dK, dV through the forward's selection).

    Reported on its own line (not the forward's metric). Setup, outside the timed region: one
    forward for O, LSE and the selection, and a seeded dO. Algorithmic work: 10 * D flops per
    unmasked (query, key) pair (S, dP, dQ, dK and dV products once each; the kernels recompute
    S and dP in both passes, 14 * D actual).
    """
    import torch
    import block_sparse_long_pisa_b200 as pisa
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = rank_workload(bench_workload(args), rank)
    shape = pisa.Shape.of(w)
    q, k, v = (workloads.device_tensor(w, t, dev) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, dev)
    o, lse, idx = pisa.forward(shape, q, k, v, ws, idx=True)
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1000)
    do = torch.randn(tuple(q.shape), generator=g).to(torch.bfloat16).to(dev)
    bws = torch.zeros(pisa.backward_workspace_size(shape), dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream(dev)
    launches = [0]

    def step():
        pisa.sparse_attention_backward(shape, q, k, v, o, lse, do, idx, ws=bws, dQ=dq, dK=dk, dV=dv)
        launches[0] += pisa.last_launch_count()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    launches[0] = 0
    clock = ClockSampler(local)
    if rank == 0:
        clock.start()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = clock.stop() if rank == 0 else None
    pisa.raise_on_device_error(ws, "backward")
    ms_step = max_over_ranks(t0.elapsed_time(t1) / args.steps, world)
    pairs = pisa.attention_pairs(idx.cpu().numpy(), shape)
    flops = 10.0 * w.head_dim * pairs
    pk, how = peaks()
    achieved = flops / (ms_step / 1e3) / 1e12
    if rank != 0:
        return
    line = {
        "metric": f"sparse-attn backward tokens/s on {w.name} (dQ, dK, dV through the forward's selection)",
        "value": whole_job_tokens_per_s(w.batch * w.seq_q, world, ms_step),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy, bf16 RNE)", "config": config_dict(w, world),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / pk["bf16_tflops"], "flops_per_step": flops,
                     "peak_source": f"{how} bf16 dense (burst)", "traffic": None},
        "gpu_launches": launches[0], "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def scored_candidates(shape, sizes) -> int:
    """Candidates the descent scores for the whole problem (host count, no GPU data needed)."""
    f, K = shape.factor, shape.topk
    total = 0
    nqb = shape.n_qblocks
    for i in range(nqb):
        last = i if (shape.causal and not shape.decode) else shape.n_blocks - 1
        width = [f ** l for l in range(len(sizes))]
        l0 = next((l for l in range(len(sizes) - 1, -1, -1) if last // width[l] + 1 > K), -1)
        if l0 < 0:
            continue
        total += last // width[l0] + 1 + l0 * K * f
    return total * shape.batch * shape.hsel


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(workloads.WORKLOADS),
                    help="prefill workload to time (default: the N=128K GQA workload)")
    ap.add_argument("--seq", type=int, default=0, help="override the sequence length (smaller profiling cases)")
    ap.add_argument("--backward", action="store_true", help="time the backward step instead of the forward")
    ap.add_argument("--per-qhead", action="store_true",
                    help="forward with one selection per query head (select_per_qhead = 1); no CPU baseline")
    args = ap.parse_args()
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.backward:
            run_backward(args, world, rank, local)
        elif workloads.WORKLOADS[args.workload].decode:
            run_decode(args, world, rank, local)
        else:
            run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
