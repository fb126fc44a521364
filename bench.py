"""Benchmark of the block-sparse video attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload hunyuan|wan13b|wan14b|...] [--report [--only PREFIX]]

One step = one pass of the whole path over one attention call of the HunyuanVideo-720p-
shaped workload (B=1, 24 heads, d=128, 33x45x80 latent grid = 118,800 tokens in 2160 tiles;
every (head, query tile) keeps a budget of key tiles proportional to exp(entropy) of its
pooled-score softmax, normalised to 19% of all tile pairs, as the decayed window of the
largest radius that fits the budget topped up by pooled score): reorder Q, K, V to
tile-major, build the block mask, block-sparse attention with the output and LSE written
back in raster order. It is the largest of the benchmark's single-GPU calls at about 20%
retained tiles. Inputs are synthetic (seeded generator) and resident in HBM (2.2 GB of
raster Q/K/V, larger than the 126 MB L2) when the timed region starts.

The metric is effective TFLOP/s: 4*64*64*d FLOPs per retained (query tile, key tile) pair,
divided by the device time of the step; `ms_per_step` gives the time per call.
Under torchrun each rank runs its own copy of the call (independent problems, weak
scaling, no collective on the data path); the time is the max over ranks.

--impl reference times the CPU oracle (test infrastructure) on a bounded sample of the
same workload on the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "hunyuan"          # default; --workload picks another benchmark call
METRIC = "sparse-attn ms/call & effective TFLOP/s at ~20% tiles; % of B200 BF16 peak"
NOMINAL_BF16_TFLOPS = 2250.0


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="benchmark call of the step (hunyuan: tau = 0.19; wan13b, wan14b, wan5b, tiny)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--report", action="store_true",
                    help="per-stage timings of every benchmark workload (one JSON line each); "
                         "not the headline measurement")
    ap.add_argument("--only", default=None, help="with --report: workloads whose name starts with this")
    return ap.parse_args()


def _dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_scalar(x: float, op: str, world: int, device=None) -> float:
    """max or sum of a per-rank scalar over all ranks (identity on one rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(bf16=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"],
                    hbm=d["hbm_gbs"], source="measured")
    return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


def _tile_valid_counts(g):
    """Valid tokens of every tile (edge tiles of a grid that is not a multiple of 4 hold
    fewer than 64)."""
    import numpy as np
    nT, nY, nX = (g.T + 3) // 4, (g.Hs + 3) // 4, (g.Ws + 3) // 4
    vt = np.minimum(4, g.T - 4 * np.arange(nT))
    vy = np.minimum(4, g.Hs - 4 * np.arange(nY))
    vx = np.minimum(4, g.Ws - 4 * np.arange(nX))
    return (vt[:, None, None] * vy[None, :, None] * vx[None, None, :]).reshape(-1)


def _valid_token_flops(g, mask_i32):
    """4 d sum over retained (query tile, key tile) pairs of n_valid(q) n_valid(k): the
    FLOPs of the valid tokens only, printed beside the tile-granular headline."""
    import numpy as np
    bits = mask_i32.cpu().numpy().view(np.uint32)                   # [B, H, NQT, NW]
    nv = _tile_valid_counts(g).astype(np.float64)
    words = np.arange(g.NT) // 32
    sh = np.arange(g.NT) % 32
    keep = (bits[..., words] >> sh) & 1                              # [B, H, NQT, NKT]
    return 4.0 * g.d * float(np.einsum("bhqk,q,k->", keep.astype(np.float64), nv, nv))


def _mask_bytes(g):
    """Algorithmic bytes of the mask build from pooled means: qbar and kbar read once, the
    bitmask and kv_count written (the pooling itself rides on the reorder's pass)."""
    return 2 * g.B * g.H * g.NT * g.d * 4 + g.B * g.H * g.NT * (g.NW + 1) * 4


def _workload_text(w):
    grid = (f"B={w.B} heads={w.H} d={w.d} grid {w.T}x{w.Hs}x{w.Ws} ({w.N} tokens, "
            f"{w.NT} tiles of 4x4x4)")
    names = {"hunyuan": "HunyuanVideo-720p-shaped", "wan13b": "Wan-1.3B-480p-shaped",
             "wan14b": "Wan-14B-720p-shaped", "wan5b": "Wan2.2-5B-shaped", "tiny": "Tiny"}
    kinds = {0: "cube window", 1: "decayed window", 2: "token-level circular window"}
    if w.budget_mode == 1:
        rule = (f"entropy budget tau={w.budget_target} of key tiles per (head, query tile): "
                "decayed window of the largest radius that fits the budget, topped up by "
                "pooled score")
    elif w.budget_mode == 2:
        rule = (f"rho={w.dense_fraction} dense query tiles, {kinds[w.window_kind]} "
                f"r={w.radius} + tiles up to pooled mass theta={w.budget_target}")
    else:
        rule = (f"rho={w.dense_fraction} dense query tiles, {kinds[w.window_kind]} "
                f"r={w.radius} + top-{w.topk}")
    return f"{names.get(w.name, w.name)} attention call: {grid}, {rule}"


def _workload_desc(w, retention):
    raster_mb = 3 * w.B * w.N * w.H * w.d * 2 / 1e6
    return {
        "workload": _workload_text(w),
        "global_batch": w.B,
        "seq_len": w.N,
        "retained_tile_fraction": round(retention, 4),
        "l2": f"inputs larger than L2 (raster Q/K/V {raster_mb:.0f} MB > 126 MB)",
        "parallelism": "independent call per rank (weak scaling)",
    }


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region (rank 0)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpus):
        self.gpus = gpus
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", ",".join(str(g) for g in self.gpus)],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        with open(self.tmp.name) as f:
            lines = [ln.strip() for ln in f if ln.strip()]
        os.unlink(self.tmp.name)
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def _attn_source_hash():
    h = hashlib.sha256()
    for f in ("attn.cu", "sm100_ptx.cuh", "tmem_ops.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "block_sparse_attention_major_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic(workload):
    """DRAM bytes per attention launch from the committed ncu summary of this workload, if
    it is current."""
    p = os.path.join(ROOT, "profiles", f"attn_kernel_{workload}_traffic.json")
    if not os.path.exists(p):
        return None, "no ncu capture of this workload's attention launch"
    with open(p) as f:
        d = json.load(f)
    if d.get("attn_source_sha256_16") != _attn_source_hash():
        return None, "kernel changed since the ncu capture"
    return d.get("dram_bytes_per_launch"), d.get("source")


# ------------------------------------------------------------------------------ CPU oracle
def _oracle_sample(w, q, k, v, diff, head, n_rows, seconds):
    """Oracle path for one head, bounded in time: reorder and mask of the head (all its query
    tiles), then attention of seeded-shuffled query tiles of the head until `seconds` of
    attention have been spent (at least n_rows tiles).

    Returns (seconds charged, retained tile pairs attended, rows attended, setup seconds):
    the attention time plus the setup time in proportion to the head's retained pairs that
    were attended, so that attending every row would charge the whole setup."""
    import numpy as np
    from oracle import bsa_oracle as O
    t0 = time.perf_counter()
    qh, kh, vh = (O.to_f64(x[:, :, head:head + 1]) for x in (q, k, v))
    qt, kt, vt = (O.reorder(x, w.T, w.Hs, w.Ws) for x in (qh, kh, vh))
    m = O.build_mask(qt, kt, diff.numpy(), T=w.T, Hs=w.Hs, Ws=w.Ws, window_kind=w.window_kind,
                     radius=w.radius, topk=w.topk, dense_fraction=w.dense_fraction,
                     budget_mode=w.budget_mode, budget_target=w.budget_target)
    t_setup = time.perf_counter() - t0
    counts = m["mask"][0, 0].sum(-1)
    order = np.random.default_rng(7).permutation(w.NT)
    t_attn, pairs, n = 0.0, 0, 0
    while n < w.NT and (n < n_rows or t_attn < seconds):
        i = int(order[n])
        t1 = time.perf_counter()
        O.attention_tiles(qt, kt, vt, m["mask"], [(0, 0, i)], T=w.T, Hs=w.Hs, Ws=w.Ws)
        t_attn += time.perf_counter() - t1
        pairs += int(counts[i])
        n += 1
    return t_attn + t_setup * pairs / int(counts.sum()), pairs, n, t_setup


def _blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((x.get("num_threads", 1) for x in info if x.get("user_api") == "blas"), default=1)
    except Exception:
        return len(os.sched_getaffinity(0))


def run_reference(args):
    """Oracle timed on the host cores, rank 0 only.

    Setup (timed once): reorder of Q, K, V and the mask of head 0 of the call (the oracle's
    mask construction loops over every row in Python; one head keeps the run to minutes).
    Each step then attends a chunk of head 0's query tiles (a seeded shuffle), taking rows
    until the step's time budget of about 120 s / (steps + warmup) is used. A step is charged
    its attention time plus the setup time in proportion to the retained tile pairs it
    attended, so that attending every row of the head would charge the whole setup.
    """
    rank, world, _ = _dist_env()
    if rank != 0:
        return 0
    import numpy as np
    from bsa_synth import WORKLOADS, generate_difficulty, generate_qkv
    from oracle import bsa_oracle as O
    w = WORKLOADS[args.workload]
    q, k, v = generate_qkv(w)
    diff = generate_difficulty(w)
    t0 = time.perf_counter()
    qt, kt, vt = (O.reorder(O.to_f64(x[:, :, :1]), w.T, w.Hs, w.Ws) for x in (q, k, v))
    m = O.build_mask(qt, kt, diff.numpy(), T=w.T, Hs=w.Hs, Ws=w.Ws, window_kind=w.window_kind,
                     radius=w.radius, topk=w.topk, dense_fraction=w.dense_fraction,
                     budget_mode=w.budget_mode, budget_target=w.budget_target)
    t_setup = time.perf_counter() - t0
    counts = m["mask"].sum(-1)
    pairs_head = int(counts.sum())
    flop_pair = 4 * 64 * 64 * w.d
    rows = [(0, 0, i) for i in range(w.NT)]
    order = np.random.default_rng(7).permutation(len(rows))
    budget = min(5.0, max(0.05, 120.0 / (args.steps + args.warmup)))
    cursor = 0
    times, flops = [], []
    for s in range(args.warmup + args.steps):
        t_attn, pairs = 0.0, 0
        while t_attn < budget:
            b, h, i = rows[order[cursor % len(rows)]]
            cursor += 1
            t1 = time.perf_counter()
            O.attention_tiles(qt, kt, vt, m["mask"], [(b, h, i)], T=w.T, Hs=w.Hs, Ws=w.Ws)
            t_attn += time.perf_counter() - t1
            pairs += int(counts[b, h, i])
        if s >= args.warmup:
            times.append(t_attn + t_setup * pairs / pairs_head)
            flops.append(pairs * flop_pair)
    total_t = sum(times)
    value = sum(flops) / total_t / 1e12
    ms = 1e3 * total_t / len(times)
    sample = (f"oracle on head 0 of {w.H}: reorder + mask ({t_setup:.1f} s, charged to the steps "
              f"by retained pairs) and, per step, attention of seeded-shuffled query tiles of "
              f"head 0 for about {budget:.2f} s; value = FLOPs of the attended retained tile "
              "pairs / charged time")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _workload_desc(w, pairs_head / counts.size / w.NT),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------ GPU path
def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import block_sparse_attention_major_b200 as bsa
    from bsa_synth import WORKLOADS, generate_difficulty, generate_qkv

    rank, world, local = _dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_scalar(x, "max", world, dev)

    def sum_over_ranks(x: float) -> float:
        return reduce_scalar(x, "sum", world, dev)

    w = WORKLOADS[args.workload]
    q_h, k_h, v_h = generate_qkv(w)
    diff_h = generate_difficulty(w)
    g = bsa.Geometry(w.B, w.H, w.d, w.T, w.Hs, w.Ws)
    p = bsa.MaskParams(w.window_kind, w.radius, w.topk, w.dense_fraction, w.budget_mode,
                       w.budget_target)
    q, k, v, diff = (x.to(dev) for x in (q_h, k_h, v_h, diff_h))
    bufs = bsa.Buffers(g, dev)
    stream = torch.cuda.current_stream(dev)

    # one untimed call to learn the retained tile count (the mask is deterministic)
    bsa.forward(g, p, q, k, v, diff, bufs)
    torch.cuda.synchronize(dev)
    if bsa.read_error(bufs.ws) != 0:
        raise SystemExit("kernel error word set")
    retained = int(bufs.kv_count.sum().item())
    mask_snapshot = bufs.mask.clone()          # the dense comparison below rewrites the mask
    dense_pairs = g.B * g.H * g.NT * g.NT
    flops_call = 4.0 * 64 * 64 * g.d * retained
    retention = retained / dense_pairs

    # ---------------------------------------------------------------- device-timed steps
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    attn_ev = [(ev(), ev()) for _ in range(args.steps)]
    for _ in range(args.warmup):
        bsa.forward(g, p, q, k, v, diff, bufs)
    sampler = ClockSampler(list(range(world))) if rank == 0 else None
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    n0 = bsa.launch_count()
    t_start, t_end = ev(), ev()
    t_start.record(stream)
    for s in range(args.steps):
        bsa.reorder_pool(g, q, bufs.qt, bufs.qbar)
        bsa.reorder_pool(g, k, bufs.kt, bufs.kbar)
        bsa.reorder(g, v, bufs.vt)
        bsa.build_mask_pooled(g, p, bufs.qbar, bufs.kbar, diff, bufs.mask, bufs.kv_count, bufs.ws)
        attn_ev[s][0].record(stream)
        bsa.sparse_attn_fwd(g, bufs.qt, bufs.kt, bufs.vt, bufs.mask, bufs.kv_count, None,
                            bufs.out, bufs.lse, bufs.ws)
        attn_ev[s][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    launches = bsa.launch_count() - n0
    barrier()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end))
    attn_each = np.array([a.elapsed_time(b) for a, b in attn_ev])
    attn_ms = float(np.mean(attn_each))
    attn_pct = {f"p{q}": float(np.percentile(attn_each, q)) for q in (10, 50, 90)}
    attn_ms = max_over_ranks(attn_ms)
    ms_step = elapsed_ms / args.steps
    total_flops = sum_over_ranks(flops_call) * args.steps
    value = total_flops / (elapsed_ms * 1e-3) / 1e12
    if bsa.read_error(bufs.ws) != 0:
        raise SystemExit("kernel error word set")

    # ---------------------------------------------------------------- end to end (host buffers)
    # Every step copies its inputs from pinned host memory and reads its output and LSE back.
    # Two sets of device inputs and outputs let the copy in of step s+1 (one stream) and the
    # copy back of step s-1 (another stream) run on the copy engines while step s's kernels
    # run; events order every reuse of a buffer.
    e2e = None
    if not args.no_e2e:
        q_p, k_p, v_p, d_p = (x.pin_memory() for x in (q_h, k_h, v_h, diff_h))
        ins = [tuple(torch.empty_like(x, device=dev) for x in (q_h, k_h, v_h, diff_h)) for _ in range(2)]
        outb = [bufs, bsa.Buffers(g, dev)]
        outs = [(torch.empty(bufs.out.shape, dtype=bufs.out.dtype).pin_memory(),
                 torch.empty(bufs.lse.shape, dtype=bufs.lse.dtype).pin_memory()) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        e2e_steps = max(3, min(args.steps, 60))

        def e2e_run(n, start):
            s_in.wait_event(start)
            s_out.wait_event(start)
            computed, returned = [None, None], [None, None]
            for step in range(n):
                j = step % 2
                qd, kd, vd, dd = ins[j]
                with torch.cuda.stream(s_in):
                    if computed[j] is not None:          # step - 2 has read these inputs
                        s_in.wait_event(computed[j])
                    for dst, src in zip((qd, kd, vd, dd), (q_p, k_p, v_p, d_p)):
                        dst.copy_(src, non_blocking=True)
                    arrived = ev()
                    arrived.record(s_in)
                stream.wait_event(arrived)
                if returned[j] is not None:              # step - 2's output has been read back
                    stream.wait_event(returned[j])
                bsa.forward(g, p, qd, kd, vd, dd, outb[j])
                computed[j] = ev()
                computed[j].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(computed[j])
                    outs[j][0].copy_(outb[j].out, non_blocking=True)
                    outs[j][1].copy_(outb[j].lse, non_blocking=True)
                    returned[j] = ev()
                    returned[j].record(s_out)
            for r in returned:
                if r is not None:
                    stream.wait_event(r)

        w0 = ev()
        w0.record(stream)
        e2e_run(args.warmup, w0)
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        a, b = ev(), ev()
        a.record(stream)
        e2e_run(e2e_steps, a)
        b.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b))
        h2d = sum(x.numel() * x.element_size() for x in (q_h, k_h, v_h, diff_h))
        d2h = outs[0][0].numel() * outs[0][0].element_size() + outs[0][1].numel() * outs[0][1].element_size()
        e2e = {"value": sum_over_ranks(flops_call) * e2e_steps / (e2e_ms * 1e-3) / 1e12,
               "unit": "TFLOP/s", "ms_per_step": e2e_ms / e2e_steps,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "overlap": "copy in of step s+1 and copy back of step s-1 overlap step s's kernels"}
        if bsa.read_error(outb[1].ws) != 0:
            raise SystemExit("kernel error word set")
        del ins, outb

    # ---------------------------------------------------------------- own dense path (rho = 1)
    pd = bsa.MaskParams(w.window_kind, w.radius, w.topk, 1.0, 0, 0.0)
    bsa.build_mask(g, pd, bufs.qt, bufs.kt, diff, bufs.mask, bufs.kv_count, bufs.ws)
    for _ in range(3):
        bsa.sparse_attn_fwd(g, bufs.qt, bufs.kt, bufs.vt, bufs.mask, bufs.kv_count, None,
                            bufs.out, bufs.lse, bufs.ws)
    torch.cuda.synchronize(dev)
    a, b = ev(), ev()
    nd = 10
    a.record(stream)
    for _ in range(nd):
        bsa.sparse_attn_fwd(g, bufs.qt, bufs.kt, bufs.vt, bufs.mask, bufs.kv_count, None,
                            bufs.out, bufs.lse, bufs.ws)
    b.record(stream)
    torch.cuda.synchronize(dev)
    dense_ms = max_over_ranks(a.elapsed_time(b) / nd)
    dense_tflops = 4.0 * 64 * 64 * g.d * dense_pairs / (dense_ms * 1e-3) / 1e12

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = _peaks()
    # The sustained GEMM peak was reached at power-capped clocks; it is the denominator only
    # when this run was power-capped too (or clocked well below max), else the burst peak.
    capped = bool(clocks) and ("sw_power_cap" in clocks["reasons"]
                               or clocks["sm_mhz"] < 0.9 * clocks["sm_max_mhz"])
    peak_kind = "sustained" if capped else "burst"
    peak = peaks["bf16_sustained"] if capped else peaks["bf16"]
    other = peaks["bf16"] if capped else peaks["bf16_sustained"]
    attn_tflops = flops_call / (attn_ms * 1e-3) / 1e12
    valid_flops = _valid_token_flops(g, mask_snapshot)
    traffic, traffic_src = _traffic(args.workload)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": _workload_desc(w, retention),
        "attn_ms_per_call": attn_ms,
        "attn_ms_per_call_percentiles": attn_pct,
        "attn_effective_tflops": attn_tflops,
        "attn_valid_token_tflops": valid_flops / (attn_ms * 1e-3) / 1e12,
        "attn_frac_of_nominal_bf16_peak": attn_tflops / NOMINAL_BF16_TFLOPS,
        "dense_path": {"ms_per_call": dense_ms, "effective_tflops": dense_tflops,
                       "sparse_speedup": dense_ms / attn_ms},
        "roofline": {"kernel": "attn_kernel (+3 scheduler kernels in the same call)",
                     "bound": "tensor", "achieved": attn_tflops, "peak": peak,
                     "peak_kind": f"{peak_kind} bf16 GEMM, {peaks['source']}",
                     "unit": "TFLOP/s", "frac": attn_tflops / peak, "traffic": traffic,
                     "traffic_source": traffic_src,
                     "frac_of_other_peak": {"peak": other, "frac": attn_tflops / other,
                                            "kind": "burst" if capped else "sustained"}},
        "gpu_launches": launches,
        "clocks": clocks,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline and world == 1:
        t_cpu, pairs, n_rows, t_setup = _oracle_sample(w, q_h, k_h, v_h, diff_h, 0, 64, 8.0)
        line["cpu_baseline"] = {
            "value": pairs * 4.0 * 64 * 64 * w.d / t_cpu / 1e12, "unit": "TFLOP/s",
            "cores": _blas_threads(), "kind": "oracle",
            "sample": (f"oracle path for head 0 of {w.H}: reorder and mask of all {w.NT} query "
                       f"tiles ({t_setup:.1f} s, charged by the share of retained pairs "
                       f"attended), attention of {n_rows} seeded-shuffled query tiles: "
                       f"{pairs} retained tile pairs in {t_cpu:.1f} s charged")}
    print(json.dumps(line), flush=True)
    return 0


def _report_workloads():
    from bsa_synth import HUNYUAN_TAU_SWEEP, WAN5B_RHO_SWEEP, WORKLOADS
    out = [("tiny", WORKLOADS["tiny"]), ("wan13b", WORKLOADS["wan13b"])]
    out += [(f"wan5b_rho{r}", WORKLOADS["wan5b"].with_(dense_fraction=r)) for r in WAN5B_RHO_SWEEP]
    out.append(("wan14b", WORKLOADS["wan14b"]))
    out += [(f"hunyuan_tau{t}", WORKLOADS["hunyuan"].with_(budget_target=t)) for t in HUNYUAN_TAU_SWEEP]
    # cumulative-mass selection on the 1.3B-shaped call (its window and dense share)
    out += [(f"wan13b_mass{t}", WORKLOADS["wan13b"].with_(budget_mode=2, budget_target=t)) for t in (0.5, 0.8)]
    return out


def run_report(args):
    """Per-stage device times of every benchmark workload on one GPU."""
    import torch

    import block_sparse_attention_major_b200 as bsa
    from bsa_synth import generate_difficulty, generate_qkv

    dev = torch.device("cuda", 0)
    peaks = _peaks()
    torch.cuda.set_device(dev)
    cache = {}
    for name, w in _report_workloads():
        if args.only and not name.startswith(args.only):
            continue
        key = (w.H, w.d, w.T, w.Hs, w.Ws, w.seed, w.sink_frac)
        if key not in cache:
            cache.clear()
            cache[key] = tuple(x.to(dev) for x in (*generate_qkv(w), generate_difficulty(w)))
        q, k, v, diff = cache[key]
        g = bsa.Geometry(w.B, w.H, w.d, w.T, w.Hs, w.Ws)
        p = bsa.MaskParams(w.window_kind, w.radius, w.topk, w.dense_fraction, w.budget_mode,
                           w.budget_target)
        b = bsa.Buffers(g, dev)
        bsa.forward(g, p, q, k, v, diff, b)
        torch.cuda.synchronize()
        retained = int(b.kv_count.sum().item())
        valid_flops = _valid_token_flops(g, b.mask)
        stages = {"reorder_qkv": lambda: (bsa.reorder_pool(g, q, b.qt, b.qbar), bsa.reorder_pool(g, k, b.kt, b.kbar),
                                          bsa.reorder(g, v, b.vt)),
                  "build_mask": lambda: bsa.build_mask_pooled(g, p, b.qbar, b.kbar, diff, b.mask, b.kv_count, b.ws),
                  "sparse_attn": lambda: bsa.sparse_attn_fwd(g, b.qt, b.kt, b.vt, b.mask, b.kv_count, None,
                                                             b.out, b.lse, b.ws)}
        res, pct = {}, {}
        for st, fn in stages.items():
            for _ in range(max(3, args.warmup)):
                fn()
            n = max(5, min(args.steps, 30))
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
            torch.cuda.synchronize()
            for e0, e1 in evs:
                e0.record()
                fn()
                e1.record()
            torch.cuda.synchronize()
            each = [e0.elapsed_time(e1) for e0, e1 in evs]
            res[st] = sum(each) / n
            if st == "sparse_attn":
                srt = sorted(each)
                pct = {f"p{q}": srt[min(n - 1, int(round(q / 100 * (n - 1))))] for q in (10, 50, 90)}
        err = bsa.read_error(b.ws)
        flops = 4.0 * 64 * 64 * g.d * retained
        dense_pairs = g.B * g.H * g.NT * g.NT
        # own dense path: the same attention kernel with every tile retained
        pd = bsa.MaskParams(w.window_kind, max(w.radius, 0), w.topk, 1.0, 0, 0.0)
        bsa.build_mask(g, pd, b.qt, b.kt, diff, b.mask, b.kv_count, b.ws)
        for _ in range(2):
            bsa.sparse_attn_fwd(g, b.qt, b.kt, b.vt, b.mask, b.kv_count, None, b.out, b.lse, b.ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nd = 3
        torch.cuda.synchronize()
        e0.record()
        for _ in range(nd):
            bsa.sparse_attn_fwd(g, b.qt, b.kt, b.vt, b.mask, b.kv_count, None, b.out, b.lse, b.ws)
        e1.record()
        torch.cuda.synchronize()
        dense_ms = e0.elapsed_time(e1) / nd
        # raster read + tile-major write of Q, K, V, and the pooled means of Q and K
        qkv_bytes = 3 * (g.B * g.N * g.H * g.d * 2 + g.B * g.H * g.NT * 64 * g.d * 2) + 2 * g.B * g.H * g.NT * g.d * 4
        print(json.dumps({
            "workload": name, "B": g.B, "H": g.H, "d": g.d, "grid": [g.T, g.Hs, g.Ws], "tiles": g.NT,
            "retained_tile_fraction": retained / dense_pairs, "ms": res,
            "ms_step": sum(res.values()),
            # a step whose mask is rebuilt every m calls and reused in between (forward's
            # rebuild_mask): the measured stage times with the mask build amortised
            "ms_step_mask_rebuilt_every": {m: res["reorder_qkv"] + res["sparse_attn"] + res["build_mask"] / m
                                           for m in (1, 2, 4, 8)},
            "attn_effective_tflops": flops / (res["sparse_attn"] * 1e-3) / 1e12,
            "step_effective_tflops": flops / (sum(res.values()) * 1e-3) / 1e12,
            "reorder_gbs": qkv_bytes / (res["reorder_qkv"] * 1e-3) / 1e9,
            "reorder_frac_of_8tbs": qkv_bytes / (res["reorder_qkv"] * 1e-3) / 8e12,
            "reorder_frac_of_measured_copy": qkv_bytes / (res["reorder_qkv"] * 1e-3) / (peaks["hbm"] * 1e9),
            "mask_gbs": _mask_bytes(g) / (res["build_mask"] * 1e-3) / 1e9,
            "mask_frac_of_8tbs": _mask_bytes(g) / (res["build_mask"] * 1e-3) / 8e12,
            "attn_valid_token_tflops": valid_flops / (res["sparse_attn"] * 1e-3) / 1e12,
            "attn_ms_percentiles": pct,
            "dense_ms": dense_ms,
            "dense_effective_tflops": 4.0 * 64 * 64 * g.d * dense_pairs / (dense_ms * 1e-3) / 1e12,
            "sparse_speedup_vs_own_dense": dense_ms / res["sparse_attn"],
            "kernel_error_word": err}), flush=True)
        del b
        torch.cuda.empty_cache()
    return 0


def main():
    args = _args()
    if args.impl == "reference":
        return run_reference(args)
    if args.report:
        return run_report(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
