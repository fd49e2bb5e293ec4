"""Benchmark: one TurboQuant decode step per step, on B200.

Workload (Llama-3.1-8B-shaped single layer, the configuration the headline
metric is quoted on): batch 1, 32 query heads / 8 KV heads, head_dim 128,
32768 cached tokens; K and V are bf16 N(0,1) times a per-(head, channel)
LogNormal(0, 0.5) scale, compressed with TurboQuant_mse b=4.

A step is the whole hot path for one new token, one tq_append_decode_attention
call: encode the new token's K and V (norm, sign flips + FWHT, Lloyd-Max
indices, bit-packing) into the cache tail, then decode attention over all
32768 packed tokens (query rotation, scores from the codes, online softmax, PV
in the rotated basis, split merge, one inverse rotation).  value =
KV-tokens/s = B * N / step time.

The cache is replicated 8x (8 x 35.7 MB > 126 MB L2) and step s uses copy
s % 8, so every step streams its cache from HBM.  Steps are replayed from a
CUDA graph of 8 steps; the time is taken with CUDA events on the launching
stream, bracketed by a barrier and a device synchronize, max over ranks.

--impl reference times the CPU oracle (oracle/, NumPy) on a bounded sample of
the same step; that leg is the reported baseline, not the optimisation target.

Multi-GPU (torchrun): each rank runs an independent replica of the step on
its own GPU (the path shards by batch / KV head with no data exchange), so
scaling is weak and value sums the ranks' tokens over the slowest rank's time.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attention KV-tokens/s and encode vectors/s on 1 B200; % of HBM roofline"
B, HQ, HKV, D, N = 1, 32, 8, 128, 32768
KBITS, VBITS = 4, 4
COPIES = 8
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# DRAM bytes (read + write) of one decode split-kernel launch on this
# workload, from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum),
# reported only while the decode source is the one it was taken on.
TRAFFIC = {"bytes": 35774976, "source_sha256": "f9f3e6ad80b24e86ffc882a923d0c951bb453cd93ac53a7431e927a72c738390"}


def traffic_bytes():
    import hashlib
    with open(os.path.join(ROOT, "kv_cache_vector_13_b200", "csrc", "tq_decode.cu"), "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    return TRAFFIC["bytes"] if h == TRAFFIC["source_sha256"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup(backend="nccl"):
    """(rank, local rank, world size) from the torchrun environment; joins the
    process group when there is more than one rank (short timeout, so ranks
    that wait on a missing peer end with an error)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws == 1:
        return 0, 0, 1
    import datetime
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), device_id=None)
    return rank, local, ws


def max_over_ranks(times, dist, device):
    """Element-wise maximum of a list of times over all ranks (every rank
    gets the result); the identity without a process group."""
    if dist is None:
        return list(times)
    import torch
    tt = torch.tensor(times, device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return tt.tolist()


def job_value(world_size, ms_per_step):
    """Whole-job KV-tokens/s: every rank decodes B * N tokens per step, and
    the job's step time is the slowest rank's."""
    return world_size * B * N / (ms_per_step * 1e-3)


# ------------------------------------------------------------------ our leg

def run_ours(args):
    import torch
    from kv_cache_vector_13_b200 import api, inputs

    rank, local, ws = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if ws > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()

    kq = api.Quantizer(D, KBITS, "mse", seed_rot=10, device=dev)
    vq = api.Quantizer(D, VBITS, "mse", seed_rot=11, device=dev)
    K, V = inputs.llama8b_kv(N=N, seed=2 + rank, device=dev)
    kc0, vc0 = api.encode(kq, K), api.encode(vq, V)
    del K, V

    def clone(c):
        return api.PackedCache(*(None if t is None else t.clone() for t in (c.codes, c.norms, c.qjl, c.rnorms)))

    kcs = [kc0] + [clone(kc0) for _ in range(COPIES - 1)]
    vcs = [vc0] + [clone(vc0) for _ in range(COPIES - 1)]
    g = torch.Generator(device=dev).manual_seed(100 + rank)
    q = torch.randn((B, HQ, D), generator=g, device=dev).to(torch.bfloat16)
    k_new = torch.randn((B, HKV, 1, D), generator=g, device=dev).to(torch.bfloat16)
    v_new = torch.randn((B, HKV, 1, D), generator=g, device=dev).to(torch.bfloat16)
    op = api.DecodeAttention(kq, vq, B, HQ, HKV, N, device=dev)
    tails = [(api.PackedCache(kc.codes[:, :, N - 1:N], kc.norms[:, :, N - 1:N]),
              api.PackedCache(vc.codes[:, :, N - 1:N], vc.norms[:, :, N - 1:N])) for kc, vc in zip(kcs, vcs)]
    stream = torch.cuda.Stream(device=dev)

    def step(c, decode_only=False):
        # one decode step: tq_append_decode_attention encodes the new token's
        # K and V into the cache tail and attends over the cache (four
        # kernels, each allowed to start while the one before it finishes)
        if decode_only:
            op(q, kcs[c], vcs[c], stream=stream)
        else:
            op.append_step(q, k_new, v_new, tails[c][0], tails[c][1], kcs[c], vcs[c], stream=stream)

    with torch.cuda.stream(stream):
        for s in range(max(args.warmup, 3)):
            step(s % COPIES)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for c in range(COPIES):
                step(c)
        graph_dec = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_dec, stream=stream):
            for c in range(COPIES):
                step(c, decode_only=True)
        for _ in range(2):
            graph.replay()
            graph_dec.replay()
        torch.cuda.synchronize()

    K_steps = args.steps
    reps, rem = divmod(K_steps, COPIES)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    with clocks:
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(reps):
                graph.replay()
            for c in range(rem):
                step(c)
            ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
    t_ms = ev0.elapsed_time(ev1)

    # the dominant kernels (prep + split of tq_decode_attention), live
    d_reps = max(1, reps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(d_reps):
            graph_dec.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    dec_ms = e0.elapsed_time(e1) / (d_reps * COPIES)

    # end to end through the public API with host buffers (pinned), per step:
    # H2D of the step's inputs (q, k_new, v_new), the step, D2H of the output
    # the step's inputs (q, k_new, v_new, all bf16) staged in one pinned host
    # buffer and one device buffer, so each step copies them with one H2D copy
    parts = (q, k_new, v_new)
    sizes = [t.numel() for t in parts]
    hin = torch.empty(sum(sizes), dtype=torch.bfloat16).pin_memory()
    din = torch.empty(sum(sizes), dtype=torch.bfloat16, device=dev)
    off = 0
    views = []
    for t, n in zip(parts, sizes):
        hin[off:off + n].copy_(t.reshape(-1).cpu())
        views.append(din[off:off + n].view(t.shape))
        off += n
    dq, dk, dv = views
    hout = torch.empty((B, HQ, D), dtype=torch.float32).pin_memory()
    e2e_steps = min(K_steps, 2000)

    def e2e_step(c):
        din.copy_(hin, non_blocking=True)
        op.append_step(dq, dk, dv, tails[c][0], tails[c][1], kcs[c], vcs[c], stream=stream)
        hout.copy_(op.out, non_blocking=True)

    # e2e: each step is one CUDA-graph replay of [H2D copy of the inputs from
    # pinned memory, tq_append_decode_attention, D2H copy of the output],
    # then a host synchronize (how a serving loop runs a decode step);
    # e2e_eager issues the same three calls without a graph
    with torch.cuda.stream(stream):
        for c in range(COPIES):
            e2e_step(c)
        torch.cuda.synchronize()
        e2e_graphs = []
        for c in range(COPIES):
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph, stream=stream):
                e2e_step(c)
            e2e_graphs.append(gph)
        for gph in e2e_graphs:
            gph.replay()
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        for s in range(e2e_steps):
            e2e_graphs[s % COPIES].replay()
            stream.synchronize()
    e2e_s = time.perf_counter() - t0
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        for s in range(e2e_steps):
            e2e_step(s % COPIES)
            stream.synchronize()
    e2e_eager_s = time.perf_counter() - t0
    barrier()

    t_ms, dec_ms, e2e_s, e2e_eager_s = max_over_ranks([t_ms, dec_ms, e2e_s, e2e_eager_s], dist, dev)

    enc_info = bench_encode(api, inputs, torch, dev, stream, args.encode_variant) if rank == 0 else None
    base = None
    if rank == 0 and not args.no_cpu_baseline:
        base = cpu_baseline_decode(budget_s=args.cpu_seconds)
    if rank == 0:
        pk, pk_kind = peaks()
        dec_bytes = B * HKV * N * (kq.record_bytes + vq.record_bytes) + q.numel() * 2 + B * HQ * D * 4
        achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
        ms_step = t_ms / K_steps
        val = job_value(ws, ms_step)
        line = {
            "metric": METRIC, "value": val, "unit": "KV-tokens/s", "n_gpus": ws, "steps": K_steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 encode; f16xf16->f32 mma decode",
            "data": "synthetic",
            "config": {"workload": "llama3.1-8b-shaped decode step (append 1 token + attend): B=1 Hq=32 Hkv=8 "
                                   "d=128 N=32768, K/V TurboQuant_mse b=4, randomized Hadamard",
                       "global_batch": B * ws, "seq_len": N, "parallelism": f"replicas x{ws}",
                       "l2": f"{COPIES} rotating cache copies ({COPIES * dec_bytes / 1e6:.0f} MB > 126 MB L2)"},
            "roofline": {"kernel": "tq_decode_attention (prep + split)", "bound": "hbm",
                         "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "peak_kind": pk_kind,
                         "bytes_per_launch": dec_bytes, "ms_per_launch": dec_ms,
                         "traffic": args.traffic if args.traffic is not None else traffic_bytes()},
            "encode": enc_info,
            "cpu_baseline": base,
            "e2e": {"value": ws * B * N * e2e_steps / e2e_s, "unit": "KV-tokens/s",
                    "h2d_bytes_per_step": hin.numel() * hin.element_size(),
                    "d2h_bytes_per_step": hout.numel() * 4, "steps": e2e_steps,
                    "mode": "per step: CUDA-graph replay of (H2D copy, tq_append_decode_attention, D2H copy), "
                            "host synchronize"},
            "e2e_eager": {"value": ws * B * N * e2e_steps / e2e_eager_s, "unit": "KV-tokens/s",
                          "mode": "the same three calls issued per step without a graph"},
            "gpu_launches": 4 * K_steps,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        del graph, graph_dec
        dist.barrier()
        dist.destroy_process_group()


def bench_encode(api, inputs, torch, dev, stream, variant="mse4"):
    """Encode throughput: 2^20 unit vectors, d=128, fp32 input (the encode
    sweep's d=128 cell), TurboQuant_mse b=4 (or TurboQuant_prod b=3 with
    variant="prod3"), 2 rotating input copies (1 GB > L2)."""
    n, d = 1 << 20, 128
    if variant == "prod3":
        qz = api.Quantizer(d, 3, "prod", seed_rot=0, seed_qjl=1, device=dev)
    else:
        qz = api.Quantizer(d, 4, "mse", seed_rot=0, device=dev)
    xs = [inputs.unit_vectors(n, d, seed=i, device=dev) for i in range(2)]
    outs = [api.empty_cache(qz, 1, 1, n, dev) for _ in range(2)]
    with torch.cuda.stream(stream):
        for i in range(3):
            api.encode(qz, xs[i % 2], out=outs[i % 2], stream=stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 50
        e0.record(stream)
        for i in range(reps):
            api.encode(qz, xs[i % 2], out=outs[i % 2], stream=stream)
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    byts = n * (d * 4 + qz.record_bytes)
    pk, _ = peaks()
    gbs = byts / (ms * 1e-3) / 1e9
    name = "TurboQuant_prod b=3" if variant == "prod3" else "TurboQuant_mse b=4"
    return {"workload": f"2^20 unit vectors d=128 fp32, {name}", "vectors_per_s": n / (ms * 1e-3),
            "ms_per_launch": ms, "bytes_per_launch": byts, "achieved_gbs": gbs, "frac": gbs / pk["hbm_gbs"]}


# ------------------------------------------------------------- CPU oracle

def cpu_baseline_decode(budget_s=15.0, steps=None):
    """Time the oracle on a bounded sample of the step: for one KV head (4
    query heads) of the 8, encode the new token and attend over the 32768
    tokens; repeat over KV heads until ``budget_s`` of CPU work, and scale
    the rate to the full layer (8 KV heads)."""
    import numpy as np
    import torch
    from kv_cache_vector_13_b200 import inputs
    from oracle import attention as OA
    from oracle import quantizer as OQ
    try:
        from threadpoolctl import threadpool_info
        blas_threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        blas_threads = 1
    cores = len(os.sched_getaffinity(0))
    kq = OQ.Quantizer(D, KBITS, "mse", seed_rot=10)
    vq = OQ.Quantizer(D, VBITS, "mse", seed_rot=11)
    K, V = inputs.llama8b_kv(N=N, seed=2, H=1, device="cpu")
    Kh = K[0, 0].float().numpy()
    Vh = V[0, 0].float().numpy()
    kc = {k: v[None, None] for k, v in OQ.encode(kq, Kh, aux=False).items()}
    vc = {k: v[None, None] for k, v in OQ.encode(vq, Vh, aux=False).items()}
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, HQ // HKV, D)).astype(np.float32)
    knew = rng.standard_normal((1, D)).astype(np.float32)
    done, t0 = 0, time.perf_counter()
    n_steps = 0
    while True:
        OQ.encode(kq, knew, aux=False)
        OQ.encode(vq, knew, aux=False)
        OA.decode_attention(kq, vq, q, kc, vc)
        done += 1
        n_steps += 1
        el = time.perf_counter() - t0
        if (steps is not None and n_steps >= steps) or (steps is None and el >= budget_s):
            break
    per_kv_head = el / done
    step_s = per_kv_head * HKV
    return {"value": B * N / step_s, "unit": "KV-tokens/s", "cores": cores, "blas_threads": blas_threads,
            "kind": "oracle",
            "sample": f"{done} x (1 of 8 KV heads: oracle encode of the new K,V token + float64 decode attention "
                      f"of 4 query heads over N=32768 TurboQuant_mse b=4 tokens), scaled x8 to the layer; "
                      f"{el:.1f} s of CPU time"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    warm = max(args.warmup, 3)
    cpu_baseline_decode(steps=warm)
    t0 = time.perf_counter()
    base = cpu_baseline_decode(steps=args.ref_steps or min(args.steps, 20))
    el = time.perf_counter() - t0
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    line = {"impl": "reference", "metric": METRIC, "value": base["value"], "unit": "KV-tokens/s",
            "n_gpus": ws, "steps": args.ref_steps or min(args.steps, 20), "warmup": warm,
            "ms_per_step": B * N / base["value"] * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "llama3.1-8b-shaped decode step (append 1 token + attend): B=1 Hq=32 Hkv=8 "
                                   "d=128 N=32768, K/V TurboQuant_mse b=4, randomized Hadamard",
                       "global_batch": B, "seq_len": N, "parallelism": "cpu oracle"},
            "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": "KV-tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": el}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40000)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-steps", type=int, default=0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per decode call from an ncu capture of this build, if any")
    ap.add_argument("--encode-variant", default="mse4", choices=["mse4", "prod3"],
                    help="codec of the encode-throughput measurement")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
