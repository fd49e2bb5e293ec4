"""Benchmark: one TurboQuant decode step per step, on B200.

Workload (the largest decode configuration that fits one GPU): batched
decode, batch 16, 32 query heads / 8 KV heads, head_dim 128, 131072 cached
tokens per sequence; K, V bf16 N(0,1) with 3 seeded channels per KV head
(2% of 128) scaled x8; keys TurboQuant_prod b=3 (2-bit Lloyd-Max codes +
1-bit QJL sketch of the residual), values TurboQuant_mse b=3.  The packed
cache is 1.81 GB, far larger than the 126 MB L2, so every step streams it
from HBM.

A step is the whole hot path for one new token per sequence, one
tq_append_decode_attention call: encode the new token's K and V (norm, sign
flips + FWHT, Lloyd-Max indices, bit-packing, residual + QJL signs) into the
cache tail, then decode attention over all 131072 packed tokens of all 16
sequences (query rotation, scores from the codes, online softmax, PV in the
rotated basis, split merge, one inverse rotation).  value = KV-tokens/s =
B * N / step time.  Steps are timed with CUDA events on the launching stream,
bracketed by a barrier and a device synchronize, max over ranks.

The line also carries, as extra keys, the decode call on the 70B-shaped
long-context configuration (B=1, 64/8 heads, N=2^20, prod-4 K, mse-4 V) and
on the Llama-3.1-8B-shaped one (B=1, 32/8 heads, N=32768, mse-4 K and V; 8
rotating cache copies so that it does not sit in L2), and the encode
throughput on the encode sweep's d=128 cells.

--impl reference times the CPU oracle (oracle/, NumPy) on a bounded sample of
the same step; that leg is the reported baseline, not the optimisation target.

Multi-GPU (torchrun): each rank runs an independent replica of the step on
its own GPU (the path shards by batch / KV head with no data exchange), so
scaling is weak and value sums the ranks' tokens over the slowest rank's time.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attention KV-tokens/s and encode vectors/s on 1 B200; % of HBM roofline"
D = 128
# workloads: sizes, quantizers (bits, variant, seed_rot[, seed_qjl]) and the
# seeded generator of their K/V (kv_cache_vector_13_b200.inputs)
WORKLOADS = {
    "batched": dict(
        B=16, Hq=32, Hkv=8, N=131072, k=(3, "prod", 20, 21), v=(3, "mse", 22), gen="outlier_kv", seed=3, copies=1,
        desc="batched decode step (append 1 token + attend)", data="bf16 K,V N(0,1) with 2% outlier channels x8",
        rot="randomized Hadamard"),
    "long70b": dict(
        B=1, Hq=64, Hkv=8, N=1 << 20, k=(4, "prod", 30, 31), v=(4, "mse", 32), gen="student_kv", seed=5, copies=1,
        desc="70B-shaped long-context decode", data="bf16 K,V 0.5*StudentT(3)*LogNormal(0,1) channel scales",
        rot="randomized Hadamard"),
    "llama8b": dict(
        B=1, Hq=32, Hkv=8, N=32768, k=(4, "mse", 10), v=(4, "mse", 11), gen="llama8b_kv", seed=2, copies=8,
        desc="Llama-3.1-8B-shaped decode", data="bf16 K,V N(0,1)*LogNormal(0,0.5) channel scales",
        rot="randomized Hadamard"),
}
HEADLINE = "batched"


def workload(key, batch=None):
    """The workload's parameters (batch optionally overridden, for smaller
    profiling captures) with its full name."""
    w = dict(WORKLOADS[key])
    if batch:
        w["B"] = batch
    n = w["N"]
    nstr = f"2^{n.bit_length() - 1}" if n & (n - 1) == 0 and n >= 1 << 20 else str(n)
    w["name"] = (f"{w['desc']}: B={w['B']} Hq={w['Hq']} Hkv={w['Hkv']} d={D} N={nstr}, {w['data']}; "
                 f"K TurboQuant_{w['k'][1]} b={w['k'][0]}, V TurboQuant_{w['v'][1]} b={w['v'][0]}, {w['rot']}")
    return w


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# DRAM bytes (read + write) of one decode split-kernel launch on the headline
# workload, from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum),
# reported only for that workload and while the decode sources are the ones
# it was taken on.
# Captured at B = 2 (reads 230,536,192 B, writes 4,043,520 B): reads scaled by
# the 8x units of B = 16 (B = 4 read 2.02x the B = 2 bytes), writes kept.
TRAFFIC = {"workload": ("batched", 16), "bytes": 8 * 230536192 + 4043520,
           "source_sha256": "be1a913840ea164638a20dcb50b885af95c308fb41ae4683bc8ee9649f68d1a5"}
DECODE_SOURCES = ("tq_decode.cu", "tq_decode_split.cuh", "tq_decode_regs.cu")


def decode_source_sha256():
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        with open(os.path.join(ROOT, "kv_cache_vector_13_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def traffic_bytes(key, B):
    if (key, B) != TRAFFIC["workload"]:
        return None
    return TRAFFIC["bytes"] if decode_source_sha256() == TRAFFIC["source_sha256"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms while the
    GPU runs the warm-up and timed steps."""

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
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
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


def job_value(world_size, ms_per_step, B, N):
    """Whole-job KV-tokens/s: every rank decodes B * N tokens per step, and
    the job's step time is the slowest rank's."""
    return world_size * B * N / (ms_per_step * 1e-3)


# ------------------------------------------------------------------ our leg

class Setup:
    """One workload on the device: quantizers, packed caches (encoded by
    tq_encode from the seeded bf16 K/V, then the inputs are freed), the
    decode operator and the tail views of token N-1."""

    def __init__(self, api, inputs, torch, dev, key, seed_shift=0, batch=None):
        w = workload(key, batch)
        self.w, self.key = w, key
        self.B, self.Hq, self.Hkv, self.N = w["B"], w["Hq"], w["Hkv"], w["N"]
        kb, kvar, ksr, *kqs = w["k"]
        vb, vvar, vsr = w["v"]
        self.kq = api.Quantizer(D, kb, kvar, seed_rot=ksr, seed_qjl=kqs[0] if kqs else 1, device=dev)
        self.vq = api.Quantizer(D, vb, vvar, seed_rot=vsr, device=dev)
        K, V = getattr(inputs, w["gen"])(N=self.N, B=self.B, seed=w["seed"] + seed_shift, device=dev)
        kc0, vc0 = api.encode(self.kq, K), api.encode(self.vq, V)
        del K, V
        torch.cuda.synchronize()

        def clone(c):
            return api.PackedCache(*(None if t is None else t.clone() for t in (c.codes, c.norms, c.qjl, c.rnorms)))

        self.kcs = [kc0] + [clone(kc0) for _ in range(w["copies"] - 1)]
        self.vcs = [vc0] + [clone(vc0) for _ in range(w["copies"] - 1)]
        g = torch.Generator(device=dev).manual_seed(100 + seed_shift)
        self.q = torch.randn((self.B, self.Hq, D), generator=g, device=dev).to(torch.bfloat16)
        self.k_new = torch.randn((self.B, self.Hkv, D), generator=g, device=dev).to(torch.bfloat16)
        self.v_new = torch.randn((self.B, self.Hkv, D), generator=g, device=dev).to(torch.bfloat16)
        self.op = api.DecodeAttention(self.kq, self.vq, self.B, self.Hq, self.Hkv, self.N, device=dev)

        def tail(c):
            return api.PackedCache(*(None if t is None else t[:, :, self.N - 1:self.N]
                                     for t in (c.codes, c.norms, c.qjl, c.rnorms)))

        self.tails = [(tail(kc), tail(vc)) for kc, vc in zip(self.kcs, self.vcs)]
        torch.cuda.synchronize()  # everything above runs on the default stream; the steps on another

    @property
    def copies(self):
        return len(self.kcs)

    def decode_bytes(self):
        """Algorithmic bytes of one decode call: the packed K and V records of
        every cached token, the bf16 query and the fp32 output."""
        return (self.B * self.Hkv * self.N * (self.kq.record_bytes + self.vq.record_bytes)
                + self.q.numel() * 2 + self.B * self.Hq * D * 4)

    def step(self, c, stream, q=None, k_new=None, v_new=None):
        # one decode step: tq_append_decode_attention encodes the new token's
        # K and V into the cache tail and attends over the cache (four
        # kernels, each allowed to start while the one before it finishes)
        self.op.append_step(self.q if q is None else q, self.k_new if k_new is None else k_new,
                            self.v_new if v_new is None else v_new, self.tails[c][0], self.tails[c][1],
                            self.kcs[c], self.vcs[c], stream=stream)

    def decode(self, c, stream):
        self.op(self.q, self.kcs[c], self.vcs[c], stream=stream)


def time_decode_calls(torch, s, stream, reps):
    """Live CUDA-event time of one tq_decode_attention call (ms), averaged
    over `reps` back-to-back calls that cycle through the cache copies."""
    torch.cuda.synchronize()  # inputs made on the default stream are complete
    with torch.cuda.stream(stream):
        for c in range(max(3, s.copies)):
            s.decode(c % s.copies, stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(reps):
            s.decode(i % s.copies, stream)
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


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

    stream = torch.cuda.Stream(device=dev)
    s = Setup(api, inputs, torch, dev, args.workload, seed_shift=rank, batch=args.batch)
    K_steps = args.steps

    # warm-up: at least W steps, and at least half a second of them, while the
    # clock sampler already runs (so its samples see the GPU under load)
    clocks = ClockSampler(local)
    with clocks:
        with torch.cuda.stream(stream):
            t_w = time.perf_counter()
            n_warm = 0
            while n_warm < max(args.warmup, 3) or time.perf_counter() - t_w < 0.5:
                s.step(n_warm % s.copies, stream)
                n_warm += 1
                if n_warm % 8 == 0:
                    torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for i in range(K_steps):
                s.step(i % s.copies, stream)
            ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
    t_ms = ev0.elapsed_time(ev1)

    # the dominant kernels (prep + split of tq_decode_attention), live
    dec_ms = time_decode_calls(torch, s, stream, max(10, min(K_steps, 200)))
    # the same call through the bulk-copy staging feed (an extra record; the
    # register feed above is the default)
    staged_ms = None
    if not args.no_extras and ws == 1:
        prev = api.set_decode_feed(True)
        try:
            staged_ms = time_decode_calls(torch, s, stream, max(10, min(K_steps, 100)))
            api.check(stream)
        finally:
            api.set_decode_feed(prev)

    # end to end through the public API with host buffers, every step: H2D of
    # the step's inputs (q, k_new, v_new, bf16, one pinned buffer), the step,
    # D2H of the fp32 output, host synchronize
    parts = (s.q, s.k_new, s.v_new)
    sizes = [t.numel() for t in parts]
    hin = torch.empty(sum(sizes), dtype=torch.bfloat16).pin_memory()
    din = torch.empty(sum(sizes), dtype=torch.bfloat16, device=dev)
    off, views = 0, []
    for t, n in zip(parts, sizes):
        hin[off:off + n].copy_(t.reshape(-1).cpu())
        views.append(din[off:off + n].view(t.shape))
        off += n
    dq, dk, dv = views
    hout = torch.empty((s.B, s.Hq, D), dtype=torch.float32).pin_memory()

    def e2e_step(c):
        din.copy_(hin, non_blocking=True)
        s.step(c, stream, dq, dk, dv)
        hout.copy_(s.op.out, non_blocking=True)
        stream.synchronize()

    with torch.cuda.stream(stream):
        for c in range(3):
            e2e_step(c % s.copies)
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        for i in range(K_steps):
            e2e_step(i % s.copies)
    e2e_s = time.perf_counter() - t0
    barrier()

    t_ms, dec_ms, e2e_s = max_over_ranks([t_ms, dec_ms, e2e_s], dist, dev)
    line = None
    if rank == 0:
        pk, pk_kind = peaks()
        ms_step = t_ms / K_steps
        dec_bytes = s.decode_bytes()
        achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": job_value(ws, ms_step, s.B, s.N), "unit": "KV-tokens/s", "n_gpus": ws,
            "steps": K_steps, "warmup": n_warm, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 encode; f16xf16->f32 mma decode",
            "data": "synthetic",
            "config": {"workload": s.w["name"], "global_batch": s.B * ws, "seq_len": s.N,
                       "parallelism": f"replicas x{ws}",
                       "l2": f"packed cache {dec_bytes / 1e9:.2f} GB per step, larger than the 126 MB L2"},
            "roofline": {"kernel": "tq_decode_attention (prep + split)", "bound": "hbm",
                         "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "peak_kind": pk_kind,
                         "bytes_per_launch": dec_bytes, "ms_per_launch": dec_ms,
                         "traffic": args.traffic if args.traffic is not None else traffic_bytes(s.key, s.B)},
            "e2e": {"value": ws * s.B * s.N * K_steps / e2e_s, "unit": "KV-tokens/s",
                    "h2d_bytes_per_step": hin.numel() * hin.element_size(),
                    "d2h_bytes_per_step": hout.numel() * 4, "steps": K_steps,
                    "mode": "per step: H2D copy of (q, k_new, v_new) from pinned memory, "
                            "tq_append_decode_attention, D2H copy of the output, host synchronize"},
            "gpu_launches": 4 * K_steps,
            "clocks": clocks.summary(),
        }
    del s
    torch.cuda.empty_cache()

    if rank == 0:
        pk, _ = peaks()
        if not args.no_extras and ws == 1:
            extras = {}
            for key in (k for k in WORKLOADS if k != args.workload):
                e = Setup(api, inputs, torch, dev, key)
                ms = time_decode_calls(torch, e, stream, 40)
                by = e.decode_bytes()
                extras[key] = {"workload": e.w["name"], "ms_per_call": ms, "kv_tokens_per_s": e.B * e.N / (ms * 1e-3),
                               "bytes_per_call": by, "achieved_gbs": by / (ms * 1e-3) / 1e9,
                               "frac": by / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
                del e
                torch.cuda.empty_cache()
            line["decode_other_workloads"] = extras
            line["encode"] = [bench_encode(api, inputs, torch, dev, stream, v) for v in ENCODE_VARIANTS]
            with ClockSampler(local) as nclk:
                line["next_rows"] = bench_next_rows(api, inputs, torch, dev, stream)
            line["next_rows"]["clocks"] = nclk.summary()
            if staged_ms is not None:
                line["next_rows"]["decode_bulk_staged"] = {
                    "workload": line["config"]["workload"] + "; records fed through shared-memory rings filled by "
                                "bulk asynchronous copies (cp.async.bulk, mbarrier waits)",
                    "ms_per_call": staged_ms, "bytes_per_call": line["roofline"]["bytes_per_launch"],
                    "achieved_gbs": line["roofline"]["bytes_per_launch"] / (staged_ms * 1e-3) / 1e9,
                    "frac": line["roofline"]["bytes_per_launch"] / (staged_ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
        if not args.no_cpu_baseline and ws == 1:
            line["cpu_baseline"] = cpu_baseline_decode(args.workload, args.batch, budget_s=args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


ENCODE_VARIANTS = ("mse4", "prod3", "mse3_bf16", "prod3_bf16")


def _time_calls(torch, stream, fn, reps, warm=3):
    """Live CUDA-event time (ms) of one fn(i) call, averaged over `reps`
    back-to-back calls on `stream` after `warm` untimed ones."""
    torch.cuda.synchronize()  # inputs made on the default stream are complete
    with torch.cuda.stream(stream):
        for i in range(warm):
            fn(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(reps):
            fn(i)
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def bench_next_rows(api, inputs, torch, dev, stream):
    """The three kernels past the decode step, each on a synthetic workload
    larger than L2: the dense (Haar) rotation encode on tensor cores, top-k
    vector search over a packed database, and decode over an outlier-channel
    split cache (the pages' 32 channels at 3 bits + 96 at 2)."""
    pk, _ = peaks()
    out = {}
    n, d = 1 << 20, 128
    # dense rotation encode: 2^20 unit vectors fp32, TurboQuant_mse b=4
    qz = api.Quantizer(d, 4, "mse", seed_rot=7, device=dev, rotation="dense")
    xs = [inputs.unit_vectors(n, d, seed=10 + i, device=dev) for i in range(2)]
    cs = [api.empty_cache(qz, 1, 1, n, dev) for _ in xs]
    ms = _time_calls(torch, stream, lambda i: api.encode(qz, xs[i % 2], out=cs[i % 2], stream=stream), 30)
    by = n * (4 * d + qz.record_bytes)
    out["dense_encode"] = {"workload": "2^20 unit vectors d=128 fp32, TurboQuant_mse b=4, dense Haar rotation",
                           "vectors_per_s": n / (ms * 1e-3), "ms_per_launch": ms, "bytes_per_launch": by,
                           "achieved_gbs": by / (ms * 1e-3) / 1e9, "frac": by / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    del xs, cs
    # search: 2^21 records (mse-4, 68 B each: 143 MB), 32 queries, top-10
    n_db, n_q, k = 1 << 21, 32, 10
    qz = api.Quantizer(d, 4, "mse", seed_rot=8, device=dev)
    db = api.encode(qz, inputs.vectors(n_db, d, seed=20, device=dev))
    qs = inputs.vectors(n_q, d, seed=21, device=dev)
    srch = api.Search(qz, n_q, n_db, device=dev)
    ms = _time_calls(torch, stream, lambda i: srch(qs, db, k, stream=stream), 20)
    by = n_db * qz.record_bytes
    out["search"] = {"workload": f"top-{k} of {n_q} fp32 queries over 2^21 packed records d=128 "
                                 "TurboQuant_mse b=4", "scores_per_s": n_db * n_q / (ms * 1e-3),
                     "ms_per_call": ms, "bytes_per_call": by, "achieved_gbs": by / (ms * 1e-3) / 1e9,
                     "frac": by / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    del db
    # split decode: B=1, 32/8 heads, N=32768, 32 outlier channels at 3 bits +
    # 96 at 2 bits for K and V (2.25 bits per channel), 8 rotating copies
    B, Hq, Hkv, N = 1, 32, 8, 32768
    K, V = inputs.outlier_kv(N=N, B=B, seed=4, device=dev)
    ms_ch = K[0, 0, :256].float().pow(2).mean(0)
    ch = torch.sort(torch.topk(ms_ch, 32).indices).values.cpu()
    kq = api.SplitQuantizer(d, ch, 3, 2, "mse", seed_rot=40, device=dev)
    vq = api.SplitQuantizer(d, ch, 3, 2, "mse", seed_rot=42, device=dev)
    kcs = [api.encode_split(kq, K) for _ in range(8)]
    vcs = [api.encode_split(vq, V) for _ in range(8)]
    del K, V
    q = inputs.queries(B, Hq, device=dev)
    op = api.DecodeAttentionSplit(kq, vq, B, Hq, Hkv, N, device=dev)
    ms = _time_calls(torch, stream, lambda i: op(q, kcs[i % 8], vcs[i % 8], stream=stream), 20)
    rec = sum(g.record_bytes for g in kq.groups) + sum(g.record_bytes for g in vq.groups)
    by = B * Hkv * N * rec
    out["split_decode"] = {"workload": "outlier-channel split decode: B=1 Hq=32 Hkv=8 d=128 N=32768, K and V "
                                       "32 channels at 3 bits + 96 at 2 bits (2.25 bits), dense rotations",
                           "kv_tokens_per_s": B * N / (ms * 1e-3), "ms_per_call": ms, "bytes_per_call": by,
                           "achieved_gbs": by / (ms * 1e-3) / 1e9, "frac": by / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    return out


def run_encode_only(variant):
    """Only the encode measurement of one variant (for profiler captures)."""
    import torch
    from kv_cache_vector_13_b200 import api, inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    print(json.dumps({"encode": bench_encode(api, inputs, torch, dev, stream, variant)}), flush=True)


def bench_encode(api, inputs, torch, dev, stream, variant="mse4"):
    """Encode throughput on 2^20 vectors, d=128, 2 rotating inputs (larger
    than L2 together): "mse4" / "prod3" are the encode sweep's d=128 cells
    (unit vectors, fp32, TurboQuant_mse b=4 / TurboQuant_prod b=3);
    "mse3_bf16" / "prod3_bf16" encode bf16 rows like the decode workloads'
    values / keys."""
    n, d = 1 << 20, 128
    if variant in ("prod3", "prod3_bf16"):
        qz = api.Quantizer(d, 3, "prod", seed_rot=0, seed_qjl=1, device=dev)
    elif variant == "mse3_bf16":
        qz = api.Quantizer(d, 3, "mse", seed_rot=0, device=dev)
    else:
        qz = api.Quantizer(d, 4, "mse", seed_rot=0, device=dev)
    if variant.endswith("_bf16"):
        xs = [inputs.vectors(n, d, seed=i, device=dev).to(torch.bfloat16) for i in range(4)]
    else:
        xs = [inputs.unit_vectors(n, d, seed=i, device=dev) for i in range(2)]
    outs = [api.empty_cache(qz, 1, 1, n, dev) for _ in range(len(xs))]
    torch.cuda.synchronize()  # the inputs and the quantizer are made on the default stream
    clocks = ClockSampler(dev.index or 0)
    with clocks, torch.cuda.stream(stream):
        for i in range(3):
            api.encode(qz, xs[i % len(xs)], out=outs[i % len(xs)], stream=stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 50
        e0.record(stream)
        for i in range(reps):
            api.encode(qz, xs[i % len(xs)], out=outs[i % len(xs)], stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    byts = n * (d * xs[0].element_size() + qz.record_bytes)
    pk, _ = peaks()
    gbs = byts / (ms * 1e-3) / 1e9
    names = {"mse4": "2^20 unit vectors d=128 fp32, TurboQuant_mse b=4",
             "prod3": "2^20 unit vectors d=128 fp32, TurboQuant_prod b=3",
             "mse3_bf16": "2^20 N(0,1) vectors d=128 bf16, TurboQuant_mse b=3",
             "prod3_bf16": "2^20 N(0,1) vectors d=128 bf16, TurboQuant_prod b=3"}
    return {"workload": names[variant], "vectors_per_s": n / (ms * 1e-3), "ms_per_launch": ms,
            "bytes_per_launch": byts, "achieved_gbs": gbs, "frac": gbs / pk["hbm_gbs"], "clocks": clocks.summary()}


# ------------------------------------------------------------- CPU oracle

CPU_TOKENS = 8192  # cached tokens of the oracle's sample slice


def cpu_baseline_decode(key=HEADLINE, batch=None, budget_s=15.0, steps=None):
    """Time the oracle on a bounded sample of the workload's step: one
    (batch, KV head) slice of CPU_TOKENS cached tokens drawn like the
    workload's, with its quantizers; a sample step encodes the new token's K
    and V and attends the slice's query heads over it.  The rate in
    token-heads/s is scaled to the workload's KV-tokens/s (a step processes
    B * Hkv * N token-heads)."""
    import numpy as np
    from kv_cache_vector_13_b200 import inputs
    from oracle import attention as OA
    from oracle import quantizer as OQ
    try:
        from threadpoolctl import threadpool_info
        blas_threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        blas_threads = 1
    w = workload(key, batch)
    cores = len(os.sched_getaffinity(0))
    kb, kvar, ksr, *kqs = w["k"]
    vb, vvar, vsr = w["v"]
    kq = OQ.Quantizer(D, kb, kvar, seed_rot=ksr, seed_qjl=kqs[0] if kqs else 1)
    vq = OQ.Quantizer(D, vb, vvar, seed_rot=vsr)
    K, V = getattr(inputs, w["gen"])(N=CPU_TOKENS, B=1, seed=w["seed"], device="cpu")
    kc = {k: v[None, None] for k, v in OQ.encode(kq, K[0, 0].float().numpy(), aux=False).items()}
    vc = {k: v[None, None] for k, v in OQ.encode(vq, V[0, 0].float().numpy(), aux=False).items()}
    g = w["Hq"] // w["Hkv"]
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, g, D)).astype(np.float32)
    knew = rng.standard_normal((1, D)).astype(np.float32)
    done, t0 = 0, time.perf_counter()
    while True:
        OQ.encode(kq, knew, aux=False)
        OQ.encode(vq, knew, aux=False)
        OA.decode_attention(kq, vq, q, kc, vc)
        done += 1
        el = time.perf_counter() - t0
        if (steps is not None and done >= steps) or (steps is None and el >= budget_s):
            break
    token_heads_per_s = done * CPU_TOKENS / el
    return {"value": token_heads_per_s / w["Hkv"], "unit": "KV-tokens/s", "cores": cores,
            "blas_threads": blas_threads, "kind": "oracle",
            "sample": f"{done} x (one (batch, KV head) slice of {CPU_TOKENS} tokens drawn like the workload: "
                      f"oracle encode of the new K,V token + float64 decode attention of {g} query heads, "
                      f"{kvar}-{kb} keys, {vvar}-{vb} values), scaled by token-heads to B={w['B']} x Hkv={w['Hkv']} x "
                      f"N={w['N']}; {el:.1f} s of CPU time"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    warm = max(args.warmup, 3)
    cpu_baseline_decode(args.workload, args.batch, steps=warm)
    n = args.ref_steps or min(args.steps, 20)
    t0 = time.perf_counter()
    base = cpu_baseline_decode(args.workload, args.batch, steps=n)
    el = time.perf_counter() - t0
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    w = workload(args.workload, args.batch)
    line = {"impl": "reference", "metric": METRIC, "value": base["value"], "unit": "KV-tokens/s",
            "n_gpus": ws, "steps": n, "warmup": warm,
            "ms_per_step": w["B"] * w["N"] / base["value"] * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w["name"], "global_batch": w["B"], "seq_len": w["N"],
                       "parallelism": "cpu oracle"},
            "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": "KV-tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": el}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=list(WORKLOADS),
                    help="the timed step's workload (the others are reported as extra keys)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiler captures)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other decode workloads and the encode measurements")
    ap.add_argument("--ref-steps", type=int, default=0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per decode call from an ncu capture of this build, if any")
    ap.add_argument("--encode-only", default=None, choices=list(ENCODE_VARIANTS),
                    help="measure only this encode variant (for profiler captures)")
    args = ap.parse_args()
    if args.encode_only:
        run_encode_only(args.encode_only)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
