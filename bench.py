"""Benchmark of the block-quantized attention hot path on B200.

One step = one pass of the whole prefill path on the INT8 causal problem
(B=1, H=32, N=4096, D=128, bf16 inputs with outlier channels, shared seeded
rotation): rotate+quantize Q (blocks of 128), K and V (blocks of 256), then
quantized attention. value = algorithmic INT8 operations of the attention
(4*D per unmasked query/key pair) / step time, in TOPS, whole job (all
ranks). Inputs are resident in HBM; L2 is flushed before every timed step
(256 MB written, then read back). The same line carries the decode KV bandwidth (INT8 and
packed-INT4 caches) and the FP8 long-sequence prefill measured in the same
run, each with its roofline fraction.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

--impl reference times the CPU oracle (the reference arm of this repo) on a
bounded sample of the same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np

METRIC = "prefill quantized-attention TFLOPS and decode KV GB/s on 1 B200, % of roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


def prefill_ops(B, H, N, D, causal):
    pairs = N * (N + 1) // 2 if causal else N * N
    return 4.0 * D * B * H * pairs


def decode_bytes(p):
    if p.kv_dtype == 2:   # INT8
        nkb = -(-p.L // p.kv_block)
        kv = 2 * p.B * p.Hkv * p.L * p.D
        sc = 2 * p.B * p.Hkv * nkb * 4
    else:
        kv = 2 * p.B * p.Hkv * p.L * p.D // 2
        sc = 2 * p.B * p.Hkv * p.L * (p.D // p.group) * 2
    qo = 2 * p.B * p.Hq * p.D * 2
    return kv + sc + qo


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi samples (200 ms) of this GPU while the timed region runs."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", "--query-gpu=" + self.Q, "--format=csv,noheader,nounits", "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.out.close()

    def summary(self, max_fallback):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 8:
                    rows.append(f)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": max_fallback, "reasons": ["unsampled"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[0]) for r in rows if num(r[0]) is not None]
        mx = max([num(r[1]) for r in rows if num(r[1]) is not None] or [max_fallback])
        power = [num(r[2]) for r in rows if num(r[2]) is not None]
        load = [s for s, pw in zip(sm, power) if pw is not None and pw > 200] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def gpu_arm(args):
    import torch
    import torch.distributed as dist

    import block_quantized_precision_b200 as qa
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    pk, pk_kind = peaks()
    hbm_peak = pk["hbm_gbs"]
    int8_peak = 2.0 * pk["bf16_tflops"]        # INT8/FP8 dense = 2 x bf16 dense (nominal ratio)
    fp32_peak = 148 * 128 * 2 * pk.get("sm_max_mhz", 1965.0) * 1e6 / 1e12   # FMA pipe, TFLOP/s
    launches = [0]

    def cu(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    # ---------------- the step: INT8 causal prefill path ----------------
    p = synth.INT8_CAUSAL
    d = synth.make_prefill(p)
    host = {n: torch.from_numpy(d[n].view(np.int16)).pin_memory() for n in ("q", "k", "v")}
    x = {n: host[n].to(dev).view(torch.bfloat16) for n in host}
    rot = cu(d["rot"])
    nqb, nkb = -(-p.N // 128), -(-p.N // 256)
    shp = p.shape()
    bufs = {
        "qc": torch.empty(shp, dtype=torch.uint8, device=dev), "qs": torch.empty((p.B, p.H, nqb), device=dev),
        "kc": torch.empty(shp, dtype=torch.uint8, device=dev), "ks": torch.empty((p.B, p.H, nkb), device=dev),
        "vc": torch.empty(shp, dtype=torch.uint8, device=dev), "vs": torch.empty((p.B, p.H, nkb), device=dev),
        "out": torch.empty(shp, dtype=torch.bfloat16, device=dev),
    }
    out_host = torch.empty(shp, dtype=torch.bfloat16).pin_memory()
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)

    def l2_flush():
        # Write 256 MB, then read it back: the read evicts everything else and
        # the written lines are cleaned before the timed kernels start, so no
        # dirty lines are written back inside them.
        flush.zero_()
        flush.sum()
    ops = prefill_ops(p.B, p.H, p.N, p.D, p.causal)
    qkv_out = [(bufs["qc"], bufs["qs"]), (bufs["kc"], bufs["ks"]), (bufs["vc"], bufs["vs"])]
    # The step runs as one CUDA graph (captured once): the launches of a step
    # reach the GPU back to back, with no host time between them. An event
    # node between the quantization and the prefill times both in every step.
    ev_mid = torch.cuda.Event(enable_timing=True, external=True)

    def step_body(st):
        # one call quantizes Q, K and V (the Q and K rotations concurrently on
        # the library's internal streams, joined back into this stream), then
        # the prefill
        qa.qattn_rotate_block_quant_qkv(x["q"], x["k"], x["v"], p.layout, rot, p.code_dtype, out=qkv_out, stream=st)
        ev_mid.record(st)
        qa.qattn_prefill(bufs["qc"], bufs["qs"], bufs["kc"], bufs["ks"], bufs["vc"], bufs["vs"], p.code_dtype,
                         p.layout, p.causal, out=bufs["out"], stream=st)

    def k1_alone(nm, st):
        # one of the three quantizations by itself on the whole GPU: the
        # per-kernel rooflines of the rotation and the V quantization
        qa.qattn_rotate_block_quant(x[nm], p.layout, rot if nm != "v" else None, 128 if nm == "q" else 256,
                                    p.code_dtype, bufs[nm + "c"], bufs[nm + "s"], stream=st)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    g_step = capture_graph(step_body, args.warmup)
    g_alone = {nm: capture_graph(lambda st, nm=nm: k1_alone(nm, st), 2) for nm in ("q", "k", "v")}
    for _ in range(args.warmup):
        l2_flush()
        g_step.replay()
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(dev)
    uuid = "GPU-" + str(props.uuid) if getattr(props, "uuid", None) else None
    per = []
    with ClockSampler(uuid) as clk:
        barrier()
        for i in range(args.steps):
            l2_flush()
            e0.record(stream)
            g_step.replay()
            e1.record(stream)
            e1.synchronize()
            per.append((e0.elapsed_time(ev_mid), ev_mid.elapsed_time(e1)))
        barrier()
    clocks = clk.summary(pk.get("sm_max_mhz", 1965.0))
    step_launches = 4 * args.steps                  # 3 quantization kernels + the prefill per step
    per = np.array(per)
    step_ms = per.sum(axis=1)
    ms = max_over_ranks(float(step_ms.mean()), world, dev)
    value = job_rate(ops, world, ms)
    kern_ms = per.mean(axis=0)
    # the three quantizations one at a time (graphs of one call each, the
    # same flush before each), for their own rooflines and for the gain of
    # running them in one call
    alone = {nm: time_graph(g_alone[nm], args.steps, args.warmup, stream, l2_flush) for nm in ("q", "k", "v")}
    assert qa.qattn_device_error() == qa.QATTN_OK
    qk_rows = p.B * p.H * p.N
    elems = qk_rows * p.D
    k1_bytes, k1_flop = 3 * 3 * elems, 2 * 2 * elems * p.D
    k1_floor_ms = max(k1_bytes / (hbm_peak * 1e9), k1_flop / (fp32_peak * 1e12)) * 1e3
    kernels = {
        "rotq_q": {"ms": alone["q"], "bound": "alu", "achieved": qk_rows * p.D * p.D * 2 / (alone["q"] * 1e-3) / 1e12,
                   "peak": fp32_peak, "unit": "TFLOP/s", "timed": "alone (graph of one call)"},
        "rotq_k": {"ms": alone["k"], "bound": "alu", "achieved": qk_rows * p.D * p.D * 2 / (alone["k"] * 1e-3) / 1e12,
                   "peak": fp32_peak, "unit": "TFLOP/s", "timed": "alone (graph of one call)"},
        "quant_v": {"ms": alone["v"], "bound": "hbm", "achieved": qk_rows * p.D * 3 / (alone["v"] * 1e-3) / 1e9,
                    "peak": hbm_peak, "unit": "GB/s", "timed": "alone (graph of one call)"},
        "quant_qkv": {"ms": kern_ms[0], "bound": "alu (FP32 FMA) / hbm, the larger time", "floor_ms": k1_floor_ms,
                      "frac": k1_floor_ms / kern_ms[0], "timed": "in the step graph (three launches, one call)",
                      "ms_three_alone": sum(alone.values())},
        "prefill": {"ms": kern_ms[1], "bound": "tensor", "achieved": ops / (kern_ms[1] * 1e-3) / 1e12,
                    "peak": int8_peak, "unit": "TOPS", "timed": "in the step graph"},
    }
    for k in kernels.values():
        if "frac" not in k:
            k["frac"] = k["achieved"] / k["peak"]
        k["ms"] = float(k["ms"])
        k["frac"] = float(k["frac"])
    dom = max((n for n in kernels if n != "quant_qkv"), key=lambda n: kernels[n]["ms"])
    traffic = load_traffic(dom)
    roof = {"kernel": dom, "bound": kernels[dom]["bound"], "achieved": round(kernels[dom]["achieved"], 2),
            "peak": kernels[dom]["peak"], "unit": kernels[dom]["unit"], "frac": round(kernels[dom]["frac"], 4),
            "traffic": traffic, "peak_source": pk_kind + " (burst)"}

    # ---------------- end to end through the C ABI with host buffers ----------------
    # qattn_attention_path_host: pinned host inputs in, pinned host output
    # out, the copies of one group of heads overlapped with the compute of
    # another (default 8 groups); the timed region holds the whole call.
    host_bf = {n: host[n].view(torch.bfloat16) for n in host}
    ws = torch.empty(qa.qattn_attention_path_host_workspace_size(p.B, p.H, p.N, p.D, p.layout, 0),
                     dtype=torch.uint8, device=dev)
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        qa.qattn_attention_path_host(host_bf["q"], host_bf["k"], host_bf["v"], rot, p.layout, p.code_dtype,
                                     p.causal, out=out_host, workspace=ws, stream=stream)
        e1.record(stream)
        e1.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    assert qa.qattn_device_error() == qa.QATTN_OK
    h2d = sum(host[n].numel() * 2 for n in host)
    d2h = out_host.numel() * 2
    te = max_over_ranks(float(np.mean(e2e_ms)), world, dev)
    e2e = {"value": round(job_rate(ops, world, te), 3), "unit": "TOPS",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(te, 4),
           "api": "qattn_attention_path_host (host buffers, 8 head groups, copies overlapped with compute)"}

    keep = {"int8_causal": {"problem": p, "data": d,
                            "out": bufs["out"].view(torch.int16).cpu().numpy().view(np.uint16)}}
    extra = {}
    if not args.no_extra:
        extra = extra_measurements(args, dev, stream, qa, synth, hbm_peak, int8_peak, fp32_peak, flush=l2_flush,
                                   keep=keep)

    cpu, errors = None, None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(p, d, args.cpu_seconds)
        errors = parity_errors(keep)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "ms_percentiles": {"p10": round(float(np.percentile(step_ms, 10)), 4),
                           "p50": round(float(np.percentile(step_ms, 50)), 4),
                           "p90": round(float(np.percentile(step_ms, 90)), 4)},
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded; shapes and distributions of the stated problem)",
        "config": {"workload": p.name, "B": p.B, "H": p.H, "N": p.N, "D": p.D, "layout": "BNSD", "causal": True,
                   "codes": "int8", "rotation": "seeded orthogonal 128x128 on Q and K",
                   "l2": "flushed before every timed step (256 MB written, then read)", "parallelism": "replicas" if world > 1 else "1 GPU"},
        "roofline": roof,
        "kernels": {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv) for kk, vv in v.items()} for k, v in kernels.items()},
        "e2e": e2e,
        "gpu_launches": int(step_launches),
        "clocks": clocks,
        "extra": extra,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if errors is not None:
        line["errors"] = errors
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of the ranks' values of x (x itself on one rank): the
    job's time is its slowest rank's. `device` holds the reduction tensor
    (the GPU with NCCL, the CPU with gloo)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(ops_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput in TOPS: every rank processes ops_per_rank in
    the (max-over-ranks) time ms."""
    return world * ops_per_rank / (ms * 1e-3) / 1e12


def load_traffic(kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu
    capture (profiles/traffic.json), or None when there is none or the
    kernel's source has changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f).get(kernel)
        src = open(os.path.join(ROOT, t["source"]), "rb").read()
        if hashlib.sha256(src).hexdigest()[:16] != t["sha256_16"]:
            return None
        return t["bytes"]
    except Exception:
        return None


def extra_measurements(args, dev, stream, qa, synth, hbm_peak, int8_peak, fp32_peak, flush=None, keep=None):
    """Decode, KV append, the FP8 long prefill (first class: its own roofline
    and its rotation/quantization reported apart), mixed and INT4 prefill.
    `keep` (a dict) receives the outputs that the CPU leg samples for the
    error figures."""
    import torch
    res = {}
    keep = {} if keep is None else keep
    pk_bf16 = int8_peak / 2.0
    n = max(5, args.steps // 2)

    def timeit(fn, reps, flush=None):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            if flush is not None:
                flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return float(np.mean(ts))

    def timeit_back_to_back(fn, reps):
        # reps calls between two events: the host's per-call work overlaps the
        # GPU's, so this is the launches' average device duration
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) / reps

    # decode, INT8 and packed INT4 caches (inputs far larger than L2)
    for key, p in (("decode_int8kv", synth.INT8_KV_DECODE), ("decode_int4kv", synth.INT4_KV_DECODE)):
        dd = synth.make_decode(p)
        q = torch.from_numpy(dd["q"].view(np.int16)).to(dev).view(torch.bfloat16)
        k = torch.from_numpy(dd["k"]).to(dev)
        v = torch.from_numpy(dd["v"]).to(dev)
        if p.kv_dtype == synth.INT8:
            ks, vs, kvt = torch.from_numpy(dd["k_scales"]).to(dev), torch.from_numpy(dd["v_scales"]).to(dev), qa.QATTN_INT8
        else:
            ks = torch.from_numpy(dd["k_scales"].view(np.int16)).to(dev).view(torch.float16)
            vs = torch.from_numpy(dd["v_scales"].view(np.int16)).to(dev).view(torch.float16)
            kvt = qa.QATTN_INT4_PACKED
        out = torch.empty((p.B, p.Hq, 1, p.D), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(16, qa.qattn_decode_workspace_size(p.B, p.Hq, p.Hkv, p.L, p.D)), dtype=torch.uint8, device=dev)
        fn = lambda: qa.qattn_decode_kvq(q, k, v, ks, vs, kvt, kv_block=p.kv_block, group=p.group, out=out, workspace=ws)
        ms_single = timeit(fn, n)
        ms = timeit_back_to_back(fn, 10)
        by = decode_bytes(p)
        gbs = by / (ms * 1e-3) / 1e9
        gbs_single = by / (ms_single * 1e-3) / 1e9
        res[key] = {"workload": p.name, "ms": round(ms, 4), "GB/s": round(gbs, 1), "bytes": by,
                    "timing": "10 calls back to back between two events (cache far larger than L2)",
                    "ms_single_call": round(ms_single, 4), "GB/s_single_call": round(gbs_single, 1),
                    "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                                 "frac": round(gbs / hbm_peak, 4), "frac_single_call": round(gbs_single / hbm_peak, 4),
                                 "traffic": load_traffic(key)}}
        keep[key] = {"problem": p, "data": {nm: dd[nm] for nm in ("q", "k_scales", "v_scales")},
                     "k": dd["k"], "v": dd["v"], "out": out.view(torch.int16).cpu().numpy().view(np.uint16)}
        del k, v, dd
        torch.cuda.empty_cache()

    # KV-cache quantize-on-append: a 256-token chunk of new K rows written
    # into the INT8 cache of the INT8 decode problem (block-aligned: one
    # fresh block per (b, h_kv)) and into the INT4 cache of the INT4 problem
    for key, p, kvt in (("kv_append_int8", synth.INT8_KV_DECODE, qa.QATTN_INT8),
                        ("kv_append_int4", synth.INT4_KV_DECODE, qa.QATTN_INT4_PACKED)):
        n_new, L0 = 256, 1024
        g = torch.Generator(device=dev).manual_seed(7)
        xn = torch.randn((p.B, p.Hkv, n_new, p.D), generator=g, device=dev).to(torch.bfloat16)
        if kvt == qa.QATTN_INT8:
            cache = torch.zeros((p.B, p.Hkv, L0 + n_new, p.D), dtype=torch.int8, device=dev)
            scl = torch.zeros((p.B, p.Hkv, (L0 + n_new) // 256), dtype=torch.float32, device=dev)
            by = xn.numel() * 2 + xn.numel() + p.B * p.Hkv * 4
        else:
            cache = torch.zeros((p.B, p.Hkv, L0 + n_new, p.D // 2), dtype=torch.uint8, device=dev)
            scl = torch.zeros((p.B, p.Hkv, L0 + n_new, p.D // p.group), dtype=torch.float16, device=dev)
            by = xn.numel() * 2 + xn.numel() // 2 + p.B * p.Hkv * n_new * (p.D // p.group) * 2
        fn = lambda: qa.qattn_kv_append(xn, cache, scl, L0, kvt, group=p.group)
        ms = timeit(fn, n, flush)
        gbs = by / (ms * 1e-3) / 1e9
        res[key] = {"workload": "%s, append %d tokens at %d" % (p.name, n_new, L0), "ms": round(ms, 4),
                    "GB/s": round(gbs, 1), "bytes": by,
                    "roofline": {"bound": "hbm", "peak": hbm_peak, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4)}}
        del cache, scl, xn

    # KV-cache append at bandwidth scale: a 4096-token prefill's K and V
    # written into empty caches of the decode problems' shapes (block-aligned:
    # no earlier codes to requantize); bytes = new rows read once + codes and
    # scales written once
    for key, p, kvt in (("kv_append_prefill_int8", synth.INT8_KV_DECODE, qa.QATTN_INT8),
                        ("kv_append_prefill_int4", synth.INT4_KV_DECODE, qa.QATTN_INT4_PACKED)):
        n_new = 4096
        g = torch.Generator(device=dev).manual_seed(8)
        xs = [torch.randn((p.B, p.Hkv, n_new, p.D), generator=g, device=dev).to(torch.bfloat16) for _ in range(2)]
        if kvt == qa.QATTN_INT8:
            caches = [torch.zeros((p.B, p.Hkv, n_new, p.D), dtype=torch.int8, device=dev) for _ in range(2)]
            scls = [torch.zeros((p.B, p.Hkv, n_new // 256), dtype=torch.float32, device=dev) for _ in range(2)]
        else:
            caches = [torch.zeros((p.B, p.Hkv, n_new, p.D // 2), dtype=torch.uint8, device=dev) for _ in range(2)]
            scls = [torch.zeros((p.B, p.Hkv, n_new, p.D // p.group), dtype=torch.float16, device=dev)
                    for _ in range(2)]
        by = sum(xs[i].numel() * 2 + caches[i].numel() + scls[i].numel() * scls[i].element_size() for i in range(2))

        def fn(xs=xs, caches=caches, scls=scls, kvt=kvt, p=p):
            for i in range(2):
                qa.qattn_kv_append(xs[i], caches[i], scls[i], 0, kvt, group=p.group)
        ms = timeit(fn, n, flush)
        gbs = by / (ms * 1e-3) / 1e9
        res[key] = {"workload": "%s shape, K and V of a %d-token prefill into empty caches" % (p.name, n_new),
                    "ms": round(ms, 4), "GB/s": round(gbs, 1), "bytes": by,
                    "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                                 "frac": round(gbs / hbm_peak, 4), "traffic": load_traffic(key)}}
        del xs, caches, scls
        torch.cuda.empty_cache()

    # FP8 long-sequence prefill path (inputs larger than L2)
    p = synth.FP8_LONG
    d = synth.make_prefill(p)
    x = {nm: torch.from_numpy(d[nm].view(np.int16)).to(dev).view(torch.bfloat16) for nm in ("q", "k", "v")}
    rot = torch.from_numpy(d["rot"]).to(dev)
    codes = {nm: qa.qattn_rotate_block_quant(x[nm], p.layout, rot if nm != "v" else None,
                                            128 if nm == "q" else 256, p.code_dtype) for nm in ("q", "k", "v")}
    out = torch.empty(p.shape(), dtype=torch.bfloat16, device=dev)
    pf = lambda: qa.qattn_prefill(codes["q"][0], codes["q"][1], codes["k"][0], codes["k"][1], codes["v"][0],
                                  codes["v"][1], p.code_dtype, p.layout, p.causal, out=out)
    ms_pf = timeit(pf, n)
    # the quantizations and the path as CUDA graphs (no host time between launches)
    k1_ms = {}
    for nm in ("q", "k", "v"):
        g = capture_graph(lambda st, nm=nm: qa.qattn_rotate_block_quant(
            x[nm], p.layout, rot if nm != "v" else None, 128 if nm == "q" else 256, p.code_dtype, codes[nm][0],
            codes[nm][1], stream=st), 2)
        k1_ms[nm] = time_graph(g, n, 3, stream)
        del g

    def qkv(st):
        qa.qattn_rotate_block_quant_qkv(x["q"], x["k"], x["v"], p.layout, rot, p.code_dtype,
                                        out=[codes["q"], codes["k"], codes["v"]], stream=st)
    g = capture_graph(qkv, 2)
    ms_qkv = time_graph(g, n, 3, stream)
    del g

    def full(st):
        qkv(st)
        qa.qattn_prefill(codes["q"][0], codes["q"][1], codes["k"][0], codes["k"][1], codes["v"][0], codes["v"][1],
                         p.code_dtype, p.layout, p.causal, out=out, stream=st)
    g = capture_graph(full, 2)
    ms_full = time_graph(g, n, 3, stream)
    del g
    ops = prefill_ops(p.B, p.H, p.N, p.D, p.causal)
    tf = ops / (ms_pf * 1e-3) / 1e12
    # K1 (rotate + quantize Q and K, quantize V): 3 bytes per element of each
    # tensor (2 read, 1 written) and D FMAs per element of Q and K
    elems = p.B * p.H * p.N * p.D
    k1_bytes, k1_fma = 3 * 3 * elems, 2 * elems * p.D
    k1_total = sum(k1_ms.values())
    k1_floor_ms = max(k1_bytes / (hbm_peak * 1e9), 2 * k1_fma / (fp32_peak * 1e12)) * 1e3
    res["prefill_fp8_long"] = {"workload": p.name, "ms_prefill": round(ms_pf, 4), "ms_path": round(ms_full, 4),
                               "TFLOPS_prefill": round(tf, 1),
                               "TFLOPS_path": round(ops / (ms_full * 1e-3) / 1e12, 1),
                               "roofline": {"kernel": "prefill", "bound": "tensor", "achieved": round(tf, 1),
                                            "peak": int8_peak, "unit": "TFLOP/s", "frac": round(tf / int8_peak, 4),
                                            "traffic": load_traffic("prefill_fp8_long"),
                                            "peak_source": "measured bf16 burst x 2 (FP8:bf16 nominal ratio)"},
                               "k1": {"ms_rotq_q": round(k1_ms["q"], 4), "ms_rotq_k": round(k1_ms["k"], 4),
                                      "ms_quant_v": round(k1_ms["v"], 4), "ms_total": round(k1_total, 4),
                                      "ms_one_call": round(ms_qkv, 4),
                                      "bytes": k1_bytes, "fma": k1_fma,
                                      "GB/s": round(k1_bytes / (k1_total * 1e-3) / 1e9, 1),
                                      "TFLOP/s_rotation": round(2 * k1_fma / ((k1_ms["q"] + k1_ms["k"]) * 1e-3) / 1e12, 2),
                                      "roofline": {"bound": "alu (FP32 FMA) / hbm, the larger time",
                                                   "floor_ms": round(k1_floor_ms, 4),
                                                   "frac": round(k1_floor_ms / ms_qkv, 4),
                                                   "frac_one_at_a_time": round(k1_floor_ms / k1_total, 4)}}}
    keep["prefill_fp8_long"] = {"problem": p, "data": d, "out": out.view(torch.int16).cpu().numpy().view(np.uint16)}
    del x, codes, out

    # The tiny FP8 problem (parity only: launch-bound)
    p = synth.TINY_FP8
    d = synth.make_prefill(p)
    x = {nm: torch.from_numpy(d[nm].view(np.int16)).to(dev).view(torch.float16) for nm in ("q", "k", "v")}
    codes = {nm: qa.qattn_rotate_block_quant(x[nm], p.layout, None, 128 if nm == "q" else 256, p.code_dtype)
             for nm in ("q", "k", "v")}
    out = qa.qattn_prefill(*codes["q"], *codes["k"], *codes["v"], p.code_dtype, p.layout, p.causal)
    torch.cuda.synchronize()
    keep["tiny_fp8"] = {"problem": p, "data": d, "out": out.view(torch.int16).cpu().numpy().view(np.uint16)}
    del x, codes, out

    # Mixed precision on the INT8 causal problem: Q/K INT8 (rotated), V in
    # packed INT4 or e4m3 (L2 flushed before every timed call)
    p = synth.INT8_CAUSAL
    d = synth.make_prefill(p)
    x = {nm: torch.from_numpy(d[nm].view(np.int16)).to(dev).view(torch.bfloat16) for nm in ("q", "k", "v")}
    rot = torch.from_numpy(d["rot"]).to(dev)
    qk = {nm: qa.qattn_rotate_block_quant(x[nm], p.layout, rot, 128 if nm == "q" else 256, qa.QATTN_INT8)
          for nm in ("q", "k")}
    out = torch.empty(p.shape(), dtype=torch.bfloat16, device=dev)
    ops = prefill_ops(p.B, p.H, p.N, p.D, p.causal)
    for key, vt in (("prefill_mixed_int4v", qa.QATTN_INT4_PACKED), ("prefill_mixed_fp8v", qa.QATTN_FP8_E4M3)):
        vcodes = qa.qattn_rotate_block_quant(x["v"], p.layout, None, 256, vt)
        qv = lambda: qa.qattn_rotate_block_quant(x["v"], p.layout, None, 256, vt, vcodes[0], vcodes[1])
        ms_qv = timeit(qv, n, flush)
        pf = lambda: qa.qattn_prefill_mixed(qk["q"][0], qk["q"][1], qk["k"][0], qk["k"][1], vcodes[0], vcodes[1],
                                            qa.QATTN_INT8, vt, p.layout, p.causal, out=out)
        ms_pf = timeit(pf, n, flush)
        v_bytes = x["v"].numel() * 2 + vcodes[0].numel()
        tops = ops / (ms_pf * 1e-3) / 1e12
        res[key] = {"workload": "%s, V %s" % (p.name, "int4 packed" if vt == qa.QATTN_INT4_PACKED else "e4m3"),
                    "ms_prefill": round(ms_pf, 4), "TOPS_prefill": round(tops, 1),
                    "ms_quant_v": round(ms_qv, 4), "GB/s_quant_v": round(v_bytes / (ms_qv * 1e-3) / 1e9, 1),
                    "roofline": {"bound": "tensor", "peak": int8_peak, "unit": "TOPS", "frac": round(tops / int8_peak, 4)}}
        if vt == qa.QATTN_INT4_PACKED:
            # the other order: V widened to INT8 codes by its own HBM-bound
            # pass, then the INT8 prefill (both timed, one flush before)
            vw = qa.qattn_widen_int4(vcodes[0])
            pw = lambda: (qa.qattn_widen_int4(vcodes[0], out=vw),
                          qa.qattn_prefill(qk["q"][0], qk["q"][1], qk["k"][0], qk["k"][1], vw, vcodes[1],
                                           qa.QATTN_INT8, p.layout, p.causal, out=out))
            ms_pw = timeit(pw, n, flush)
            tops_w = ops / (ms_pw * 1e-3) / 1e12
            res[key]["widened_first"] = {"ms": round(ms_pw, 4), "TOPS": round(tops_w, 1),
                                         "frac": round(tops_w / int8_peak, 4),
                                         "calls": "qattn_widen_int4(V), qattn_prefill INT8"}
            del vw

    # The dequantize-first comparison path on the same codes: bf16 = code x
    # scale written to HBM, then attention on the 16-bit tensor-core path
    # (P unquantized); timed beside the INT8 prefill
    cq = {nm: qa.qattn_rotate_block_quant(x[nm], p.layout, rot if nm != "v" else None, 128 if nm == "q" else 256,
                                          qa.QATTN_INT8) for nm in ("q", "k", "v")}
    deq = {nm: torch.empty(p.shape(), dtype=torch.bfloat16, device=dev) for nm in ("q", "k", "v")}
    dq = lambda: [qa.qattn_dequant_bf16(*cq[nm], qa.QATTN_INT8, p.layout, 128 if nm == "q" else 256, out=deq[nm])
                  for nm in ("q", "k", "v")]
    ab = lambda: qa.qattn_attention_bf16(deq["q"], deq["k"], deq["v"], p.layout, p.causal, out=out)
    i8 = lambda: qa.qattn_prefill(*cq["q"], *cq["k"], *cq["v"], qa.QATTN_INT8, p.layout, p.causal, out=out)
    ms_dq, ms_ab, ms_i8 = timeit(dq, n, flush), timeit(ab, n, flush), timeit(i8, n, flush)
    dq_bytes = 3 * x["q"].numel() * 3
    res["ablation_dequant_bf16"] = {
        "workload": "%s: INT8 codes dequantized to bf16, then bf16 attention (P unquantized)" % p.name,
        "ms_dequant": round(ms_dq, 4), "GB/s_dequant": round(dq_bytes / (ms_dq * 1e-3) / 1e9, 1),
        "ms_attention_bf16": round(ms_ab, 4), "TFLOPS_attention_bf16": round(ops / (ms_ab * 1e-3) / 1e12, 1),
        "ms_path": round(ms_dq + ms_ab, 4), "ms_int8_prefill": round(ms_i8, 4),
        "int8_speedup_over_path": round((ms_dq + ms_ab) / ms_i8, 3),
        "roofline": {"kernel": "attn_bf16", "bound": "tensor", "peak": pk_bf16, "unit": "TFLOP/s",
                     "achieved": round(ops / (ms_ab * 1e-3) / 1e12, 1),
                     "frac": round(ops / (ms_ab * 1e-3) / 1e12 / pk_bf16, 4),
                     "traffic": load_traffic("attn_bf16"), "peak_source": "measured bf16 burst (cuBLAS)"}}
    del cq, deq

    # INT4 Q/K/V on the same problem (Q/K rotated), widened to INT8 on chip
    c4 = {nm: qa.qattn_rotate_block_quant(x[nm], p.layout, rot if nm != "v" else None, 128 if nm == "q" else 256,
                                          qa.QATTN_INT4_PACKED) for nm in ("q", "k", "v")}
    pf4 = lambda: qa.qattn_prefill_mixed(*c4["q"], *c4["k"], *c4["v"], qa.QATTN_INT4_PACKED, qa.QATTN_INT4_PACKED,
                                         p.layout, p.causal, out=out)
    ms_pf4 = timeit(pf4, n, flush)

    def full4():
        for nm in ("q", "k", "v"):
            qa.qattn_rotate_block_quant(x[nm], p.layout, rot if nm != "v" else None, 128 if nm == "q" else 256,
                                        qa.QATTN_INT4_PACKED, c4[nm][0], c4[nm][1])
        pf4()
    ms_full4 = timeit(full4, n, flush)
    tops4 = ops / (ms_pf4 * 1e-3) / 1e12
    # The other order: each packed tensor widened to INT8 codes by its own
    # HBM-bound pass (the widened codes stay in L2), then the INT8 prefill;
    # its path quantizes Q/K/V in one call
    w4 = {nm: qa.qattn_widen_int4(c4[nm][0]) for nm in ("q", "k", "v")}

    def widen4():
        for nm in ("q", "k", "v"):
            qa.qattn_widen_int4(c4[nm][0], out=w4[nm])

    def pw4():
        widen4()
        qa.qattn_prefill(w4["q"], c4["q"][1], w4["k"], c4["k"][1], w4["v"], c4["v"][1], qa.QATTN_INT8, p.layout,
                         p.causal, out=out)

    def full4w():
        qa.qattn_rotate_block_quant_qkv(x["q"], x["k"], x["v"], p.layout, rot, qa.QATTN_INT4_PACKED,
                                        out=[c4["q"], c4["k"], c4["v"]])
        pw4()
    ms_w4, ms_pw4, ms_full4w = timeit(widen4, n, flush), timeit(pw4, n, flush), timeit(full4w, n, flush)
    w_bytes = 3 * sum(c4[nm][0].numel() for nm in ("q", "k", "v"))
    tops4w = ops / (ms_pw4 * 1e-3) / 1e12
    res["prefill_int4_qkv"] = {"workload": "%s, Q/K/V int4 packed" % p.name,
                               "order": "widen to INT8 first (qattn_widen_int4 x3), then the INT8 prefill",
                               "ms_prefill": round(ms_pw4, 4), "TOPS_prefill": round(tops4w, 1),
                               "ms_widen": round(ms_w4, 4), "GB/s_widen": round(w_bytes / (ms_w4 * 1e-3) / 1e9, 1),
                               "ms_path": round(ms_full4w, 4),
                               "TOPS_path": round(ops / (ms_full4w * 1e-3) / 1e12, 1),
                               "roofline": {"bound": "tensor", "peak": int8_peak, "unit": "TOPS",
                                            "frac": round(tops4w / int8_peak, 4)},
                               "on_chip": {"ms_prefill": round(ms_pf4, 4), "TOPS_prefill": round(tops4, 1),
                                           "frac": round(tops4 / int8_peak, 4), "ms_path": round(ms_full4, 4),
                                           "calls": "qattn_prefill_mixed INT4/INT4 (widened inside the kernel); "
                                                    "path: three qattn_rotate_block_quant calls"}}
    del w4
    return res


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(p, d, heads, row_chunk=128):
    """The oracle on `heads` of the workload: its own rotate+quantize of Q,
    K, V and quantized attention for every row of those heads (row_chunk
    rows per parallel job; None: one job per head)."""
    import oracle
    hs = [(0, h) for h in range(heads)]
    oq = oracle.rotate_block_quant(d["q"], p.in_dtype, p.layout, d["rot"], 128, p.code_dtype, heads=hs)
    ok_ = oracle.rotate_block_quant(d["k"], p.in_dtype, p.layout, d["rot"], 256, p.code_dtype, heads=hs)
    ov = oracle.rotate_block_quant(d["v"], p.in_dtype, p.layout, None, 256, p.code_dtype, heads=hs)
    rows = {(b, h): list(range(p.N)) for (b, h) in hs}
    oracle.prefill_rows(*oq, *ok_, *ov, p.code_dtype, p.layout, p.causal, rows, row_chunk=row_chunk)


def cpu_baseline(p, d, target_s):
    """The oracle on the whole workload when that fits the time budget (it
    takes a few seconds on 8 cores), else on as many heads as fit."""
    import oracle
    oracle.build()
    cores = oracle.threads()
    t0 = time.perf_counter()
    oracle_sample(p, d, 1)
    one = time.perf_counter() - t0
    heads = int(max(1, min(p.H, target_s / max(one, 1e-3))))
    t0 = time.perf_counter()
    oracle_sample(p, d, heads)
    dt = time.perf_counter() - t0
    ops = prefill_ops(1, heads, p.N, p.D, p.causal)
    # one thread: one head as a single job (its rotation and all its rows in
    # one call each), the same work per head as above
    t0 = time.perf_counter()
    oracle_sample(p, d, 1, row_chunk=None)
    dt1 = time.perf_counter() - t0
    ops1 = prefill_ops(1, 1, p.N, p.D, p.causal)
    return {"value": round(ops / dt / 1e12, 6), "unit": "TOPS", "cores": cores, "kind": "oracle",
            "sample": "%d of %d heads of %s (all rows: rotate+quantize Q/K/V and quantized attention), %.1f s"
                      % (heads, p.H, p.name, dt),
            "value_1thread": round(ops1 / dt1 / 1e12, 6), "cores_1thread": 1,
            "sample_1thread": "1 head of %s on one thread, %.1f s" % (p.name, dt1)}


def _v_absmax(vc, vs, p, b, h):
    """max |dequantized V| of head (b, h) (the tolerance's scale)."""
    import synth
    codes = vc[b, h] if p.layout == synth.BNSD else vc[b, :, h]
    if p.code_dtype == synth.INT8:
        vals = np.abs(codes.view(np.int8).astype(np.float64))
    else:
        import oracle
        vals = np.abs(oracle.e4m3_decode(codes).astype(np.float64))
    blk = np.arange(codes.shape[0]) // p.kv_block
    return float((vals.max(axis=1) * vs[b, h, blk].astype(np.float64)).max())


def _bf16(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _prefill_errors(entry, heads, rows):
    """Sampled rows of a GPU prefill output against the oracle (same codes,
    same algorithm) and against float64 attention on the unquantized inputs;
    errors relative to max |V| of the head (dequantized)."""
    import oracle
    import synth
    p, d, out = entry["problem"], entry["data"], entry["out"]
    hs = [(0, h) for h in heads]
    oq = oracle.rotate_block_quant(d["q"], p.in_dtype, p.layout, d["rot"], 128, p.code_dtype, heads=hs)
    ok_ = oracle.rotate_block_quant(d["k"], p.in_dtype, p.layout, d["rot"], 256, p.code_dtype, heads=hs)
    ov = oracle.rotate_block_quant(d["v"], p.in_dtype, p.layout, None, 256, p.code_dtype, heads=hs)
    rbh = {bh: list(rows) for bh in hs}
    ref = oracle.prefill_rows(*oq, *ok_, *ov, p.code_dtype, p.layout, p.causal, rbh)
    exact = oracle.exact_rows(d["q"], d["k"], d["v"], p.in_dtype, p.layout, p.causal, rbh)
    e_or, e_ex = [], []
    for (b, h) in hs:
        got = _bf16(out[b, h] if p.layout == synth.BNSD else out[b, :, h])[list(rows)]
        vmax = _v_absmax(ov[0], ov[1], p, b, h)
        e_or.append(np.abs(got - _bf16(ref[(b, h)][0])) / vmax)
        e_ex.append(np.abs(got - exact[(b, h)]) / vmax)
    e_or, e_ex = np.concatenate(e_or), np.concatenate(e_ex)
    return {"rows": "%d rows of heads %s" % (len(rows), heads), "max_abs_vs_oracle": float(e_or.max()),
            "mean_abs_vs_oracle": float(e_or.mean()), "max_abs_vs_fp64": float(e_ex.max()),
            "mean_abs_vs_fp64": float(e_ex.mean()), "within_tolerance": bool(e_or.max() <= 1e-2 and e_or.mean() <= 1e-3),
            "scale": "max |dequantized V| of the head"}


def _decode_dequant(p, k, scales, b, hk):
    """float64 K or V rows [L, D] of cache head (b, hk), codes x scales."""
    import synth
    if p.kv_dtype == synth.INT8:
        blk = np.arange(p.L) // p.kv_block
        return k[b, hk].astype(np.float64) * scales[b, hk, blk].astype(np.float64)[:, None]
    raw = k[b, hk]
    lo = ((raw & 0xF).astype(np.int16) ^ 8) - 8
    hi = ((raw >> 4).astype(np.int16) ^ 8) - 8
    codes = np.empty((p.L, p.D), np.float64)
    codes[:, 0::2], codes[:, 1::2] = lo, hi
    sc = scales[b, hk].view(np.float16).astype(np.float64)            # [L, D / group]
    return codes * np.repeat(sc, p.group, axis=1)


def _decode_errors(entry, pairs):
    """Sampled (b, h_q) outputs of a GPU decode against the oracle (query
    quantized to INT8 per head, as the method reads it) and against float64
    attention with the unquantized bf16 query over the dequantized cache (the
    cost of that query quantization shows in the second figure)."""
    import oracle
    p, dd, out = entry["problem"], entry["data"], entry["out"]
    ref, _ = oracle.decode(dd["q"], entry["k"], entry["v"], dd["k_scales"], dd["v_scales"], p.kv_dtype, p.Hkv,
                           heads=pairs, kv_block=p.kv_block, group=p.group)
    e_or, e_ex = [], []
    for (b, h) in pairs:
        hk = h // (p.Hq // p.Hkv)
        K = _decode_dequant(p, entry["k"], dd["k_scales"], b, hk)
        V = _decode_dequant(p, entry["v"], dd["v_scales"], b, hk)
        q = _bf16(dd["q"][b, h, 0])
        s = K @ q / np.sqrt(p.D)
        w = np.exp(s - s.max())
        exact = (w @ V) / w.sum()
        got = _bf16(out[b, h, 0])
        vmax = float(np.abs(V).max())
        e_or.append(np.abs(got - _bf16(ref[b, h, 0])) / vmax)
        e_ex.append(np.abs(got - exact) / vmax)
    e_or, e_ex = np.concatenate(e_or), np.concatenate(e_ex)
    return {"rows": "(b, h_q) pairs %s" % (pairs,), "max_abs_vs_oracle": float(e_or.max()),
            "mean_abs_vs_oracle": float(e_or.mean()), "max_abs_vs_fp64_unquantized_query": float(e_ex.max()),
            "mean_abs_vs_fp64_unquantized_query": float(e_ex.mean()),
            "within_tolerance": bool(e_or.max() <= 1e-2 and e_or.mean() <= 1e-3),
            "scale": "max |dequantized V| of the head"}


def parity_errors(keep):
    """Error figures of this run's GPU outputs, one entry per stated problem
    (computed on the host after the timed regions)."""
    res = {}
    try:
        if "tiny_fp8" in keep:
            res["tiny_fp8"] = _prefill_errors(keep["tiny_fp8"], [0, 1], range(256))
        if "int8_causal" in keep:
            res["int8_causal"] = _prefill_errors(keep["int8_causal"], [0, 31],
                                                 list(range(64)) + list(range(4032, 4096)))
        if "prefill_fp8_long" in keep:
            res["fp8_long"] = _prefill_errors(keep["prefill_fp8_long"], [0, 23],
                                              list(range(64)) + list(range(16320, 16384)))
        if "decode_int8kv" in keep:
            res["int8kv_decode"] = _decode_errors(keep["decode_int8kv"], [(0, 0), (17, 5), (33, 31), (63, 12)])
        if "decode_int4kv" in keep:
            res["int4kv_decode"] = _decode_errors(keep["decode_int4kv"], [(0, 0), (5, 9), (11, 30), (15, 17)])
    except Exception as e:      # a report, never a reason to lose the bench line
        res["error"] = repr(e)
    return res


def reference_arm(args):
    """Reference arm: the CPU oracle as it stands, each step a bounded sample
    (args.ref_heads heads, every row) of the same workload."""
    import synth
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    p = synth.INT8_CAUSAL
    d = synth.make_prefill(p)
    import oracle
    oracle.build()
    cores = oracle.threads()
    heads = args.ref_heads
    for _ in range(args.warmup):
        oracle_sample(p, d, heads)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_sample(p, d, heads)
        ts.append(time.perf_counter() - t0)
    ms = float(np.mean(ts)) * 1e3
    ops = prefill_ops(1, heads, p.N, p.D, p.causal)
    value = ops / (ms * 1e-3) / 1e12
    sample = "%d of %d heads of %s per step (all rows: rotate+quantize Q/K/V and quantized attention)" % (
        heads, p.H, p.name)
    line = {"metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": p.name, "B": p.B, "H": p.H, "N": p.N, "D": p.D, "layout": "BNSD", "causal": True},
            "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)



def capture_graph(fn, warm):
    """A CUDA graph of the launches fn(stream) makes, captured after `warm`
    eager runs on a side stream (capture wants warmed-up callers)."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(max(1, warm)):
            fn(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn(torch.cuda.current_stream())
    torch.cuda.synchronize()
    return g


def time_graph(g, reps, warm, stream, flush=None):
    """Mean device time (ms) of graph replays, each after flush(): CUDA events
    on the replaying stream around each replay."""
    import torch
    ts = []
    for i in range(warm + reps):
        if flush is not None:
            flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        b.synchronize()
        if i >= warm:
            ts.append(a.elapsed_time(b))
    return float(np.mean(ts))

def profile_case(args):
    """Runs one workload (warmup + steps launches, no timing, no JSON): the
    command line that the ncu summaries under profiles/ were captured with."""
    import torch

    import block_quantized_precision_b200 as qa
    import synth
    dev = torch.device("cuda", 0)
    c = args.case
    if c.startswith("kv_append"):
        # the bandwidth-scale append: K of a 4096-token prefill into an empty
        # cache of the decode problem's shape
        p = synth.INT8_KV_DECODE if c == "kv_append_int8" else synth.INT4_KV_DECODE
        kvt = qa.QATTN_INT8 if c == "kv_append_int8" else qa.QATTN_INT4_PACKED
        g = torch.Generator(device=dev).manual_seed(8)
        xn = torch.randn((p.B, p.Hkv, 4096, p.D), generator=g, device=dev).to(torch.bfloat16)
        if kvt == qa.QATTN_INT8:
            cache = torch.zeros((p.B, p.Hkv, 4096, p.D), dtype=torch.int8, device=dev)
            scl = torch.zeros((p.B, p.Hkv, 16), dtype=torch.float32, device=dev)
        else:
            cache = torch.zeros((p.B, p.Hkv, 4096, p.D // 2), dtype=torch.uint8, device=dev)
            scl = torch.zeros((p.B, p.Hkv, 4096, p.D // p.group), dtype=torch.float16, device=dev)
        for _ in range(args.warmup + args.steps):
            qa.qattn_kv_append(xn, cache, scl, 0, kvt, group=p.group)
    elif c == "step_int8":
        # the benchmark step as bench.py times it: one quantization call and
        # the prefill, captured as a CUDA graph after eager warm-up runs
        p = synth.INT8_CAUSAL
        d = synth.make_prefill(p)
        x = {n: torch.from_numpy(d[n].view(np.int16)).to(dev).view(torch.bfloat16) for n in ("q", "k", "v")}
        rot = torch.from_numpy(d["rot"]).to(dev)
        shp = p.shape()
        nqb, nkb = -(-p.N // 128), -(-p.N // 256)
        c3 = [(torch.empty(shp, dtype=torch.uint8, device=dev), torch.empty((p.B, p.H, nb), device=dev))
              for nb in (nqb, nkb, nkb)]
        out = torch.empty(shp, dtype=torch.bfloat16, device=dev)

        def body(st):
            qa.qattn_rotate_block_quant_qkv(x["q"], x["k"], x["v"], p.layout, rot, p.code_dtype, out=c3, stream=st)
            qa.qattn_prefill(*c3[0], *c3[1], *c3[2], p.code_dtype, p.layout, p.causal, out=out, stream=st)
        g = capture_graph(body, args.warmup)
        for _ in range(args.warmup + args.steps):
            g.replay()
    elif c == "ablation_bf16":
        # the dequantize-first comparison path on the INT8 causal problem
        p = synth.INT8_CAUSAL
        d = synth.make_prefill(p)
        x = {n: torch.from_numpy(d[n].view(np.int16)).to(dev).view(torch.bfloat16) for n in ("q", "k", "v")}
        rot = torch.from_numpy(d["rot"]).to(dev)
        for _ in range(args.warmup + args.steps):
            deq = []
            for n in ("q", "k", "v"):
                cs = qa.qattn_rotate_block_quant(x[n], p.layout, rot if n != "v" else None, 128 if n == "q" else 256,
                                                 qa.QATTN_INT8)
                deq.append(qa.qattn_dequant_bf16(*cs, qa.QATTN_INT8, p.layout, 128 if n == "q" else 256))
            qa.qattn_attention_bf16(*deq, p.layout, p.causal)
    elif c.startswith("decode"):
        p = synth.INT8_KV_DECODE if c == "decode_int8kv" else synth.INT4_KV_DECODE
        dd = synth.make_decode(p)
        q = torch.from_numpy(dd["q"].view(np.int16)).to(dev).view(torch.bfloat16)
        k, v = torch.from_numpy(dd["k"]).to(dev), torch.from_numpy(dd["v"]).to(dev)
        if p.kv_dtype == synth.INT8:
            ks, vs, kvt = torch.from_numpy(dd["k_scales"]).to(dev), torch.from_numpy(dd["v_scales"]).to(dev), qa.QATTN_INT8
        else:
            ks = torch.from_numpy(dd["k_scales"].view(np.int16)).to(dev).view(torch.float16)
            vs = torch.from_numpy(dd["v_scales"].view(np.int16)).to(dev).view(torch.float16)
            kvt = qa.QATTN_INT4_PACKED
        for _ in range(args.warmup + args.steps):
            qa.qattn_decode_kvq(q, k, v, ks, vs, kvt, kv_block=p.kv_block, group=p.group)
    else:
        p = synth.FP8_LONG if c == "prefill_fp8" else synth.INT8_CAUSAL
        # prefill_int4v: the INT8 causal problem with V in packed INT4;
        # prefill_int4: with Q, K and V in packed INT4; prefill_int4_widened:
        # the same codes widened to INT8 first, then the INT8 prefill
        int4 = ("prefill_int4v", "prefill_int4", "prefill_int4_widened")
        vt = qa.QATTN_INT4_PACKED if c in int4 else p.code_dtype
        qkt = qa.QATTN_INT4_PACKED if c in int4[1:] else p.code_dtype
        d = synth.make_prefill(p)
        x = {n: torch.from_numpy(d[n].view(np.int16)).to(dev).view(torch.bfloat16) for n in ("q", "k", "v")}
        rot = torch.from_numpy(d["rot"]).to(dev)
        for _ in range(args.warmup + args.steps):
            qc = qa.qattn_rotate_block_quant(x["q"], p.layout, rot, 128, qkt)
            kc = qa.qattn_rotate_block_quant(x["k"], p.layout, rot, 256, qkt)
            vc = qa.qattn_rotate_block_quant(x["v"], p.layout, None, 256, vt)
            if c == "prefill_int4_widened":
                qa.qattn_prefill(qa.qattn_widen_int4(qc[0]), qc[1], qa.qattn_widen_int4(kc[0]), kc[1],
                                 qa.qattn_widen_int4(vc[0]), vc[1], qa.QATTN_INT8, p.layout, p.causal)
            else:
                qa.qattn_prefill_mixed(*qc, *kc, *vc, qkt, vt, p.layout, p.causal)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    print("case %s: ok" % c)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the decode / FP8 measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--ref-heads", type=int, default=4, help="heads per reference-arm step")
    ap.add_argument("--case", default=None,
                    choices=["step_int8", "prefill_int8", "prefill_fp8", "prefill_int4v", "prefill_int4",
                             "prefill_int4_widened", "decode_int8kv", "decode_int4kv", "kv_append_int8",
                             "kv_append_int4", "ablation_bf16"],
                    help="run one workload only (for profiler captures); prints no JSON")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.case:
        profile_case(args)
    elif args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
