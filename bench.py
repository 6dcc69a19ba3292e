#!/usr/bin/env python3
"""Benchmark of the CSA/HCA hybrid-attention hot path: CSA decode at 1M context.

Workload (N=1): 8 sequences x 1048576 raw tokens -> 262144 compressed CSA entries each,
128 query heads over one KV head (d = 128), lightning indexer with 16 heads x 64 dims in
MXFP4, BF16 index scores, top-1024, 128-token raw window, KV rows in E4M3 (non-RoPE dims,
per-row scale) + BF16 (RoPE dims).  One step = one decode query per sequence through the
whole path: quantise q_I -> index scores -> top-k -> sparse attention (+ split merge).

Data-parallel over sequences: with N GPUs every rank runs its own 8 sequences (weak
scaling, no data-path collective); the timing is the max over ranks.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle instead.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA decode queries/s at 1M ctx; achieved HBM GB/s and % of roofline"
UNIT = "queries/s"
FALLBACK_HBM_GBS = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def workload():
    from synth.configs import CSA_1M
    return CSA_1M


def bytes_per_query(cfg):
    """Algorithmic HBM bytes of one decode query (the whole step, per sequence)."""
    kI = cfg.Nc * (cfg.dI // 2 + cfg.dI // 32)           # MXFP4 index keys: 34 B / entry
    rows = (cfg.k + cfg.W) * (cfg.d // 2 + 4 + cfg.d)     # gathered split rows: 196 B / row
    qo = 2 * cfg.H * cfg.d * 2 + cfg.HI * cfg.dI * 2 + cfg.HI * 4 + 4   # q in, o out, q_I, w
    return kI + rows + qo


def rank_sequences(n_per_rank, rank):
    """Global ids of the sequences rank `rank` decodes (weak scaling: a fixed number per
    rank, disjoint across ranks, no data-path exchange)."""
    return list(range(rank * n_per_rank, (rank + 1) * n_per_rank))


def max_over_ranks(x, world, device):
    """The slowest rank's value (a device-side all-reduce MAX); x itself when world == 1."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# DRAM traffic of one decode indexer launch as measured once with ncu (dram__bytes_read.sum +
# dram__bytes_write.sum of one launch over 16 sequences, `--kernel indexer --batch 16`), per
# sequence.  It is reported only while the indexer source is byte-identical to the source that
# was profiled (its hash below); after any change it is null until the next capture.
INDEXER_TRAFFIC = {"source_sha256_16": "13421fb6350a5216",
                   "bytes_per_seq": (142.652672e6 + 4.876544e6) / 16}


def indexer_traffic(B):
    import hashlib
    src = os.path.join(ROOT, "heavily_compressed_long_b200", "csrc", "indexer.cu")
    with open(src, "rb") as fh:
        h = hashlib.sha256(fh.read()).hexdigest()[:16]
    return B * INDEXER_TRAFFIC["bytes_per_seq"] if h == INDEXER_TRAFFIC["source_sha256_16"] else None


def indexer_bytes_per_launch(cfg, B):
    """Algorithmic bytes of one indexer launch: MXFP4 keys read + bf16 scores written."""
    return B * cfg.Nc * (cfg.dI // 2 + cfg.dI // 32 + 2)


# ------------------------------------------------------------------------------------------
# clocks sampled during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sms, maxs, util_sms, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax, util = float(parts[1]), float(parts[2]), float(parts[4])
            except ValueError:
                continue
            sms.append(sm)
            maxs.append(smax)
            if util >= 50:
                util_sms.append(sm)
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        src = util_sms or sms
        return {"sm_mhz": statistics.median(src) if src else None,
                "sm_max_mhz": max(maxs) if maxs else None,
                "reasons": sorted(reasons), "samples": len(self.lines),
                "samples_under_load": len(util_sms)}


# ------------------------------------------------------------------------------------------
# CPU oracle timing (the baseline / reference arm)

def oracle_query_sample(cfg, seed_b, n_keys):
    """Inputs of one decode query restricted to the first n_keys compressed entries, as the
    oracle consumes them (quantised by the oracle)."""
    import numpy as np
    import oracle
    from synth import gen
    from synth.configs import scaled
    c = scaled(cfg, B=1)
    kI = gen.index_keys(scaled(cfg, L=4 * n_keys), [seed_b])
    kp, ks = oracle.quant_mxfp4(kI)
    kvc = gen.comp_kv(cfg, [seed_b], n_keys)
    cn, cs, cr = oracle.quant_kv_fp8(kvc)
    raw = gen.raw_kv(cfg, [seed_b], cfg.L - cfg.W, cfg.L)
    rn, rs, rr = oracle.quant_kv_fp8(raw)
    q, qI, w = gen.queries(c, [seed_b]), gen.index_queries(c, [seed_b]), gen.head_weights(c, [seed_b])
    pos = np.full((1, 1), 4 * n_keys - 1, np.int32)      # every sampled entry visible
    return dict(kp=kp, ks=ks, cn=cn, cs=cs, cr=cr, rn=rn, rs=rs, rr=rr, q=q, qI=qI, w=w, pos=pos,
                n_keys=n_keys)


def oracle_step(cfg, s):
    import oracle
    qp, qs = oracle.quant_mxfp4(s["qI"])
    sc = oracle.index_scores(oracle.FMT_MXFP4, qp, s["w"], s["kp"], s["pos"], cfg.m, qI_sf=qs,
                             kI_sf=s["ks"], bf16_scores=True)
    idx = oracle.topk(sc, s["pos"], cfg.m, cfg.k)
    okc = oracle.KV(oracle.FMT_FP8SPLIT, s["cn"], s["n_keys"], scale=s["cs"], rope=s["cr"])
    # window rows are stored as a ring of W slots holding tokens L-W .. L-1; with the sampled
    # query position 4*n_keys-1 the window reads the ring's slots through the same t mod W map
    okr = oracle.KV(oracle.FMT_FP8SPLIT, s["rn"], cfg.W, scale=s["rs"], rope=s["rr"])
    return oracle.csa_attn(s["q"], okc, idx, okr, cfg.W, s["pos"])


def time_oracle(cfg, seconds, min_steps=1, frac=1.0):
    """Run oracle decode queries (each over frac of the entries) for about `seconds`."""
    n_keys = max(cfg.k + 1, int(cfg.Nc * frac))
    s = oracle_query_sample(cfg, 0, n_keys)
    oracle_step(cfg, s)                                   # warm (thread pool, pages)
    t0 = time.perf_counter()
    n = 0
    while n < min_steps or time.perf_counter() - t0 < seconds:
        oracle_step(cfg, s)
        n += 1
    dt = time.perf_counter() - t0
    f = n_keys / cfg.Nc
    return n, dt, f, n_keys


def cpu_threads():
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v and v.isdigit() else os.cpu_count()


# ------------------------------------------------------------------------------------------

def run_reference(args, rank, world):
    """The oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    cfg = workload()
    K, Wm = args.steps, args.warmup
    # each step is one query over a sample of the entries sized so the run stays ~2 minutes
    est = 1.5                                          # s per full 1M query (order of magnitude)
    frac = min(1.0, 90.0 / max(1, (K + Wm)) / est)
    n_keys = max(cfg.k + 1, int(cfg.Nc * frac))
    s = oracle_query_sample(cfg, 0, n_keys)
    for _ in range(Wm):
        oracle_step(cfg, s)
    t0 = time.perf_counter()
    for _ in range(K):
        oracle_step(cfg, s)
    dt = time.perf_counter() - t0
    f = n_keys / cfg.Nc
    value = K * f / dt
    sample = (f"each step: one decode query over the first {n_keys} of {cfg.Nc} compressed "
              f"entries (fraction {f:.4f}), full top-k and attention; queries/s scaled by the fraction")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": Wm, "ms_per_step": 1e3 * dt / max(K, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "B_per_gpu": cfg.B, "L": cfg.L, "Nc": cfg.Nc,
                       "H": cfg.H, "HI": cfg.HI, "k": cfg.k, "W": cfg.W},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def build_inputs(cfg, B, rank, n_sets, device):
    """Device-resident inputs of n_sets independent decode problems (GPU-generated values,
    quantised by libhcl).  Returns pipelines and the per-step host-side query tensors."""
    import torch
    from heavily_compressed_long_b200 import api
    from heavily_compressed_long_b200.api import HCL_BF16, HCL_MXFP4, KV
    from heavily_compressed_long_b200.pipeline import CsaDecode
    Nc, W, L, d, HI, dI = cfg.Nc, cfg.W, cfg.L, cfg.d, cfg.HI, cfg.dI
    sets = []
    for s in range(n_sets):
        g = torch.Generator(device=device)
        g.manual_seed(cfg.seed + 7919 * rank + 104729 * s)
        kI_p = torch.empty(B, Nc, dI // 2, dtype=torch.uint8, device=device)
        kI_s = torch.empty(B, Nc, dI // 32, dtype=torch.uint8, device=device)
        c_n = torch.empty(B, Nc, d // 2, dtype=torch.uint8, device=device)
        c_s = torch.empty(B, Nc, dtype=torch.float32, device=device)
        c_r = torch.empty(B, Nc, d // 2, dtype=torch.bfloat16, device=device)
        for b in range(B):
            x = torch.randn(Nc, dI, generator=g, device=device).to(torch.bfloat16)
            api.hcl_quant_mxfp4(x, kI_p[b], kI_s[b])
            x = torch.randn(Nc, d, generator=g, device=device).to(torch.bfloat16)
            api.hcl_quant_kv_fp8(x, c_n[b], c_s[b], c_r[b])
            del x
        ring = torch.randn(B, W, d, generator=g, device=device).to(torch.bfloat16)
        r_n = torch.empty(B, W, d // 2, dtype=torch.uint8, device=device)
        r_s = torch.empty(B, W, dtype=torch.float32, device=device)
        r_r = torch.empty(B, W, d // 2, dtype=torch.bfloat16, device=device)
        api.hcl_quant_kv_fp8(ring, r_n, r_s, r_r)
        q = torch.randn(B, 1, cfg.H, d, generator=g, device=device).to(torch.bfloat16)
        qI = torch.randn(B, 1, HI, dI, generator=g, device=device).to(torch.bfloat16)
        w = torch.rand(B, 1, HI, generator=g, device=device)
        pos = torch.full((B, 1), L - 1, dtype=torch.int32, device=device)
        pipe = CsaDecode(q, qI, w, kI_p, KV(c_n, c_s, c_r), Nc, KV(r_n, r_s, r_r), L, W, pos,
                         m=cfg.m, k=cfg.k, op_fmt=HCL_MXFP4, score_fmt=HCL_BF16, kI_sf=kI_s)
        sets.append(pipe)
    return sets


def run_hcl(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from heavily_compressed_long_b200 import api
    from heavily_compressed_long_b200._lib import lib
    lib()                                               # fail loudly without libhcl.so
    cfg = workload()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    B = cfg.B
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    per_set = B * cfg.Nc * (cfg.dI // 2 + cfg.dI // 32)
    n_sets = max(2, -(-4 * l2 // per_set))              # streamed bytes per cycle >= 4 x L2
    sets = build_inputs(cfg, B, rank, n_sets, device)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()

    # eager warm-up (attributes, first-launch costs), then capture one graph per input set and
    # one graph of a whole cycle (one step on every set, in order), so that a run of K steps
    # is K // n_sets cycle replays plus single-step replays: few host launches per step
    with torch.cuda.stream(stream):
        for p in sets:
            p.step(stream=stream)
    torch.cuda.synchronize()
    graphs = []
    for p in sets:
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            p.step(stream=stream)
        graphs.append(gr)
    cycle = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cycle, stream=stream):
        for p in sets:
            p.step(stream=stream)
    torch.cuda.synchronize()

    def run_steps(n):
        """n decode steps, rotating over the input sets from set 0."""
        for _ in range(n // n_sets):
            cycle.replay()
        for i in range(n % n_sets):
            graphs[i].replay()

    def barrier():
        if world > 1:
            dist.barrier()

    def maxv(x):
        return max_over_ranks(x, world, device)

    K, Wm = args.steps, args.warmup
    with torch.cuda.stream(stream):
        run_steps(Wm)
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        run_steps(K)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    step_ms = maxv(e0.elapsed_time(e1) / K)

    # dominant kernel alone: the indexer, back to back over the rotating sets
    from heavily_compressed_long_b200.api import HCL_MXFP4
    with torch.cuda.stream(stream):
        for p in sets:
            api.hcl_quant_mxfp4(p.qI, p.qI_packed, p.qI_sf, stream=stream)
    torch.cuda.synchronize()
    n_idx = max(50, min(K, 2000))

    def run_indexer(i):
        p = sets[i % n_sets]
        api.hcl_csa_index_scores(HCL_MXFP4, p.qI_packed, p.w, p.kI, p.q_pos, p.m, p.scores,
                                 Nc=p.Nc, qI_sf=p.qI_sf, kI_sf=p.kI_sf, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(2 * n_sets):
            run_indexer(i)
    i0, i1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    i0.record(stream)
    with torch.cuda.stream(stream):
        for i in range(n_idx):
            run_indexer(i)
    i1.record(stream)
    torch.cuda.synchronize()
    idx_ms = maxv(i0.elapsed_time(i1) / n_idx)

    # end to end through the C ABI with host buffers: H2D of the step's queries, the fused
    # decode-step call, D2H of the outputs -- every step
    hq = [torch.empty_like(p.q, device="cpu").pin_memory() for p in sets]
    hqi = [torch.empty_like(p.qI, device="cpu").pin_memory() for p in sets]
    hw = [torch.empty_like(p.w, device="cpu").pin_memory() for p in sets]
    hpos = [torch.empty_like(p.q_pos, device="cpu").pin_memory() for p in sets]
    hout = [torch.empty_like(p.out, device="cpu").pin_memory() for p in sets]
    for j, p in enumerate(sets):
        hq[j].copy_(p.q)
        hqi[j].copy_(p.qI)
        hw[j].copy_(p.w)
        hpos[j].copy_(p.q_pos)
    h2d = hq[0].numel() * 2 + hqi[0].numel() * 2 + hw[0].numel() * 4 + hpos[0].numel() * 4
    d2h = hout[0].numel() * 2

    # One graph per cycle of input sets: the H2D copies of every set's inputs on a copy stream,
    # each set's C-ABI decode step on the main stream once its inputs have landed, and its D2H
    # copy on a third stream once that step is done -- copies overlap the other sets' steps,
    # and every step still moves its own inputs in and its output out.
    h2d_st, d2h_st = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in sets]
    ev_step = [torch.cuda.Event() for _ in sets]

    def e2e_cycle():
        h2d_st.wait_stream(stream)
        d2h_st.wait_stream(stream)
        with torch.cuda.stream(h2d_st):
            for j, p in enumerate(sets):
                p.q.copy_(hq[j], non_blocking=True)
                p.qI.copy_(hqi[j], non_blocking=True)
                p.w.copy_(hw[j], non_blocking=True)
                p.q_pos.copy_(hpos[j], non_blocking=True)
                ev_in[j].record(h2d_st)
        for j, p in enumerate(sets):
            stream.wait_event(ev_in[j])
            p.step(stream=stream)
            ev_step[j].record(stream)
            with torch.cuda.stream(d2h_st):
                d2h_st.wait_event(ev_step[j])
                hout[j].copy_(p.out, non_blocking=True)
        stream.wait_stream(h2d_st)
        stream.wait_stream(d2h_st)

    with torch.cuda.stream(stream):
        e2e_cycle()                      # eager once (first-use costs)
    torch.cuda.synchronize()
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=stream):
        e2e_cycle()
    torch.cuda.synchronize()
    n_cyc = max(3, min(K, 2000) // n_sets)
    n_e2e = n_cyc * n_sets
    with torch.cuda.stream(stream):
        for _ in range(max(1, Wm // n_sets)):
            g_e2e.replay()
    torch.cuda.synchronize()
    barrier()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(n_cyc):
            g_e2e.replay()
    x1.record(stream)
    torch.cuda.synchronize()
    barrier()
    del g_e2e
    e2e_ms = maxv(x0.elapsed_time(x1) / n_e2e)
    clocks = sampler.stop() if sampler else None
    extra = {}
    if rank == 0 and world == 1 and not args.no_extra:
        extra["cache_append"] = measure_cache_append(sets[0], device, stream)
        del sets[1:]                      # room for the prefill workload
        torch.cuda.empty_cache()
        extra["prefill"] = measure_prefill(device, stream)
    status = int(sum(int(p.status.item()) for p in sets))

    # CPU baseline: the oracle on the host cores, a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, dt, f, n_keys = time_oracle(cfg, args.cpu_seconds, frac=args.cpu_frac)
        cpu = {"value": n * f / dt, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{n} decode queries, each over the first {n_keys} of {cfg.Nc} entries "
                         f"(fraction {f:.3f}), full top-k and attention; scaled by the fraction"}

    if rank == 0:
        hbm, src = peaks()
        q_per_step = B * world
        value = q_per_step / (step_ms * 1e-3)
        bpq = bytes_per_query(cfg)
        step_gbs = B * bpq / (step_ms * 1e-3) / 1e9
        idx_bytes = indexer_bytes_per_launch(cfg, B)
        idx_gbs = idx_bytes / (idx_ms * 1e-3) / 1e9
        launches = sets[0].launches_per_step()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": Wm, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "mxfp4+e4m3+bf16 (fp32 accumulate)",
            "data": "synthetic: seeded N(0,1) on device, MXFP4 / E4M3 quantised by libhcl",
            "config": {"workload": cfg.name, "B_per_gpu": B, "L": cfg.L, "Nc": cfg.Nc, "H": cfg.H,
                       "HI": cfg.HI, "dI": cfg.dI, "k": cfg.k, "W": cfg.W,
                       "parallelism": f"dp{world} (sequences)",
                       "l2": f"{n_sets} rotating input sets ({n_sets * per_set / 1e6:.0f} MB of index "
                             f"keys streamed per cycle vs {l2 / 1e6:.0f} MB L2)",
                       "timing": "CUDA graph per input set, CUDA events, max over ranks"},
            "step_hbm_gbs": step_gbs,
            "step_frac_of_hbm": step_gbs / hbm,
            "bytes_per_query": bpq,
            "roofline": {"bound": "hbm", "kernel": "indexer (tcgen05 kind::mxf4)",
                         "achieved": idx_gbs, "peak": hbm, "unit": "GB/s", "frac": idx_gbs / hbm,
                         "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else "fallback 6.65 TB/s",
                         "bytes_per_launch": idx_bytes, "ms_per_launch": idx_ms,
                         "share_of_step": idx_ms / step_ms, "traffic": indexer_traffic(B),
                         "traffic_source": "ncu capture at 16 sequences, scaled per sequence"},
            "e2e": {"value": q_per_step / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "path": "hcl_csa_decode_step (C ABI) per step with its pinned H2D input copies "
                            "and D2H output copy, one CUDA graph per cycle of input sets, copies on "
                            "their own streams overlapping other sets' steps"},
            "gpu_launches": K * launches,
            "device_status": status,
            "clocks": clocks,
        }
        line.update(extra)
        if cpu:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    for gr in graphs:
        del gr
    graphs.clear()
    del cycle


def _time_ms(fn, stream, reps, warm=2):
    """Average device time of fn() (enqueued on `stream`) over reps calls, CUDA events."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warm):
            fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_cache_append(p, device, stream, steps=128):
    """Per-step cost of the decode-time cache append of a CSA layer for the decode workload's
    sequences (raw window and entries as split FP8 rows, MXFP4 index keys; one CSA entry every
    4 tokens), B tokens per step: one launch, graph-replayed over `steps` consecutive positions."""
    import torch
    from heavily_compressed_long_b200 import api
    B, d = p.B, p.q.shape[-1]
    g = torch.Generator(device=device)
    g.manual_seed(11)
    stage_kv = torch.randn(B, 128, d, generator=g, device=device).to(torch.bfloat16)
    stage_g = torch.randn(B, 128, d, generator=g, device=device).to(torch.bfloat16)
    kv_new = torch.randn(steps, B, d, generator=g, device=device).to(torch.bfloat16)
    g_new = torch.randn(steps, B, d, generator=g, device=device).to(torch.bfloat16)
    kI_new = torch.randn(steps, B, 64, generator=g, device=device).to(torch.bfloat16)
    bias = 0.1 * torch.randn(8, generator=g, device=device)
    t0 = p.L
    ts = [torch.full((B,), t0 + s, dtype=torch.int32, device=device) for s in range(steps)]

    def run_all():
        for s in range(steps):
            api.hcl_cache_append(kv_new[s], g_new[s], ts[s], stage_kv, stage_g, p.raw, kvc=p.kvc,
                                 bias_csa=bias, m=p.m, kI_new=kI_new[s], kI=p.kI, kI_sf=p.kI_sf,
                                 stream=stream)

    with torch.cuda.stream(stream):
        run_all()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=stream):
        run_all()
    ms = _time_ms(gr.replay, stream, 3, warm=1) / steps
    del gr
    return {"us_per_step": ms * 1e3, "sequences": B, "launches_per_step": 1,
            "what": "hcl_cache_append: raw window row + staging rings every step, CSA entry "
                    "(split FP8) + MXFP4 index key every 4th step"}


def measure_prefill(device, stream):
    """The chunked-prefill workload (4096 new tokens on a 262144-token context, 64 heads, CSA
    top-1024 + HCA, 128-token window): the prefill indexer alone (TFLOP/s vs the measured bf16
    dense peak), the HCA prefill attention alone, and the whole CSA/HCA layer pair (ms)."""
    import torch
    from heavily_compressed_long_b200 import api
    from heavily_compressed_long_b200.api import HCL_BF16, KV
    from heavily_compressed_long_b200.pipeline import HcaLayer, PairPrefill
    from synth.configs import PAIR_PREFILL as cfg
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed)
    L, d, Tq, H, HI, dI, Nc, Nh = cfg.L, cfg.d, cfg.Tq, cfg.H, cfg.HI, cfg.dI, cfg.Nc, cfg.Nh
    bf = lambda *sh: torch.randn(*sh, generator=g, device=device).to(torch.bfloat16)
    kv, gate = bf(1, L, d), bf(1, L, d)
    q_csa, q_hca = bf(1, Tq, H, d), bf(1, Tq, H, d)
    qI, kI = bf(1, Tq, HI, dI), bf(1, Nc, dI)
    w = torch.rand(1, Tq, HI, generator=g, device=device)
    b_csa = 0.1 * torch.randn(2 * cfg.m, generator=g, device=device)
    b_hca = 0.1 * torch.randn(cfg.mh, generator=g, device=device)
    pos = torch.arange(cfg.first_pos, cfg.first_pos + Tq, dtype=torch.int32, device=device).unsqueeze(0).contiguous()
    comp_c = torch.zeros(1, Nc, d, dtype=torch.bfloat16, device=device)
    comp_h = torch.zeros(1, Nh, d, dtype=torch.bfloat16, device=device)
    pp = PairPrefill(kv, gate, b_csa, b_hca, comp_c, comp_h, q_csa, q_hca, qI, w, kI, pos,
                     cfg.first_pos, m=cfg.m, mh=cfg.mh, k=cfg.k, W=cfg.W, score_fmt=HCL_BF16)
    with torch.cuda.stream(stream):
        pp.compress_prior(stream=stream)
    torch.cuda.synchronize()
    pair_ms = _time_ms(lambda: pp.step(stream=stream), stream, 5)
    idx_ms = _time_ms(lambda: api.hcl_csa_index_scores(HCL_BF16, qI, w, kI, pos, cfg.m, pp.scores,
                                                       stream=stream), stream, 10)
    hca = HcaLayer(q_hca, KV(comp_h), Nh, cfg.mh, KV(kv), L, cfg.W, pos)
    hca_ms = _time_ms(lambda: hca.step(stream=stream), stream, 10)
    peak = bf16_peak()
    idx_flops = 2.0 * HI * dI * sum(min(Nc, (p_ + 1) // cfg.m) for p_ in range(cfg.first_pos, cfg.first_pos + Tq))
    rows = sum(min(Nh, (p_ + 1) // cfg.mh) + min(cfg.W, p_ + 1) for p_ in range(cfg.first_pos, cfg.first_pos + Tq))
    hca_flops = 4.0 * H * d * rows
    return {"workload": cfg.name,
            "layer_pair_ms": pair_ms,
            "indexer": {"ms": idx_ms, "tflops": idx_flops / idx_ms / 1e9,
                        "frac_of_bf16_peak": idx_flops / idx_ms / 1e9 / peak,
                        "flops": idx_flops, "note": "2 x 16 heads x 64 per visible (query, entry) pair; masked pairs not counted"},
            "hca_attention": {"ms": hca_ms, "tflops": hca_flops / hca_ms / 1e9,
                              "frac_of_bf16_peak": hca_flops / hca_ms / 1e9 / peak, "flops": hca_flops,
                              "note": "4 flops per (query, head, visible row, dim)"},
            "peak_tflops": peak, "peak_source": "MEASURED_PEAKS.json bf16_tflops (burst)"}


def run_prefill_indexer(args, local_rank):
    """The lightning indexer on the chunked-prefill shape (4096 new queries x 16 heads x 64
    against 66560 compressed entries, bf16 operands, bf16 scores, entry-causal): a dense
    tensor-core contraction.  Prints TFLOP/s against the measured bf16 dense peak."""
    import torch
    from heavily_compressed_long_b200 import api
    from heavily_compressed_long_b200.api import HCL_BF16
    from synth.configs import PAIR_PREFILL as cfg
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed)
    Tq, HI, dI, Nc = cfg.Tq, cfg.HI, cfg.dI, cfg.Nc
    qI = torch.randn(1, Tq, HI, dI, generator=g, device=device).to(torch.bfloat16)
    kI = torch.randn(1, Nc, dI, generator=g, device=device).to(torch.bfloat16)
    w = torch.rand(1, Tq, HI, generator=g, device=device)
    pos = torch.arange(cfg.first_pos, cfg.first_pos + Tq, dtype=torch.int32,
                       device=device).unsqueeze(0).contiguous()
    scores = torch.empty(1, Tq, Nc, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.Stream(device)

    def launch():
        api.hcl_csa_index_scores(HCL_BF16, qI, w, kI, pos, cfg.m, scores, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup)):
            launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            launch()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    # useful work: the visible (query, entry) pairs only (masked tiles are computed but not
    # counted)
    flops = 2.0 * HI * dI * sum(min(Nc, (p_ + 1) // cfg.m) for p_ in range(cfg.first_pos, cfg.first_pos + Tq))
    peak = 1662.1
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            peak = float(json.load(f)["bf16_tflops"])
    print(json.dumps({"kernel": "indexer_prefill", "workload": f"{cfg.name} indexer",
                      "ms_per_launch": ms, "flops_per_launch": flops,
                      "achieved_tflops": flops / ms / 1e9, "peak_tflops": peak,
                      "frac": flops / ms / 1e9 / peak,
                      "scores_bytes": Tq * Nc * 2}), flush=True)


def run_hca_shape_micro(args, local_rank):
    """The compressors and the HCA prefill attention alone on the HCA workload's shapes (4
    sequences x 65536 raw tokens; 2048 queries x 16 heads per sequence for the attention), one
    kernel back to back from a CUDA graph.  Prints achieved GB/s (compressors: kv + gate read,
    entries written) or TFLOP/s (attention: 4 flops per (query, head, row, dim) over the rows
    each query sees)."""
    import torch
    from heavily_compressed_long_b200 import api
    from heavily_compressed_long_b200.api import KV
    from synth.configs import HCA_64K as cfg
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed)
    B, L, d, mh, W, Tq, H = cfg.B, cfg.L, cfg.d, cfg.mh, cfg.W, cfg.Tq, cfg.H
    kv = torch.randn(B, L, d, generator=g, device=device).to(torch.bfloat16)
    gate = torch.randn(B, L, d, generator=g, device=device).to(torch.bfloat16)
    stream = torch.cuda.Stream(device)
    if args.kernel == "compress_csa":
        m, n_ent = cfg.m, -(-L // cfg.m)
        bias = 0.1 * torch.randn(2 * m, generator=g, device=device)
        out = torch.empty(B, n_ent, d, dtype=torch.bfloat16, device=device)
        launch = lambda: api.hcl_csa_compress(kv, gate, bias, m, out, stream=stream)
        nbytes, flops = 2 * kv.numel() * 2 + out.numel() * 2, None
    elif args.kernel == "compress_hca":
        n_ent = -(-L // mh)
        bias = 0.1 * torch.randn(mh, generator=g, device=device)
        out = torch.empty(B, n_ent, d, dtype=torch.bfloat16, device=device)
        launch = lambda: api.hcl_hca_compress(kv, gate, bias, mh, out, stream=stream)
        nbytes, flops = 2 * kv.numel() * 2 + out.numel() * 2, None
    else:
        Nh = -(-L // mh)
        ent = torch.randn(B, Nh, d, generator=g, device=device).to(torch.bfloat16)
        q = torch.randn(B, Tq, H, d, generator=g, device=device).to(torch.bfloat16)
        pos = torch.arange(L - Tq, L, dtype=torch.int32, device=device).repeat(B, 1).contiguous()
        layer = None
        from heavily_compressed_long_b200.pipeline import HcaLayer
        layer = HcaLayer(q, KV(ent), Nh, mh, KV(kv), L, W, pos)
        launch = lambda: layer.step(stream=stream)
        rows = sum(min(Nh, (p + 1) // mh) + min(W, p + 1) for p in range(L - Tq, L))
        nbytes, flops = None, 4.0 * B * H * d * rows
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            launch()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(args.steps):
            launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    del graph
    line = {"kernel": args.kernel, "workload": f"{cfg.name} shapes", "ms_per_launch": ms,
            "launches": args.steps}
    if nbytes:
        hbm, src = peaks()
        line.update({"bytes_per_launch": nbytes, "achieved_gbs": nbytes / ms / 1e6,
                     "peak_gbs": hbm, "frac": nbytes / ms / 1e6 / hbm, "peak_source": src})
    else:
        line.update({"flops_per_launch": flops, "achieved_tflops": flops / ms / 1e9,
                     "frac_of_bf16_peak": flops / ms / 1e9 / bf16_peak()})
    print(json.dumps(line), flush=True)


def bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


def run_kernel_micro(args, local_rank):
    """One kernel alone on one input set of `--batch` sequences (indexer: larger than L2),
    for profiling: times back-to-back launches with CUDA events and prints a JSON line."""
    import torch
    from heavily_compressed_long_b200 import api
    from heavily_compressed_long_b200.api import HCL_MXFP4
    if args.kernel == "indexer_prefill":
        return run_prefill_indexer(args, local_rank)
    if args.kernel in ("compress_csa", "compress_hca", "hca_prefill"):
        return run_hca_shape_micro(args, local_rank)
    cfg = workload()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    B = args.batch
    (p,) = build_inputs(cfg, B, 0, 1, device)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        api.hcl_quant_mxfp4(p.qI, p.qI_packed, p.qI_sf, stream=stream)
        p.step_parts(stream=stream)
    torch.cuda.synchronize()

    def launch():
        if args.kernel == "indexer":
            api.hcl_csa_index_scores(HCL_MXFP4, p.qI_packed, p.w, p.kI, p.q_pos, p.m, p.scores,
                                     Nc=p.Nc, qI_sf=p.qI_sf, kI_sf=p.kI_sf, stream=stream)
        elif args.kernel == "topk":
            api.hcl_csa_topk(p.scores, p.q_pos, p.m, p.k, p.idx, stream=stream)
        elif args.kernel == "step":
            p.step(stream=stream)
        else:
            api.hcl_csa_sparse_attn(p.q, p.kvc, p.Nc, p.idx, p.raw, p.L, p.W, p.q_pos, p.out,
                                    lse=p.lse, ws=p.attn_ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            launch()
    torch.cuda.synchronize()
    # the launches are replayed from a CUDA graph so host-side call overhead does not leave
    # the device idle between them (device time per launch)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(args.steps):
            launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    del graph
    hbm, src = peaks()
    nbytes = indexer_bytes_per_launch(cfg, B) if args.kernel == "indexer" else None
    line = {"kernel": args.kernel, "workload": f"{cfg.name} with B={B}", "ms_per_launch": ms,
            "launches": args.steps}
    if nbytes:
        line.update({"bytes_per_launch": nbytes, "achieved_gbs": nbytes / ms / 1e6,
                     "peak_gbs": hbm, "frac": nbytes / ms / 1e6 / hbm, "peak_source": src})
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default=None,
                    choices=["indexer", "topk", "attn", "step", "indexer_prefill", "compress_csa",
                             "compress_hca", "hca_prefill"],
                    help="time one kernel alone (profiling aid) instead of the whole step")
    ap.add_argument("--batch", type=int, default=16, help="sequences for --kernel")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="hcl", choices=["hcl", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--cpu-frac", type=float, default=1.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the cache-append and prefill measurements added to the line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.kernel:
        run_kernel_micro(args, local_rank)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_hcl(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
