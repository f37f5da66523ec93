#!/usr/bin/env python
"""Benchmark of one denoising step of sink-aware, query-predicted,
block-sparse bidirectional attention on the 32-layer, 32K-context workload.

Workload (per GPU): LLaDA-8B attention shape, 32 layers x 32 heads, head dim
128, 32768 cached context tokens, decode block of 32, batch 4.  Layers 0-1
attend densely; layer 2 finds the 4 sinks (attention mass) that layers 2-31
reuse; sparse layers keep the top-128 of 512 blocks plus the sink blocks.
Synthetic bf16 inputs drawn by the seeded generator (`synth`), resident in
HBM (68.7 GB of KV cache) before the timed region.

A step = the cache refresh of one layer (a finished 32-token decode block
joins the cached context of one layer: written into the pools with its
block's pooled key recomputed, dl_cache_write; the 32 layers of a 32-step
block amortised one layer per step) + query prediction + 32 layers
(pooled-key scores, sinks at layer 2, selection, attention).  K steps are
captured in one CUDA graph and timed with CUDA events on the launch stream;
each attention call and each cache write is bracketed by graph event nodes to
time them over the same region.

The same line carries sub-records for the other workloads (single-layer
steps at 8K and 16K, the chunked 32K prefix, the tiny fp32 layer), each timed
as a CUDA-graph replay with the L2 flushed before it, and the whole-layer
pooled-key rebuild that a cache whose context K/V are recomputed needs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the fp64 CPU oracle (the reference arm) on a bounded
sample of the same workload.  Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "sparse-attn denoise steps/s and KV-tokens/s at 32K; % of HBM/tensor roofline"
WORKLOAD = "llada32k_step"
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic of the dominant kernel from one ncu capture at the benchmark's
# size (dram__bytes_read.sum + dram__bytes_write.sum of one sparse-layer
# launch, batch 4: 557.87 + 4.88 MB).  Reported only while the kernel's
# sources hash to the captured build.
TRAFFIC_CAPTURE = {"sha": "a1aa471f8011b5dd", "bytes_per_launch": 557.874688e6 + 4.879104e6,
                   "sources": ["attn_tc_kt.cu", "tc_common.cuh", "sm100.cuh"]}


def captured_traffic():
    import hashlib
    h = hashlib.sha256()
    for f in TRAFFIC_CAPTURE["sources"]:
        with open(os.path.join(ROOT, "long_context_diffusion_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return TRAFFIC_CAPTURE["bytes_per_launch"] if h.hexdigest()[:16] == TRAFFIC_CAPTURE["sha"]         else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock, power and throttle reasons of one GPU via NVML every
    20 ms while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index: int):
        self.samples, self._stop, self.ok = [], threading.Event(), False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:
                pr = torch.cuda.get_device_properties(index)
                bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - NVML missing
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                rs = self._reasons(self.h)
                self.samples.append((sm, pw, rs))
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sms = [s[0] for s in self.samples]
        reasons = sorted({n for _, _, r in self.samples for n, bit in self.REASONS.items()
                          if r & bit})
        return {"sm_mhz": float(statistics.median(sms)), "sm_max_mhz": int(self.max_mhz),
                "reasons": reasons, "samples": len(sms),
                "power_w_max": float(max(s[1] for s in self.samples))}


# ---------------------------------------------------------------- inputs
def make_inputs(wl, device, kv_heads=None):
    """All layers' tensors of the workload, drawn on the device; with
    kv_heads = (g0, g1) only those KV heads (and their query heads) are kept,
    as one rank of a head-sharded run holds them."""
    pt = synth.page_permutation(wl).to(device)
    layers = []
    for l in range(wl.n_layers):
        q = synth.make_q_dec(wl, l, device)
        kd, vd = synth.make_kv_dec(wl, l, device)
        kp, vp = synth.make_layer_kv(wl, l, q, device, pt.cpu())
        x = dict(q=q, kd=kd, vd=vd, kp=kp, vp=vp)
        if kv_heads is not None:
            g0, g1 = kv_heads
            x = dict(q=q[:, g0 * wl.G:g1 * wl.G].contiguous(), kd=kd[:, g0:g1].contiguous(),
                     vd=vd[:, g0:g1].contiguous(), kp=kp[:, g0:g1].contiguous(),
                     vp=vp[:, g0:g1].contiguous())
            del q, kd, vd, kp, vp
        layers.append(x)
    confs, masks = zip(*(synth.confidence(wl, b) for b in range(wl.batch)))
    conf = torch.stack(confs).to(device)
    masked = torch.stack(masks).to(device)
    return layers, pt, conf, masked


def attn_bytes(wl, n_ctx_tokens_per_bg):
    """Algorithmic HBM bytes of one attention call: every attended context
    K and V row once, the decode K/V, Q, O and the LSE."""
    e = 2  # bf16
    kv_ctx = sum(n_ctx_tokens_per_bg) * wl.d * e * 2
    dec = wl.batch * wl.H_kv * wl.L_q * wl.d * e * 2
    q = wl.batch * wl.H * wl.L_q * wl.d * e
    o = wl.batch * wl.L_q * wl.H * wl.d * e + wl.batch * wl.H * wl.L_q * 4
    return kv_ctx + dec + q + o


def attn_flops(wl, n_ctx_tokens_per_bg):
    keys = sum(n + wl.L_q for n in n_ctx_tokens_per_bg)
    return 4.0 * wl.d * keys * wl.G * wl.L_q


def cache_write_bytes(wl, start, n_new):
    """Algorithmic HBM bytes of one dl_cache_write over all (b, g): the new K
    and V rows read and written, the touched blocks' other rows read back,
    and their pooled keys written."""
    e = 2
    j0, j1 = start // wl.B, (start + n_new - 1) // wl.B
    rows = sum(min(wl.B, wl.L_ctx - j * wl.B) for j in range(j0, j1 + 1))
    key_b = wl.d * 4 + wl.d * 5 + 4  # pooled key, its five digit planes, its exponent word
    per_bg = n_new * wl.d * e * 4 + (rows - n_new) * wl.d * e + (j1 - j0 + 1) * key_b
    return wl.batch * wl.H_kv * per_bg


def _graph_time_us(fn, device, reps, flush_l2=True):
    """Median device time of one CUDA-graph replay of fn (captured on a side
    stream), the L2 flushed (a 256 MiB write) before each replay."""
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        out = fn(side)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        out = fn(side)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    times = []
    for r in range(reps + 3):
        with torch.cuda.stream(side):
            if flush_l2:
                flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(side)
            g.replay()
            e1.record(side)
        torch.cuda.synchronize(device)
        if r >= 3:
            times.append(e0.elapsed_time(e1) * 1e3)
    del g
    return float(statistics.median(times)), out


def workload_record(name, device, pk, reps=30):
    """One step of a single-layer or chunked workload: median graph-replay
    time, algorithmic bytes, and the fraction of the measured and nominal
    HBM rooflines."""
    import long_context_diffusion_b200 as dl
    from long_context_diffusion_b200 import pipeline
    wl = synth.workload(name)
    inp = synth.make_step_inputs(wl, device=device)
    e = 4 if wl.dtype == "fp32" else 2
    desc = dl.make_desc(wl.batch, wl.H, wl.H_kv, wl.d, wl.L_ctx, wl.L_q, wl.B, wl.n_pages,
                        wl.n_slots, dl.DL_FP32 if wl.dtype == "fp32" else dl.DL_BF16)
    ws = pipeline.workspace(desc, device)
    n_units = wl.n_chunks if wl.chunked else wl.n_blk
    Kbar = torch.empty((wl.batch, wl.H_kv, n_units, wl.d), dtype=torch.float32, device=device)
    Kdig = Kexp = None
    if wl.chunked:  # chunk keys belong to the cache build, not to the step
        Kdig, Kexp = dl.key_digit_buffers(wl.batch, wl.H_kv, wl.n_chunks, wl.d, device)
        dl.dl_pool_keys(desc, inp.k_pool, inp.page_table, wl.n_chunks, wl.chunk_stride, 1,
                        wl.chunk_content, Kbar, Kdig=Kdig, Kexp=Kexp)

        def fn(st):
            return pipeline.chunked_step(desc, inp.q_dec, inp.k_pool, inp.v_pool, inp.page_table,
                                         inp.k_dec, inp.v_dec, n_chunks=wl.n_chunks,
                                         stride=wl.chunk_stride, content=wl.chunk_content,
                                         topK_chunks=wl.topK_chunks, topT=wl.topT_tokens,
                                         Kbar=Kbar, Kexp=Kexp, ws=ws, stream=st)
    else:
        Kdig, Kexp = dl.key_digit_buffers(wl.batch, wl.H_kv, wl.n_blk, wl.d, device)
        dl.dl_pool_keys(desc, inp.k_pool, inp.page_table, wl.n_blk, wl.B, 0, wl.B, Kbar,
                        Kdig=Kdig, Kexp=Kexp)
        sinks = inp.sinks_planted[:, :wl.sinks_given].contiguous() if wl.sinks_given else None

        def fn(st):
            return pipeline.layer_step(desc, inp.q_dec, inp.k_pool, inp.v_pool, inp.page_table,
                                       inp.k_dec, inp.v_dec, topK=wl.topK,
                                       conf_prev=inp.conf_prev, still_masked=inp.still_masked,
                                       k=wl.k, w=wl.w, sink_pos=sinks, Kbar=Kbar, Kdig=Kdig,
                                       Kexp=Kexp, ws=ws, stream=st)
    us, out = _graph_time_us(fn, device, reps)
    if dl.dl_get_status() != dl.DL_OK:
        raise RuntimeError(f"device status after the {name} step")
    q_b = inp.q_dec.numel() * e
    dec_b = inp.k_dec.numel() * e * 2
    o_b = out.O.numel() * e + out.lse.numel() * 4
    if wl.chunked:
        kc = int(out.chunk_cnt.sum().item())
        n_tok = int(out.tok_cnt.sum().item())
        ctx_tokens = n_tok / (wl.batch * wl.H_kv)
        nbytes = (Kbar.numel() * 4 + q_b + kc * wl.chunk_content * wl.d * e +
                  n_tok * wl.d * e * 2 + dec_b + o_b)
    else:
        cnt = out.blk_cnt.view(-1).cpu().tolist()
        idx = out.blk_idx.view(len(cnt), -1).cpu()
        toks = 0
        for r, c in enumerate(cnt):
            last = int((idx[r, :c] == wl.n_blk - 1).sum().item())
            toks += int(c) * wl.B - last * (wl.n_blk * wl.B - wl.L_ctx)
        ctx_tokens = toks / (wl.batch * wl.H_kv)
        # the int8 tensor-core selection reads the digit planes; the fp64 one Kbar
        fast = wl.dtype == "bf16" and wl.d == 128 and wl.G * min(wl.L_q, wl.k * (2 * wl.w + 1)) \
            <= 24 and wl.n_blk <= 512
        key_b = Kdig.numel() + Kexp.numel() * 4 if fast else Kbar.numel() * 4
        nbytes = (key_b + q_b + wl.batch * wl.H_kv * wl.n_blk * 8 +
                  toks * wl.d * e * 2 + dec_b + o_b)
    t = us * 1e-6
    return {"workload": name, "us_per_step": us, "steps_per_s": 1.0 / t,
            "kv_tokens_per_s": wl.batch * (ctx_tokens + wl.L_q) / t,
            "bytes": int(nbytes), "achieved_GBps": nbytes / t / 1e9,
            "frac_of_measured": nbytes / t / 1e9 / pk["hbm_gbs"],
            "frac_of_nominal_8tbs": nbytes / t / 1e9 / NOMINAL_HBM_GBS,
            "timing": f"median of {reps} CUDA-graph replays, L2 flushed before each"}


# ---------------------------------------------------------------- oracle arm
def oracle_sample(wl, seconds_budget=8.0):
    """Times the fp64 oracle on a bounded sample of the step and scales it to
    one full step.  Sample: one sequence, a few KV heads, one dense layer, one
    sparse layer (sinks given) and the sink search over those heads."""
    import oracle
    from oracle import steps as S
    heads = 2
    b, layer_d, layer_s = 0, 0, wl.first_sparse_layer
    q = synth.make_q_dec(wl.replace(batch=1), layer_s)
    qd = synth.make_q_dec(wl.replace(batch=1), layer_d)
    scale = S.scale_for(wl.d)

    def kv(layer, qq):
        k, v = synth.make_logical_kv(wl.replace(batch=1), layer, b, 0, heads, qq)
        return k, v

    kd_full, vd_full = synth.make_kv_dec(wl.replace(batch=1), layer_s)
    conf, masked = synth.confidence(wl, b)
    q_idx = S.predict_queries(conf, masked, wl.k, wl.w)
    t_dense = t_sparse = t_sink = 0.0
    n_rep = 0
    t_all = time.perf_counter()
    while True:
        k_d, v_d = kv(layer_d, qd)
        t0 = time.perf_counter()
        pool_k = k_d.view(heads, wl.n_blk, wl.B, wl.d).permute(1, 0, 2, 3).contiguous()
        pool_v = v_d.view(heads, wl.n_blk, wl.B, wl.d).permute(1, 0, 2, 3).contiguous()
        pt = np.arange(wl.n_blk)
        S.dense_attention(qd[0, :heads], pool_k, pool_v, pt, wl.L_ctx, wl.B,
                          kd_full[0, :heads], vd_full[0, :heads], scale)
        t_dense += time.perf_counter() - t0
        k_s, v_s = kv(layer_s, q)
        t0 = time.perf_counter()
        pool_k = k_s.view(heads, wl.n_blk, wl.B, wl.d).permute(1, 0, 2, 3).contiguous()
        pool_v = v_s.view(heads, wl.n_blk, wl.B, wl.d).permute(1, 0, 2, 3).contiguous()
        sinks = synth.sink_positions(wl, b)
        r = oracle.layer_step(q[:, :heads], pool_k, pool_v, pt[None], kd_full[:, :heads],
                              vd_full[:, :heads], wl.L_ctx, wl.B, wl.topK,
                              q_idx=oracle.step._pad([q_idx], wl.L_q),
                              q_cnt=np.array([len(q_idx)]), sink_pos=np.array([sinks]))
        t_sparse += time.perf_counter() - t0
        t0 = time.perf_counter()
        S.find_sinks(q[0, :heads], S.f64(k_s), S.f64(kd_full[0, :heads]), q_idx, wl.detect_sinks,
                     scale)
        t_sink += time.perf_counter() - t0
        n_rep += 1
        if time.perf_counter() - t_all > seconds_budget or n_rep >= 3:
            break
    t_dense, t_sparse, t_sink = t_dense / n_rep, t_sparse / n_rep, t_sink / n_rep
    per_seq_heads = wl.H_kv / heads * wl.batch
    n_dense = wl.first_sparse_layer
    n_sparse = wl.n_layers - wl.first_sparse_layer
    t_step = per_seq_heads * (n_dense * t_dense + n_sparse * t_sparse + t_sink)
    del r
    cores = torch.get_num_threads()
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        cores = max([i.get("num_threads", 1) for i in info] + [cores])
    except Exception:
        pass
    sample = (f"sequence 0, KV heads 0-{heads - 1} of {wl.H_kv}: one dense layer, one sparse "
              f"layer (pool, score, select, attend) and the sink search, x{n_rep}; scaled by "
              f"{per_seq_heads:.0f} (heads x batch) and by layer counts "
              f"({n_dense} dense, {n_sparse} sparse, 1 sink search)")
    return 1.0 / t_step, cores, sample, t_step


def run_reference(args):
    # The oracle arm never touches the GPU library: the package (which loads
    # libdlsparse.so on import) is not imported here.
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    wl = synth.workload(WORKLOAD)
    times = []
    for i in range(args.warmup + args.steps):
        v, cores, sample, t_step = oracle_sample(wl, seconds_budget=1.0)
        if i >= args.warmup:
            times.append(t_step)
    t = float(np.mean(times))
    value = 1.0 / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl),
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_of(wl, parallelism="replicas"):
    return {"workload": WORKLOAD, "layers": wl.n_layers, "batch_per_gpu": wl.batch,
            "parallelism": parallelism,
            "heads": wl.H, "kv_heads": wl.H_kv, "head_dim": wl.d, "context": wl.L_ctx,
            "decode_block": wl.L_q, "block": wl.B, "topK": wl.topK, "sinks": wl.detect_sinks,
            "dense_layers": wl.first_sparse_layer, "predict_k": wl.k, "window": wl.w,
            "l2": "inputs larger than L2 (68.7 GB resident KV per GPU, 23 GB read per step)"}


# ---------------------------------------------------------------- our arm
def run_ours(args):
    from long_context_diffusion_b200 import runtime
    rank, world, local, device = runtime.init()
    import long_context_diffusion_b200 as dl
    from long_context_diffusion_b200 import pipeline

    wl_full = synth.workload(WORKLOAD, n_layers=args.layers, batch=args.batch)
    torch.manual_seed(0)
    desc = dl.make_desc(wl_full.batch, wl_full.H, wl_full.H_kv, wl_full.d, wl_full.L_ctx,
                        wl_full.L_q, wl_full.B, wl_full.n_pages, wl_full.n_slots, dl.DL_BF16)
    heads = args.shard == "heads" or args.shard_sim > 1
    kv_heads, sink_group, wl = None, None, wl_full
    if heads:
        # this rank holds only its KV heads; the sink mass is all-reduced
        from long_context_diffusion_b200 import sharded
        # --shard-sim W: rank 0's share of a head split over W GPUs, run alone
        hs = (sharded.HeadShard.of(desc, 0, args.shard_sim) if args.shard_sim > 1
              else sharded.HeadShard.of(desc, rank, world))
        desc, kv_heads = hs.desc, (hs.g0, hs.g1)
        wl = wl_full.replace(H=hs.desc.H, H_kv=hs.desc.H_kv)
        if world > 1 and args.shard_sim <= 1:
            import torch.distributed as dist
            sink_group = dist.group.WORLD
    t_gen = time.time()
    layers, pt, conf, masked = make_inputs(wl_full, device, kv_heads)
    t_gen = time.time() - t_gen
    L = wl.n_layers
    step = pipeline.DenoiseStep(desc, L, wl.first_sparse_layer, wl.topK, wl.detect_sinks, wl.k,
                                wl.w, torch.bfloat16, device, sink_group=sink_group)
    Kbar = [step.key_cache() for _ in range(L)]  # (pooled keys, digits, exponents) per layer
    stream = torch.cuda.Stream(device)
    args_of = lambda: (conf, masked, [x["q"] for x in layers], [x["kp"] for x in layers],  # noqa
                       [x["vp"] for x in layers], pt, [x["kd"] for x in layers],
                       [x["vd"] for x in layers], Kbar)

    # the finished decode block joins the context as its last L_q positions
    start = torch.full((wl.batch,), wl.L_ctx - wl.L_q, dtype=torch.int32, device=device)
    cw_events = []

    def commit(i, kd, vd, events=None):
        ev = step._begin(events, stream)
        step.commit_block(kd, vd, start, layers[i % L]["kp"], layers[i % L]["vp"], pt,
                          Kbar[i % L], stream)
        step._end(events, ev, i % L, stream)

    def one_step(i, events=None, cw=None):
        commit(i, layers[i % L]["kd"], layers[i % L]["vd"], cw)
        step.run(*args_of(), stream=stream, attn_events=events)

    with torch.cuda.stream(stream):
        for l in range(L):  # the cache refresh that precedes a block of steps
            step.refresh_pooled_keys(l, layers[l]["kp"], pt, Kbar[l], stream)
        one_step(0)
    torch.cuda.synchronize(device)
    st = dl.dl_get_status(stream)
    if st != dl.DL_OK:
        raise RuntimeError(f"device status {st} after the first step")

    K, W = args.steps, args.warmup
    g_warm = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, stream=stream):
        one_step(0)
    events = []
    g_timed = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_timed, stream=stream):
        for i in range(K):
            one_step(i, events, cw_events)
    for _ in range(W):
        g_warm.replay()
    torch.cuda.synchronize(device)

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    runtime.barrier(device)
    torch.cuda.synchronize(device)
    dl.dl_read_counters()  # cleared: the counts below are the timed steps'
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            g_timed.replay()
            ev1.record(stream)
        torch.cuda.synchronize(device)
    runtime.barrier(device)
    sel_fast, sel_fallback = dl.dl_read_counters()
    ms_total = ev0.elapsed_time(ev1)
    ms_total = runtime.max_over_ranks(ms_total, device)
    ms_step = ms_total / K
    st = dl.dl_get_status(stream)
    if st != dl.DL_OK:
        raise RuntimeError(f"device status {st} after the timed steps")

    # selected context tokens per (b, g) of each layer, from the returned counts
    n_blk = wl.n_blk
    ctx_tokens = []
    for l in range(L):
        if l < wl.first_sparse_layer:
            ctx_tokens.append([wl.L_ctx] * (wl.batch * wl.H_kv))
        else:
            cnt = step.blk_cnt[l].view(-1).cpu().tolist()
            idx = step.blk_idx[l].view(wl.batch * wl.H_kv, -1).cpu()
            toks = []
            for r, c in enumerate(cnt):
                blocks = idx[r, :c]
                last = (blocks == n_blk - 1).sum().item()
                toks.append(int(c) * wl.B - last * (n_blk * wl.B - wl.L_ctx))
            ctx_tokens.append(toks)
    attn_b = [attn_bytes(wl, t) for t in ctx_tokens]
    attn_f = [attn_flops(wl, t) for t in ctx_tokens]
    # KV tokens attended per step, averaged over the KV heads (of the whole
    # model when the heads are sharded)
    tok_sum = runtime.sum_over_ranks(float(sum(sum(t) for t in ctx_tokens)), device) \
        if heads else float(sum(sum(t) for t in ctx_tokens))
    kv_tokens = tok_sum / wl_full.H_kv + L * wl.batch * wl.L_q

    # dominant kernel: the sparse-layer attention calls, over the timed region
    sparse_ms, dense_ms = [], []
    for layer, s, e in events:
        (sparse_ms if layer >= wl.first_sparse_layer else dense_ms).append(
            (layer, s.elapsed_time(e)))
    sp_bytes = sum(attn_b[l] for l, _ in sparse_ms)
    sp_time = sum(t for _, t in sparse_ms) / 1e3
    sp_flops = sum(attn_f[l] for l, _ in sparse_ms)
    dn_bytes = sum(attn_b[l] for l, _ in dense_ms)
    dn_time = sum(t for _, t in dense_ms) / 1e3
    pk, pk_kind = peaks()
    achieved = sp_bytes / sp_time / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / pk["hbm_gbs"], "traffic": captured_traffic(),
            "kernel": "dl_sparse_attn (sparse layers)", "launches": len(sparse_ms),
            "bytes_per_launch": sp_bytes / max(1, len(sparse_ms)),
            "avg_launch_us": sp_time / max(1, len(sparse_ms)) * 1e6,
            "tflops": sp_flops / sp_time / 1e12, "peak_kind": f"{pk_kind} (copy)",
            "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS}

    # step-level roofline: algorithmic bytes of every kernel of one step
    e2b = 2
    cw_b = cache_write_bytes(wl, wl.L_ctx - wl.L_q, wl.L_q)
    # the selection reads the pooled keys as five int8 digit planes + one exponent word
    kbar_b = wl.batch * wl.H_kv * n_blk * (wl.d * 5 + 4)
    q_b = wl.batch * wl.H * wl.L_q * wl.d * e2b
    # sink search: K counted once (the kernels stream it twice: the row LSEs
    # must be known before any column mass can be summed)
    sink_b = wl.batch * wl.H_kv * (wl.L_ctx + wl.L_q) * wl.d * e2b + q_b
    n_sparse = L - wl.first_sparse_layer
    score_b = n_sparse * (kbar_b + q_b + wl.batch * wl.H_kv * n_blk * 8)
    step_bytes = cw_b + sink_b + score_b + sum(attn_b)
    step_flops = sum(attn_f)
    t_roof_meas = max(step_bytes / (pk["hbm_gbs"] * 1e9), step_flops / (pk["bf16_tflops"] * 1e12))
    t_roof_nom = max(step_bytes / (NOMINAL_HBM_GBS * 1e9),
                     step_flops / (NOMINAL_BF16_TFLOPS * 1e12))
    t_step = ms_step / 1e3

    # end to end: every step's inputs copied in from pinned host memory and
    # its results copied back, inside the timed graph.  Copies run on their own
    # streams, double-buffered: the inputs of step i+1 go up and the results
    # of step i-1 come down while step i computes.
    def job_rate(seconds_per_step):
        # replicas: every rank steps its own batch; heads: the ranks share one step
        return (1.0 if heads else float(world)) / seconds_per_step if seconds_per_step else 0.0

    e2e = None
    if not args.no_e2e:
        keys = ("q", "kd", "vd")
        dev_in = [{"conf": conf, "masked": masked,
                   **{(l, k): layers[l][k] for l in range(L) for k in keys}}]
        dev_in.append({n: t.clone() for n, t in dev_in[0].items()})
        h_in = {n: t.cpu().pin_memory() for n, t in dev_in[0].items()}
        outs = [(l, "O") for l in range(L)] + [(l, "lse") for l in range(L)] + \
               [(l, "blk") for l in range(L)]

        def out_of(key):
            l, k = key
            return {"O": step.O, "lse": step.lse, "blk": step.blk_idx}[k][l]

        staging = [{key: torch.empty_like(out_of(key)) for key in outs} for _ in range(2)]
        h_out = [{key: torch.empty_like(out_of(key), device="cpu").pin_memory() for key in outs}
                 for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in h_in.values())
        d2h = sum(t.numel() * t.element_size() for t in h_out[0].values())
        cs_in, cs_out = torch.cuda.Stream(device), torch.cuda.Stream(device)

        def args_set(j):
            d = dev_in[j]
            return (d["conf"], d["masked"], [d[(l, "q")] for l in range(L)],
                    [x["kp"] for x in layers], [x["vp"] for x in layers], pt,
                    [d[(l, "kd")] for l in range(L)], [d[(l, "vd")] for l in range(L)], Kbar)

        def e2e_steps():
            fork = torch.cuda.Event()
            fork.record(stream)
            cs_in.wait_event(fork)
            cs_out.wait_event(fork)
            in_ready, in_free, out_done = [None, None], [None, None], [None, None]

            def upload(i):
                j = i % 2
                with torch.cuda.stream(cs_in):
                    if in_free[j] is not None:
                        cs_in.wait_event(in_free[j])
                    for n, t in h_in.items():
                        dev_in[j][n].copy_(t, non_blocking=True)
                    in_ready[j] = torch.cuda.Event()
                    in_ready[j].record(cs_in)

            upload(0)
            for i in range(K):
                j = i % 2
                if i + 1 < K:
                    upload(i + 1)
                stream.wait_event(in_ready[j])
                commit(i, dev_in[j][(i % L, "kd")], dev_in[j][(i % L, "vd")])
                step.run(*args_set(j), stream=stream)
                in_free[j] = torch.cuda.Event()
                in_free[j].record(stream)
                if out_done[j] is not None:
                    stream.wait_event(out_done[j])
                for key in outs:
                    staging[j][key].copy_(out_of(key), non_blocking=True)
                staged = torch.cuda.Event()
                staged.record(stream)
                with torch.cuda.stream(cs_out):
                    cs_out.wait_event(staged)
                    for key in outs:
                        h_out[j][key].copy_(staging[j][key], non_blocking=True)
                    out_done[j] = torch.cuda.Event()
                    out_done[j].record(cs_out)
            join = torch.cuda.Event()
            join.record(cs_in)
            stream.wait_event(join)
            join2 = torch.cuda.Event()
            join2.record(cs_out)
            stream.wait_event(join2)

        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e, stream=stream):
            e2e_steps()
        g_e2e.replay()
        torch.cuda.synchronize(device)
        runtime.barrier(device)
        torch.cuda.synchronize(device)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            g_e2e.replay()
            ev1.record(stream)
        torch.cuda.synchronize(device)
        runtime.barrier(device)
        e2e_ms = runtime.max_over_ranks(ev0.elapsed_time(ev1), device) / K
        e2e = {"value": job_rate(e2e_ms / 1e3), "unit": "steps/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms,
               "overlap": "inputs of step i+1 and results of step i-1 copied while step i "
                          "computes (double-buffered, own copy streams)"}
        del g_e2e

    launches_per_step = count_launches(wl)
    value = job_rate(t_step)
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if heads else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(wl_full, (f"heads{args.shard_sim}, rank 0 alone: no all-reduce"
                                      if args.shard_sim > 1 else f"heads{world}")
                            if heads else "replicas"),
        "kv_tokens_per_s": kv_tokens * (1 if heads else world) / t_step,
        "kv_tokens_per_step": kv_tokens,
        "roofline": roof,
        "step_roofline": {"bytes": step_bytes, "flops": step_flops,
                          "frac_of_measured": t_roof_meas / t_step,
                          "frac_of_nominal": t_roof_nom / t_step,
                          "t_roof_measured_ms": t_roof_meas * 1e3,
                          "t_roof_nominal_ms": t_roof_nom * 1e3,
                          "dense_attn_GBps": dn_bytes / dn_time / 1e9 if dn_time else None},
        "clocks": clk.summary(),
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
        "block_select_int8": {"certified": sel_fast, "fp64_fallback": sel_fallback,
                              "per_step": (sel_fast + sel_fallback) / K},
        "gen_seconds": t_gen,
    }
    # cache refresh on the timed path: one decode block joining one layer
    cw_us = [s_.elapsed_time(e_) * 1e3 for _, s_, e_ in cw_events]
    cw_b = cache_write_bytes(wl, wl.L_ctx - wl.L_q, wl.L_q)
    cw_mean = sum(cw_us) / max(1, len(cw_us))
    line["cache_write"] = {
        "call": "dl_cache_write", "n_new": wl.L_q, "start": wl.L_ctx - wl.L_q,
        "avg_us": cw_mean, "launches": len(cw_us), "bytes_per_call": cw_b,
        "achieved_GBps": cw_b / (cw_mean * 1e-6) / 1e9 if cw_mean > 0 else None}
    # whole-layer pooled-key rebuild (a cache whose context K/V are recomputed)
    with torch.cuda.stream(stream):
        ts = []
        for r in range(6):
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            step.refresh_pooled_keys(r % L, layers[r % L]["kp"], pt, Kbar[r % L], stream)
            b_.record(stream)
            ts.append((a_, b_))
    torch.cuda.synchronize(device)
    pool_us = [a_.elapsed_time(b_) * 1e3 for a_, b_ in ts[1:]]
    pool_b = wl.batch * wl.H_kv * (wl.L_ctx * wl.d * 2 + wl.n_blk * (wl.d * 9 + 4))
    pm = sum(pool_us) / len(pool_us)
    line["full_layer_pool"] = {"call": "dl_pool_keys", "avg_us": pm, "bytes": pool_b,
                               "achieved_GBps": pool_b / (pm * 1e-6) / 1e9,
                               "step_ms_if_amortised_per_step": ms_step + (pm - cw_mean) / 1e3}
    # sinks kept across the steps of one decode block: a block of L_q steps
    # (one position unmasked per step), the first step finds the sinks and
    # the others keep them; each step commits one layer's block as above
    n_blk_steps = wl.L_q
    g_blk = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_blk, stream=stream):
        for i in range(n_blk_steps):
            commit(i, layers[i % L]["kd"], layers[i % L]["vd"])
            step.run(*args_of(), stream=stream, find_sinks=(i == 0))
    g_blk.replay()
    torch.cuda.synchronize(device)
    runtime.barrier(device)
    blk_ms = []
    for _ in range(2):
        with torch.cuda.stream(stream):
            ev0.record(stream)
            g_blk.replay()
            ev1.record(stream)
        torch.cuda.synchronize(device)
        blk_ms.append(ev0.elapsed_time(ev1))
    runtime.barrier(device)
    blk_ms = runtime.max_over_ranks(min(blk_ms), device)
    del g_blk
    line["decode_block"] = {
        "steps": n_blk_steps, "sinks": "found at the block's first step, kept by the others",
        "ms_per_step": blk_ms / n_blk_steps, "steps_per_s": job_rate(blk_ms / n_blk_steps / 1e3),
        "ms_per_step_keeping_sinks": (blk_ms - ms_step) / max(1, n_blk_steps - 1)}
    if not args.no_configs:
        line["workloads"] = {n: workload_record(n, device, pk)
                             for n in ("tiny", "llada8k", "dream16k", "chunked32k")}
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        v, cores, sample, _ = oracle_sample(synth.workload(WORKLOAD))
        line["cpu_baseline"] = {"value": v, "unit": "steps/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    del g_timed, g_warm
    if rank == 0:
        print(json.dumps(line))
    runtime.finalize()
    return 0


def count_launches(wl):
    """Kernels of this library launched per step (from the call sequence):
    the cache write, the prediction, attention and combine per layer, the
    certified sink search, and one score + select kernel per sparse layer when
    the group's rows fit a fused kernel (else three)."""
    n_sparse = wl.n_layers - wl.first_sparse_layer
    # sinks: LSE pass + combine, mass, top-n, and the certification (bound,
    # band count, band final, fp64 LSE, merge, candidate masses, pick: the
    # last four return at once when the cut is certified)
    pool, predict, attn, sinks = 1, 1, 2, 11
    rows = wl.G * min(wl.L_q, wl.k * (2 * wl.w + 1))
    fused = rows <= 32 and wl.n_blk <= 512
    score_select = 1 if fused else 3
    return pool + predict + wl.first_sparse_layer * attn + sinks + n_sparse * (
        score_select + attn)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the sub-records of the other workloads")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="replicas: each GPU steps its own batch (weak scaling); heads: the "
                         "GPUs split the KV heads of one batch and all-reduce the sink mass "
                         "(strong scaling)")
    ap.add_argument("--shard-sim", type=int, default=0,
                    help="one GPU runs rank 0's share of a head split over this many GPUs, "
                         "without the sink-mass all-reduce (the per-rank compute of a "
                         "head-sharded step)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours" and args.layers == 32:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
