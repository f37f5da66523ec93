"""One kernel of the denoising step, on one synthetic layer, for profiling.

    python bench_cases.py --case attn_sparse --reps 3
    python bench_cases.py --case block_select --reps 3
    python bench_cases.py --case sinks --reps 3
    python bench_cases.py --case chunk_step --reps 20

Builds one sparse layer of the 32K workload (batch 4, 32 KV heads, 32K context:
about 2.1 GB of K/V pages on the device), runs the steps before the profiled
call once, then calls it `reps` times (the first is a warm-up) and prints its
mean time from CUDA events.  Meant to sit under `ncu -k ... -s 1 -c 1`.

`workload --workload NAME` times one single-layer step of a small workload
(tiny, llada8k or dream16k; as the bench's `workloads` sub-records: CUDA-graph
replays with L2 flushed before each) and prints its median time.

`chunk_step` instead times the chunked-prefix step (32 chunks of a BOS and
1024 content tokens in permuted 64-token pages, 64 decode queries, top-8
chunks, top-256 tokens per chunk): chunk scores, chunk selection, token
selection and the gathered attention, with the chunk keys built beforehand
(they belong to the cache refresh), and reports the step's algorithmic bytes
per second.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import torch  # noqa: E402

import synth  # noqa: E402
from long_context_diffusion_b200 import _abi as A  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=["attn_sparse", "attn_dense", "block_select", "pool", "sinks",
                                       "chunk_step", "workload"], required=True)
    ap.add_argument("--workload", default="dream16k", help="for --case workload")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--fp64-select", action="store_true",
                    help="dl_block_select on the fp64 kernel (DL_FLAG_SCORE_FP64)")
    args = ap.parse_args()
    dev = torch.device("cuda", 0)
    if args.case == "chunk_step":
        return chunk_step(args.reps, dev)
    if args.case == "workload":
        import bench
        rec = bench.workload_record(args.workload, dev, bench.peaks()[0], reps=args.reps)
        print(json.dumps({k: rec[k] for k in ("workload", "us_per_step", "bytes",
                                              "frac_of_measured")}))
        return None
    wl = synth.workload("llada32k_step", n_layers=3, batch=args.batch)
    layer = wl.first_sparse_layer
    pt = synth.page_permutation(wl).to(dev)
    q = synth.make_q_dec(wl, layer, dev)
    kd, vd = synth.make_kv_dec(wl, layer, dev)
    kp, vp = synth.make_layer_kv(wl, layer, q, dev, pt.cpu())
    confs, masks = zip(*(synth.confidence(wl, b) for b in range(wl.batch)))
    conf, masked = torch.stack(confs).to(dev), torch.stack(masks).to(dev)
    desc = A.make_desc(wl.batch, wl.H, wl.H_kv, wl.d, wl.L_ctx, wl.L_q, wl.B, wl.n_pages,
                       wl.n_slots, A.DL_BF16)
    ws = torch.empty(A.dl_workspace_size(desc), dtype=torch.uint8, device=dev)
    q_idx = torch.empty((wl.batch, wl.L_q), dtype=torch.int32, device=dev)
    q_cnt = torch.empty((wl.batch,), dtype=torch.int32, device=dev)
    A.dl_predict_queries(conf, masked, wl.k, wl.w, q_idx, q_cnt)
    Kbar = torch.empty((wl.batch, wl.H_kv, wl.n_blk, wl.d), dtype=torch.float32, device=dev)
    Kdig, Kexp = A.key_digit_buffers(wl.batch, wl.H_kv, wl.n_blk, wl.d, dev)
    A.dl_pool_keys(desc, kp, pt, wl.n_blk, wl.B, 0, wl.B, Kbar, Kdig=Kdig, Kexp=Kexp)
    if args.fp64_select:
        A.dl_set_kernel_flags(A.DL_FLAG_SCORE_FP64)
    sinks = torch.empty((wl.batch, wl.detect_sinks), dtype=torch.int32, device=dev)
    A.dl_find_sinks(desc, q, q_idx, q_cnt, kp, pt, kd, wl.detect_sinks, sinks, ws, Kexp=Kexp)
    max_sel = min(wl.topK, wl.n_blk) + wl.detect_sinks
    score = torch.empty((wl.batch, wl.H_kv, wl.n_blk), dtype=torch.float64, device=dev)
    blk = torch.empty((wl.batch, wl.H_kv, max_sel), dtype=torch.int32, device=dev)
    cnt = torch.empty((wl.batch, wl.H_kv), dtype=torch.int32, device=dev)
    O = torch.empty((wl.batch, wl.L_q, wl.H, wl.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.batch, wl.H, wl.L_q), dtype=torch.float32, device=dev)

    max_q = min(wl.L_q, wl.k * (2 * wl.w + 1))  # the bound DenoiseStep passes

    def block_select():
        A.dl_block_select(desc, q, q_idx, q_cnt, Kbar, wl.n_blk, wl.B, wl.topK, sinks, score,
                          blk, cnt, ws, max_q=max_q, Kdig=Kdig, Kexp=Kexp)

    calls = {
        "block_select": block_select,
        "attn_sparse": lambda: A.dl_sparse_attn(desc, q, kp, vp, pt, blk, cnt, kd, vd, O, lse,
                                                ws),
        "attn_dense": lambda: A.dl_sparse_attn(desc, q, kp, vp, pt, None, None, kd, vd, O, lse,
                                               ws),
        "pool": lambda: A.dl_pool_keys(desc, kp, pt, wl.n_blk, wl.B, 0, wl.B, Kbar, Kdig=Kdig,
                                       Kexp=Kexp),
        "sinks": lambda: A.dl_find_sinks(desc, q, q_idx, q_cnt, kp, pt, kd, wl.detect_sinks,
                                         sinks, ws, Kexp=Kexp),
    }
    if args.case.startswith("attn"):
        block_select()
    fn = calls[args.case]
    torch.cuda.synchronize()
    A.dl_read_counters()
    times = []
    for _ in range(args.reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    st = A.dl_get_status()
    if st != A.DL_OK:
        raise RuntimeError(f"device status {st}")
    fast, fallback = A.dl_read_counters()
    print(json.dumps({"case": args.case, "batch": wl.batch, "us_per_call": times,
                      "mean_us_after_first": sum(times[1:]) / max(1, len(times) - 1),
                      "int8_select_fast": fast, "int8_select_fallback": fallback}))


def chunk_step(reps: int, dev):
    from long_context_diffusion_b200 import pipeline
    wl = synth.workload("chunked32k")
    inp = synth.make_step_inputs(wl, device=dev)
    desc = A.make_desc(wl.batch, wl.H, wl.H_kv, wl.d, wl.L_ctx, wl.L_q, wl.B, wl.n_pages,
                       wl.n_slots, A.DL_BF16)
    ws = torch.empty(A.dl_workspace_size(desc), dtype=torch.uint8, device=dev)
    Kbar = torch.empty((wl.batch, wl.H_kv, wl.n_chunks, wl.d), dtype=torch.float32, device=dev)
    Kdig, Kexp = A.key_digit_buffers(wl.batch, wl.H_kv, wl.n_chunks, wl.d, dev)
    A.dl_pool_keys(desc, inp.k_pool, inp.page_table, wl.n_chunks, wl.chunk_stride, 1,
                   wl.chunk_content, Kbar, Kdig=Kdig, Kexp=Kexp)

    def fn():
        return pipeline.chunked_step(desc, inp.q_dec, inp.k_pool, inp.v_pool, inp.page_table,
                                     inp.k_dec, inp.v_dec, n_chunks=wl.n_chunks,
                                     stride=wl.chunk_stride, content=wl.chunk_content,
                                     topK_chunks=wl.topK_chunks, topT=wl.topT_tokens,
                                     Kbar=Kbar, Kexp=Kexp, ws=ws)
    out = fn()
    torch.cuda.synchronize()
    # algorithmic bytes per step: pooled chunk keys, Q, the content K rows of
    # the selected chunks (token scores), K and V of the gathered tokens and of
    # the decode block, O and LSE written
    esz = 2
    kc = int(out.chunk_cnt.sum().item())
    n_tok = int(out.tok_cnt.sum().item())
    nbytes = (Kbar.numel() * 4 + inp.q_dec.numel() * esz + kc * wl.chunk_content * wl.d * esz +
              n_tok * wl.d * esz * 2 + inp.k_dec.numel() * esz * 2 + out.O.numel() * esz +
              out.lse.numel() * 4)
    # one graph replay per timed step, so that host launch overhead is not timed
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # larger than L2
    times = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    st = A.dl_get_status()
    if st != A.DL_OK:
        raise RuntimeError(f"device status {st}")
    mean = sum(times[1:]) / max(1, len(times) - 1)
    print(json.dumps({"case": "chunk_step", "workload": "chunked32k", "us_per_call": times,
                      "mean_us_after_first": mean, "bytes_per_step": nbytes,
                      "achieved_GBps": nbytes / (mean * 1e-6) / 1e9}))


if __name__ == "__main__":
    main()
