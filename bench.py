"""Benchmark of the KVarN hot path on B200.

Workload (one "step"): Qwen3-4B-shaped long-horizon decode -- batch 8, 32 query / 8 kv heads,
head_dim 128, bf16, 36 layer caches at a 32K context.  A step is one full block period: 128
consecutive decode tokens, each running, for every layer, kvarn_append_token (which quantises the
filled 128-token tail on the last token: rotation, 4 normalisation sweeps, 2-bit packing) and then
kvarn_decode_attention over the whole 2-bit cache.  Each step starts from 32640 cached tokens
(255 blocks) and ends at 32768, so every (layer, sequence, kv head) quantises exactly one K and one
V block per step.  The line also reports bulk quantisation GB/s on the Llama-3-8B-shaped prefill
(batch 32 x 32 layers x 8 kv heads x 8192 tokens x 128, bf16).

Alongside (keys of the same line) it times the other model shapes on one GPU: the tiny single-head case
(256 tokens x 64, fp32), the Qwen3-4B decode step at batch 1 and context 4153 (36 layers in one graph), the
Phi-3-mini MHA decode with quantise-on-append (batch 16, 32 heads, head_dim 96, context 16384), and the
share of a block period spent quantising blocks at contexts 1024 and 32768.

With --gpus N > 1 and no launcher environment, the script starts N ranks itself (torch.distributed.run on
127.0.0.1); every rank runs the same step on a batch of its own.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvarn|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "KV quantize GB/s + fused 2-bit decode-attn tokens/s, % of HBM roofline"
UNIT = "tokens/s"
S, HQ, HKV, D, LAYERS = 8, 32, 8, 128, 36
T_BLK = 128
CTX0 = 32768 - T_BLK          # tokens cached when a step starts
QB_SEQS, QB_TOKENS = 32 * 32, 8192  # bulk quantise: batch 32 x 32 layers folded into sequences
WORKLOAD = ("Qwen3-4B-shaped long-horizon decode: batch 8, 32 q / 8 kv heads, head_dim 128, bf16, "
            "36 layer caches, context 32641..32768 (one 128-token block period per step: 128 x 36 x "
            "(append+quantise-on-fill, decode attention))")
QB_WORKLOAD = "Llama-3-8B-shaped bulk prefill quantise: 32 batch x 32 layers x 8 kv heads x 8192 tokens x 128, bf16"
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one decode launch at context 32705 for this
# batch, from one ncu capture of `bench.py --profile decode` with the current decode kernel; None whenever
# the decode kernel has changed since the last capture.
DECODE_TRAFFIC_BYTES = 220170496 + 4353280
# The same for one bulk-quantisation launch of `bench.py --profile quantize` (16 of the 1024 sequences); the
# traffic grows with the sequences, so the full workload's is 64 times this.
QUANT_TRAFFIC_BYTES_16SEQ = 537332992 + 97235968


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def record_alg_bytes(d: int) -> int:
    """Bytes of one 128-token record that decode must read: 2-bit codes, binary16 (s, m) per token and
    32-channel group, binary16 r per token and c per channel (6656 at D = 128, 5056 at D = 96)."""
    return T_BLK * d // 4 + (d // 32) * T_BLK * 2 * 2 + T_BLK * 2 + d * 2


def decode_bytes(n_tokens: int, seqs: int = S, hkv: int = HKV, hq: int = HQ, d: int = D, in_bytes: int = 2) -> int:
    """Algorithmic HBM bytes of one decode launch at context n for the whole batch.

    Per (sequence, kv head): both records (K and V) of every full block, plus 2 x D input-dtype values of
    every tail token; per query head: q (input dtype) read and out (fp32) written."""
    nb, nt = n_tokens // T_BLK, n_tokens % T_BLK
    per_kv = nb * 2 * record_alg_bytes(d) + nt * 2 * d * in_bytes
    return seqs * hkv * per_kv + seqs * hq * d * (in_bytes + 4)


# FP32-pipe operations per element that the quantiser's arithmetic needs at 4 sweeps, counted from the method:
# per sweep, the row step scales by 1/c, shifts, and adds to a sum and a sum of squares (4 operations), and the
# column step does the same with 1/r (4 more): 32 for 4 sweeps; then Y = x / (r c) (2 multiplies), the group's
# min and max (2), the level (1 FMA), its rounding (1 add) and clamp (2), and the bf16 widening (1): 9 more.
# The Hadamard rotation runs on the tensor cores and is not counted.
QUANT_FP32_OPS_PER_ELEM = 41
FP32_LANES_PER_SM = 128  # FP32 operations per clock per SM (4 sub-partitions x 32 lanes)


def quant_bytes(n_elems: int) -> int:
    """Algorithmic bytes of bulk quantisation: bf16 read + record bytes written (2.40625 B/elem)."""
    return n_elems * 2 + (n_elems // (T_BLK * D)) * 6656


def shared_lengths(caches, n: int):
    """Point every cache's sequence-length vector into one [layers, S] tensor, so that one copy resets all
    layers inside a captured step.  Returns (that tensor, a copy holding n everywhere)."""
    seqs = caches[0].n_tokens.numel()
    dev = caches[0].n_tokens.device
    n_all = torch.full((len(caches), seqs), n, dtype=torch.int32, device=dev)
    for layer, c in enumerate(caches):
        c.n_tokens = n_all[layer]
    return n_all, n_all.clone()


def graph_ms(graph, reps: int, warmup: int = 3, flush=None) -> float:
    """Median device time of one replay of a captured graph, by CUDA events on the replaying stream.
    With flush (a tensor larger than L2), it is overwritten before each replay, outside the events."""
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush.add_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def capture(fn, dev):
    """A CUDA graph of fn() captured on a side stream (fn runs once eagerly first, which checks every call)."""
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    torch.cuda.synchronize()
    return g


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def spawn_ranks(n: int, argv) -> int:
    """Run this script as n ranks under torch.distributed.run (one node, rendezvous on 127.0.0.1); the
    ranks find WORLD_SIZE / RANK / LOCAL_RANK in their environment.  Returns the launcher's exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def run_stub(args):
    """A CPU stand-in for the step, on gloo: every rank times a seeded numpy workload of its own between
    barriers; the job's time is the slowest rank's.  Prints the contract line with "stub": true."""
    import numpy as np

    from bit_kv_cache_token_b200 import dp
    world, rank, _ = dp.world_from_env()
    dp.init(world, "gloo")
    a = np.random.default_rng(dp.rank_seed(2, rank)).standard_normal((256, 256))
    for _ in range(args.warmup):
        a @ a
    dp.barrier(world)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        a = np.tanh(a @ a / 16.0)
    my_ms = (time.perf_counter() - t0) * 1e3
    dp.barrier(world)
    ms = dp.max_over_ranks(my_ms, world)
    rank_ms = dp.gather_floats(my_ms, world)
    if rank == 0:
        print(json.dumps({"metric": METRIC, "value": dp.aggregate_rate(args.steps, ms / 1e3, world),
                          "unit": "stub steps/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                          "vs_baseline": None, "dtype": "f64", "data": "synthetic", "stub": True,
                          "config": {"workload": "CPU stand-in step (256 x 256 matmul)", "parallelism": f"dp{world}"},
                          "rank_ms": rank_ms}), flush=True)
    dp.finish(world)


def _dist_setup(args):
    from bit_kv_cache_token_b200 import dp
    world, rank, local = dp.world_from_env()
    torch.cuda.set_device(local if world > 1 else 0)
    dp.init(world, "nccl", torch.device("cuda", local))
    return world, rank, local


def _barrier(world):
    from bit_kv_cache_token_b200 import dp
    dp.barrier(world)


def _max_over_ranks(x: float, world: int) -> float:
    from bit_kv_cache_token_b200 import dp
    return dp.max_over_ranks(x, world, "cuda")


def run_kvarn(args, world, rank, local):
    from bit_kv_cache_token_b200 import kvarn, synth

    dev = torch.device("cuda", local)
    cfg = kvarn.Config(S, HKV, D, max_blocks=32768 // T_BLK, hadamard=D, sweeps=4, dtype=kvarn.KVARN_BF16)
    from bit_kv_cache_token_b200 import dp
    seed = dp.rank_seed(2, rank)
    # ---- caches: 36 layers prefilled to CTX0 tokens through the bulk quantiser
    caches = []
    for layer in range(LAYERS):
        k, v = synth.layer_kv(seed, layer, S, HKV, CTX0, D, n_outliers=4, sigma_k=0.5, device=dev)
        c = kvarn.KVCache(cfg, device=dev)
        kvarn.quantize_blocks(cfg, k, v, c)
        caches.append(c)
        del k, v
    torch.cuda.synchronize()
    n_all, n_reset = shared_lengths(caches, CTX0)
    # ---- the step's new tokens (distinct per sub-step and layer), outputs, workspace
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 77)
    qs = torch.randn(T_BLK, LAYERS, S, HQ, D, generator=g, device=dev).to(torch.bfloat16)
    ks = torch.empty(T_BLK, LAYERS, S, HKV, D, dtype=torch.bfloat16, device=dev)
    vs = torch.empty_like(ks)
    for layer in range(LAYERS):
        k, v = synth.layer_kv(seed, layer, S, HKV, T_BLK, D, n_outliers=4, first_position=CTX0, device=dev)
        ks[:, layer] = k.permute(2, 0, 1, 3)
        vs[:, layer] = v.permute(2, 0, 1, 3)
        del k, v
    outs = torch.empty(T_BLK, LAYERS, S, HQ, D, dtype=torch.float32, device=dev)
    ws = kvarn.decode_workspace(cfg, HQ, dev)

    def step(qs_=qs, ks_=ks, vs_=vs, outs_=outs):
        n_all.copy_(n_reset)  # every layer back to CTX0 tokens (one copy: the lengths share a tensor)
        for j in range(T_BLK):
            for layer, c in enumerate(caches):
                kvarn.append_token(cfg, ks_[j, layer], vs_[j, layer], c)
                kvarn.decode_attention(cfg, qs_[j, layer], c, max_tokens=32768, out=outs_[j, layer], workspace=ws)

    # ---- capture one step in a CUDA graph (9216 kernels), warm up
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        step()  # eager run once (also validates every call)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    status = sum(int(c.status.item()) for c in caches)
    if status:
        raise RuntimeError(f"device status flagged during warm-up: {status}")

    clocks = ClockSampler(local)
    clocks.start()
    _barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        graph.replay()
    t1.record()
    torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    my_ms = t0.elapsed_time(t1)
    ms_total = _max_over_ranks(my_ms, world)
    rank_ms = dp.gather_floats(my_ms, world, dev)
    ms_step = ms_total / args.steps
    value = dp.aggregate_rate(S * T_BLK * args.steps, ms_total / 1e3, world)

    # ---- decode alone, for its roofline: the 36 decode launches of one sub-step (context CTX0 + 65) captured
    # as a graph of their own, timed by events around whole replays (nothing between the launches)
    probe_j = 64
    n_all.fill_(CTX0 + probe_j + 1)
    dgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(dgraph, stream=stream):
        for layer, c in enumerate(caches):
            kvarn.decode_attention(cfg, qs[probe_j, layer], c, max_tokens=32768, out=outs[probe_j, layer],
                                   workspace=ws)
    dec_avg_ms = graph_ms(dgraph, reps=10) / LAYERS
    del dgraph
    dbytes = decode_bytes(CTX0 + probe_j + 1)
    peak, peak_kind = _peaks()
    achieved = dbytes / (dec_avg_ms / 1e3) / 1e9
    # the step holds exactly these decodes plus the appends, so launch time x launches cannot exceed it
    consistent = dec_avg_ms * LAYERS * T_BLK <= ms_step

    # ---- end to end through the API: every step copies its inputs in from pinned host memory and its outputs
    # back, as a serving loop does; with two buffer sets (and a graph for each) the copies of the neighbouring
    # steps overlap this step's compute on their own streams
    h_q = torch.empty(qs.shape, dtype=qs.dtype, pin_memory=True).copy_(qs)
    h_k = torch.empty(ks.shape, dtype=ks.dtype, pin_memory=True).copy_(ks)
    h_v = torch.empty(vs.shape, dtype=vs.dtype, pin_memory=True).copy_(vs)
    h_out = [torch.empty(outs.shape, dtype=outs.dtype, pin_memory=True) for _ in range(2)]
    sets = [(qs, ks, vs, outs), tuple(torch.empty_like(t) for t in (qs, ks, vs, outs))]
    graph_b = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_b, stream=stream):
        step(*sets[1])
    graphs = [graph, graph_b]
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n, e_start=None, e_end=None):
        if e_start is not None:
            e_start.record(h2d_s)
        for i in range(n):
            b = i % 2
            q_, k_, v_, o_ = sets[b]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev_run[b])  # the step two back has read these inputs
                q_.copy_(h_q, non_blocking=True); k_.copy_(h_k, non_blocking=True); v_.copy_(h_v, non_blocking=True)
                ev_in[b].record(h2d_s)
            with torch.cuda.stream(stream):
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])  # and its outputs have been read back
                graphs[b].replay()
                ev_run[b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_run[b])
                h_out[b].copy_(o_, non_blocking=True)
                ev_out[b].record(d2h_s)
        if e_end is not None:
            d2h_s.wait_stream(stream)
            e_end.record(d2h_s)

    e2e_steps(2)
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps(args.steps, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = dp.aggregate_rate(S * T_BLK * args.steps, e2e_ms / 1e3, world)
    got, want = h_out[(args.steps - 1) % 2], sets[(args.steps - 1) % 2][3].cpu()
    e2e_check = "the last step's outputs read back equal the device's"
    if not torch.equal(got, want):
        bad = (got != want) & ~(torch.isnan(got) & torch.isnan(want))
        where = bad.reshape(T_BLK, LAYERS, -1).any(dim=2).nonzero()[:8].tolist()
        e2e_check = (f"MISMATCH: {int(bad.sum())} outputs differ, {int(torch.isnan(got).sum())} NaN read back, "
                     f"{int(torch.isnan(want).sum())} NaN on the device; first (sub-step, layer): {where}")
        print(f"bench: end-to-end check: {e2e_check}", file=sys.stderr, flush=True)
    h2d = (qs.numel() + ks.numel() + vs.numel()) * 2
    d2h = outs.numel() * 4
    del graph, graph_b, graphs
    caches.clear()
    del qs, ks, vs, outs, ws, h_q, h_k, h_v, h_out, sets
    torch.cuda.empty_cache()

    # ---- bulk quantise GB/s (Llama-3-8B-shaped prefill)
    quant = None
    if not args.skip_quant:
        quant = run_bulk_quant(args, dev, seed, peak)
    ablation = None if args.skip_ablation or rank != 0 else run_ablation(dev)
    multi = None if args.skip_ablation or rank != 0 else run_multi_query(dev, peak)
    shapes = {}
    if not args.skip_shapes and rank == 0:
        shapes["tiny"] = run_tiny(dev)
        shapes["qwen3_4b_batch1_step"] = run_qwen_b1(dev, peak)
        shapes["phi3_mini_mha"] = run_phi(dev, peak)
        shapes["quantise_share"] = quantise_share(dev, ms_step)

    return dict(value=value, ms_step=ms_step, clocks=clk, dec_avg_ms=dec_avg_ms, dbytes=dbytes, achieved=achieved,
                peak=peak, peak_kind=peak_kind, e2e_value=e2e_value, h2d=h2d, d2h=d2h, e2e_check=e2e_check,
                quant=quant, ablation=ablation, multi=multi,
                launches=args.steps * T_BLK * LAYERS * 2, rank_ms=rank_ms, consistent=consistent, shapes=shapes)


def run_bulk_quant(args, dev, seed, peak):
    from bit_kv_cache_token_b200 import kvarn, synth
    nseq = QB_SEQS if not args.small else 64
    cfg = kvarn.Config(nseq, HKV, D, max_blocks=QB_TOKENS // T_BLK, hadamard=D, sweeps=4, dtype=kvarn.KVARN_BF16)
    k = torch.empty(nseq, HKV, QB_TOKENS, D, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    per = 32  # sequences generated per chunk (one layer of the batch)
    for i in range(0, nseq, per):
        kk, vv = synth.layer_kv(seed + 3, i // per, min(per, nseq - i), HKV, QB_TOKENS, D, n_outliers=4,
                                sigma_k=0.7, device=dev)
        k[i:i + per] = kk
        v[i:i + per] = vv
        del kk, vv
    cache = kvarn.KVCache(cfg, device=dev)
    for _ in range(2):
        kvarn.quantize_blocks(cfg, k, v, cache)
    torch.cuda.synchronize()
    reps = 5
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        kvarn.quantize_blocks(cfg, k, v, cache)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    n_elems = 2 * k.numel()
    nbytes = quant_bytes(n_elems)
    gbs = nbytes / (ms / 1e3) / 1e9
    st = int(cache.status.item())
    del k, v, cache
    torch.cuda.empty_cache()
    props = torch.cuda.get_device_properties(dev)
    clk_mhz = 1965.0  # clocks.max.sm of the B200: the highest clock gives the highest (most demanding) peak
    alu_peak = props.multi_processor_count * FP32_LANES_PER_SM * clk_mhz * 1e6 / 1e12  # T operations / s
    alu_achieved = n_elems * QUANT_FP32_OPS_PER_ELEM / (ms / 1e3) / 1e12
    return dict(workload=QB_WORKLOAD if not args.small else QB_WORKLOAD + " (reduced to 64 sequences)",
                ms=ms, gbs=gbs, bytes=nbytes, frac=gbs / peak, status=st,
                alu={"bound": "alu", "achieved": alu_achieved, "peak": alu_peak, "unit": "Top/s",
                     "frac": alu_achieved / alu_peak, "ops_per_element": QUANT_FP32_OPS_PER_ELEM,
                     "peak_source": f"{props.multi_processor_count} SMs x {FP32_LANES_PER_SM} FP32 lanes x "
                                    f"{clk_mhz:.0f} MHz (derived)",
                     "hbm_frac_at_alu_peak": alu_peak * 1e12 / QUANT_FP32_OPS_PER_ELEM * (nbytes / n_elems) / 1e9 / peak})


# ------------------------------------------------------------------- the other model shapes
def run_tiny(dev):
    """Tiny single head: K, V of 256 tokens x 64 (fp32; 2 outlier channels, token 0 x 8), Hadamard 64, two
    blocks, 4 sweeps; one decode query.  Times one quantisation of both blocks and one decode (per launch,
    from a graph of 50 back-to-back launches; everything is L2-resident at this size)."""
    from bit_kv_cache_token_b200 import kvarn, synth
    cfg = kvarn.Config(1, 1, 64, max_blocks=2, hadamard=64, sweeps=4, dtype=kvarn.KVARN_F32)
    k, v = synth.layer_kv(0, 0, 1, 1, 256, 64, n_outliers=2, dtype=torch.float32, device=dev)
    q = synth.queries(0, 1, 1, 64, dtype=torch.float32, device=dev)
    c = kvarn.KVCache(cfg, device=dev)
    ws = kvarn.decode_workspace(cfg, 1, dev)
    out = torch.empty(1, 1, 64, dtype=torch.float32, device=dev)
    n = 50
    gq = capture(lambda: [kvarn.quantize_blocks(cfg, k, v, c) for _ in range(n)], dev)
    gd = capture(lambda: [kvarn.decode_attention(cfg, q, c, max_tokens=256, out=out, workspace=ws)
                          for _ in range(n)], dev)
    res = {"workload": "tiny single head: 256 tokens x head_dim 64, fp32, Hadamard 64, 2 blocks, 4 sweeps, "
                       "1 decode query", "quantize_us": graph_ms(gq, 10) * 1e3 / n,
           "decode_us": graph_ms(gd, 10) * 1e3 / n, "status": int(c.status.item()),
           "l2": "resident (tiny); per-launch time from 50 launches in one graph"}
    del gq, gd
    return res


def run_qwen_b1(dev, peak):
    """Qwen3-4B-shaped decode step at batch 1: 36 layers x (append one token, decode attention) at context
    4153 (32 blocks + a 57-token tail), captured as one graph and replayed with L2 flushed before each step."""
    from bit_kv_cache_token_b200 import kvarn, synth
    n0, layers = 4153, LAYERS
    cfg = kvarn.Config(1, HKV, D, max_blocks=64, hadamard=D, sweeps=4, dtype=kvarn.KVARN_BF16)
    caches = []
    for layer in range(layers):
        k, v = synth.layer_kv(21, layer, 1, HKV, n0, D, n_outliers=4, device=dev)
        c = kvarn.KVCache(cfg, device=dev)
        kvarn.quantize_blocks(cfg, k, v, c)
        caches.append(c)
    n_all, n_reset = shared_lengths(caches, n0)
    kn = torch.empty(layers, 1, HKV, D, dtype=torch.bfloat16, device=dev)
    vn = torch.empty_like(kn)
    for layer in range(layers):
        k, v = synth.layer_kv(21, layer, 1, HKV, 1, D, n_outliers=4, first_position=n0, device=dev)
        kn[layer], vn[layer] = k[:, :, 0], v[:, :, 0]
    q = synth.queries(22, layers, HQ, D, device=dev).reshape(layers, 1, HQ, D)
    out = torch.empty(layers, 1, HQ, D, dtype=torch.float32, device=dev)
    ws = kvarn.decode_workspace(cfg, HQ, dev)

    def step():
        n_all.copy_(n_reset)
        for layer, c in enumerate(caches):
            kvarn.append_token(cfg, kn[layer], vn[layer], c)
            kvarn.decode_attention(cfg, q[layer], c, max_tokens=4224, out=out[layer], workspace=ws)

    g = capture(step, dev)
    flush = torch.zeros(64 << 20, dtype=torch.float32, device=dev)  # 256 MB, twice L2
    us = graph_ms(g, 20, flush=flush) * 1e3
    by = layers * decode_bytes(n0 + 1, seqs=1)
    st = sum(int(c.status.item()) for c in caches)
    del g, flush
    return {"workload": "Qwen3-4B-shaped decode step, batch 1: 36 layers x (append + decode attention) at context "
                        "4153 (32 blocks + 57-token tail), one CUDA graph, L2 flushed before each step",
            "step_us": us, "tokens_per_s": 1e6 / us, "kernel_launches": layers * 2,
            "decode_bytes_per_step": by, "gbs": by / (us * 1e-6) / 1e9, "frac": by / (us * 1e-6) / 1e9 / peak,
            "status": st}


def run_phi(dev, peak):
    """Phi-3-mini-shaped MHA: batch 16, 32 heads (no GQA), head_dim 96 with a Hadamard of 3 blocks x 32, bf16,
    32 layers at context 16383 + 1.  Times: decode attention alone (32 launches in a graph), the appends of the
    token that fills block 128 (quantise-on-append of every (sequence, head) unit, 32 launches in a graph), and
    the whole token step (32 x (append + decode)).  Outlier channels sit on both sides of the Hadamard block
    boundaries (channels 31, 32, 63, 64)."""
    from bit_kv_cache_token_b200 import kvarn, synth
    S4, H4, D4, L4, n0 = 16, 32, 96, 32, 16383
    cfg = kvarn.Config(S4, H4, D4, max_blocks=128, hadamard=32, sweeps=4, dtype=kvarn.KVARN_BF16)
    caches = []
    for layer in range(L4):
        k, v = synth.layer_kv(31, layer, S4, H4, n0, D4, outlier_channels=(31, 32, 63, 64), device=dev)
        c = kvarn.KVCache(cfg, device=dev)
        kvarn.quantize_blocks(cfg, k, v, c)
        caches.append(c)
        del k, v
    n_all, n_reset = shared_lengths(caches, n0)
    kn = torch.empty(L4, S4, H4, D4, dtype=torch.bfloat16, device=dev)
    vn = torch.empty_like(kn)
    for layer in range(L4):
        k, v = synth.layer_kv(31, layer, S4, H4, 1, D4, outlier_channels=(31, 32, 63, 64), first_position=n0,
                              device=dev)
        kn[layer], vn[layer] = k[:, :, 0], v[:, :, 0]
    q = synth.queries(32, L4 * S4, H4, D4, device=dev).reshape(L4, S4, H4, D4)
    out = torch.empty(L4, S4, H4, D4, dtype=torch.float32, device=dev)
    ws = kvarn.decode_workspace(cfg, H4, dev)

    def appends():
        n_all.copy_(n_reset)
        for layer, c in enumerate(caches):
            kvarn.append_token(cfg, kn[layer], vn[layer], c)

    def decodes():
        for layer, c in enumerate(caches):
            kvarn.decode_attention(cfg, q[layer], c, max_tokens=16384, out=out[layer], workspace=ws)

    def step():
        n_all.copy_(n_reset)
        for layer, c in enumerate(caches):
            kvarn.append_token(cfg, kn[layer], vn[layer], c)
            kvarn.decode_attention(cfg, q[layer], c, max_tokens=16384, out=out[layer], workspace=ws)

    ga = capture(appends, dev)
    app_us = graph_ms(ga, 10) * 1e3 / L4
    del ga
    gd = capture(decodes, dev)  # after the appends: every sequence holds 16384 tokens, 128 full blocks
    dec_us = graph_ms(gd, 10) * 1e3 / L4
    del gd
    gs = capture(step, dev)
    step_us = graph_ms(gs, 10) * 1e3
    del gs
    by = decode_bytes(n0 + 1, seqs=S4, hkv=H4, hq=H4, d=D4)
    st = sum(int(c.status.item()) for c in caches)
    caches.clear()
    torch.cuda.empty_cache()
    return {"workload": "Phi-3-mini-shaped MHA decode: batch 16, 32 heads, head_dim 96 (Hadamard 3 x 32), bf16, "
                        "32 layers, context 16384 (the token that fills block 128 is appended and quantised)",
            "decode_us_per_layer": dec_us, "decode_gbs": by / (dec_us * 1e-6) / 1e9,
            "decode_frac": by / (dec_us * 1e-6) / 1e9 / peak, "decode_bytes_per_layer": by,
            "decode_tokens_per_s": S4 / (L4 * dec_us * 1e-6),
            "append_quantise_us_per_layer": app_us, "step_us": step_us, "step_tokens_per_s": S4 / (step_us * 1e-6),
            "status": st, "l2": "inputs larger than L2: 32 layers x 683 MB of records per token"}


def append_costs(dev, n_filled: int = 1023, n_plain: int = 1000):
    """Per-launch time of kvarn_append_token for the Qwen3-4B-shaped batch (8 sequences x 8 kv heads, bf16):
    an append that fills the tail (and so quantises one K and one V block per unit) and one that does not;
    36 layers' appends in one graph.  The quantisation work does not depend on the context."""
    from bit_kv_cache_token_b200 import kvarn, synth
    cfg = kvarn.Config(S, HKV, D, max_blocks=8, hadamard=D, sweeps=4, dtype=kvarn.KVARN_BF16)
    caches = []
    for layer in range(LAYERS):
        k, v = synth.layer_kv(41, layer, S, HKV, n_filled, D, n_outliers=4, device=dev)
        c = kvarn.KVCache(cfg, device=dev)
        kvarn.quantize_blocks(cfg, k, v, c)
        caches.append(c)
    n_all, _ = shared_lengths(caches, n_filled)
    kn, vn = synth.layer_kv(41, 99, S, HKV, 1, D, n_outliers=4, first_position=n_filled, device=dev)
    kn, vn = kn[:, :, 0].contiguous(), vn[:, :, 0].contiguous()
    res = {}
    for name, n in (("fill_us", n_filled), ("plain_us", n_plain)):
        def appends(n=n):
            n_all.fill_(n)
            for c in caches:
                kvarn.append_token(cfg, kn, vn, c)
        g = capture(appends, dev)
        res[name] = graph_ms(g, 10) * 1e3 / LAYERS
        del g
    res["status"] = sum(int(c.status.item()) for c in caches)
    return res


def run_block_period(dev, ctx_end: int):
    """Device time of one block period (128 tokens x 36 layers x (append, decode)) for the Qwen3-4B-shaped
    batch of 8 ending at context ctx_end, captured as one graph."""
    from bit_kv_cache_token_b200 import kvarn, synth
    n0 = ctx_end - T_BLK
    cfg = kvarn.Config(S, HKV, D, max_blocks=ctx_end // T_BLK, hadamard=D, sweeps=4, dtype=kvarn.KVARN_BF16)
    caches = []
    for layer in range(LAYERS):
        k, v = synth.layer_kv(51, layer, S, HKV, n0, D, n_outliers=4, device=dev)
        c = kvarn.KVCache(cfg, device=dev)
        kvarn.quantize_blocks(cfg, k, v, c)
        caches.append(c)
    n_all, n_reset = shared_lengths(caches, n0)
    ks = torch.empty(T_BLK, LAYERS, S, HKV, D, dtype=torch.bfloat16, device=dev)
    vs = torch.empty_like(ks)
    for layer in range(LAYERS):
        k, v = synth.layer_kv(51, layer, S, HKV, T_BLK, D, n_outliers=4, first_position=n0, device=dev)
        ks[:, layer] = k.permute(2, 0, 1, 3)
        vs[:, layer] = v.permute(2, 0, 1, 3)
    qs = synth.queries(52, T_BLK * LAYERS * S, HQ, D, device=dev).reshape(T_BLK, LAYERS, S, HQ, D)
    outs = torch.empty(T_BLK, LAYERS, S, HQ, D, dtype=torch.float32, device=dev)
    ws = kvarn.decode_workspace(cfg, HQ, dev)

    def step():
        n_all.copy_(n_reset)
        for j in range(T_BLK):
            for layer, c in enumerate(caches):
                kvarn.append_token(cfg, ks[j, layer], vs[j, layer], c)
                kvarn.decode_attention(cfg, qs[j, layer], c, max_tokens=ctx_end, out=outs[j, layer], workspace=ws)

    g = capture(step, dev)
    ms = graph_ms(g, 3)
    del g
    return ms


def quantise_share(dev, ms_step_32k: float):
    """Share of a block period spent quantising blocks, at the two ends of the long-horizon growth (context
    1024 and 32768): 36 layers' block quantisations per period (the filling append's extra time over a plain
    append) over the period's device time.  The pages quote 0.18 % (1.9 ms of normalisation in 1050 ms of
    token generation, Qwen3-4B)."""
    ap = append_costs(dev)
    quant_ms = LAYERS * (ap["fill_us"] - ap["plain_us"]) / 1e3
    ms_1k = run_block_period(dev, 1024)
    return {"workload": "Qwen3-4B-shaped batch 8, one block period (128 tokens x 36 layers x (append + decode))",
            "append_fill_us": ap["fill_us"], "append_plain_us": ap["plain_us"],
            "quantise_ms_per_period": quant_ms, "period_ms_1k": ms_1k, "period_ms_32k": ms_step_32k,
            "share_1k": quant_ms / ms_1k, "share_32k": quant_ms / ms_step_32k, "pages_share": 0.0018,
            "status": ap["status"]}


# --------------------------------------------------------------------------- oracle (CPU)
def oracle_sample(max_threads: int = 16):
    """Time the fp64 oracle on a bounded sample of the step and extrapolate to tokens/s.

    Sample: one layer, P (sequence, kv head) pairs, P = min(host cores, 16), one pair per thread.
    (a) decode at context CTX0+65: dequantise all 255 K and V records, explicit softmax attention over
    32705 tokens for the 4 query heads of the pair; (b) one K and one V block quantisation per pair
    (append quantises once per 128 tokens).  Per generated token the full step needs 36 x 64 decodes
    and 36 x 64 x 2 / 128 block quantisations, which the per-thread times are scaled to."""
    import concurrent.futures

    import numpy as np

    import oracle
    from bit_kv_cache_token_b200 import synth

    oracle.build()
    P = max(1, min(os.cpu_count() or 1, max_threads))
    n = CTX0 + 65
    nb, nt = n // T_BLK, n % T_BLK
    k, v = synth.layer_kv(2, 0, 1, P, n, D, n_outliers=4, dtype=torch.bfloat16)
    q = synth.queries(5, 1, 4 * P, D)
    kx, vx = k[0].double().numpy(), v[0].double().numpy()
    raw_k = k[0].contiguous().view(torch.int16).numpy().view(np.uint16)
    raw_v = v[0].contiguous().view(torch.int16).numpy().view(np.uint16)

    def records(h):  # untimed set-up: the cache this pair's decode reads, quantised by the oracle
        return (oracle.quantize_many(raw_k[h, :nb * T_BLK], "bf16", T_BLK, D, D, nthreads=1)[0],
                oracle.quantize_many(raw_v[h, :nb * T_BLK], "bf16", T_BLK, D, D, nthreads=1)[0])

    with concurrent.futures.ThreadPoolExecutor(P) as ex:
        recs = list(ex.map(records, range(P)))

    def decode_pair(h):
        kt = np.zeros((1, T_BLK, D)); vt = np.zeros((1, T_BLK, D))
        kt[0, :nt] = kx[h, nb * T_BLK:n]; vt[0, :nt] = vx[h, nb * T_BLK:n]
        oracle.decode_from_cache(q[0, 4 * h:4 * h + 4].double().numpy(), recs[h][0][None], recs[h][1][None],
                                 kt, vt, n, T_BLK, D, 1 / math.sqrt(D))

    def quant_pair(h):
        oracle.quantize_many(raw_k[h, :T_BLK], "bf16", T_BLK, D, D, nthreads=1)
        oracle.quantize_many(raw_v[h, :T_BLK], "bf16", T_BLK, D, D, nthreads=1)

    with concurrent.futures.ThreadPoolExecutor(P) as ex:
        t0 = time.perf_counter()
        list(ex.map(decode_pair, range(P)))
        t1 = time.perf_counter()
        list(ex.map(quant_pair, range(P)))
        t2 = time.perf_counter()
    # wall time of P concurrent units = time per unit per thread
    t_dec, t_q = t1 - t0, t2 - t1
    decodes = LAYERS * S * HKV
    quants = LAYERS * S * HKV * 2 / T_BLK
    t_token = decodes / P * t_dec + quants / (2 * P) * t_q
    return dict(value=S / t_token, unit=UNIT, cores=P, kind="oracle",
                sample=f"1 of 36 layers x {P} of 64 (sequence, kv head) pairs: one decode token at context {n} "
                       f"({t_dec:.2f} s) and one K + one V block quantisation per pair ({t_q:.2f} s), one pair per "
                       f"thread on {P} threads; extrapolated to 36 x 64 decodes + 36 x 64 x 2/128 quantisations "
                       f"per token for the 8-sequence batch")


# ------------------------------------------------------------------- ablation of the two stages
def run_ablation(dev):
    """Magnitude / direction error of the stored K and V per token, for the full encoding and with the rotation,
    the normalisation or both switched off (one Qwen3-4B-shaped layer: 8 sequences x 8 kv heads x 4096 tokens,
    bf16), measured by kvarn_token_errors on the GPU; plus that kernel's time."""
    from bit_kv_cache_token_b200 import kvarn, synth
    k, v = synth.layer_kv(9, 0, S, HKV, 4096, D, n_outliers=4, device=dev)
    out = {}
    for name, hb, sw in (("kvarn", D, 4), ("no_rotation", 0, 4), ("no_normalisation", D, 0), ("plain_rtn", 0, 0)):
        cfg = kvarn.Config(S, HKV, D, max_blocks=4096 // T_BLK, hadamard=hb, sweeps=sw, dtype=kvarn.KVARN_BF16)
        c = kvarn.KVCache(cfg, device=dev)
        kvarn.quantize_blocks(cfg, k, v, c)
        ek, ev = kvarn.token_errors(cfg, k, v, c)
        torch.cuda.synchronize()
        row = {}
        for tn, e in (("k", ek), ("v", ev)):
            e = e.reshape(-1, 2)
            row[f"{tn}_magnitude_mean"] = float(e[:, 0].mean())
            row[f"{tn}_direction_mean"] = float(e[:, 1].mean())
            row[f"{tn}_magnitude_p99"] = float(torch.quantile(e[:, 0], 0.99))
            row[f"{tn}_direction_p99"] = float(torch.quantile(e[:, 1], 0.99))
        out[name] = row
        if name == "kvarn":
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(10):
                kvarn.token_errors(cfg, k, v, c)
            e1.record()
            torch.cuda.synchronize()
            out["token_errors_ms"] = e0.elapsed_time(e1) / 10
    out["workload"] = "Qwen3-4B-shaped layer: 8 sequences x 8 kv heads x 4096 tokens x 128, bf16"
    return out


# ------------------------------------------------------------------- several query tokens at once
def run_multi_query(dev, peak):
    """One Qwen3-4B-shaped layer at 32705 cached tokens: decode of the last token alone versus the last two
    tokens at once (speculative verification); 2 queries x GQA 4 fill the 8 rows of the tensor-core tiles."""
    from bit_kv_cache_token_b200 import kvarn, synth
    cfg = kvarn.Config(S, HKV, D, max_blocks=32768 // T_BLK, hadamard=D, dtype=kvarn.KVARN_BF16)
    caches = []
    for layer in range(4):  # distinct layers so that L2 cannot hold the working set
        k, v = synth.layer_kv(11, layer, S, HKV, CTX0 + 65, D, device=dev)
        c = kvarn.KVCache(cfg, device=dev)
        kvarn.quantize_blocks(cfg, k, v, c)
        caches.append(c)
        del k, v
    res = {}
    for Q in (1, 2):
        q = synth.queries(12, S * Q, HQ, D, device=dev).reshape(S, Q, HQ, D)
        ws = kvarn.decode_workspace(cfg, Q * HQ, dev)
        out = torch.empty(q.shape, dtype=torch.float32, device=dev)
        for c in caches:
            kvarn.decode_attention_multi(cfg, q, c, max_tokens=32768, out=out, workspace=ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        e0.record()
        for _ in range(reps):
            for c in caches:
                kvarn.decode_attention_multi(cfg, q, c, max_tokens=32768, out=out, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (reps * len(caches))
        gbs = decode_bytes(CTX0 + 65) / (us * 1e-6) / 1e9
        res[f"q{Q}"] = {"us_per_launch": us, "us_per_query_token": us / Q, "gbs": gbs, "frac": gbs / peak}
    res["workload"] = "Qwen3-4B-shaped layer, batch 8, 32705 cached tokens; the last 1 or 2 tokens as queries"
    return res


# ------------------------------------------------------------------- small profiling cases
def run_profile_case(case: str):
    """Small cases for ncu captures: 3 launches of one kernel on inputs larger than L2.

    decode:   one Qwen3-4B-shaped layer (batch 8, 8 kv / 32 q heads, 32705 cached tokens, 219 MB).
    quantize: bulk quantisation of 16 sequences x 8 kv heads x 8192 tokens (537 MB in, 1.6 GB held).
    append:   append with quantise-on-fill for the same layer (tail completes on every launch)."""
    from bit_kv_cache_token_b200 import kvarn, synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if case in ("decode", "append"):
        cfg = kvarn.Config(S, HKV, D, max_blocks=32768 // T_BLK, hadamard=D, dtype=kvarn.KVARN_BF16)
        k, v = synth.layer_kv(2, 0, S, HKV, CTX0 + 65, D, device=dev)
        c = kvarn.KVCache(cfg, device=dev)
        kvarn.quantize_blocks(cfg, k, v, c)
        q = synth.queries(3, S, HQ, D, device=dev)
        ws = kvarn.decode_workspace(cfg, HQ, dev)
        kk, vv = k[:, :, -1].contiguous(), v[:, :, -1].contiguous()
        del k, v
        for _ in range(3):
            if case == "decode":
                kvarn.decode_attention(cfg, q, c, max_tokens=32768, workspace=ws)
            else:
                c.n_tokens.fill_(CTX0 - 1)
                kvarn.append_token(cfg, kk, vv, c)
    else:
        cfg = kvarn.Config(16, HKV, D, max_blocks=QB_TOKENS // T_BLK, hadamard=D, dtype=kvarn.KVARN_BF16)
        k, v = synth.layer_kv(5, 0, 16, HKV, QB_TOKENS, D, sigma_k=0.7, device=dev)
        c = kvarn.KVCache(cfg, device=dev)
        for _ in range(3):
            kvarn.quantize_blocks(cfg, k, v, c)
    torch.cuda.synchronize()
    print(f"profile case {case} done", flush=True)


# -------------------------------------------------------------------------------- main
def check_line(line: dict) -> list[str]:
    """Internal consistency of a bench line; the list of what does not hold (empty when all do)."""
    bad = []
    rf = line.get("roofline", {})
    if rf.get("launch_ms") is not None and rf.get("launches_per_step"):
        if rf["launch_ms"] * rf["launches_per_step"] > line["ms_per_step"]:
            bad.append("decode launch_ms x launches_per_step exceeds ms_per_step")
    if rf.get("achieved") and rf.get("peak") and abs(rf["frac"] - rf["achieved"] / rf["peak"]) > 1e-9:
        bad.append("roofline frac is not achieved / peak")
    if rf.get("launch_ms") and rf.get("algorithmic_bytes_per_launch"):
        gbs = rf["algorithmic_bytes_per_launch"] / (rf["launch_ms"] / 1e3) / 1e9
        if abs(gbs - rf["achieved"]) > 1e-6 * gbs:
            bad.append("roofline achieved is not bytes / launch time")
    if len(line.get("rank_ms", [None])) != line.get("n_gpus", 1):
        bad.append("rank_ms does not hold one time per rank")
    if line.get("rank_ms") and abs(max(line["rank_ms"]) / line["steps"] - line["ms_per_step"]) > 1e-6 * line["ms_per_step"]:
        bad.append("ms_per_step is not the slowest rank's time per step")
    return bad


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kvarn", choices=["kvarn", "reference"])
    ap.add_argument("--skip-quant", action="store_true", help="skip the bulk quantise measurement")
    ap.add_argument("--small", action="store_true", help="reduced bulk quantise size (quick checks)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-ablation", action="store_true", help="skip the ablation and multi-query measurements")
    ap.add_argument("--skip-shapes", action="store_true", help="skip the tiny, batch-1, Phi-3 and quantise-share keys")
    ap.add_argument("--stub", action="store_true",
                    help="CPU-only stand-in step on gloo (tests the rank launch and the JSON line without a GPU)")
    ap.add_argument("--profile", choices=["decode", "quantize", "append"], default=None,
                    help="run a small case of one kernel for ncu and exit")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args.profile)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))
    if args.stub:
        run_stub(args)
        return

    world, rank, local = _dist_setup(args) if args.impl == "kvarn" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)

    if args.impl == "reference":
        if rank != 0:
            return
        runs = []
        for _ in range(args.warmup):
            oracle_sample()
        for _ in range(args.steps):
            runs.append(oracle_sample())
        val = statistics.median(r["value"] for r in runs)
        line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": 0, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": S * T_BLK / val * 1e3, "higher_is_better": True, "scaling": "weak",  # ms_per_step: extrapolated from the sample
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {"workload": WORKLOAD, "global_batch": S, "seq_len": 32768},
                "cpu_baseline": {k: runs[-1][k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        line["cpu_baseline"]["value"] = val
        print(json.dumps(line), flush=True)
        return

    r = run_kvarn(args, world, rank, local)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample()
    if rank == 0:
        q = r["quant"]
        line = {
            "metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": S * world, "seq_len": 32768, "layers": LAYERS,
                       "q_heads": HQ, "kv_heads": HKV, "head_dim": D, "tokens_per_step": S * T_BLK * world,
                       "parallelism": f"dp{world} (independent batches, no collective)",
                       "numerics": "bf16 inputs, 2-bit records with binary16 scales, fp32 arithmetic (tensor-core "
                                   "operands as fp16 hi/lo pairs, fp32 accumulation)",
                       "l2": "inputs larger than L2: each decode launch streams ~219 MB of cache, 7.9 GB per token"},
            "roofline": {"bound": "hbm", "kernel": "decode_kernel", "achieved": r["achieved"], "peak": r["peak"],
                         "unit": "GB/s", "frac": r["achieved"] / r["peak"], "traffic": DECODE_TRAFFIC_BYTES,
                         "peak_source": r["peak_kind"], "algorithmic_bytes_per_launch": r["dbytes"],
                         "launch_ms": r["dec_avg_ms"], "launches_per_step": T_BLK * LAYERS,
                         "launch_ms_source": "the 36 decode launches of one sub-step (context 32705) as their own "
                                             "CUDA graph, median replay / 36",
                         "launch_ms_x_launches_within_step": r["consistent"]},
            "e2e": {"value": r["e2e_value"], "unit": UNIT, "h2d_bytes_per_step": r["h2d"],
                    "d2h_bytes_per_step": r["d2h"], "check": r["e2e_check"]},
            "gpu_launches": r["launches"],
            "clocks": r["clocks"],
        }
        if q:
            line["quantize"] = {"workload": q["workload"], "gbs": q["gbs"], "ms": q["ms"], "frac": q["frac"],
                                "algorithmic_bytes": q["bytes"], "peak": r["peak"], "status": q["status"],
                                "roofline_alu": q["alu"],
                                "traffic": QUANT_TRAFFIC_BYTES_16SEQ * (QB_SEQS // 16) if not args.small else None,
                                "traffic_source": "ncu capture of 16 sequences, scaled by 64 (traffic grows with the "
                                                  "sequences)"}
        if r["ablation"]:
            line["ablation"] = r["ablation"]
        if r["multi"]:
            line["multi_query_decode"] = r["multi"]
        line.update(r["shapes"])
        line["rank_ms"] = r["rank_ms"]
        if cpu:
            line["cpu_baseline"] = cpu
        for msg in check_line(line):
            print(f"bench: inconsistent line: {msg}", file=sys.stderr, flush=True)
        print(json.dumps(line), flush=True)
    from bit_kv_cache_token_b200 import dp
    dp.finish(world)


if __name__ == "__main__":
    main()
