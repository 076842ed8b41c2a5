"""Benchmark of the KVarN hot path on B200.

Workload (one "step"): Qwen3-4B-shaped long-horizon decode -- batch 8, 32 query / 8 kv heads,
head_dim 128, bf16, 36 layer caches at a 32K context.  A step is one full block period: 128
consecutive decode tokens, each running, for every layer, kvarn_append_token (which quantises the
filled 128-token tail on the last token: rotation, 4 normalisation sweeps, 2-bit packing) and then
kvarn_decode_attention over the whole 2-bit cache.  Each step starts from 32640 cached tokens
(255 blocks) and ends at 32768, so every (layer, sequence, kv head) quantises exactly one K and one
V block per step.  The line also reports bulk quantisation GB/s on the Llama-3-8B-shaped prefill
(batch 32 x 32 layers x 8 kv heads x 8192 tokens x 128, bf16).

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
# batch, from one ncu capture of `bench.py --profile decode` with the current decode kernel; reset it to None
# whenever the decode kernel changes until it is captured again.
DECODE_TRAFFIC_BYTES = 219929856 + 4410112


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def decode_bytes(n_tokens: int) -> int:
    """Algorithmic HBM bytes of one decode launch at context n for the whole batch.

    Per (sequence, kv head): both 6656-byte records (K and V: 2-bit codes 4096 B, (s, m) pairs
    2048 B, r 256 B, c 256 B) of every full block, plus 2 x D bf16 values of every tail token;
    per query head: q (bf16) read and out (fp32) written."""
    nb, nt = n_tokens // T_BLK, n_tokens % T_BLK
    per_kv = nb * 2 * 6656 + nt * 2 * D * 2
    return S * HKV * per_kv + S * HQ * D * (2 + 4)


def quant_bytes(n_elems: int) -> int:
    """Algorithmic bytes of bulk quantisation: bf16 read + record bytes written (2.40625 B/elem)."""
    return n_elems * 2 + (n_elems // (T_BLK * D)) * 6656


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
    n_reset = torch.full((S,), CTX0, dtype=torch.int32, device=dev)
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
    # external events become event-record nodes of the captured graph, so they time each replay
    ev_pairs = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
                for _ in range(LAYERS)]
    probe_j = 64  # sub-step whose decode launches are bracketed with events

    def step(qs_=qs, ks_=ks, vs_=vs, outs_=outs, probe=True):
        for c in caches:
            c.n_tokens.copy_(n_reset)
        for j in range(T_BLK):
            for layer, c in enumerate(caches):
                kvarn.append_token(cfg, ks_[j, layer], vs_[j, layer], c)
                if probe and j == probe_j:
                    ev_pairs[layer][0].record()
                kvarn.decode_attention(cfg, qs_[j, layer], c, max_tokens=32768, out=outs_[j, layer], workspace=ws)
                if probe and j == probe_j:
                    ev_pairs[layer][1].record()

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
    dec_ms = []
    t0.record()
    for _ in range(args.steps):
        graph.replay()
        # per-launch decode durations of this replay (events are graph nodes)
    t1.record()
    torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    for a, b in ev_pairs:
        dec_ms.append(a.elapsed_time(b))  # last replay's probe launches
    ms_total = _max_over_ranks(t0.elapsed_time(t1), world)
    ms_step = ms_total / args.steps
    value = dp.aggregate_rate(S * T_BLK * args.steps, ms_total / 1e3, world)

    # decode-only roofline: events around each layer's decode at sub-step probe_j (context CTX0+probe_j+1)
    dec_avg_ms = statistics.mean(dec_ms)
    dbytes = decode_bytes(CTX0 + probe_j + 1)
    peak, peak_kind = _peaks()
    achieved = dbytes / (dec_avg_ms / 1e3) / 1e9

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
        step(*sets[1], probe=False)
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
    if not torch.equal(h_out[(args.steps - 1) % 2], sets[(args.steps - 1) % 2][3].cpu()):
        raise RuntimeError("end-to-end outputs read back do not match the device outputs")
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

    return dict(value=value, ms_step=ms_step, clocks=clk, dec_avg_ms=dec_avg_ms, dbytes=dbytes, achieved=achieved,
                peak=peak, peak_kind=peak_kind, e2e_value=e2e_value, h2d=h2d, d2h=d2h, quant=quant, ablation=ablation, multi=multi,
                launches=args.steps * T_BLK * LAYERS * 2)


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
    nbytes = quant_bytes(2 * k.numel())
    gbs = nbytes / (ms / 1e3) / 1e9
    st = int(cache.status.item())
    del k, v, cache
    torch.cuda.empty_cache()
    return dict(workload=QB_WORKLOAD if not args.small else QB_WORKLOAD + " (reduced to 64 sequences)",
                ms=ms, gbs=gbs, bytes=nbytes, frac=gbs / peak, status=st)


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
    ap.add_argument("--profile", choices=["decode", "quantize", "append"], default=None,
                    help="run a small case of one kernel for ncu and exit")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args.profile)
        return
    if args.warmup < 3:
        args.warmup = 3

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
                         "launch_ms": r["dec_avg_ms"]},
            "e2e": {"value": r["e2e_value"], "unit": UNIT, "h2d_bytes_per_step": r["h2d"],
                    "d2h_bytes_per_step": r["d2h"]},
            "gpu_launches": r["launches"],
            "clocks": r["clocks"],
        }
        if q:
            line["quantize"] = {"workload": q["workload"], "gbs": q["gbs"], "ms": q["ms"], "frac": q["frac"],
                                "algorithmic_bytes": q["bytes"], "peak": r["peak"], "status": q["status"]}
        if r["ablation"]:
            line["ablation"] = r["ablation"]
        if r["multi"]:
            line["multi_query_decode"] = r["multi"]
        if cpu:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    from bit_kv_cache_token_b200 import dp
    dp.finish(world)


if __name__ == "__main__":
    main()
