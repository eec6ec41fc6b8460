"""Benchmark of the quantized-KV decode step (KVQuant hot path) on B200.

One step = for every layer: quantize-append one new token (K and V) into the
3-bit cache, then decode attention of one query per sequence over the whole
cache (QK with NUQ lookup + RoPE + key outliers, split-K softmax merge, PV with
value outliers).  Default workload: LLaMA-7B shape, 32 layers x 32 heads x
head_dim 128, 1,048,576 cached tokens, batch 1, 3-bit NUQ, 0.5% outliers,
synthetic seeded inputs.  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV tokens/s in quantized decode attention; achieved HBM GB/s vs peak"
UNIT = "KV tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default="llama7b_1m_32layers")
    p.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    p.add_argument("--splits", type=int, default=0)
    p.add_argument("--path", default="split", choices=["split", "one-call", "fused"],
                   help="split: kvq_decode_qk + kvq_softmax_merge + kvq_decode_pv; one-call: "
                        "kvq_decode_attention (the same kernels); fused: "
                        "kvq_decode_attention_fused (one kernel per split, no logits)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-fp16", action="store_true")
    p.add_argument("--no-graph", action="store_true",
                   help="time the per-layer calls only (by default the headline is the whole "
                        "step, every layer's append and attention, replayed as one CUDA graph "
                        "through kvq_step_launch)")
    p.add_argument("--layers", type=int, default=0, help="override the workload's layer count")
    p.add_argument("--tokens", type=int, default=0, help="override the cached token count")
    p.add_argument("--bits", type=int, default=0, help="override the workload's code width")
    p.add_argument("--shard", default="tokens", choices=["tokens", "replicas"],
                   help="N > 1: tokens = one sequence of N x T tokens, rank r holding tokens "
                        "[r T, (r+1) T) (partials all-gathered and merged per layer); replicas = "
                        "an independent sequence per rank")
    return p.parse_args()


# ----------------------------------------------------------------------------- helpers

def rank_layer_key(layer: int, rank: int) -> int:
    """Synthetic-data key of a layer on a rank: every rank holds a different sequence."""
    return layer + 4096 * rank


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time; every rank calls this at the same point."""
    if world == 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(tokens_per_rank: float, world: int, ms: float) -> float:
    """Whole-job KV tokens/s: every rank processed tokens_per_rank in at most ms."""
    return tokens_per_rank * world / (ms / 1e3)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # the timed region starts once the sampler runs (first sample, at most 5 s)
            t_end = time.time() + 5.0
            while not self.lines and time.time() < t_end and self.proc.poll() is None:
                time.sleep(0.02)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def src_hash(kernel_file):
    with open(os.path.join(ROOT, "long_context_decode_nuq_b200", "csrc", kernel_file), "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def traffic_for(kernel, units):
    """Per-launch DRAM bytes from the committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        d = json.load(fh)
    e = d.get(kernel)
    if not e or e.get("src_sha") != src_hash(e["file"]):
        return None
    return e["dram_bytes_per_unit"] * units


# ----------------------------------------------------------------------------- algorithmic bytes

OUTLIER_ENTRY_BYTES = 4  # one packed uint32 per outlier: (fp16 bits << 16) | (t % 64) << 7 | c


def expected_outliers_per_token(w):
    """Expected outlier entries per cached token of one layer (all kv heads).

    Keys: a channel keeps 2k of its N calibration values as outliers, k = floor(f*N/2 + 1/2),
    i.e. about f*n per token over the n = Hkv*D channels; values: each token row keeps 2k_v,
    k_v = floor(f*n/2 + 1/2).
    """
    kv = math.floor(w.f * w.n / 2 + 0.5)
    return w.f * w.n, 2 * kv


def cache_bytes_per_token(w, outlier_bytes=OUTLIER_ENTRY_BYTES, params=True):
    """Stored bytes per token of one layer: K and V codes, outlier entries, value (off, half).

    The per-channel key scales and the chunk pointers are per sequence, not per token.
    """
    k_out, v_out = expected_outliers_per_token(w)
    codes = 2 * w.n * w.bits / 8
    return codes + outlier_bytes * (k_out + v_out) + (8 if params else 0)


def bytes_model(w, T, kcount, vcount, path, outlier_bytes=OUTLIER_ENTRY_BYTES, logits=True):
    """Algorithmic bytes of one layer's decode (attention part) over T tokens of each of the
    w.B sequences; kcount and vcount are the outlier entries of all the sequences.

    Key side (QK): packed key codes, key-outlier entries (outlier_bytes each: position and
    value), key chunk pointers (one list per kv head); value side (PV): packed value codes,
    value-outlier entries, value token params (8 B/token), value chunk pointers.  The split
    path (kvq_decode_qk / kvq_softmax_merge / kvq_decode_pv) also writes and reads fp32 logits
    (4 B per token per query head, each way), and so does kvq_decode_attention, which runs the
    same kernels; the fused path (kvq_decode_attention_fused) moves no logits.
    """
    code_row = w.Hkv * w.D * w.bits // 8
    nch = (T + 63) // 64 + 1
    k_bytes = w.B * (T * code_row + 4 * nch * w.Hkv) + outlier_bytes * kcount
    v_bytes = w.B * (T * code_row + 8 * T + 4 * nch * w.Hkv) + outlier_bytes * vcount
    logit = 4 * w.Hq * T * w.B if logits else 0
    if path == "split":
        return {"qk": k_bytes + logit, "pv": v_bytes + logit, "total": k_bytes + v_bytes + 2 * logit}
    if path == "one-call":
        return {"attn": k_bytes + v_bytes + 2 * logit, "total": k_bytes + v_bytes + 2 * logit}
    return {"attn": k_bytes + v_bytes, "total": k_bytes + v_bytes}


# ----------------------------------------------------------------------------- CPU oracle

def cpu_oracle_sample(w, budget_s=12.0, layer=0):
    """Time the CPU oracle's decode (dequantize + binary64 attention) on a bounded
    sample of the workload: one layer, all heads, T_s tokens; returns KV tokens/s."""
    import oracle as O
    import synth
    T_s = 1024 if w.Hkv >= 16 else 4096
    ws = synth.workload(w.name, B=1, T=T_s)
    idx = (np.zeros((1, 1, 1, 1), dtype=np.int64), np.arange(T_s)[None, :, None, None],
           np.arange(w.Hkv)[None, None, :, None], np.arange(w.D)[None, None, None, :])
    K16 = synth.gen_k(ws, layer, *idx)
    V16 = synth.gen_v(ws, layer, *idx)
    cbK = O.fit_codebook(synth.codebook_samples_k(ws, layer), w.f, w.bits)
    cbV = O.fit_codebook(synth.codebook_samples_v(ws, layer), w.f, w.bits)
    c = O.QuantizedCache(1, w.Hkv, w.bits, T_s, w.f, T_s * w.Hkv * w.D, T_s * w.Hkv * w.D)
    c.prefill(K16, V16, [T_s], cbK, cbV)
    q = synth.gen_q(ws, layer)[0]
    reps, t0 = 0, time.perf_counter()
    while True:
        Kh, Vh = c.dequantize(0, cbK, cbV)
        O.decode_attention(q, T_s, Kh, Vh, w.rope_theta)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return reps * T_s / el, f"1 layer x {w.Hkv} kv heads x {T_s} tokens, {reps} repetitions, {el:.1f} s"


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import synth
    w = synth.workload(args.workload)
    steps_t = []
    samples = []
    for _ in range(args.warmup):
        cpu_oracle_sample(w, budget_s=2.0)
    for _ in range(args.steps):
        v, smp = cpu_oracle_sample(w, budget_s=4.0)
        steps_t.append(v)
        samples.append(smp)
    val = statistics.median(steps_t)
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Philox4x32-10, LLaMA-shaped)",
        "config": {"workload": w.name, "layers": w.layers, "B": w.B, "kv_heads": w.Hkv,
                   "head_dim": w.D, "T": w.T, "bits": w.bits, "outlier_frac": w.f},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": samples[-1],
                         "extrapolated": "KV tokens/s of a sampled slice, not a run of the "
                                         "whole workload"},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def run_kvq(args, rank, world):
    import torch
    import torch.distributed as dist
    import long_context_decode_nuq_b200 as K
    import synth
    from synth.gpu import DeviceGen

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    over = {}
    if args.layers:
        over["layers"] = args.layers
    if args.tokens:
        over["T"] = args.tokens
    if args.bits:
        over["bits"] = args.bits
    w = synth.workload(args.workload, **over)
    steps_total = args.warmup + args.steps
    e2e_steps = min(args.steps, 10)
    sharded = world > 1 and args.shard == "tokens"
    shard_n = world if sharded else 1
    if w.T + steps_total + 16 > w.T_gen:
        w = synth.workload(args.workload, appends=1, steps=steps_total + 16, **over)
    layers = w.layers
    T0 = w.T  # tokens held by this rank's caches
    # the generator's token extent: the whole sequence when sharded (rank r holds its tokens
    # [r T0, (r+1) T0), the last rank appends at positions N T0 + s)
    w_gen = synth.workload(args.workload, appends=1, steps=steps_total + e2e_steps + 16,
                           **{**over, "T": shard_n * T0})
    t_base = rank * T0 if sharded else 0          # position of this rank's first token
    pos0 = shard_n * T0                            # position of the first appended token
    appends_here = (not sharded) or rank == world - 1
    # the graph-replayed step (not with token sharding, whose merge is a collective) runs first
    use_graph = not args.no_graph and not sharded
    graph_steps = steps_total if use_graph else 0
    T_max = T0 + graph_steps + steps_total + e2e_steps + 64
    # outlier lists are per (sequence, kv head): a key channel keeps ~f*T outliers, a token's
    # 2k value outliers spread over the Hkv heads; capacities are multiples of 8
    ceil8 = lambda x: (int(x) + 7) // 8 * 8  # noqa: E731
    kout_cap = ceil8(T_max * w.f * w.D * 1.25 + 4096)
    vout_cap = ceil8(T_max * 2 * math.floor(w.f * w.n / 2 + 0.5) / w.Hkv * 1.5 + 4096)
    cfg = K.make_cfg(w.B, w.Hq, w.Hkv, w.bits, T_max, w.f, w.rope_theta, kout_cap, vout_cap)
    # replicas: a different synthetic sequence per rank; sharded: one sequence split across ranks
    layer_key = lambda l: rank_layer_key(l, 0 if sharded else rank)  # noqa: E731

    # replicas of the whole cache so that the timed inputs exceed L2 by a wide margin
    one_cache_bytes = sum(K.kvq_layout(cfg).values()) * layers
    R = 1 if one_cache_bytes * 1 > 4 * L2_BYTES else int(math.ceil(4 * L2_BYTES / one_cache_bytes))

    t_setup = time.time()
    kstage = torch.empty((w.B, T0, w.Hkv, w.D), dtype=torch.float16, device=dev)
    vstage = torch.empty_like(kstage)
    caches, cbs = [], []
    kfirst = None
    fit_ws = torch.empty(K.kvq_fit_workspace(32, 128), dtype=torch.uint8, device=dev)
    qws = torch.empty(K.kvq_quantize_workspace(cfg, T0, 1), dtype=torch.uint8, device=dev)
    prefill_ms = []
    for r in range(R):
        for l in range(layers):
            gen = DeviceGen(w_gen, layer_key(l) + 100000 * r, device=dev)
            gen.fill_k(kstage, t_base, T0)
            gen.fill_v(vstage, t_base, T0)
            cb = []
            for samples in (synth.codebook_samples_k(w, layer_key(l)),
                            synth.codebook_samples_v(w, layer_key(l))):
                s = torch.from_numpy(samples.view(np.int16).copy()).to(dev)
                lev = torch.empty(1 << w.bits, dtype=torch.float32, device=dev)
                bnd = torch.empty((1 << w.bits) - 1, dtype=torch.float32, device=dev)
                K.kvq_fit_codebook(s, w.f, w.bits, lev, bnd,
                                   torch.empty(K.kvq_fit_workspace(*samples.shape),
                                               dtype=torch.uint8, device=dev))
                cb.append(K.Codebook(lev, bnd))
            c = K.Cache(cfg, device=dev)
            K.kvq_cache_reset(c)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            K.kvq_quantize_append(c, cb[0], cb[1], kstage, vstage, T0, None, 1, qws)
            e1.record()
            torch.cuda.synchronize()
            prefill_ms.append(e0.elapsed_time(e1))
            st = K.kvq_get_status(c)
            if st:
                raise RuntimeError(f"cache status {st} after prefill of layer {l}")
            caches.append(c)
            cbs.append(cb)
    setup_s = time.time() - t_setup
    if args.no_fp16:  # the staged K/V of the last layer serve only the fp16 comparison
        del kstage, vstage
        torch.cuda.empty_cache()
    kcount = int(caches[0].kcount.cpu().sum())  # all sequences of the layer
    vcount = int(caches[0].vcount.cpu().sum())

    # per-step inputs: appended token K/V and queries, per layer (device and pinned host)
    nL = layers * R
    knew = torch.empty((nL, steps_total, w.B, 1, w.Hkv, w.D), dtype=torch.float16, device=dev)
    vnew = torch.empty_like(knew)
    qall = torch.empty((nL, steps_total, w.B, w.Hq, w.D), dtype=torch.float16, device=dev)
    for i in range(nL):
        r, l = divmod(i, layers)
        gen = DeviceGen(w_gen, layer_key(l) + 100000 * r, device=dev)
        for s in range(steps_total):
            tmp = torch.empty((w.B, 1, w.Hkv, w.D), dtype=torch.float16, device=dev)
            gen.fill_k(tmp, pos0 + s, 1)
            knew[i, s] = tmp
            gen.fill_v(tmp, pos0 + s, 1)
            vnew[i, s] = tmp
            gen.fill_q(qall[i, s], step=s)
    # the per-layer region appends after the graph region's tokens
    qpos = torch.tensor([[pos0 + graph_steps + s] * w.B for s in range(steps_total)],
                        dtype=torch.int32, device=dev)
    sdec = None
    if sharded:
        from long_context_decode_nuq_b200.shard import ShardedDecode
        sdec = ShardedDecode(cfg, world, rank, dev)
    S = args.splits or K.kvq_decode_splits(cfg, T_max)
    aws = torch.empty(K.kvq_quantize_workspace(cfg, 1, 0), dtype=torch.uint8, device=dev)
    dws = torch.empty(K.kvq_decode_workspace(cfg, T_max, S), dtype=torch.uint8, device=dev)
    BH = w.B * w.Hq
    logits = torch.empty((w.B, w.Hq, T_max), dtype=torch.float32, device=dev)
    stats = torch.empty((w.B, w.Hq, S, 2), dtype=torch.float32, device=dev)
    qkws = torch.empty(K.kvq_decode_qk_workspace(cfg, T_max), dtype=torch.uint8, device=dev)
    mlb = torch.empty((w.B, w.Hq, 2), dtype=torch.float32, device=dev)
    part = torch.empty((w.B, w.Hq, S, w.D), dtype=torch.float32, device=dev)
    outs = torch.empty((nL, w.B, w.Hq, w.D), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    ev_pool = []

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        ev_pool.append(e)
        return e

    def local_len(s):
        return T0 + graph_steps + s + 1 if appends_here else T0

    def layer_step(i, s, timing):
        c = caches[i]
        cbK, cbV = cbs[i]
        max_len = local_len(s)
        marks = [ev(), ev(), ev(), ev(), ev()] if timing else None
        if timing:
            marks[0].record()
        if appends_here:
            K.kvq_quantize_append(c, cbK, cbV, knew[i, s], vnew[i, s], 1, None, 0, aws)
        if timing:
            marks[1].record()
        if sharded:
            if timing:
                marks[2].record()
                marks[3].record()
            sdec(c, cbK, cbV, qall[i, s], qpos[s], max_len, t_base, outs[i], dws, S)
        elif args.path == "split":
            K.kvq_decode_qk(c, cbK, qall[i, s], qpos[s], max_len, logits, stats, S, qkws)
            if timing:
                marks[2].record()
            K.kvq_softmax_merge(cfg, stats, S, mlb)
            if timing:
                marks[3].record()
            K.kvq_decode_pv(c, cbV, logits, mlb, max_len, outs[i], part, S)
        else:
            if timing:
                marks[2].record()
                marks[3].record()
            if args.path == "fused":
                K.kvq_decode_attention_fused(c, cbK, cbV, qall[i, s], qpos[s], max_len, outs[i],
                                             dws, S)
            else:
                K.kvq_decode_attention(c, cbK, cbV, qall[i, s], qpos[s], max_len, outs[i], dws, S)
        if timing:
            marks[4].record()
        return marks

    # ---- the whole step (every layer's append + attention) replayed as one CUDA graph
    appended = [0] * R  # tokens appended so far to each replica's caches

    def step_record(s, r, qp):
        """Packed kvq_step input record: per layer k, v, q (fp16 bytes), then qpos (int32 [B],
        padded to 16 bytes)."""
        parts = []
        for i in range(r * layers, (r + 1) * layers):
            parts += [knew[i, s].reshape(-1).view(torch.uint8),
                      vnew[i, s].reshape(-1).view(torch.uint8),
                      qall[i, s].reshape(-1).view(torch.uint8)]
        qp_t = torch.zeros((w.B * 4 + 15) // 16 * 4, dtype=torch.int32, device=dev)
        qp_t[:w.B] = qp
        parts.append(qp_t.view(torch.uint8))
        return torch.cat(parts)

    graph = None
    if use_graph:
        g_max_len = T0 + graph_steps + steps_total + e2e_steps  # bounds every graph launch
        g_in = torch.empty(K.kvq_step_input_bytes(cfg, layers, 1), dtype=torch.uint8, device=dev)
        g_ws = torch.empty(K.kvq_step_workspace(cfg, 1, g_max_len, S,
                                                1 if args.path == "fused" else 0),
                           dtype=torch.uint8, device=dev)
        gsteps = [K.kvq_step_create(cfg, caches[r * layers:(r + 1) * layers],
                                    [cb[0] for cb in cbs[r * layers:(r + 1) * layers]],
                                    [cb[1] for cb in cbs[r * layers:(r + 1) * layers]], 1,
                                    g_max_len, g_in, outs[r * layers:(r + 1) * layers], g_ws, S,
                                    1 if args.path == "fused" else 0)
                  for r in range(R)]
        # the launch schedule: warm-up launches every replica per step, a timed step one
        plan = [(s, r) for s in range(args.warmup) for r in range(R)] + [
            (s, s % R) for s in range(args.warmup, steps_total)]
        recs, g_tok = [], []
        for s, r in plan:
            recs.append(step_record(s, r, pos0 + appended[r]))
            appended[r] += 1
            g_tok.append(T0 + appended[r])
        recs = torch.stack(recs)
        n_warm = args.warmup * R
        torch.cuda.synchronize()
        for j in range(n_warm):
            K.kvq_step_launch(gsteps[plan[j][1]], recs[j])
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(dev.index) as clk_g:
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record()
            for j in range(n_warm, len(plan)):
                K.kvq_step_launch(gsteps[plan[j][1]], recs[j])
            g1.record()
            torch.cuda.synchronize()
        g_ms = g0.elapsed_time(g1)
        for c in caches:
            if K.kvq_get_status(c):
                raise RuntimeError("cache status set after the graph-replayed steps")
        graph = {"ms": g_ms, "tokens": w.B * layers * sum(g_tok[n_warm:]), "clk": clk_g}
        del recs

    # ---- the same step as per-layer calls, with events between the kernels of each layer
    # warm-up
    for s in range(args.warmup):
        for i in range(nL):
            layer_step(i, s, False)
        for r in range(R):
            appended[r] += 1
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    marks = []
    with ClockSampler(dev.index) as clk:
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t_start.record()
        m_tok, m_len = [], []
        for s in range(args.warmup, steps_total):
            rep = s % R
            for i in range(rep * layers, (rep + 1) * layers):
                marks.append(layer_step(i, s, True))
            appended[rep] += 1  # the sequence grows (on the last rank when sharded)
            m_len.append(T0 + appended[rep] if appends_here else T0)
            m_tok.append(w.B * layers * (shard_n * T0 + appended[rep]) *
                         (1 if sharded else world))
        t_end.record()
        torch.cuda.synchronize()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    if world > 1:
        dist.barrier()
    n_layer_steps = len(marks)
    # KV tokens attended over the whole job: replicas, each rank its own sequence; sharded,
    # one sequence of N T0 + appended tokens
    m_value = sum(m_tok) / (elapsed_ms / 1e3)
    if graph is not None:
        graph["ms"] = max_over_ranks(graph["ms"], world, dev)
        value = graph["tokens"] * world / (graph["ms"] / 1e3)
        ms_per_step = graph["ms"] / args.steps
    else:
        value, ms_per_step = m_value, elapsed_ms / args.steps
    # per-kernel times
    t_app = sum(m[0].elapsed_time(m[1]) for m in marks)
    t_qk = sum(m[1].elapsed_time(m[2]) for m in marks)
    t_merge = sum(m[2].elapsed_time(m[3]) for m in marks)
    t_pv = sum(m[3].elapsed_time(m[4]) for m in marks)
    Tmid = int(round(statistics.mean(m_len)))  # this rank's cache length, mid-region
    bm = bytes_model(w, Tmid, kcount, vcount, "one-call" if sharded else args.path)
    hbm, peak_kind = peaks()
    if args.path == "split" and not sharded:
        kernels = {"k_qk": (t_qk, bm["qk"], "kvq_decode.cu"), "k_pv": (t_pv, bm["pv"], "kvq_decode.cu")}
    else:
        kernels = {"k_attn": (t_pv, bm["attn"], "kvq_decode.cu")}
    dom = max(kernels, key=lambda k: kernels[k][0])
    dom_ms = kernels[dom][0] / n_layer_steps
    dom_bytes = kernels[dom][1]
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    step_attn_ms = (t_qk + t_merge + t_pv) / n_layer_steps
    attn_gbs = bm["total"] / (step_attn_ms / 1e3) / 1e9

    # ---- end-to-end through the public API with host buffers: every step copies its inputs
    # from pinned host memory and reads its outputs back (replica 0, fresh positions)
    e2e_app = []
    for j in range(e2e_steps):
        appended[0] += 1
        e2e_app.append(appended[0])
    e2e_tokens = w.B * layers * sum(shard_n * T0 + a for a in e2e_app) * (1 if sharded else world)
    h_out = torch.empty((layers, w.B, w.Hq, w.D), dtype=torch.float32).pin_memory()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph is not None:
        h_rec = torch.stack([step_record(args.warmup + j, 0, pos0 + a - 1)
                             for j, a in enumerate(e2e_app)]).cpu().pin_memory()
        h2d = h_rec[0].numel()
        d2h = h_out.numel() * 4
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e_s.record()
        for j in range(e2e_steps):
            K.kvq_step_launch(gsteps[0], h_rec[j])
            h_out.copy_(outs[:layers], non_blocking=True)
        e_e.record()
        torch.cuda.synchronize()
    else:
        h_q = torch.empty_like(qall, device="cpu").pin_memory()
        h_k = torch.empty_like(knew, device="cpu").pin_memory()
        h_v = torch.empty_like(vnew, device="cpu").pin_memory()
        h_q.copy_(qall)
        h_k.copy_(knew)
        h_v.copy_(vnew)
        d_q = torch.empty((layers, w.B, w.Hq, w.D), dtype=torch.float16, device=dev)
        d_k = torch.empty((layers, w.B, 1, w.Hkv, w.D), dtype=torch.float16, device=dev)
        d_v = torch.empty_like(d_k)
        qpos_e2e = torch.tensor([[pos0 + a - 1] * w.B for a in e2e_app], dtype=torch.int32,
                                device=dev)
        h2d = (d_q.numel() + d_k.numel() + d_v.numel()) * 2
        d2h = h_out.numel() * 4
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e_s.record()
        for j in range(e2e_steps):
            s = args.warmup + j
            ml_len = T0 + e2e_app[j] if appends_here else T0
            d_q.copy_(h_q[:layers, s], non_blocking=True)
            d_k.copy_(h_k[:layers, s], non_blocking=True)
            d_v.copy_(h_v[:layers, s], non_blocking=True)
            for i in range(layers):
                c = caches[i]
                if appends_here:
                    K.kvq_quantize_append(c, cbs[i][0], cbs[i][1], d_k[i], d_v[i], 1, None, 0,
                                          aws)
                if sharded:
                    sdec(c, cbs[i][0], cbs[i][1], d_q[i], qpos_e2e[j], ml_len, t_base, outs[i],
                         dws, S)
                elif args.path == "split":
                    K.kvq_decode_qk(c, cbs[i][0], d_q[i], qpos_e2e[j], ml_len, logits, stats, S,
                                    qkws)
                    K.kvq_softmax_merge(cfg, stats, S, mlb)
                    K.kvq_decode_pv(c, cbs[i][1], logits, mlb, ml_len, outs[i], part, S)
                elif args.path == "fused":
                    K.kvq_decode_attention_fused(c, cbs[i][0], cbs[i][1], d_q[i], qpos_e2e[j],
                                                 ml_len, outs[i], dws, S)
                else:
                    K.kvq_decode_attention(c, cbs[i][0], cbs[i][1], d_q[i], qpos_e2e[j], ml_len,
                                           outs[i], dws, S)
            h_out.copy_(outs[:layers], non_blocking=True)
        e_e.record()
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_s.elapsed_time(e_e), world, dev)
    e2e_value = e2e_tokens / (e2e_ms / 1e3)
    if graph is not None:
        for st in gsteps:
            K.kvq_step_destroy(st)

    # ---- uncompressed fp16 comparison kernel on one layer (last staged K/V)
    fp16 = None
    if not args.no_fp16:
        lens = torch.full((w.B,), T0, dtype=torch.int32, device=dev)
        fws = torch.empty(K.kvq_decode_workspace(cfg, T0, S), dtype=torch.uint8, device=dev)
        fout = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device=dev)
        qp0 = torch.full((w.B,), T0, dtype=torch.int32, device=dev)
        for _ in range(3):
            K.kvq_fp16_decode_attention(cfg, kstage, vstage, T0, lens, qall[0, 0], qp0, T0, fout,
                                        fws, S)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nrep = 5
        f0.record()
        for _ in range(nrep):
            K.kvq_fp16_decode_attention(cfg, kstage, vstage, T0, lens, qall[0, 0], qp0, T0, fout,
                                        fws, S)
        f1.record()
        torch.cuda.synchronize()
        fms = f0.elapsed_time(f1) / nrep
        fbytes = 2 * w.B * T0 * w.Hkv * w.D * 2
        f_gbs = fbytes / (fms / 1e3) / 1e9
        hbm_peak = peaks()[0]
        # the ratio is quoted only next to the fp16 kernel's own fraction of peak: a slow fp16
        # kernel would inflate it; the fp16 cache's time at peak bandwidth bounds it honestly
        fp16 = {"ms_per_layer": fms, "GB/s": f_gbs, "frac_of_peak": f_gbs / hbm_peak,
                "kv_tokens_per_s": w.B * T0 / (fms / 1e3),
                "quantized_ms_per_layer": step_attn_ms,
                "speedup_quantized_vs_fp16": fms / step_attn_ms,
                "speedup_vs_fp16_at_peak": (fbytes / (hbm_peak * 1e9) * 1e3) / step_attn_ms,
                "layers_timed": 1}

    # ---- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, smp = cpu_oracle_sample(w)
        cpu = {"value": v_cpu, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": smp, "extrapolated": "KV tokens/s of a sampled slice (one layer, "
               "1,024 tokens), not a run of the whole workload"}

    if rank != 0:
        return 0
    # append of one token: the short-append kernel (up to 32 kv heads), else begin, statistics,
    # scan, write, final; split kernels: qk (tables, qk, key outliers, split stats), merge, pv
    # (pv, value outliers, split sum); fused: tables, fused kernel, merge; sharded: the split
    # kernels and the conversion to a partial, then one merge of the gathered partials.  The
    # graph replays exactly these launches.
    fused_path = args.path == "fused" and not sharded
    launches_per_layer_step = ((1 if w.Hkv <= 32 else 5) if appends_here else 0) + (
        3 if fused_path else 8) + (2 if sharded else 0)
    per_layer_calls = {"value": m_value, "ms_per_step": elapsed_ms / args.steps,
                       "clocks": clk.summary()}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded Philox4x32-10; LLaMA-7B-shaped K/V distributions)",
        "config": {"workload": w.name, "layers": layers, "B": w.B, "q_heads": w.Hq,
                   "kv_heads": w.Hkv, "head_dim": w.D, "T_cached": T0, "bits": w.bits,
                   "outlier_frac": w.f, "rope_theta": w.rope_theta,
                   "path": "sharded (partial + all-gather + merge)" if sharded else args.path,
                   "splits": S, "cache_replicas": R,
                   "step": ("one CUDA graph per step: every layer's append + attention "
                            "(kvq_step_create / kvq_step_launch; the step's packed inputs "
                            "copied in by each launch)") if graph is not None
                           else "per-layer calls",
                   "parallelism": (f"token-sharded x{world}: one sequence of {shard_n * T0} "
                                   "tokens, rank r holding [r T, (r+1) T)") if sharded
                                  else (f"replicas x{world}" if world > 1 else "1 GPU"),
                   "l2": f"inputs {one_cache_bytes * R / 1e9:.1f} GB > 126 MB L2, not flushed"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm,
                     "unit": "GB/s", "frac": achieved / hbm, "peak_source": peak_kind,
                     "traffic": traffic_for(dom, Tmid),
                     "algorithmic_bytes_per_launch": dom_bytes,
                     "avg_launch_ms": dom_ms},
        "attention_step": {"ms_per_layer": step_attn_ms, "GB/s": attn_gbs,
                           "frac_of_peak": attn_gbs / hbm, "bytes_per_layer": bm["total"]},
        "kernels_ms_per_layer": {"append": t_app / n_layer_steps, "qk": t_qk / n_layer_steps,
                                 "merge": t_merge / n_layer_steps, "pv": t_pv / n_layer_steps},
        "prefill": {"ms_per_layer": statistics.median(prefill_ms), "tokens": T0,
                    "setup_s": setup_s},
        "outliers_per_layer": {"k": kcount, "v": vcount},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "fp16_attention": fp16,
        "cpu_baseline": cpu,
        "per_layer_calls": per_layer_calls if graph is not None else None,
        "gpu_launches": launches_per_layer_step * n_layer_steps,
        "clocks": graph["clk"].summary() if graph is not None else clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        return run_kvq(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
