#!/usr/bin/env python
"""Benchmark of one DiffusionGemma denoising round (dg_denoise_step) on B200.

Workload (default, "full"): the full-size single step — 30 layers, d_model
2816, 16 query / 8 KV heads x 176, 128 experts top-8 (SwiGLU, ffn 704), vocab
262144, self-conditioning projection, random-init bf16 weights N(0, 0.02)
(seeded generator), a causally encoded context of 1024 random tokens, one
256-token canvas (batch 1).  A step is one dg_denoise_step: embedding and
self-conditioning input, 30 transformer layers, LM head with vocabulary
statistics and Gumbel sampling, expected embedding, canvas update.

Prints one JSON line (rank 0).  value = denoise steps/s summed over ranks
(replicas, one per GPU; no collective on the data path).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # full-size single step: 30 layers, self-conditioning, context 1024, batch 1
    "full": dict(cfg=dict(n_layers=30, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=176,
                          n_experts=128, top_k=8, d_ff=704, vocab=262144, self_cond=True),
                 ctx=1024, batch=1),
    # single-layer full-width step: context 2048, no self-conditioning
    "layer1": dict(cfg=dict(n_layers=1, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=176,
                            n_experts=128, top_k=8, d_ff=704, vocab=262144, self_cond=False),
                   ctx=2048, batch=1),
    # one full-width layer with a small vocabulary (1.9 GB of weights): the
    # workload for hardware-counter captures of the layer kernels
    "moe1": dict(cfg=dict(n_layers=1, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=176,
                          n_experts=128, top_k=8, d_ff=704, vocab=16384, self_cond=False),
                 ctx=1024, batch=1),
    # the same with the self-conditioning product and expected embedding (vocabulary 16384):
    # the workload for captures of the LM-head / expected-embedding kernels
    "moe1sc": dict(cfg=dict(n_layers=1, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=176,
                            n_experts=128, top_k=8, d_ff=704, vocab=16384, self_cond=True),
                   ctx=1024, batch=1),
    # one full-width layer with 16 experts and the full vocabulary, self-conditioning (3.3 GB of
    # weights): the workload for captures of the vocabulary-phase kernels at their real width
    "vocab1": dict(cfg=dict(n_layers=1, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=176,
                            n_experts=16, top_k=8, d_ff=704, vocab=262144, self_cond=True),
                   ctx=1024, batch=1),
    # tiny: 2 layers, d 256, 16 experts top-2, vocab 4096, context 64
    "tiny": dict(cfg=dict(n_layers=2, d_model=256, n_q_heads=8, n_kv_heads=8, head_dim=32, n_experts=16,
                          top_k=2, d_ff=512, vocab=4096, self_cond=False),
                 ctx=64, batch=1),
}
METRIC = "denoise steps/s on 256-token canvas"
UNIT = "steps/s"
CANVAS = 256
MAX_STEPS = 48
SEED = 7


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm_gbs=j["hbm_gbs"], bf16_tflops=j["bf16_tflops"],
                    bf16_tflops_sustained=j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def step_cost(cfg, batch, ctx, distinct_per_layer):
    """Algorithmic FLOPs and HBM bytes of one denoising round."""
    d, hd, Hq, Hkv, E, k, f, V, L = (cfg[x] for x in ("d_model", "head_dim", "n_q_heads", "n_kv_heads",
                                                      "n_experts", "top_k", "d_ff", "vocab", "n_layers"))
    T = batch * CANVAS
    qkv_rows = (Hq + 2 * Hkv) * hd
    keys = ctx + CANVAS
    flops = 0.0
    bytes_ = 0.0
    for l in range(L):
        macs = T * (qkv_rows * d + d * Hq * hd + E * d + k * 3 * f * d)
        flops += 2.0 * macs + 4.0 * batch * CANVAS * Hq * hd * keys
        bytes_ += 2.0 * (qkv_rows * d + d * Hq * hd + E * d)
        bytes_ += distinct_per_layer[l] * 3 * f * d * 2.0
        bytes_ += 2.0 * batch * Hkv * keys * hd * 2  # K and V of the context and the canvas
    flops += 2.0 * T * V * d  # LM head
    bytes_ += V * d * 2.0
    if cfg["self_cond"]:
        flops += 2.0 * T * V * d + 2.0 * T * d * d
        bytes_ += V * d * 2.0 + d * d * 2.0
    return flops, bytes_


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"dg_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            try:
                sm.append(float(r[1].split()[0]))
                smax.append(float(r[2].split()[0]))
            except (ValueError, IndexError):
                continue
            for nm, v in zip(names, r[5:9]):
                if "Active" in v and "Not" not in v:
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in ("discrete_diffusion_moe_b200/csrc/gemm_tc.cuh", "discrete_diffusion_moe_b200/csrc/gemm_pair.cuh",
                "discrete_diffusion_moe_b200/csrc/epilogues.cuh", "discrete_diffusion_moe_b200/csrc/common.cuh",
                "discrete_diffusion_moe_b200/csrc/moe_pair.cuh"):
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, distinct_mean):
    """DRAM bytes per launch of the dominant kernel, scaled from the committed
    ncu capture of one launch on the one-layer workload, or None when missing
    or taken on a different kernel source.  The capture's bytes beyond the
    launch's expert-independent part (the permuted inputs and the outputs of
    the same 256 canvas tokens) grow with the distinct experts the launch
    streams, so a full-size launch is that part plus the rest times the
    round's mean distinct experts per layer over the capture's count."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    j = json.load(open(p))
    e = j.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash() or not distinct_mean:
        return None
    measured = e["read_bytes"] + e["write_bytes"]
    fixed = e["fixed_bytes"]
    return fixed + (measured - fixed) * distinct_mean / e["distinct_experts"]


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, timed on a bounded sample of the workload

def oracle_setup(wl, threads):
    """The oracle's inputs for timing one step of the workload (generated, not
    timed: weights and tokens are inputs): the model, a context KV cache of the
    workload's length (synthetic keys / values, as the GPU's encode would
    leave), the canvas and its embedding."""
    import oracle
    import synth
    from oracle import decode as OD
    c = wl["cfg"]
    ocfg = oracle.ModelConfig(**c)
    W = oracle.Weights(ocfg, seed=0, threads=threads, keep_chunks=True)
    ctx = wl["ctx"]
    kv = oracle.KVCache(ocfg, 1, ctx + CANVAS)
    for l in range(c["n_layers"]):
        kv.k[l][:, :ctx] = synth.f32_tensor(ctx * c["n_kv_heads"] * c["head_dim"], 3, 900 + 2 * l, 1.0).reshape(
            1, ctx, c["n_kv_heads"], c["head_dim"])
        kv.v[l][:, :ctx] = synth.f32_tensor(ctx * c["n_kv_heads"] * c["head_dim"], 3, 901 + 2 * l, 1.0).reshape(
            1, ctx, c["n_kv_heads"], c["head_dim"])
    kv.length = ctx
    toks = OD.init_canvas(SEED, 0, 1, CANVAS, c["vocab"])
    x0 = W.emb_rows(toks).reshape(1, CANVAS, c["d_model"])
    return ocfg, W, kv, x0


def oracle_tail_sample(wl, W, x, threads, n_pos=8, chunk=16384):
    """Seconds of the oracle's vocabulary phase of one step, from timed
    samples: the LM head over one 16384-id block (x V / 16384), the statistics
    and Gumbel sample of n_pos positions (x 256 / n_pos) and the expected
    embedding over one 16384-id block (x V / 16384).  Returns (seconds, desc)."""
    import numpy as np
    import oracle
    import synth
    from oracle import sampler as OS
    from oracle.model import lm_logits
    c = wl["cfg"]
    vcfg = oracle.ModelConfig(**dict(c, n_layers=1, vocab=chunk))
    Wv = oracle.Weights(vcfg, seed=0, threads=threads, keep_chunks=True)
    Wv.lm_chunk(0, chunk)
    Wv.emb_chunk(0, chunk)
    t0 = time.perf_counter()
    lm_logits(vcfg, Wv, x.reshape(CANVAS, -1), chunk=chunk)
    t1 = time.perf_counter()
    rng_logits = synth.f32_tensor(n_pos * c["vocab"], 5, 902, 1.0).reshape(n_pos, c["vocab"])
    for i in range(n_pos):
        OS.position_stats(rng_logits[i])
        OS.position_sample(rng_logits[i], np.float32(1.25), SEED, 0, 0, 0, i)
        OS.selfcond_probs(rng_logits[i])
    t2 = time.perf_counter()
    t3 = t2
    if c["self_cond"]:
        p_all = np.full((CANVAS, chunk), 1.0 / c["vocab"])
        t2 = time.perf_counter()
        OS.expected_embedding(p_all, Wv, chunk=chunk)
        t3 = time.perf_counter()
    reps = c["vocab"] / chunk
    sec = (t1 - t0) * reps + (t2 - t1) * (CANVAS / n_pos) + (t3 - t2) * reps
    desc = (f"LM head over {chunk} of {c['vocab']} ids (x{reps:g}), statistics and Gumbel sample of {n_pos} of "
            f"256 positions (x{CANVAS // n_pos})" + (f", expected embedding over {chunk} ids (x{reps:g})"
                                                   if c["self_cond"] else ""))
    return sec, desc


def oracle_sample(wl, threads, distinct):
    """The oracle's seconds per step from timed samples: layer 0's attention
    block, router and experts timed separately (seconds per routed expert
    from its experts block), every layer costed as attention + router +
    (its measured distinct experts) x (seconds per expert), plus the timed
    vocabulary-phase samples.  `distinct`: experts per layer of the GPU's
    own round (None: a one-layer workload, whose layer 0 is timed whole).
    Returns (seconds per step, description, wall seconds)."""
    import numpy as np
    from oracle import model as OM
    c = wl["cfg"]
    w0 = time.perf_counter()
    ocfg, W, kv, x0 = oracle_setup(dict(wl, cfg=dict(c, n_layers=1)), threads)
    lw = W.layer(0)
    t0 = time.perf_counter()
    xm = OM.attention_block(ocfg, lw, x0, kv.k[0], kv.v[0], wl["ctx"], causal=False, append=False)
    t1 = time.perf_counter()
    OM.router_block(ocfg, lw, xm)
    t2 = time.perf_counter()
    x1, (idx, _, _, _) = OM.moe_block(ocfg, lw, xm)
    t3 = time.perf_counter()
    e0 = len(np.unique(np.asarray(idx)))
    t_attn, t_route = t1 - t0, t2 - t1
    t_exp = max(0.0, (t3 - t2) - t_route) / max(e0, 1)
    tail, tdesc = oracle_tail_sample(wl, W, x1, threads)
    if distinct is None:
        layers = t1 - t0 + t3 - t2
        desc = (f"oracle (numpy float64): the layer timed whole (attention {t_attn:.2f} s, router {t_route:.2f} s, "
                f"{e0} experts {t3 - t2 - t_route:.2f} s); {tdesc}; inputs generated outside the timing")
        return layers + tail, desc, time.perf_counter() - w0
    layers = sum(t_attn + t_route + e * t_exp for e in distinct)
    desc = (f"oracle (numpy float64): layer 0 timed (attention {t_attn:.2f} s, router {t_route:.2f} s, "
            f"{e0} experts {t3 - t2 - t_route:.2f} s); each of the {c['n_layers']} layers costed as attention + "
            f"router + its routed experts (the GPU round's distinct experts per layer, mean "
            f"{sum(distinct) / len(distinct):.1f}) x {t_exp:.3f} s; {tdesc}; inputs generated outside the timing")
    return layers + tail, desc, time.perf_counter() - w0


def oracle_cfg(c):
    import oracle
    return oracle.ModelConfig(**c)


def oracle_other_configs(cores, full_width=True):
    """The oracle on the smaller configurations, on the host cores: the tiny
    model's whole 4-round loop (seed 1234, lock above 0.9) on all cores and on
    one thread, the same loop on the plain C++ oracle (one thread), and one
    full-width layer at context 2048 (timed as the main line's sample, the
    layer whole).  Returns a list of cpu_baseline-style entries with their
    workload named."""
    from threadpoolctl import threadpool_limits
    from oracle import decode as OD
    from oracle import sampler as OS
    out = []
    wl = WORKLOADS["tiny"]
    c = wl["cfg"]
    for threads in (cores, 1):
        with threadpool_limits(limits=threads):
            ocfg, W, kv, _ = oracle_setup(wl, threads)
            state = OD.new_state(OD.init_canvas(1234, 0, 1, CANVAS, c["vocab"]), c["d_model"])
            sc = OS.SamplerConfig(max_steps=4, lock_threshold=0.9, seed=1234)
            W.layer(0)
            t0 = time.perf_counter()
            for s_ in range(4):
                OD.denoise_step(ocfg, W, kv, state, sc, 0, s_, keep_logits=False)
            sec = time.perf_counter() - t0
        out.append({"workload": "tiny 2-layer model (d 256, 16 experts top-2, vocab 4096), context 64, "
                                "the whole 4-round loop",
                    "value": 4.0 / sec, "unit": UNIT, "cores": threads, "kind": "oracle",
                    "sample": "every round of the loop computed and timed (weights generated outside the timing)"})
    # the plain C++ oracle (one thread, plain loops) on the same loop
    from oracle import cpp
    import synth
    m = cpp.Model(oracle_cfg(c), seed=0)
    cache = cpp.Cache(m.cfg, 1, wl["ctx"] + CANVAS)
    cpp.encode_context(m, cache, synth.context_tokens(1, wl["ctx"], 1234, c["vocab"]).astype("int64"))
    import numpy as np
    st = {"tokens": cpp.init_canvas(1234, 0, 1, CANVAS, c["vocab"]), "sc": np.zeros((1, CANVAS, c["d_model"])),
          "prev_argmax": np.full((1, CANVAS), -1, np.int64), "done": np.zeros(1, np.uint8),
          "locked": np.zeros((1, CANVAS), np.uint8)}
    samp = cpp.sampler(max_steps=4, lock_threshold=0.9, seed=1234)
    t0 = time.perf_counter()
    for s_ in range(4):
        cpp.denoise_step(m, cache, st, samp, 0, s_)
    sec = time.perf_counter() - t0
    out.append({"workload": "tiny 2-layer model (d 256, 16 experts top-2, vocab 4096), context 64, "
                            "the whole 4-round loop", "value": 4.0 / sec, "unit": UNIT, "cores": 1,
                "kind": "oracle (plain C++, double, plain loops)",
                "sample": "every round of the loop computed and timed (weights and the context encode outside "
                          "the timing)"})
    if full_width:
        with threadpool_limits(limits=cores):
            per_step, desc, _ = oracle_sample(WORKLOADS["layer1"], cores, distinct=None)
        out.append({"workload": "one full-width layer, context 2048, one round", "value": 1.0 / per_step,
                    "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc})
    return out


def time_steps(dg, model, kv, cv, samp, block, steps, warm, stream):
    """Mean ms of `steps` graph-replayed rounds after `warm` untimed ones."""
    model.canvas_init(cv, block, SEED)
    s_ = 0
    for _ in range(warm):
        model.step(kv, cv, block, s_, samp, graph=True)
        s_ += 1
    import torch
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        model.step(kv, cv, block, s_, samp, graph=True)
        s_ += 1
    e1.record(stream)
    torch.cuda.synchronize()
    model.check_device()
    return e0.elapsed_time(e1) / steps


def routed_distinct(dg, cfg, model, kv, cv, samp, B, n_layers):
    """Distinct experts per layer (over all canvases) of one more round."""
    import torch
    out = dg.StepOutputs(cfg, B, routing=True)
    model.canvas_init(cv, 1, SEED)
    model.step(kv, cv, 1, 0, samp, out)
    torch.cuda.synchronize()
    ridx = out.route_idx.cpu()
    return [int(torch.unique(ridx[l]).numel()) for l in range(n_layers)]


def line_roofline(cfg_d, B, ctx, distinct, ms, peaks):
    flops, nbytes = step_cost(cfg_d, B, ctx, distinct)
    t_f = flops / (peaks["bf16_tflops_sustained"] * 1e12)
    t_b = nbytes / (peaks["hbm_gbs"] * 1e9)
    return {"flops": flops, "bytes": nbytes, "t_ms": 1000 * max(t_f, t_b), "bound": "hbm" if t_b >= t_f else "tensor",
            "frac": max(t_f, t_b) / (ms / 1000.0)}


def other_configs(dg, synth, model, wl, rank, peaks, stream, steps=5, warm=3):
    """The benchmark's other configurations, measured in the same run:
    the single-layer full-width step (context 2048, one canvas), the batch x
    context sweep on the full-size model (B canvases of 256 tokens, B in
    {1, 2, 4, 8, 16}, each with its own causal context of C in {1024, 8192,
    32768} random tokens), and the router-load probe (every layer's router on
    N(0, 1) hidden states of 256 tokens)."""
    import torch
    res = {}
    samp = dg.sampler_config(max_steps=MAX_STEPS, stop_entropy=0.5, lock_threshold=0.9, seed=SEED + rank)
    samp_topk = dg.sampler_config(max_steps=MAX_STEPS, stop_entropy=0.5, lock_threshold=0.9, seed=SEED + rank,
                                  selfcond_topk=64)
    # single-layer full-width step
    w1 = WORKLOADS["layer1"]
    c1 = w1["cfg"]
    cfg1 = dg.model_config(**c1)
    m1 = dg.Model(cfg1, 1, seed=0)
    kv1 = dg.KVCache(cfg1, 1, w1["ctx"] + CANVAS)
    m1.encode(kv1, torch.from_numpy(synth.context_tokens(1, w1["ctx"], 1234 + rank, c1["vocab"])).cuda())
    cv1 = dg.Canvas(cfg1, 1)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ms_list = []
    for _ in range(steps):        # its 3 GB of weights fit in L2 twice over: flush L2 before each round
        flush.zero_()
        ms_list.append(time_steps(dg, m1, kv1, cv1, samp, 0, 1, warm if not ms_list else 0, stream))
    ms1 = statistics.median(ms_list)
    dist1 = routed_distinct(dg, cfg1, m1, kv1, cv1, samp, 1, 1)
    res["single_layer_full_width"] = {"workload": "1 layer, d 2816, 128 experts top-8, vocab 262144, context 2048, "
                                                  "one canvas; L2 flushed before each round",
                                      "ms_per_step": ms1, "steps_per_s": 1000.0 / ms1,
                                      "distinct_experts": dist1[0],
                                      "roofline": line_roofline(c1, 1, w1["ctx"], dist1, ms1, peaks)}
    m1.close()
    del m1, kv1, cv1, flush
    torch.cuda.empty_cache()
    # batch x context sweep on the full-size model (shared weights, one context per batch)
    c = wl["cfg"]
    cfg = dg.model_config(**c)
    sweep = []
    for B in (16, 8, 4, 2, 1):
        mb = dg.Model(cfg, B, weights_of=model)
        kvb = dg.KVCache(cfg, B, 32768 + CANVAS)
        mb.encode(kvb, torch.from_numpy(synth.context_tokens(B, 32768, 1234 + rank, c["vocab"])).cuda())
        mb.check_device()
        cvb = dg.Canvas(cfg, B)
        for C in (32768, 8192, 1024):   # descending: a round's canvas keys overwrite [C, C + 256)
            kvb.s.length = C
            ms = time_steps(dg, mb, kvb, cvb, samp, 0, steps, warm, stream)
            dist = routed_distinct(dg, cfg, mb, kvb, cvb, samp, B, c["n_layers"])
            sweep.append({"batch": B, "context": C, "ms_per_step": ms, "steps_per_s": 1000.0 / ms,
                          "canvas_tok_per_s": B * CANVAS * 1000.0 / ms,
                          "distinct_experts_per_layer": sum(dist) / len(dist),
                          "roofline": line_roofline(c, B, C, dist, ms, peaks)})
            if B == 16 and C == 1024 and c.get("self_cond"):
                # the high-batch variant: expected embedding over each position's 64 largest logits
                ms_k = time_steps(dg, mb, kvb, cvb, samp_topk, 0, steps, warm, stream)
                res["selfcond_topk_variant"] = {
                    "workload": "full-size model, 16 canvases, context 1024, self-conditioning input over the "
                                "64 largest logits of each position",
                    "k": 64, "ms_per_step": ms_k, "full_vocabulary_ms_per_step": ms,
                    "canvas_tok_per_s": B * CANVAS * 1000.0 / ms_k}
        mb.close()
        del mb, kvb, cvb
        torch.cuda.empty_cache()
    res["batch_context_sweep"] = sweep
    # router-load probe: N(0, 1) hidden states of 256 tokens through every layer's router
    x = torch.from_numpy(synth.f32_tensor(CANVAS * c["d_model"], 7, 905, 1.0).reshape(CANVAS, c["d_model"])).cuda()
    idx = torch.zeros(CANVAS, c["top_k"], dtype=torch.int32, device="cuda")
    per_layer = []
    for l in range(c["n_layers"]):
        model.router_probe(l, x, idx)
        cnt = torch.bincount(idx.reshape(-1).long(), minlength=c["n_experts"]).cpu()
        per_layer.append({"distinct": int((cnt > 0).sum()), "max_load": int(cnt.max()),
                          "cv": float(cnt.float().std() / cnt.float().mean())})
    model.check_device()
    res["router_load_probe"] = {
        "inputs": "256 hidden states N(0, 1) (seeded generator), each layer's RMSNorm + router + top-8",
        "distinct_experts_mean": sum(p["distinct"] for p in per_layer) / len(per_layer),
        "max_load_mean": sum(p["max_load"] for p in per_layer) / len(per_layer),
        "load_cv_mean": sum(p["cv"] for p in per_layer) / len(per_layer),
        "per_layer_distinct": [p["distinct"] for p in per_layer]}
    return res


def max_over_ranks(x, world):
    """The largest value of x over the ranks of the job (a job's time is its
    slowest rank's).  One process per GPU: NCCL tensors live on the rank's
    GPU, gloo (the CPU tests of this path) on the host."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def reference_arm(args, wl, rank, world):
    """The oracle on the host cores.  Each step times one real layer of the
    oracle's own chain for the workload's canvas (step i runs layer i mod L on
    the stream the previous step left) plus the vocabulary-phase samples; a
    step's value is the whole round costed from them: the layers timed so
    far, each untimed layer at the mean of the timed layers past layer 0,
    plus the vocabulary phase."""
    if rank != 0:
        return 0
    import numpy as np
    from oracle import model as OM
    cores = cpu_cores()
    c = wl["cfg"]
    L = c["n_layers"]
    ocfg, W, kv, x = oracle_setup(wl, cores)
    layer_s = {}
    times, sample_s = [], []
    tail, descs = oracle_tail_sample(wl, W, x, cores)   # the vocabulary phase, timed once
    for i in range(args.warmup + args.steps):
        l = i % L
        lw = W.layer(l)                       # generated outside the timing
        t0 = time.perf_counter()
        x, _ = OM.layer_forward(ocfg, lw, x, kv.k[l], kv.v[l], wl["ctx"], causal=False, append=False)
        t1 = time.perf_counter()
        layer_s[l] = t1 - t0
        deep = [v for k, v in layer_s.items() if k > 0] or [layer_s[0]]
        est = sum(layer_s.get(k, sum(deep) / len(deep)) for k in range(L)) + tail
        if i >= args.warmup:
            times.append(est)
            sample_s.append(t1 - t0)
    v = 1.0 / statistics.mean(times)
    desc = (f"oracle (numpy float64) on {cores} cores: one real layer of its own {L}-layer chain per step "
            f"(layers 0..{min(L, args.warmup + args.steps) - 1} timed), the untimed layers at the mean of the "
            f"timed ones past layer 0; once per run: {descs}; inputs generated outside the timing")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * statistics.mean(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args, wl, world),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
                             "sample_s_per_step": statistics.mean(sample_s),
                             "note": "ms_per_step is the whole round costed from the timed samples; the "
                                     "timed work per step is sample_s_per_step"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(args, wl, world):
    c = wl["cfg"]
    return {"workload": {"full": "full-size single step (30 layers, self-conditioning, context 1024, batch 1)",
                         "layer1": "single-layer full-width step (context 2048, batch 1)",
                         "moe1": "single full-width layer, vocabulary 16384 (context 1024, batch 1)",
                         "moe1sc": "single full-width layer, vocabulary 16384, self-conditioning (context 1024, batch 1)",
                         "vocab1": "single full-width layer with 16 experts, vocabulary 262144, self-conditioning "
                                   "(context 1024)",
                         "tiny": "tiny 2-layer step (context 64, batch 1)"}[args.workload],
            "n_layers": c["n_layers"], "d_model": c["d_model"], "heads": f"{c['n_q_heads']}q/{c['n_kv_heads']}kv x {c['head_dim']}",
            "experts": f"{c['n_experts']} top-{c['top_k']} ffn {c['d_ff']}", "vocab": c["vocab"],
            "self_cond": bool(c["self_cond"]), "context": wl["ctx"], "canvas": CANVAS, "batch_per_gpu": wl["batch"],
            "global_batch": wl["batch"] * world, "parallelism": f"replicas x{world}",
            "selfcond_topk": getattr(args, "selfcond_topk", 0),
            "l2": "inputs larger than L2: every step streams the full weight set (no flush needed)"
            if args.workload != "tiny" else "L2 flushed between steps (256 MiB write)",
            "weights": "random-init bf16, seeded generator, std 0.02"}


# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="full", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode-loop", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="canvases per GPU (0: the workload's)")
    ap.add_argument("--selfcond-topk", type=int, default=0,
                    help="time the round with the self-conditioning input over each position's K largest "
                         "logits (the high-batch variant); 0 = the method")
    args = ap.parse_args()
    wl = dict(WORKLOADS[args.workload])
    if args.batch > 0:
        wl["batch"] = args.batch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return reference_arm(args, wl, rank, world)
    if args.warmup < 3:
        args.warmup = 3
    if args.warmup + args.steps >= MAX_STEPS:
        args.steps = MAX_STEPS - 1 - args.warmup

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    import discrete_diffusion_moe_b200 as dg
    import synth

    c = wl["cfg"]
    B, ctx = wl["batch"], wl["ctx"]
    cfg = dg.model_config(**c)
    stream = torch.cuda.current_stream()
    model = dg.Model(cfg, B, seed=0)
    kv = dg.KVCache(cfg, B, ctx + CANVAS)
    ctx_tok = torch.from_numpy(synth.context_tokens(B, ctx, 1234 + rank, c["vocab"])).cuda()
    model.encode(kv, ctx_tok)
    cv = dg.Canvas(cfg, B)
    model.canvas_init(cv, 0, SEED + rank)
    samp = dg.sampler_config(max_steps=MAX_STEPS, stop_entropy=0.5, lock_threshold=0.9, seed=SEED + rank,
                             selfcond_topk=args.selfcond_topk)
    model.check_device()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if args.workload == "tiny" else None

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    step_i = 0
    for _ in range(args.warmup):
        model.step(kv, cv, 0, step_i, samp, graph=True)
        step_i += 1
    barrier()

    # ---- device-timed region (graph replays, no per-kernel events) -------------------
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        if flush is not None:
            flush.zero_()
        model.step(kv, cv, 0, step_i, samp, graph=True)
        step_i += 1
    e1.record(stream)
    barrier()
    clk = clocks.stop()
    model.check_device()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    ms_per_step = ms / args.steps
    value = world * args.steps / (ms / 1000.0)

    # ---- per-kernel durations: the same rounds as direct launches with CUDA events
    # around every profiled launch on its stream (a separate pass of K rounds)
    prof = dg.dg_profile()
    model.canvas_init(cv, 3, SEED + rank)
    for s_ in range(2):
        model.step(kv, cv, 3, s_, samp)
    barrier()
    dg.check(dg.lib.dg_profile_start(model.ctx))
    for s_ in range(args.steps):
        model.step(kv, cv, 3, 2 + s_, samp)
    barrier()
    dg.check(dg.lib.dg_profile_stop(model.ctx, ctypes.byref(prof)))
    model.check_device()
    graph_kernels = prof.launches_total  # kernels per round are the same in both passes

    # ---- routing of one more round: distinct experts per layer ----------------------
    out = dg.StepOutputs(cfg, B, routing=True)
    model.canvas_init(cv, 1, SEED + rank)
    model.step(kv, cv, 1, 0, samp, out)
    torch.cuda.synchronize()
    ridx = out.route_idx.cpu()
    distinct = [int(torch.unique(ridx[l]).numel()) for l in range(c["n_layers"])]

    # ---- the decode loop (dg_decode_block): 4 blocks of up to 48 steps after a
    # prompt of the workload's context length; block appends are included, the
    # prompt encode is not ------------------------------------------------------------
    loop = None
    if not args.no_decode_loop and B == 1:
        n_blocks = 4
        kv_l = dg.KVCache(cfg, 1, ctx + n_blocks * CANVAS)
        model.encode(kv_l, ctx_tok[:1].contiguous())
        cv_l = dg.Canvas(cfg, 1)
        toks = torch.zeros(1, CANVAS, dtype=torch.int32, device="cuda")
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        barrier()
        g0.record(stream)
        passes = 0
        block_stats = []
        for blk in range(n_blocks):
            st_, _ = model.decode_block(kv_l, cv_l, blk, samp, toks)
            passes += st_[0]
            block_stats.append(model.last_block_stats)
        g1.record(stream)
        barrier()
        model.check_device()
        ms_l = g0.elapsed_time(g1)
        loop = {"blocks": n_blocks, "max_steps_per_block": MAX_STEPS, "output_tokens": n_blocks * CANVAS,
                "denoise_passes": passes, "tokens_per_pass": n_blocks * CANVAS / passes, "ms": ms_l,
                "output_tok_per_s": n_blocks * CANVAS / (ms_l / 1000.0),
                "library_tokens_per_pass": [round(b["tokens_per_pass"], 3) for b in block_stats],
                "distinct_experts_per_layer": [round(sum(b["distinct_experts"]) / len(b["distinct_experts"]), 2)
                                               for b in block_stats],
                "note": "random-init weights: predictions stay near uniform, so no position locks and the "
                        "entropy stop never fires; every block runs its full step budget"}
        del kv_l

    # ---- end to end through the public API with host buffers -------------------------
    e2e = None
    if not args.no_e2e:
        # two sets of pinned host buffers: round s reads its inputs from one set
        # and returns its results into the other, which feeds round s + 1
        h_tok = [torch.empty(B, CANVAS, dtype=torch.int32).pin_memory() for _ in range(2)]
        h_sc = [torch.empty(B, CANVAS, c["d_model"], dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        h_tok[0].copy_(cv.tokens.cpu())
        h_sc[0].copy_(cv.sc_state.cpu())
        res = dg.StepOutputs(cfg, B)
        h_res = torch.empty_like(res.packed, device="cpu").pin_memory()
        n_e2e = max(3, min(args.steps, 10))
        h2d = h_tok[0].numel() * 4 + h_sc[0].numel() * 2
        d2h = h_tok[0].numel() * 4 + h_sc[0].numel() * 2 + res.packed.numel()
        model.canvas_init(cv, 2, SEED + rank)
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for s in range(n_e2e):
            a, b_ = s & 1, (s + 1) & 1
            cv.tokens.copy_(h_tok[a], non_blocking=True)
            cv.sc_state.copy_(h_sc[a], non_blocking=True)
            model.step(kv, cv, 2, s, samp, res, graph=True)
            h_tok[b_].copy_(cv.tokens, non_blocking=True)
            h_sc[b_].copy_(cv.sc_state, non_blocking=True)
            h_res.copy_(res.packed, non_blocking=True)
            stream.synchronize()  # the host reads the round's result
        f1.record(stream)
        barrier()
        ms_e2e = max_over_ranks(f0.elapsed_time(f1), world)
        e2e = {"value": world * n_e2e / (ms_e2e / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e2e}

    peaks = load_peaks()
    extra = None
    if not args.no_other_configs and args.workload == "full":
        extra = other_configs(dg, synth, model, wl, rank, peaks, stream)
    flops, nbytes = step_cost(c, B, ctx, distinct)
    t_roof = max(flops / (peaks["bf16_tflops_sustained"] * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9))
    # dominant kernel: grouped expert gate/up projection + SwiGLU (one launch per layer)
    gu = dg.DG_PROF_EXPERT_GATE_UP
    gu_ms = prof.ms[gu] / max(prof.launches[gu], 1)
    P = B * CANVAS * c["top_k"]
    avg_distinct = sum(distinct) / len(distinct)
    gu_bytes = avg_distinct * 2 * c["d_ff"] * c["d_model"] * 2 + P * c["d_model"] * 2 + P * c["d_ff"] * 2
    # with the fused expert kernel (no separate down launches) the launch also
    # streams the down weights, reads the SwiGLU outputs and writes the fp32 outputs
    fused = prof.launches[1] == 0
    if fused:
        gu_bytes += avg_distinct * c["d_model"] * c["d_ff"] * 2 + P * c["d_ff"] * 2 + P * c["d_model"] * 4
    achieved = gu_bytes / (gu_ms / 1000.0) / 1e9
    kinds = ["expert_gate_up", "expert_down", "lm_head", "attention", "dense_proj", "expected_emb"]
    breakdown = {kinds[i]: {"ms_per_step": prof.ms[i] / args.steps, "launches_per_step": prof.launches[i] / args.steps}
                 for i in range(6)}

    if rank == 0:
        cpu = None
        cpu_other = None
        if world == 1 and not args.no_cpu_baseline:
            cores = cpu_cores()
            per_step, desc, wall = oracle_sample(wl, threads=cores, distinct=distinct)
            cpu = {"value": 1.0 / per_step, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
                   "sample_wall_s": wall}
            if args.workload == "full" and not args.no_other_configs:
                try:
                    cpu_other = oracle_other_configs(cores)
                except Exception as e:  # reported; the main line stands without these figures
                    cpu_other = {"error": f"{type(e).__name__}: {e}"}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (random-init weights, random tokens)",
            "config": workload_config(args, wl, world),
            "decode_loop": loop,
            "output_tok_per_s": {"at_48_rounds_per_block": value * CANVAS / MAX_STEPS,
                                 "projected_at_12_rounds_per_block": value * CANVAS / 12},
            "step_roofline": {"flops": flops, "bytes": nbytes, "t_ms": 1000 * t_roof,
                              "frac": t_roof / (ms_per_step / 1000.0),
                              "bound": "hbm" if nbytes / (peaks["hbm_gbs"] * 1e9) >= flops / (peaks["bf16_tflops_sustained"] * 1e12) else "tensor",
                              "peaks": f"{peaks['source']}: {peaks['hbm_gbs']} GB/s, {peaks['bf16_tflops_sustained']} TF/s sustained bf16"},
            "roofline": {"kernel": ("moe_pair_kernel<EpiSwiGLU, EpiDown> (both grouped expert products in one launch, "
                                    "CTA pairs)" if fused else
                                    "gemm_pair_kernel<EpiSwiGLU> (grouped expert gate/up + SwiGLU, CTA pairs)"),
                         "bound": "hbm",
                         "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"],
                         "traffic": ncu_traffic("expert_block" if fused else "expert_gate_up", avg_distinct),
                         "bytes_per_launch": gu_bytes, "launch_ms": gu_ms,
                         "peak_source": f"{peaks['source']} (of {peaks['source']})"},
            "kernel_breakdown": breakdown,
            "distinct_experts_per_layer": avg_distinct,
            "gpu_launches": int(graph_kernels),
            "kernel_timing": "per-kernel CUDA events in a second pass of the same rounds as direct launches",
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "cpu_baseline_other_configs": cpu_other,
            "other_configs": extra,
        }
        print(json.dumps(line), flush=True)
    model.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
