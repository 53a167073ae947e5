"""Shared helpers of the GPU-vs-oracle parity tests.

Gates (the benchmark specification): logits agree within max relative error
2e-2 per position (max |l_gpu - l_oracle| / max |l_oracle|); routing
indices, lock masks, argmax and sampled tokens agree bit for bit, a mismatch
being allowed only where the oracle's margin of that decision is below 1e-3.

Every step is checked twice.

1. Stage by stage (teacher-forced).  The oracle runs each stage on the GPU's
   own input to that stage: the layer-0 input from the GPU's canvas and
   self-conditioning state; each layer's attention block from the GPU's
   residual stream entering the layer (and the GPU's context KV cache); each
   router and each expert block from the GPU's stream after that layer's
   attention; the LM head and its statistics from the GPU's final stream; the
   canvas update from the GPU's per-position statistics; the expected
   embedding from the GPU's logits.  Every decision of every position is
   compared bit for bit, and a mismatch is allowed only where the oracle's
   margin is below 1e-3 (MARGIN, in the decision's own units) -- the strict
   gate of the specification, with no allowance for the measured difference.

2. End to end within the step (free-running).  The oracle runs the whole
   step on its own numbers from the step's inputs (the GPU's canvas and
   self-conditioning state, the oracle's own encoding of the context).  The
   chain of bf16 roundings differs from the GPU's only by fp32-versus-float64
   rounding inside the stages, and one value that rounds the other way at a
   bf16 point moves everything downstream a little, so a decision whose
   margin is above 1e-3 can come out differently at the end of a long chain.
   Such a mismatch is accepted only because stage check 1 has shown that the
   GPU took the right decision on its own input; it is counted ("upstream")
   and capped at UPSTREAM_CAP of the decisions compared at that stage.
   Expert choices are discrete: one token sent to other experts changes its
   own stream at O(1), and through the next layer's attention -- a nearly
   uniform average over hundreds of keys, of size |v| / sqrt(n) -- every
   other token of its canvas by about 1 / sqrt(n) relative.  So the oracle's
   chain compares its own routing with the GPU's at every layer (counted as
   above) and then continues with the GPU's expert choices, which keeps every
   position of the step comparable to the end: logits within 2e-2 at all
   positions, decisions as above.

Both checks report what they compared; a step that compared nothing fails.
"""

from dataclasses import dataclass, field

import numpy as np
import torch

import synth
import oracle
from oracle import decode as OD
from oracle import model as OM
from oracle import sampler as OS
from oracle.numerics import f32_round

MARGIN = 1e-3
LOGIT_REL = 2e-2
ROUTER_REL = 2e-2
UPSTREAM_CAP = 0.15

TINY = dict(n_layers=2, d_model=256, n_q_heads=8, n_kv_heads=8, head_dim=32, n_experts=16, top_k=2,
            d_ff=512, vocab=4096)
LAYER1 = dict(n_layers=1, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=176, n_experts=128, top_k=8,
              d_ff=704, vocab=262144)
FULL = dict(LAYER1, n_layers=30)
CANVAS = 256


@dataclass
class Report:
    steps: int = 0
    # stage checks (teacher-forced)
    tf_decisions: int = 0         # decisions compared bit for bit
    tf_positions: int = 0         # positions whose logits were compared
    tf_logit_rel: float = 0.0
    tf_router_rel: float = 0.0
    tf_attn_rel: float = 0.0      # attention block output against the oracle on the same input
    tf_moe_rel: float = 0.0       # expert block output against the oracle on the same input
    excused: dict = field(default_factory=dict)   # mismatches at an oracle margin below MARGIN
    # end to end within the step (free-running)
    logit_rel: float = 0.0
    router_rel: float = 0.0
    upstream: dict = field(default_factory=dict)  # free-running mismatches at margins >= MARGIN
    compared_positions: int = 0   # positions compared at the end of the free-running chain
    tainted_tokens: int = 0       # context tokens left out of the KV-cache comparison
    layer_err: list = field(default_factory=list)

    def add(self, d, what, n):
        if n:
            d[what] = d.get(what, 0) + int(n)


def rel_err(gpu, ref):
    """max |gpu - ref| / max |ref| over the last axis, maximised over the rest."""
    ref = np.asarray(ref, dtype=np.float64)
    gpu = np.asarray(gpu, dtype=np.float64)
    den = np.abs(ref).max(axis=-1)
    return float(np.max(np.abs(gpu - ref).max(axis=-1) / np.maximum(den, 1e-30)))


logit_rel_err = rel_err


def compare_decisions(name, gpu, ref, margin, rep: Report, skip=None, upstream=False, explain=None):
    """Bit-exact except where the oracle's `margin` < MARGIN (counted in
    rep.excused) or, with `upstream`, free-running mismatches whose margin is
    below `explain` -- twice the measured difference of the very values that
    decision compares -- counted in rep.upstream and capped at UPSTREAM_CAP of
    the decisions compared.  gpu / ref share a leading shape with margin (and
    skip, explain); trailing axes (routing's k slots) count as one decision.
    Returns the mask of mismatched decisions."""
    gpu = np.asarray(gpu)
    ref = np.asarray(ref)
    margin = np.asarray(margin, dtype=np.float64)
    mism = gpu != ref
    while mism.ndim > margin.ndim:
        mism = mism.any(axis=-1)
    live = np.ones(mism.shape, bool) if skip is None else ~np.asarray(skip, bool)
    mism &= live
    excused = mism & (margin < MARGIN)
    rest = mism & ~excused
    n_live = int(live.sum())
    rep.add(rep.excused, name, excused.sum())
    if upstream:
        rep.add(rep.upstream, name, rest.sum())
        if explain is not None:
            bad = rest & (margin >= np.asarray(explain, dtype=np.float64))
            assert not bad.any(), f"{name}: {int(bad.sum())} mismatches at margins above twice the measured " \
                f"difference of their inputs, first at {np.argwhere(bad)[0].tolist()}"
        cap = max(1, int(UPSTREAM_CAP * n_live))
        assert rest.sum() <= cap, f"{name}: {int(rest.sum())} of {n_live} decisions differ at margins >= " \
            f"{MARGIN} (cap {cap})"
    else:
        rep.tf_decisions += n_live
        assert not rest.any(), f"{name}: {int(rest.sum())} mismatches at margins >= {MARGIN}, first at " \
            f"{np.argwhere(rest)[0].tolist()}: gpu {gpu[rest][0]} oracle {ref[rest][0]}"
    return mism


def top2_gap(v):
    v = np.asarray(v, dtype=np.float64)
    if v.shape[-1] < 2:
        return np.full(v.shape[:-1], np.inf)
    top = np.partition(v, -2, axis=-1)[..., -2:]
    return top[..., 1] - top[..., 0]


def cumsum_margin(H, threshold):
    """Per position: distance of its cumulative entropy (in (H, index) order)
    from the budget, and the gap to its neighbours in that order."""
    H = np.asarray(H, dtype=np.float64)
    order = np.argsort(H, kind="stable")
    cs = np.cumsum(H[order])
    m = np.empty_like(H)
    gaps = np.full(H.size, np.inf)
    d = np.diff(H[order])
    gaps[:-1] = np.minimum(gaps[:-1], d)
    gaps[1:] = np.minimum(gaps[1:], d)
    m[order] = np.minimum(np.abs(cs - threshold), gaps)
    return m


def lock_margin(sc, H, pmax):
    """Oracle margin of each position's lock decision [B, N]."""
    if sc.lock_policy == OS.LOCK_PROB:
        return np.abs(np.asarray(pmax, np.float64) - sc.lock_threshold)
    return np.stack([cumsum_margin(H[b], sc.lock_threshold) for b in range(H.shape[0])])


# ---------------------------------------------------------------------------
# stage checks on the GPU's own inputs


def gpu_layer_kv(gkv, l, L0):
    """Layer l's cached context keys / values [B, L0, Hkv, hd] (float32)."""
    k, v = gkv.layer_kv(l)
    k = k[:, :, :L0].float().cpu().numpy().transpose(0, 2, 1, 3)
    v = v[:, :, :L0].float().cpu().numpy().transpose(0, 2, 1, 3)
    return np.ascontiguousarray(k), np.ascontiguousarray(v)


def tf_embedding(rep, ocfg, W, tokens_in, sc_in, g0):
    """a1: the layer-0 input from the canvas the step consumed and the
    self-conditioning state it read."""
    B, N = tokens_in.shape
    x0 = W.emb_rows(tokens_in.reshape(-1)).reshape(B * N, -1)
    if ocfg.self_cond:
        x0 = x0 + f32_round(np.asarray(sc_in, np.float64).reshape(B * N, -1) @ W.sc().T)
    x0 = f32_round(x0)
    err = rel_err(g0.reshape(B * N, -1), x0)
    assert err <= 1e-5, f"layer-0 input rel err {err}"


def tf_router(rep, ocfg, lw, l, x_mid, gi, gr):
    """Layer l's router on the GPU's stream after the attention block:
    router logits within ROUTER_REL, expert choices bit for bit (strict).
    x_mid [T, d]; gi [T, k]; gr [T, E].  Returns the oracle's routing idx
    [T, k] and the mask of (excused) mismatches."""
    T = x_mid.shape[0]
    idx, w, margin, rlog = OM.router_block(ocfg, lw, x_mid.reshape(1, T, -1))
    rlog = rlog.reshape(T, -1)
    rel = rel_err(gr, rlog)
    rep.tf_router_rel = max(rep.tf_router_rel, rel)
    assert rel <= ROUTER_REL, f"layer {l}: router logits rel err {rel} on the GPU's input"
    mism = compare_decisions(f"route[{l}]", gi, idx.reshape(T, -1), margin.reshape(T), rep)
    return idx.reshape(T, -1), mism


def tf_layer_halves(rep, ocfg, lw, l, x_in, x_mid, x_out, gi, kk, vv, L0, B):
    """Layer l's attention block on the GPU's stream entering the layer (and
    the GPU's context cache kk / vv [B, L0, Hkv, hd]), compared with the GPU's
    stream after it; and its expert block on the GPU's stream after the
    attention block, compared (for tokens whose routing agrees) with the GPU's
    stream after the layer.  x_* [T, d] of B canvases."""
    T, d = x_in.shape
    n = T // B
    xm_o = OM.attention_block(ocfg, lw, x_in.reshape(B, n, d), kk, vv, L0, causal=False, append=False)
    err = rel_err(x_mid, xm_o.reshape(T, d))
    rep.tf_attn_rel = max(rep.tf_attn_rel, err)
    assert err <= LOGIT_REL, f"layer {l}: attention block rel err {err} on the GPU's input"
    xo_o, (idx, _, _, _) = OM.moe_block(ocfg, lw, x_mid.reshape(B, n, d))
    same = (np.asarray(gi).reshape(T, -1) == idx.reshape(T, -1)).all(axis=1)
    if same.any():
        err = rel_err(x_out[same], xo_o.reshape(T, d)[same])
        rep.tf_moe_rel = max(rep.tf_moe_rel, err)
        assert err <= LOGIT_REL, f"layer {l}: expert block rel err {err} on the GPU's input"


def tf_lm_head(rep, ocfg, W, sc, x_fin, gl, g_amax, g_samp, g_H, g_pm, block, step, rows, B):
    """Final norm + LM head on the GPU's final stream at `rows` (flat token
    indices): logits within LOGIT_REL, argmax and Gumbel sample bit for bit
    (strict), entropy and max probability within the bound the logit
    difference implies.  Returns the oracle's logits [len(rows), V]."""
    rows = np.asarray(rows)
    ref = OM.lm_logits(ocfg, W, np.asarray(x_fin, np.float64)[rows])
    gl = np.asarray(gl)
    rel = rel_err(gl, ref)
    rep.tf_logit_rel = max(rep.tf_logit_rel, rel)
    assert rel <= LOGIT_REL, f"LM head: logits rel err {rel} on the GPU's final stream"
    rep.tf_positions += len(rows)
    inv_t = OS.inv_temperature_f32(step, sc.max_steps, sc.t_start, sc.t_end)
    amax = np.empty(len(rows), np.int64)
    samp = np.empty(len(rows), np.int64)
    a_gap = np.empty(len(rows))
    s_gap = np.empty(len(rows))
    for i, t in enumerate(rows):
        b, p = divmod(int(t), CANVAS)
        H, pmax, amax[i], _ = OS.position_stats(ref[i])
        samp[i], keys = OS.position_sample(ref[i], inv_t, sc.seed, b, block, step, p)
        a_gap[i] = top2_gap(ref[i])
        s_gap[i] = top2_gap(keys)
        eps = float(np.abs(gl[i].astype(np.float64) - ref[i]).max())
        spread = np.abs(ref[i] - ref[i].mean()).max()
        # a logit change of eps moves H by at most 2 eps max|l - mean l| and pmax
        # by at most a factor e^(2 eps)
        assert abs(g_H[t] - H) <= 2 * eps * spread + 1e-4, ("entropy", int(t), g_H[t], H)
        assert abs(g_pm[t] - pmax) <= (np.exp(2 * eps) - 1) * pmax + 1e-6, ("pmax", int(t), g_pm[t], pmax)
    compare_decisions("argmax", np.asarray(g_amax)[rows], amax, a_gap, rep)
    compare_decisions("sample", np.asarray(g_samp)[rows], samp, s_gap, rep)
    return ref


def tf_update(rep, ocfg, sc, out, tokens_in, prev_argmax, done_in, tokens_out, block, step, locked_in=None,
              locked_out=None):
    """a9 on the GPU's per-position statistics: lock mask, stop flag, final
    flag and the next canvas (strict); with the persistent lock also the
    committed-position mask."""
    B = tokens_in.shape[0]
    state = OD.CanvasState(tokens=tokens_in.astype(np.int64).copy(), sc=np.zeros((B, CANVAS, 1)),
                           prev_argmax=prev_argmax.astype(np.int64).copy(), done=done_in.astype(bool).copy(),
                           locked=None if locked_in is None else locked_in.astype(bool).copy())
    H = out.entropy.cpu().numpy().astype(np.float64)
    pm = out.pmax.cpu().numpy().astype(np.float64)
    amax = out.argmax.cpu().numpy().astype(np.int64)
    samp = out.sample.cpu().numpy().astype(np.int64)
    meanH, stop, final, lock = OD.update_canvas(ocfg, sc, state, block, step, H, pm, amax, samp)
    lk = out.lock.cpu().numpy().astype(bool)
    ex_l = compare_decisions("lock", lk, lock, lock_margin(sc, H, pm), rep)
    live = ~done_in.astype(bool)
    ex_s = compare_decisions("stop", out.stop.cpu().numpy().astype(bool), stop,
                             np.abs(meanH - sc.stop_entropy), rep, skip=~live)
    compare_decisions("final", out.final_round.cpu().numpy().astype(bool), final,
                      np.where(ex_s, 0.0, np.inf), rep, skip=~live)
    diff = tokens_out != state.tokens
    explained = ex_l | ex_s[:, None]
    assert not (diff & ~explained).any(), f"step {step}: next canvas differs from the update rule"
    if getattr(sc, "persistent_lock", False) and locked_out is not None:
        assert not ((locked_out.astype(bool) != state.locked) & ~explained).any(), "committed positions differ"
    return meanH, stop, final, lock


def tf_expected_embedding(rep, W, gl, ge, rows):
    """a8 on the GPU's logits at `rows`: e = bf16(sum_v bf16(p_v) E_emb[v])
    with p the expected embedding's probabilities of the GPU's logits
    (oracle.sampler.selfcond_probs); within one bf16 ulp of e plus the fp32
    accumulation of a 262144-term sum (2^-8 of max |e|)."""
    probs = np.stack([OS.selfcond_probs(gl[i]) for i in range(len(rows))])
    e = OS.expected_embedding(probs, W)
    tol = 2.0 ** -7 * np.abs(e) + 2.0 ** -8 * np.abs(e).max()
    bad = np.abs(ge - e) > tol
    assert not bad.any(), f"expected embedding differs at {int(bad.sum())} elements"


def tf_expected_embedding_topk(rep, W, gl, ge, k):
    """a8's top-k variant on the GPU's logits: the K ids are chosen on the
    bf16 logits both sides store (ties to the lower id), so the set is exact;
    e within one bf16 ulp plus the rounding of each bf16 p_v (2^-8 of max |e|)."""
    e, _ = OS.expected_embedding_topk(gl, W, k)
    tol = 2.0 ** -7 * np.abs(e) + 2.0 ** -8 * np.abs(e).max()
    bad = np.abs(ge - e) > tol
    assert not bad.any(), f"top-{k} expected embedding differs at {int(bad.sum())} elements"


# ---------------------------------------------------------------------------
# one case: context encoding, canvas initialisation, then steps


@dataclass
class Case:
    cfg: dict
    self_cond: bool = False
    ctx_len: int = 64
    batch: int = 1
    steps: int = 1
    sampler: dict = field(default_factory=dict)
    lm_std: float = None
    ctx_seed: int = 1234
    block: int = 0
    ctx_split: int = 0      # > 0: the GPU encodes the context in two calls, split there
    prefill: int = 0        # the GPU context's prefill_tokens (encode passes of that many tokens)


def _sampler(case: Case):
    kw = dict(lock_policy=OS.LOCK_PROB, lock_threshold=0.9, max_steps=max(case.steps, 1),
              stop_entropy=0.5, seed=1234)
    kw.update(case.sampler)
    return OS.SamplerConfig(**kw)


def gpu_sampler(dg, sc):
    return dg.sampler_config(lock_policy=0 if sc.lock_policy == OS.LOCK_PROB else 1,
                             lock_threshold=sc.lock_threshold, t_start=sc.t_start, t_end=sc.t_end,
                             max_steps=sc.max_steps, stop_entropy=sc.stop_entropy,
                             stop_require_stable_argmax=sc.stop_require_stable_argmax, seed=sc.seed,
                             persistent_lock=sc.persistent_lock, selfcond_topk=sc.selfcond_topk)


def check_context_kv(rep, ocfg, gkv, okv, enc_rec, B, C):
    """The context KV cache written by the causal encode, every layer.  A
    context token whose expert choice sits within MARGIN of a tie in layer j
    may route differently on the two sides: its keys and values from layer
    j + 1 on are not compared, nor (causal attention) those of the later
    tokens of its canvas from layer j + 2 on."""
    L = ocfg.n_layers
    skip = np.zeros((L, B, C), bool)
    for j, (_, _, margin, _, _) in enumerate(enc_rec):
        near = np.asarray(margin).reshape(B, C) < MARGIN
        if j + 1 < L:
            skip[j + 1:] |= near
        if j + 2 < L:
            skip[j + 2:] |= np.maximum.accumulate(near, axis=1)
    rep.tainted_tokens += int(skip[-1].sum())
    for l in range(L):
        gk, gv = gpu_layer_kv(gkv, l, C)
        keep = ~skip[l]
        for g_, o_ in ((gk, okv.k[l][:, :C]), (gv, okv.v[l][:, :C])):
            err = np.abs(g_ - o_)[keep].max() / max(np.abs(o_).max(), 1e-30)
            assert err < LOGIT_REL, f"layer {l} KV cache differs: {err}"


def run_case(case: Case, check_kv=True, verbose=True):
    """Run the case on both sides step by step and check every gate (stage
    checks and the free-running chain of each step).  Returns a Report."""
    import discrete_diffusion_moe_b200 as dg
    rep = Report()
    c = case.cfg
    V, d, k = c["vocab"], c["d_model"], c["top_k"]
    L = c["n_layers"]
    ocfg = oracle.ModelConfig(**c, self_cond=case.self_cond)
    std = {synth.KIND_LM: case.lm_std} if case.lm_std else None
    W = oracle.Weights(ocfg, seed=0, std=std)
    c_max = case.ctx_len + 256
    okv = oracle.KVCache(ocfg, case.batch, c_max)
    ctx = synth.context_tokens(case.batch, case.ctx_len, case.ctx_seed, V)
    enc_rec = []
    OD.encode_context(ocfg, W, okv, ctx, record=enc_rec)
    sc = _sampler(case)

    gcfg = dg.model_config(**c, self_cond=case.self_cond)
    model = dg.Model(gcfg, case.batch, seed=0, kind_std=std, prefill_tokens=case.prefill)
    gkv = dg.KVCache(gcfg, case.batch, c_max)
    if case.ctx_split:
        model.encode(gkv, torch.from_numpy(np.ascontiguousarray(ctx[:, :case.ctx_split]).astype(np.int32)).cuda())
        model.encode(gkv, torch.from_numpy(np.ascontiguousarray(ctx[:, case.ctx_split:]).astype(np.int32)).cuda())
    else:
        model.encode(gkv, torch.from_numpy(ctx.astype(np.int32)).cuda())
    model.check_device()
    assert gkv.length == okv.length == case.ctx_len
    if check_kv and case.ctx_len > 0:
        check_context_kv(rep, ocfg, gkv, okv, enc_rec, case.batch, case.ctx_len)

    gcv = dg.Canvas(gcfg, case.batch)
    model.canvas_init(gcv, case.block, sc.seed)
    assert np.array_equal(gcv.tokens.cpu().numpy(), OD.init_canvas(sc.seed, case.block, case.batch, 256, V)), \
        "canvas initialisation differs"

    gs = gpu_sampler(dg, sc)
    B, T = case.batch, case.batch * 256
    g_kv_ctx = [gpu_layer_kv(gkv, l, case.ctx_len) for l in range(L)]   # the GPU's context cache
    for s in range(case.steps):
        # the step's inputs (the oracle's free-running chain starts from the same ones)
        tokens_in = gcv.tokens.cpu().numpy()
        prev_in = gcv.prev_argmax.cpu().numpy()
        done_in = gcv.done.cpu().numpy().astype(bool)
        locked_in = gcv.locked.cpu().numpy().astype(bool)
        sc_in = gcv.sc_state.float().cpu().numpy().astype(np.float64)
        out = dg.StepOutputs(gcfg, B, logits=True, routing=True, hidden=True)
        model.step(gkv, gcv, case.block, s, gs, out)
        model.check_device()
        rep.steps += 1
        gh = out.hidden.cpu().numpy().astype(np.float64)          # [L + 1, T, d]
        ga = out.hidden_attn.cpu().numpy().astype(np.float64)     # [L, T, d]
        gi = out.route_idx.cpu().numpy()                          # [L, T, k]
        gr = out.route_logits.cpu().numpy().astype(np.float64)    # [L, T, E]
        gl = out.logits.cpu().numpy().reshape(T, V)
        g_amax = out.argmax.cpu().numpy().reshape(T)
        g_samp = out.sample.cpu().numpy().reshape(T)
        g_H = out.entropy.cpu().numpy().astype(np.float64).reshape(T)
        g_pm = out.pmax.cpu().numpy().astype(np.float64).reshape(T)
        toks_out = gcv.tokens.cpu().numpy()

        # ---- 1. stage checks on the GPU's own inputs ------------------------------------
        tf_embedding(rep, ocfg, W, tokens_in, sc_in, gh[0])
        tf_route_mism = []
        for l in range(L):
            lw = W.layer(l)
            kk, vv = g_kv_ctx[l]
            _, mism = tf_router(rep, ocfg, lw, l, ga[l], gi[l], gr[l])
            tf_route_mism.append(mism)
            tf_layer_halves(rep, ocfg, lw, l, gh[l], ga[l], gh[l + 1], gi[l], kk, vv, case.ctx_len, B)
        tf_lm_head(rep, ocfg, W, sc, gh[L], gl, g_amax, g_samp, g_H, g_pm, case.block, s, np.arange(T), B)
        tf_update(rep, ocfg, sc, out, tokens_in, prev_in, done_in, toks_out, case.block, s, locked_in,
                  gcv.locked.cpu().numpy())
        if case.self_cond:
            live_rows = np.nonzero(np.repeat(~done_in, 256))[0]
            if live_rows.size:
                ge = gcv.sc_state.float().cpu().numpy().astype(np.float64).reshape(T, d)
                if sc.selfcond_topk > 0:
                    tf_expected_embedding_topk(rep, W, gl[live_rows], ge[live_rows], sc.selfcond_topk)
                else:
                    tf_expected_embedding(rep, W, gl[live_rows], ge[live_rows], live_rows)

        # ---- 2. the oracle's own chain from the step's inputs ---------------------------
        state = OD.CanvasState(tokens=tokens_in.astype(np.int64).copy(), sc=sc_in.copy(),
                               prev_argmax=prev_in.astype(np.int64).copy(), done=done_in.copy(),
                               locked=locked_in.copy())
        o = OD.denoise_step(ocfg, W, okv, state, sc, case.block, s, record_routing=True,
                            force_routing=lambda l: gi[l].reshape(B, 256, k))
        rep.layer_err = [rel_err(gh[l + 1], r[3].reshape(T, d)) for l, r in enumerate(o.routing)]
        for l, (idx, w, margin, _, rlog) in enumerate(o.routing):
            rlog = rlog.reshape(T, -1)
            rep.router_rel = max(rep.router_rel, rel_err(gr[l], rlog))
            assert rep.router_rel <= ROUTER_REL, f"step {s} layer {l}: router logits rel err {rep.router_rel}"
            compare_decisions(f"route[{l}]", gi[l], idx.reshape(T, -1), margin.reshape(T), rep, upstream=True,
                              explain=2 * np.abs(gr[l] - rlog).max(axis=1))
        rep.compared_positions += T
        ol = o.logits.reshape(T, V)
        rep.logit_rel = max(rep.logit_rel, rel_err(gl, ol))
        assert rep.logit_rel <= LOGIT_REL, f"step {s}: logits rel err {rep.logit_rel}"
        inv_t = float(OS.inv_temperature_f32(s, sc.max_steps, sc.t_start, sc.t_end))
        d_l = np.abs(gl.astype(np.float64) - ol).max(axis=1)
        m_a = compare_decisions("argmax", g_amax, o.argmax.reshape(T), o.argmax_margin.reshape(T), rep,
                                upstream=True, explain=2 * d_l)
        m_s = compare_decisions("sample", g_samp, o.sample.reshape(T), o.sample_margin.reshape(T), rep,
                                upstream=True, explain=2 * d_l * inv_t + 1e-5)
        lk = out.lock.cpu().numpy().astype(bool).reshape(T)
        if sc.lock_policy == OS.LOCK_PROB:
            lx = 2 * np.abs(g_pm - o.pmax.reshape(T))
        else:
            lx = np.repeat(2 * np.abs(g_H.reshape(B, 256) - o.entropy).sum(axis=1), 256)
        m_l = compare_decisions("lock", lk, o.lock.reshape(T), lock_margin(sc, o.entropy, o.pmax).reshape(T),
                                rep, upstream=True, explain=lx)
        mH = out.mean_entropy.cpu().numpy().astype(np.float64)
        m_st = compare_decisions("stop", out.stop.cpu().numpy().astype(bool), o.stop,
                                 np.abs(o.mean_entropy - sc.stop_entropy), rep, skip=done_in, upstream=True,
                                 explain=2 * np.abs(mH - o.mean_entropy))
        diff = (toks_out != o.tokens_out).reshape(T)
        explained = m_a | m_s | m_l | np.repeat(m_st, 256)
        assert not (diff & ~explained).any(), f"step {s}: canvas differs without a differing decision"
        if verbose:
            print(f"step {s}: stage checks: {rep.tf_decisions} decisions, attention rel {rep.tf_attn_rel:.1e}, "
                  f"router rel {rep.tf_router_rel:.1e}, experts rel {rep.tf_moe_rel:.1e}, logits rel "
                  f"{rep.tf_logit_rel:.1e}; end to end: {T} positions, logits rel {rep.logit_rel:.1e}, "
                  f"router rel {rep.router_rel:.1e}, residual rel per layer "
                  f"{['%.1e' % e for e in rep.layer_err]}; excused {rep.excused}; upstream {rep.upstream}")
    model.close()
    assert rep.tf_decisions > 0 and rep.tf_positions == case.steps * T and rep.compared_positions > 0, rep
    return rep
