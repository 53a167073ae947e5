"""Shared helpers of the GPU-vs-oracle parity tests.

Gates (the benchmark specification): logits agree within max relative error
2e-2 per position (max |l_gpu - l_oracle| / max |l_oracle|); routing
indices, lock masks, argmax and sampled tokens agree bit for bit except where
the oracle's own decision margin is below 1e-3 (top-2 gap of the logits, of
the Gumbel keys, of the router logits among the first k + 1, |pmax - 0.9|,
|cumulative entropy - budget|, |mean entropy - stop threshold|).

A routing decision that legitimately differs at a near-tie sends that token
to another expert, so everything downstream of it for that canvas position
differs too.  Such positions are "tainted" from the layer of the excused
decision on: later decisions, logits and samples at a tainted position are
not compared (they are counted in the report).  Every other position must
meet all gates.
"""

from dataclasses import dataclass, field

import numpy as np
import torch

import synth
import oracle
from oracle import decode as OD
from oracle import sampler as OS

MARGIN = 1e-3
LOGIT_REL = 2e-2

TINY = dict(n_layers=2, d_model=256, n_q_heads=8, n_kv_heads=8, head_dim=32, n_experts=16, top_k=2,
            d_ff=512, vocab=4096)
LAYER1 = dict(n_layers=1, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=176, n_experts=128, top_k=8,
              d_ff=704, vocab=262144)
FULL = dict(LAYER1, n_layers=30)


@dataclass
class Report:
    steps: int = 0
    logit_rel: float = 0.0
    excused: dict = field(default_factory=dict)
    diverged_at: int = -1
    layer_err: list = field(default_factory=list)
    tainted: int = 0

    def excuse(self, what, n):
        if n:
            self.excused[what] = self.excused.get(what, 0) + int(n)


def logit_rel_err(gpu, ref):
    ref = np.asarray(ref, dtype=np.float64)
    gpu = np.asarray(gpu, dtype=np.float64)
    den = np.abs(ref).max(axis=-1)
    return float(np.max(np.abs(gpu - ref).max(axis=-1) / np.maximum(den, 1e-30)))


def compare_decisions(name, gpu, ref, margin, rep: Report, skip=None):
    """Bit-exact except where the oracle's margin < MARGIN or the position is
    in `skip` (same leading shape).  Returns the mask of excused mismatches."""
    gpu = np.asarray(gpu)
    ref = np.asarray(ref)
    mism = gpu != ref
    if skip is not None:
        sk = np.asarray(skip).reshape(np.asarray(skip).shape + (1,) * (mism.ndim - np.asarray(skip).ndim))
        mism = mism & ~np.broadcast_to(sk, mism.shape)
    excused = mism & (np.asarray(margin) < MARGIN)
    bad = mism & ~excused
    assert not bad.any(), f"{name}: {int(bad.sum())} mismatches outside the margin, " \
        f"first at {np.argwhere(bad)[0].tolist()}: gpu {gpu[bad][0]} oracle {ref[bad][0]}"
    rep.excuse(name, excused.sum())
    return excused


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


def _sampler(case: Case):
    kw = dict(lock_policy=OS.LOCK_PROB, lock_threshold=0.9, max_steps=max(case.steps, 1),
              stop_entropy=0.5, seed=1234)
    kw.update(case.sampler)
    return OS.SamplerConfig(**kw)


def run_case(case: Case, check_kv=True):
    """Run the case on both sides step by step and check every gate.
    Returns a Report."""
    import discrete_diffusion_moe_b200 as dg
    rep = Report()
    c = case.cfg
    V, d = c["vocab"], c["d_model"]
    ocfg = oracle.ModelConfig(**c, self_cond=case.self_cond)
    std = {synth.KIND_LM: case.lm_std} if case.lm_std else None
    W = oracle.Weights(ocfg, seed=0, std=std)
    c_max = case.ctx_len + 256
    okv = oracle.KVCache(ocfg, case.batch, c_max)
    ctx = synth.context_tokens(case.batch, case.ctx_len, case.ctx_seed, V)
    OD.encode_context(ocfg, W, okv, ctx)
    sc = _sampler(case)

    gcfg = dg.model_config(**c, self_cond=case.self_cond)
    model = dg.Model(gcfg, case.batch, seed=0, kind_std=std)
    gkv = dg.KVCache(gcfg, case.batch, c_max)
    model.encode(gkv, torch.from_numpy(ctx.astype(np.int32)).cuda())
    model.check_device()
    assert gkv.length == okv.length == case.ctx_len

    if check_kv:
        for l in range(c["n_layers"]):
            gk, gv = gkv.layer_kv(l)
            gk = gk[:, :, :case.ctx_len].float().cpu().numpy().transpose(0, 2, 1, 3)
            gv = gv[:, :, :case.ctx_len].float().cpu().numpy().transpose(0, 2, 1, 3)
            for g_, o_ in ((gk, okv.k[l][:, :case.ctx_len]), (gv, okv.v[l][:, :case.ctx_len])):
                err = np.abs(g_ - o_).max() / max(np.abs(o_).max(), 1e-30)
                assert err < LOGIT_REL, f"layer {l} KV cache differs: {err}"

    gcv = dg.Canvas(gcfg, case.batch)
    model.canvas_init(gcv, case.block, sc.seed)
    state = OD.new_state(OD.init_canvas(sc.seed, case.block, case.batch, 256, V), d)
    assert np.array_equal(gcv.tokens.cpu().numpy(), state.tokens), "canvas initialisation differs"

    gs = dg.sampler_config(lock_policy=0 if sc.lock_policy == OS.LOCK_PROB else 1,
                           lock_threshold=sc.lock_threshold, t_start=sc.t_start, t_end=sc.t_end,
                           max_steps=sc.max_steps, stop_entropy=sc.stop_entropy,
                           stop_require_stable_argmax=sc.stop_require_stable_argmax, seed=sc.seed)
    for s in range(case.steps):
        out = dg.StepOutputs(gcfg, case.batch, logits=True, routing=True, hidden=True)
        model.step(gkv, gcv, case.block, s, gs, out)
        model.check_device()
        o = OD.denoise_step(ocfg, W, okv, state, sc, case.block, s, record_routing=True)
        rep.steps += 1
        # residual stream after each layer (reported; the gates below decide)
        gh = out.hidden.cpu().numpy()
        rep.layer_err = [float(np.abs(gh[l + 1] - r[3].reshape(gh.shape[1:])).max()
                               / max(np.abs(r[3]).max(), 1e-30)) for l, r in enumerate(o.routing)]
        print(f"step {s}: residual-stream rel err per layer {['%.2e' % e for e in rep.layer_err]}")
        # routing per layer; an excused near-tie taints the position for later layers
        T = case.batch * 256
        gi = out.route_idx.cpu().numpy()
        taint = np.zeros(T, bool)
        for l, (idx, w, margin, _) in enumerate(o.routing):
            mrg = np.repeat(margin.reshape(T, 1), c["top_k"], axis=1)
            ex = compare_decisions(f"route[{l}]", gi[l].reshape(T, -1), idx.reshape(T, -1), mrg, rep,
                                   skip=taint)
            taint |= ex.any(axis=1)
        taint = taint.reshape(case.batch, 256)
        rep.tainted += int(taint.sum())
        ok = ~taint
        # logits of untainted positions
        gl = out.logits.cpu().numpy()
        if ok.any():
            rep.logit_rel = max(rep.logit_rel, logit_rel_err(gl[ok], o.logits[ok]))
        assert rep.logit_rel <= LOGIT_REL, f"step {s}: logits rel err {rep.logit_rel}"
        # statistics
        amax = out.argmax.cpu().numpy()
        samp = out.sample.cpu().numpy()
        ex_a = compare_decisions("argmax", amax, o.argmax, o.argmax_margin, rep, skip=taint)
        ex_s = compare_decisions("sample", samp, o.sample, o.sample_margin, rep, skip=taint)
        H = out.entropy.cpu().numpy()
        dH = np.abs(H - o.entropy)[ok]
        assert dH.size == 0 or dH.max() < 2e-2, f"entropy differs by {dH.max()}"
        pm = out.pmax.cpu().numpy()
        assert np.all((np.abs(pm - o.pmax) <= 2e-2 * o.pmax + 1e-9)[ok]), "pmax differs"
        mH = out.mean_entropy.cpu().numpy()
        assert np.abs(mH - o.mean_entropy).max() < 2e-2
        # lock mask and stop
        lk = out.lock.cpu().numpy().astype(bool)
        if sc.lock_policy == OS.LOCK_PROB:
            lmarg = np.abs(o.pmax - sc.lock_threshold)
            ex_l = compare_decisions("lock", lk, o.lock, lmarg, rep, skip=taint)
        else:
            # the cumulative rule couples all positions of a canvas: a canvas
            # with a tainted position is checked for validity instead
            lmarg = np.stack([cumsum_margin(o.entropy[b], sc.lock_threshold) for b in range(case.batch)])
            skip_c = np.repeat(taint.any(axis=1, keepdims=True), 256, axis=1)
            ex_l = compare_decisions("lock", lk, o.lock, lmarg, rep, skip=skip_c)
            ex_l = ex_l | skip_c
            for b in np.nonzero(taint.any(axis=1))[0]:
                assert H[b][lk[b]].sum() <= sc.lock_threshold + 1e-3, "cumulative lock exceeds its budget"
        compare_decisions("stop", out.stop.cpu().numpy().astype(bool), o.stop,
                          np.abs(o.mean_entropy - sc.stop_entropy), rep)
        # next canvas: identical wherever the decisions that feed it agree
        toks = gcv.tokens.cpu().numpy()
        diff = toks != o.tokens_out
        explained = ex_a | ex_s | ex_l | taint
        assert not (diff & ~explained).any(), f"step {s}: canvas differs without an excused decision"
        if diff.any() or not np.array_equal(gcv.done.cpu().numpy().astype(bool), state.done):
            rep.diverged_at = s
            break
        if case.self_cond:
            ge = gcv.sc_state.float().cpu().numpy()
            err = np.abs(ge - o.expected_emb)[ok].max() / max(np.abs(o.expected_emb).max(), 1e-30)
            assert err < 5e-2, f"step {s}: expected embedding differs by {err}"
        print(f"step {s}: tainted positions {int(taint.sum())}, excused {rep.excused}, "
              f"logit rel err {rep.logit_rel:.2e}")
    model.close()
    # near-tie routing flips must stay rare
    assert rep.tainted <= 0.1 * max(rep.steps, 1) * case.batch * 256, f"too many tainted positions: {rep}"
    return rep
