"""Shared helpers of the GPU-vs-oracle parity tests.

Gates (the benchmark specification): logits agree within max relative error
2e-2 per position (max |l_gpu - l_oracle| / max |l_oracle|); routing
indices, lock masks, argmax and sampled tokens agree bit for bit except at
near-ties.

Near-ties.  The specification allows a mismatch where the oracle's top-2
margin is below 1e-3.  Both sides round to bf16 at the same points, but their
pre-rounding values differ at the level of fp32 versus float64 accumulation,
so a few elements round the other way; with a random-init model whose
attention is nearly uniform over thousands of keys, every attention output is
a heavily cancelling average and those single-ulp flips add up to router-logit
differences of order 1e-3 at full width.  A decision is therefore excused
exactly when its input difference could have flipped it: where the oracle's
margin is below max(1e-3, 2 * the measured |GPU - oracle| difference of the
quantities the decision compares at that position).  The measured differences
are themselves gated (logits and router logits within 2e-2 relative; entropy
and max probability within the bounds the logit difference implies).

Taint.  An excused routing flip sends that token to another expert, so its
hidden state then differs at O(1): the token is tainted from that layer on,
and through the next layer's bidirectional attention its whole canvas is
tainted from the following layer on.  Tainted positions / canvases are not
compared after the taint (counted in the report); everything before, and
every untainted canvas, must meet all gates.

Cases that scale the LM head up to make positions lock scale the logit-unit
1e-3 floor by the same factor (the specification's margin is stated for
weights N(0, 0.02), logits of order 1).
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
ROUTER_REL = 2e-2

TINY = dict(n_layers=2, d_model=256, n_q_heads=8, n_kv_heads=8, head_dim=32, n_experts=16, top_k=2,
            d_ff=512, vocab=4096)
LAYER1 = dict(n_layers=1, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=176, n_experts=128, top_k=8,
              d_ff=704, vocab=262144)
FULL = dict(LAYER1, n_layers=30)


@dataclass
class Report:
    steps: int = 0
    logit_rel: float = 0.0
    router_rel: float = 0.0
    excused: dict = field(default_factory=dict)
    diverged_at: int = -1
    layer_err: list = field(default_factory=list)
    tainted_tokens: int = 0
    tainted_canvases: int = 0
    compared_positions: int = 0

    def excuse(self, what, n):
        if n:
            self.excused[what] = self.excused.get(what, 0) + int(n)


def logit_rel_err(gpu, ref):
    ref = np.asarray(ref, dtype=np.float64)
    gpu = np.asarray(gpu, dtype=np.float64)
    den = np.abs(ref).max(axis=-1)
    return float(np.max(np.abs(gpu - ref).max(axis=-1) / np.maximum(den, 1e-30)))


def compare_decisions(name, gpu, ref, ratio, rep: Report, skip=None):
    """Bit-exact except where `ratio` (oracle margin / allowed bound) < 1 or
    the position is in `skip` (same leading shape).  Returns the mask of
    excused mismatches."""
    gpu = np.asarray(gpu)
    ref = np.asarray(ref)
    mism = gpu != ref
    if skip is not None:
        sk = np.asarray(skip)
        sk = sk.reshape(sk.shape + (1,) * (mism.ndim - sk.ndim))
        mism = mism & ~np.broadcast_to(sk, mism.shape)
    excused = mism & (np.asarray(ratio) < 1.0)
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


def run_case(case: Case, check_kv=True, verbose=True):
    """Run the case on both sides step by step and check every gate.
    Returns a Report."""
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
    floor = MARGIN * (case.lm_std or 0.02) / 0.02

    gcfg = dg.model_config(**c, self_cond=case.self_cond)
    model = dg.Model(gcfg, case.batch, seed=0, kind_std=std)
    gkv = dg.KVCache(gcfg, case.batch, c_max)
    model.encode(gkv, torch.from_numpy(ctx.astype(np.int32)).cuda())
    model.check_device()
    assert gkv.length == okv.length == case.ctx_len

    if check_kv and case.ctx_len > 0:
        # A context token whose expert choice sits within MARGIN of a tie in
        # layer j may route differently on the two sides: its keys and values
        # from layer j + 1 on are not compared, nor (causal attention) those of
        # the later tokens of its canvas from layer j + 2 on.
        Bc, Cc = case.batch, case.ctx_len
        skip = np.zeros((L, Bc, Cc), bool)
        for j, (_, _, margin, _, _) in enumerate(enc_rec):
            near = np.asarray(margin).reshape(Bc, Cc) < MARGIN
            if j + 1 < L:
                skip[j + 1:] |= near
            if j + 2 < L:
                skip[j + 2:] |= np.maximum.accumulate(near, axis=1)
        rep.tainted_tokens += int(skip[-1].sum())
        for l in range(L):
            gk, gv = gkv.layer_kv(l)
            gk = gk[:, :, :case.ctx_len].float().cpu().numpy().transpose(0, 2, 1, 3)
            gv = gv[:, :, :case.ctx_len].float().cpu().numpy().transpose(0, 2, 1, 3)
            keep = ~skip[l]
            for g_, o_ in ((gk, okv.k[l][:, :case.ctx_len]), (gv, okv.v[l][:, :case.ctx_len])):
                err = np.abs(g_ - o_)[keep].max() / max(np.abs(o_).max(), 1e-30)
                assert err < LOGIT_REL, f"layer {l} KV cache differs: {err}"

    gcv = dg.Canvas(gcfg, case.batch)
    model.canvas_init(gcv, case.block, sc.seed)
    state = OD.new_state(OD.init_canvas(sc.seed, case.block, case.batch, 256, V), d)
    assert np.array_equal(gcv.tokens.cpu().numpy(), state.tokens), "canvas initialisation differs"

    gs = dg.sampler_config(lock_policy=0 if sc.lock_policy == OS.LOCK_PROB else 1,
                           lock_threshold=sc.lock_threshold, t_start=sc.t_start, t_end=sc.t_end,
                           max_steps=sc.max_steps, stop_entropy=sc.stop_entropy,
                           stop_require_stable_argmax=sc.stop_require_stable_argmax, seed=sc.seed)
    B, T = case.batch, case.batch * 256
    for s in range(case.steps):
        out = dg.StepOutputs(gcfg, B, logits=True, routing=True, hidden=True)
        model.step(gkv, gcv, case.block, s, gs, out)
        model.check_device()
        o = OD.denoise_step(ocfg, W, okv, state, sc, case.block, s, record_routing=True)
        rep.steps += 1
        gh = out.hidden.cpu().numpy()
        rep.layer_err = [float(np.abs(gh[l + 1] - r[3].reshape(gh.shape[1:])).max()
                               / max(np.abs(r[3]).max(), 1e-30)) for l, r in enumerate(o.routing)]

        # ---- routing, layer by layer -------------------------------------------------
        gi = out.route_idx.cpu().numpy()
        gr = out.route_logits.cpu().numpy().astype(np.float64)
        tok_taint = np.zeros(T, bool)   # tokens whose expert choice differed at a near-tie
        can_taint = np.zeros(B, bool)   # canvases mixed with such a token by a later layer
        flipped = np.zeros(T, bool)
        for l, (idx, w, margin, _, rlog) in enumerate(o.routing):
            rlog = rlog.reshape(T, -1)
            live = ~(np.repeat(can_taint, 256) | tok_taint)
            flipped = np.zeros(T, bool)
            if live.any():
                err_r = np.abs(gr[l] - rlog)
                rel = err_r[live].max() / max(np.abs(rlog[live]).max(), 1e-30)
                rep.router_rel = max(rep.router_rel, float(rel))
                assert rel <= ROUTER_REL, f"step {s} layer {l}: router logits rel err {rel}"
                bound = np.maximum(floor, 2.0 * err_r.max(axis=1))
                ratio = np.repeat((margin.reshape(T) / bound)[:, None], k, axis=1)
                ex = compare_decisions(f"route[{l}]", gi[l].reshape(T, -1), idx.reshape(T, -1), ratio, rep,
                                       skip=~live)
                flipped = ex.any(axis=1)
            # a flipped token differs from here on; its canvas from the next layer on
            tok_taint |= flipped
            can_taint |= tok_taint.reshape(B, 256).any(axis=1)
        # after the last layer: tokens flipped at the last layer, and every
        # position of a canvas that had a flip at an earlier layer
        last_flip = flipped.reshape(B, 256)
        pre_last = (tok_taint.reshape(B, 256) & ~last_flip).any(axis=1)
        taint = last_flip.copy()
        taint[pre_last] = True
        rep.tainted_tokens += int(taint.sum())
        rep.tainted_canvases += int(pre_last.sum())
        ok = ~taint
        rep.compared_positions += int(ok.sum())

        # ---- logits and per-position statistics ---------------------------------------
        gl = out.logits.cpu().numpy()
        eps_l = np.abs(gl.astype(np.float64) - o.logits).max(axis=-1)    # per position
        if ok.any():
            rep.logit_rel = max(rep.logit_rel, logit_rel_err(gl[ok], o.logits[ok]))
        assert rep.logit_rel <= LOGIT_REL, f"step {s}: logits rel err {rep.logit_rel}"
        inv_t = float(OS.inv_temperature_f32(s, sc.max_steps, sc.t_start, sc.t_end))
        ex_a = compare_decisions("argmax", out.argmax.cpu().numpy(), o.argmax,
                                 o.argmax_margin / np.maximum(floor, 2 * eps_l), rep, skip=taint)
        ex_s = compare_decisions("sample", out.sample.cpu().numpy(), o.sample,
                                 o.sample_margin / np.maximum(floor, 2 * eps_l * inv_t + 1e-5), rep,
                                 skip=taint)
        H = out.entropy.cpu().numpy().astype(np.float64)
        pm = out.pmax.cpu().numpy().astype(np.float64)
        eps_H = np.abs(H - o.entropy)
        eps_p = np.abs(pm - o.pmax)
        # a logit change of eps moves H by at most 2 * eps * max|l - mean l| and
        # pmax by at most a factor e^(2 eps)
        spread = np.abs(o.logits - o.logits.mean(axis=-1, keepdims=True)).max(axis=-1)
        assert np.all((eps_H <= 2 * eps_l * spread + 1e-4)[ok]), f"entropy differs by {eps_H[ok].max()}"
        assert np.all((eps_p <= (np.exp(2 * eps_l) - 1) * o.pmax + 1e-6)[ok]), "max probability differs"
        mH = out.mean_entropy.cpu().numpy().astype(np.float64)
        eps_mH = np.abs(mH - o.mean_entropy)
        # ---- lock and stop ------------------------------------------------------------
        lk = out.lock.cpu().numpy().astype(bool)
        if sc.lock_policy == OS.LOCK_PROB:
            lratio = np.abs(o.pmax - sc.lock_threshold) / np.maximum(1e-3, 2 * eps_p)
            ex_l = compare_decisions("lock", lk, o.lock, lratio, rep, skip=taint)
        else:
            # the cumulative rule couples the positions of a canvas: a canvas with a
            # tainted position is checked for validity instead
            lratio = np.stack([cumsum_margin(o.entropy[b], sc.lock_threshold)
                               / max(1e-3, 2 * eps_H[b].sum()) for b in range(B)])
            skip_c = np.repeat(taint.any(axis=1, keepdims=True), 256, axis=1)
            ex_l = compare_decisions("lock", lk, o.lock, lratio, rep, skip=skip_c) | skip_c
            for b in np.nonzero(taint.any(axis=1))[0]:
                assert H[b][lk[b]].sum() <= sc.lock_threshold + 1e-3, "cumulative lock exceeds its budget"
        compare_decisions("stop", out.stop.cpu().numpy().astype(bool), o.stop,
                          np.abs(o.mean_entropy - sc.stop_entropy) / np.maximum(1e-3, 2 * eps_mH), rep,
                          skip=taint.any(axis=1))
        # ---- next canvas: identical wherever the decisions that feed it agree ----------
        toks = gcv.tokens.cpu().numpy()
        diff = toks != o.tokens_out
        explained = ex_a | ex_s | ex_l | taint
        assert not (diff & ~explained).any(), f"step {s}: canvas differs without an excused decision"
        if case.self_cond and ok.any():
            # e = sum_v p_v E_emb[v]: a logit difference eps moves p by at most
            # (e^(2 eps) - 1) in total variation; plus bf16 roundings of p and e
            ge = gcv.sc_state.float().cpu().numpy().astype(np.float64)
            emax = np.abs(W.emb_chunk(0, V)).max()
            tol = 2 * (np.exp(2 * eps_l) - 1)[..., None] * emax + 2.0 ** -7 * np.abs(o.expected_emb) \
                + 2.0 ** -8 * np.abs(o.expected_emb).max()
            bad = (np.abs(ge - o.expected_emb) > tol) & ok[..., None]
            assert not bad.any(), f"step {s}: expected embedding differs at {int(bad.sum())} elements"
        if verbose:
            print(f"step {s}: residual rel err per layer {['%.1e' % e for e in rep.layer_err]}; "
                  f"tainted tokens {int(taint.sum())} canvases {int(pre_last.sum())}; excused {rep.excused}; "
                  f"logit rel {rep.logit_rel:.2e} router rel {rep.router_rel:.2e}")
        if diff.any() or not np.array_equal(gcv.done.cpu().numpy().astype(bool), state.done):
            rep.diverged_at = s
            break
    model.close()
    return rep
