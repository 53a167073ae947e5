"""GPU-vs-oracle parity of the full-size model (30 layers, d 2816, 16 q / 8
kv heads x 176, 128 experts top-8, ffn 704, vocab 262144) at sizes the
oracle cannot run whole: every stage is checked teacher-forced, i.e. the
oracle consumes the GPU's own inputs to that stage.

  - layers: the residual stream entering sampled layers and the layer's KV
    cache (context keys) are taken from the GPU; the oracle runs that layer
    and its router logits, routing and output stream are compared;
  - LM head: the final stream of sampled positions -> logits, argmax, Gumbel
    sample, entropy and max probability;
  - canvas update: the GPU's per-position statistics of every position ->
    lock mask, stop flag and next canvas (bit for bit);
  - self-conditioning: the next step's input x0 = E_emb[canvas] + bf16(e) W_sc
    from the GPU's state e, and e itself at sampled positions.

Gates are those of tests/parity.py (logits and router logits within max
relative error 2e-2; integer decisions bit-exact except where the oracle's
margin is below max(1e-3, twice the measured input difference)).

Workloads: the full-size single step (context 1024, self-conditioning, two
steps), the batch / context sweep corners (16 canvases x 1024, 2 x 8192,
1 x 32768), and the full decode loop (1024-token prompt, 4 blocks of up to
48 steps, stop at mean entropy < 0.5, lock at max probability > 0.9, seed 7).
"""

import numpy as np
import pytest
import torch

import synth
import oracle
from oracle import decode as OD
from oracle import model as OM
from oracle import sampler as OS
from oracle.numerics import f32_round
from parity import FULL, LOGIT_REL, MARGIN, ROUTER_REL, Report, compare_decisions, logit_rel_err

pytestmark = pytest.mark.gpu

CANVAS = 256


@pytest.fixture(scope="module")
def full():
    """One full-size model (self-conditioning, up to 16 canvases) shared by the
    tests of this module, and the oracle's lazily generated weights."""
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(**FULL, self_cond=True)
    model = dg.Model(cfg, 16, seed=0)
    ocfg = oracle.ModelConfig(**FULL, self_cond=True)
    W = oracle.Weights(ocfg, seed=0)
    yield dg, cfg, model, ocfg, W
    model.close()


def _sampler(**kw):
    a = dict(lock_policy=OS.LOCK_PROB, lock_threshold=0.9, max_steps=48, stop_entropy=0.5, seed=7)
    a.update(kw)
    return OS.SamplerConfig(**a)


def _gpu_sampler(dg, sc):
    return dg.sampler_config(lock_policy=0 if sc.lock_policy == OS.LOCK_PROB else 1,
                             lock_threshold=sc.lock_threshold, t_start=sc.t_start, t_end=sc.t_end,
                             max_steps=sc.max_steps, stop_entropy=sc.stop_entropy,
                             stop_require_stable_argmax=sc.stop_require_stable_argmax, seed=sc.seed)


def _layer_kv(gkv, l, L0):
    """This layer's cached context keys / values [B, L0, Hkv, hd] (float32)."""
    k, v = gkv.layer_kv(l)
    k = k[:, :, :L0].float().cpu().numpy().transpose(0, 2, 1, 3)
    v = v[:, :, :L0].float().cpu().numpy().transpose(0, 2, 1, 3)
    return np.ascontiguousarray(k), np.ascontiguousarray(v)


def check_layers(rep, ocfg, W, gkv, out, L0, layers, canvases, B):
    """Teacher-forced layers: the oracle runs layer l on the GPU's input stream
    and KV cache of canvas b; router logits, routing and the output stream
    are compared."""
    d, k = ocfg.d_model, ocfg.top_k
    hid = out.hidden.cpu().numpy()                  # [L + 1, T, d]
    gi = out.route_idx.cpu().numpy()                # [L, T, k]
    gr = out.route_logits.cpu().numpy().astype(np.float64)
    for l in layers:
        kk, vv = _layer_kv(gkv, l, L0)
        for b in canvases:
            rows = slice(b * CANVAS, (b + 1) * CANVAS)
            x_in = hid[l, rows].astype(np.float64)[None]
            x_out, (idx, w, margin, rlog) = OM.layer_forward(ocfg, W.layer(l), x_in, kk[b:b + 1],
                                                             vv[b:b + 1], L0, causal=False, append=False)
            rlog = rlog.reshape(CANVAS, -1)
            err_r = np.abs(gr[l, rows] - rlog)
            rel = err_r.max() / max(np.abs(rlog).max(), 1e-30)
            rep.router_rel = max(rep.router_rel, float(rel))
            assert rel <= ROUTER_REL, f"layer {l} canvas {b}: router logits rel err {rel}"
            bound = np.maximum(MARGIN, 2.0 * err_r.max(axis=1))
            ratio = np.repeat((margin.reshape(CANVAS) / bound)[:, None], k, axis=1)
            ex = compare_decisions(f"route[{l}]", gi[l, rows], idx.reshape(CANVAS, k), ratio, rep)
            flipped = ex.any(axis=1)
            ref = x_out[0]
            ok = ~flipped
            got = hid[l + 1, rows].astype(np.float64)
            err = np.abs(got[ok] - ref[ok]).max() / max(np.abs(ref[ok]).max(), 1e-30)
            rep.layer_err.append((l, b, float(err)))
            assert err <= LOGIT_REL, f"layer {l} canvas {b}: output stream rel err {err}"
            rep.tainted_tokens += int(flipped.sum())


def check_lm_head(rep, ocfg, W, out, sc, block, step, positions, floor=MARGIN):
    """Teacher-forced LM head on the GPU's final stream at (canvas, position)
    pairs: logits, argmax, Gumbel sample, entropy and max probability."""
    L = ocfg.n_layers
    T = out.hidden.shape[1]
    hid = out.hidden[L].cpu().numpy().reshape(T, -1)
    rows = np.array([b * CANVAS + p for b, p in positions])
    ref = OM.lm_logits(ocfg, W, hid[rows].astype(np.float64))
    gl = out.logits.cpu().numpy().reshape(T, -1)[rows]
    rel = logit_rel_err(gl, ref)
    rep.logit_rel = max(rep.logit_rel, rel)
    assert rel <= LOGIT_REL, f"logits rel err {rel}"
    inv_t = OS.inv_temperature_f32(step, sc.max_steps, sc.t_start, sc.t_end)
    g_amax = out.argmax.cpu().numpy()
    g_samp = out.sample.cpu().numpy()
    g_H = out.entropy.cpu().numpy().astype(np.float64)
    g_pm = out.pmax.cpu().numpy().astype(np.float64)
    for i, (b, p) in enumerate(positions):
        eps = float(np.abs(gl[i].astype(np.float64) - ref[i]).max())
        H, pmax, amax, _ = OS.position_stats(ref[i])
        srt = np.sort(ref[i].astype(np.float64))
        compare_decisions("argmax", [g_amax[b, p]], [amax], [(srt[-1] - srt[-2]) / max(floor, 2 * eps)], rep)
        samp, keys = OS.position_sample(ref[i], inv_t, sc.seed, b, block, step, p)
        ks = np.sort(keys.astype(np.float64))
        compare_decisions("sample", [g_samp[b, p]], [samp],
                          [(ks[-1] - ks[-2]) / max(floor, 2 * eps * float(inv_t) + 1e-5)], rep)
        spread = np.abs(ref[i] - ref[i].mean()).max()
        assert abs(g_H[b, p] - H) <= 2 * eps * spread + 1e-4, (b, p, g_H[b, p], H)
        assert abs(g_pm[b, p] - pmax) <= (np.exp(2 * eps) - 1) * pmax + 1e-6, (b, p, g_pm[b, p], pmax)
        rep.compared_positions += 1


def check_update(rep, ocfg, sc, out, tokens_in, prev_argmax, done_in, tokens_out, block, step):
    """Teacher-forced canvas update of every position: the oracle's lock
    mask, stop flag and next canvas from the GPU's statistics."""
    B = tokens_in.shape[0]
    state = OD.CanvasState(tokens=tokens_in.astype(np.int64).copy(), sc=np.zeros((B, CANVAS, 1)),
                           prev_argmax=prev_argmax.astype(np.int64).copy(), done=done_in.astype(bool).copy())
    H = out.entropy.cpu().numpy().astype(np.float64)
    pm = out.pmax.cpu().numpy().astype(np.float64)
    amax = out.argmax.cpu().numpy().astype(np.int64)
    samp = out.sample.cpu().numpy().astype(np.int64)
    meanH, stop, final, lock = OD.update_canvas(ocfg, sc, state, block, step, H, pm, amax, samp)
    lk = out.lock.cpu().numpy().astype(bool)
    compare_decisions("lock", lk, lock, np.full(lk.shape, np.inf), rep)
    gm = out.mean_entropy.cpu().numpy().astype(np.float64)
    compare_decisions("stop", out.stop.cpu().numpy().astype(bool), stop,
                      np.abs(meanH - sc.stop_entropy) / np.maximum(1e-3, 2 * np.abs(gm - meanH)), rep)
    assert np.array_equal(tokens_out, state.tokens), "next canvas differs"
    return state


def _run_step(dg, cfg, model, gkv, gcv, gs, block, step, logits=True):
    B = gcv.tokens.shape[0]
    tokens_in = gcv.tokens.cpu().numpy()
    prev = gcv.prev_argmax.cpu().numpy()
    done = gcv.done.cpu().numpy()
    sc_in = gcv.sc_state.float().cpu().numpy()
    out = dg.StepOutputs(cfg, B, logits=logits, routing=logits, hidden=logits)
    model.step(gkv, gcv, block, step, gs, out)
    model.check_device()
    return out, tokens_in, prev, done, sc_in


def _encode(dg, cfg, model, B, C):
    gkv = dg.KVCache(cfg, B, C + CANVAS)
    ctx = synth.context_tokens(B, C, 1234, cfg.vocab)
    model.encode(gkv, torch.from_numpy(ctx.astype(np.int32)).cuda())
    model.check_device()
    assert gkv.length == C
    return gkv


def test_full_size_step_teacher_forced(full):
    """Full-size single step: 30 layers, self-conditioning, context 1024,
    one canvas; steps 0 and 1 (step 1 consumes step 0's expected embedding)."""
    dg, cfg, model, ocfg, W = full
    rep = Report()
    sc = _sampler(max_steps=48)
    gs = _gpu_sampler(dg, sc)
    gkv = _encode(dg, cfg, model, 1, 1024)
    gcv = dg.Canvas(cfg, 1)
    model.canvas_init(gcv, 0, sc.seed)
    assert np.array_equal(gcv.tokens.cpu().numpy(), OD.init_canvas(sc.seed, 0, 1, CANVAS, cfg.vocab))
    rng = np.random.default_rng(3)
    for step in range(2):
        out, tok_in, prev, done, sc_in = _run_step(dg, cfg, model, gkv, gcv, gs, 0, step)
        # a1: the layer-0 input from the canvas and the self-conditioning state
        x0 = W.emb_rows(tok_in[0])
        if step > 0:
            x0 = x0 + f32_round(sc_in[0].astype(np.float64) @ W.sc().T)
        x0 = f32_round(x0)
        g0 = out.hidden[0].cpu().numpy().astype(np.float64)
        err0 = np.abs(g0 - x0).max() / np.abs(x0).max()
        assert err0 <= 1e-5, f"step {step}: layer-0 input rel err {err0}"
        check_layers(rep, ocfg, W, gkv, out, 1024, [0, 14, 29] if step == 0 else [29], [0], 1)
        pos = [(0, int(p)) for p in rng.choice(CANVAS, 6, replace=False)]
        check_lm_head(rep, ocfg, W, out, sc, 0, step, pos)
        check_update(rep, ocfg, sc, out, tok_in, prev, done, gcv.tokens.cpu().numpy(), 0, step)
        # a8: the expected embedding at the sampled positions from the GPU's logits
        ge = gcv.sc_state.float().cpu().numpy().astype(np.float64)[0]
        gl = out.logits.cpu().numpy()[0]
        probs = np.stack([OS.position_stats(gl[p])[3] for _, p in pos])
        e = OS.expected_embedding(probs, W)
        got = ge[[p for _, p in pos]]
        tol = 2.0 ** -7 * np.abs(e) + 2.0 ** -8 * np.abs(e).max()
        assert (np.abs(got - e) <= tol).all(), f"step {step}: expected embedding differs"
    print(f"full-size step: {rep}")


@pytest.mark.parametrize("B,C", [(16, 1024), (2, 8192), (1, 32768)])
def test_batch_context_sweep_teacher_forced(full, B, C):
    """Batch / context sweep corners: B canvases, each with its own causal
    context of C random tokens, one step; layers 0 and 29 of the first and
    last canvas, LM head at sampled positions, canvas update of all."""
    dg, cfg, model, ocfg, W = full
    rep = Report()
    sc = _sampler(max_steps=48)
    gs = _gpu_sampler(dg, sc)
    gkv = _encode(dg, cfg, model, B, C)
    gcv = dg.Canvas(cfg, B)
    model.canvas_init(gcv, 0, sc.seed)
    out, tok_in, prev, done, _ = _run_step(dg, cfg, model, gkv, gcv, gs, 0, 0)
    canv = sorted({0, B - 1})
    check_layers(rep, ocfg, W, gkv, out, C, [0, 29], canv, B)
    rng = np.random.default_rng(B * 7 + C)
    pos = [(b, int(p)) for b in canv for p in rng.choice(CANVAS, 3, replace=False)]
    check_lm_head(rep, ocfg, W, out, sc, 0, 0, pos)
    check_update(rep, ocfg, sc, out, tok_in, prev, done, gcv.tokens.cpu().numpy(), 0, 0)
    print(f"B {B} C {C}: {rep}")


def test_full_decode_loop(full):
    """Full decode loop: 1024-token prompt, 4 consecutive blocks of up to 48
    steps (stop when mean entropy < 0.5, lock at max probability > 0.9,
    uniform re-noising, seed 7).  Block 0 runs step by step with every
    canvas update checked against the oracle on the GPU's statistics, and
    dg_decode_block on an identical context must produce the same block;
    blocks 1-3 go through dg_decode_block and grow the context by 256 each."""
    dg, cfg, model, ocfg, W = full
    rep = Report()
    sc = _sampler(max_steps=48, stop_entropy=0.5, lock_threshold=0.9, seed=7)
    gs = _gpu_sampler(dg, sc)
    prompt = synth.context_tokens(1, 1024, 1234, cfg.vocab)
    # block 0, step by step
    gkv = dg.KVCache(cfg, 1, 1024 + 4 * CANVAS)
    model.encode(gkv, torch.from_numpy(prompt.astype(np.int32)).cuda())
    gkv_len = gkv.length
    gcv = dg.Canvas(cfg, 1)
    model.canvas_init(gcv, 0, sc.seed)
    steps = 0
    for step in range(sc.max_steps):
        out, tok_in, prev, done, _ = _run_step(dg, cfg, model, gkv, gcv, gs, 0, step, logits=False)
        check_update(rep, ocfg, sc, out, tok_in, prev, done, gcv.tokens.cpu().numpy(), 0, step)
        steps += 1
        if gcv.done.cpu().numpy().all():
            break
    block0 = gcv.tokens.cpu().numpy().copy()
    assert gkv.length == gkv_len  # canvas passes do not grow the context
    # the same block through dg_decode_block on a fresh, identical context
    gkv2 = dg.KVCache(cfg, 1, 1024 + 4 * CANVAS)
    model.encode(gkv2, torch.from_numpy(prompt.astype(np.int32)).cuda())
    gcv2 = dg.Canvas(cfg, 1)
    toks = torch.zeros(1, CANVAS, dtype=torch.int32, device="cuda")
    st, rounds = model.decode_block(gkv2, gcv2, 0, gs, toks)
    model.check_device()
    assert st == [steps], (st, steps)
    assert np.array_equal(toks.cpu().numpy(), block0), "dg_decode_block differs from the step-by-step block"
    assert gkv2.length == 1024 + CANVAS
    total = steps
    for blk in range(1, 4):
        st, rounds = model.decode_block(gkv2, gcv2, blk, gs, toks)
        model.check_device()
        t = toks.cpu().numpy()
        assert ((t >= 0) & (t < cfg.vocab)).all()
        assert 1 <= st[0] <= sc.max_steps
        total += st[0]
        assert gkv2.length == 1024 + (blk + 1) * CANVAS
    print(f"decode loop: {4 * CANVAS} tokens in {total} passes, {4 * CANVAS / total:.2f} tokens per pass; {rep}")
