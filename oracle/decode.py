"""Oracle: context encoding, one denoising step of the canvas, and the block
decoding loop.

The pages (the arXiv abstract page "DiffusionGemma 技术报告" and the
laozijiushiniubi.cn article "谷歌DeepMind如何将一台'逐字打稿机'改造成
'整段喷墨机'", §一, §二, §四) describe generation as: encode the prompt
causally; start a 256-token block from uniformly random tokens; refine every
position in parallel each round; lock confident positions and re-randomise
the others; stop adaptively; the block then becomes context for the next one.

One step, in order (steps a1-a9):
  a1  x0 = E_emb[canvas] (+ bf16(e_prev) W_sc^T when self-conditioning)
  a2-a6 the transformer layers over the canvas (forward_layers, no mask,
      canvas keys not kept)
  a7  LM-head logits and per-position H, pmax, argmax, Gumbel sample at T_s
  a8  the expected embedding e = sum_v softmax(l)_v E_emb[v] (next step's
      self-conditioning input)
  a9  mean entropy, stop flag, lock mask, and the next canvas: locked
      positions keep their sample, the others get uniform random tokens; on
      stop (or at the last budgeted step) the canvas becomes the argmax
      sequence and the canvas is frozen.

Canvases of a batch are independent (own context, own random stream, own stop).
"""

from dataclasses import dataclass, field

import numpy as np

from . import sampler as smp
from .model import ModelConfig, Weights, KVCache, forward_layers, lm_logits
from .numerics import f32_round
from .philox import method_draw, uniform_token, gumbel_words, PURPOSE_INIT, PURPOSE_AR_GUMBEL


@dataclass
class CanvasState:
    tokens: np.ndarray            # [B, N] int64
    sc: np.ndarray                # [B, N, d] float64 (bf16 values); zeros before step 0
    prev_argmax: np.ndarray       # [B, N] int64, -1 before step 0
    done: np.ndarray              # [B] bool
    locked: np.ndarray = None     # [B, N] bool, positions committed so far (persistent lock)


@dataclass
class StepOutput:
    logits: np.ndarray            # [B, N, V] float32
    argmax: np.ndarray            # [B, N]
    sample: np.ndarray            # [B, N]
    entropy: np.ndarray           # [B, N] float64
    pmax: np.ndarray              # [B, N] float64
    mean_entropy: np.ndarray      # [B]
    stop: np.ndarray              # [B] bool (stopped at this step)
    final: np.ndarray             # [B] bool (stopped, or the last budgeted step)
    lock: np.ndarray              # [B, N] bool
    tokens_in: np.ndarray         # [B, N] canvas the step consumed
    tokens_out: np.ndarray        # [B, N] canvas after the update
    sample_margin: np.ndarray     # [B, N] top-2 gap of the Gumbel keys
    argmax_margin: np.ndarray     # [B, N] top-2 gap of the logits
    routing: list = field(default_factory=list)  # per layer (idx [B,N,k], w [B,N,k])
    expected_emb: np.ndarray = None


def init_canvas(seed: int, block: int, batch: int, n_pos: int, vocab: int) -> np.ndarray:
    """Uniform random starting tokens (draw purpose 1)."""
    toks = np.empty((batch, n_pos), np.int64)
    for b in range(batch):
        w0, _, _, _ = method_draw(seed, PURPOSE_INIT, b, block, 0, np.arange(n_pos, dtype=np.uint64))
        toks[b] = uniform_token(w0, vocab)
    return toks


def new_state(tokens, d_model) -> CanvasState:
    B, N = tokens.shape
    return CanvasState(tokens=np.array(tokens, np.int64), sc=np.zeros((B, N, d_model)),
                       prev_argmax=np.full((B, N), -1, np.int64), done=np.zeros(B, bool),
                       locked=np.zeros((B, N), bool))


def encode_context(cfg: ModelConfig, W: Weights, kv: KVCache, tokens, record=None):
    """Causal encoding of tokens [B, n] appended at kv.length (keys stored).
    Encoding no tokens leaves the cache as it is.  `record`, if a list,
    receives the per-layer routing record of forward_layers."""
    tokens = np.asarray(tokens)
    B, n = tokens.shape
    if n == 0:
        return
    x = W.emb_rows(tokens).reshape(B, n, cfg.d_model)
    forward_layers(cfg, W, x, kv, causal=True, append=True, record=record)


def _top2_gap(v):
    v = np.asarray(v, dtype=np.float64)
    if v.size < 2:
        return np.inf
    top = np.partition(v, -2)[-2:]
    return float(top[1] - top[0])


def update_canvas(cfg: ModelConfig, sc: smp.SamplerConfig, state: CanvasState, block: int, step: int,
                  H, pmax, amax, samp, e_new=None):
    """a9 on the per-position statistics of one step (H, pmax, argmax and
    sample [B, N]): the mean entropy, the stop flag, the lock mask and the next
    canvas (locked positions keep their sample, the others get the re-noise
    draw; a stopping or last-budget canvas becomes its argmax and is frozen);
    `state` is updated in place.  With sc.persistent_lock (the masked-style
    variant) a position locked in an earlier round keeps its token and counts
    as locked.  Returns (meanH, stop, final, lock)."""
    B, N = state.tokens.shape
    V = cfg.vocab
    meanH = H.mean(axis=1)
    stop = np.zeros(B, bool)
    final = np.zeros(B, bool)
    lock = np.zeros((B, N), bool)
    persistent = bool(getattr(sc, "persistent_lock", False))
    if persistent and state.locked is None:
        state.locked = np.zeros((B, N), bool)
    for b in range(B):
        lock[b] = smp.lock_mask(H[b], pmax[b], sc.lock_policy, sc.lock_threshold)
        committed = state.locked[b].copy() if persistent else np.zeros(N, bool)
        lock[b] |= committed
        if state.done[b]:
            continue
        prev = state.prev_argmax[b] if step > 0 else None
        stop[b] = smp.stop_flag(meanH[b], sc.stop_entropy, sc.stop_require_stable_argmax, step,
                                amax[b], prev)
        final[b] = stop[b] or step == sc.max_steps - 1
        if final[b]:
            state.tokens[b] = np.where(committed, state.tokens[b], amax[b])
            state.done[b] = True
        else:
            noise = smp.renoise_tokens(sc.seed, b, block, step, N, V)
            state.tokens[b] = np.where(committed, state.tokens[b], np.where(lock[b], samp[b], noise))
        state.prev_argmax[b] = amax[b]
        if persistent:
            state.locked[b] |= lock[b]
        if cfg.self_cond and e_new is not None:
            state.sc[b] = e_new[b]
    return meanH, stop, final, lock


def denoise_step(cfg: ModelConfig, W: Weights, kv: KVCache, state: CanvasState,
                 sc: smp.SamplerConfig, block: int, step: int, keep_logits: bool = True,
                 record_routing: bool = False, force_routing=None) -> StepOutput:
    """One denoising round over every canvas of the batch; updates `state`.
    force_routing (optional): layer -> experts [B, N, k] the layer's MoE uses
    (forward_layers' force); the routing record keeps the router's own choice."""
    B, N = state.tokens.shape
    d, V = cfg.d_model, cfg.vocab
    tokens_in = state.tokens.copy()

    # a1: canvas embedding plus the self-conditioning input
    x = W.emb_rows(tokens_in).reshape(B, N, d)
    if cfg.self_cond:
        x = f32_round(x + f32_round(state.sc.reshape(B * N, d) @ W.sc().T).reshape(B, N, d))

    # a2-a6: transformer layers, bidirectional over the canvas
    routing = [] if record_routing else None
    x = forward_layers(cfg, W, x, kv, causal=False, append=False, record=routing, force=force_routing)

    # a7: logits and per-position statistics / samples
    logits = lm_logits(cfg, W, x.reshape(B * N, d)).reshape(B, N, V)
    inv_t = smp.inv_temperature_f32(step, sc.max_steps, sc.t_start, sc.t_end)
    H = np.empty((B, N))
    pmax = np.empty((B, N))
    amax = np.empty((B, N), np.int64)
    samp = np.empty((B, N), np.int64)
    s_gap = np.empty((B, N))
    a_gap = np.empty((B, N))
    topk = int(getattr(sc, "selfcond_topk", 0))
    probs = np.empty((B, N, V)) if cfg.self_cond and topk == 0 else None
    for b in range(B):
        for i in range(N):
            H[b, i], pmax[b, i], amax[b, i], p = smp.position_stats(logits[b, i])
            samp[b, i], keys = smp.position_sample(logits[b, i], inv_t, sc.seed, b, block, step, i)
            s_gap[b, i] = _top2_gap(keys)
            a_gap[b, i] = _top2_gap(logits[b, i])
            if probs is not None:
                probs[b, i] = smp.selfcond_probs(logits[b, i])

    # a8: expected embedding for the next round's self-conditioning input
    e_new = None
    if cfg.self_cond and topk > 0:
        e_new = smp.expected_embedding_topk(logits.reshape(B * N, V), W, topk)[0].reshape(B, N, d)
    elif cfg.self_cond:
        e_new = smp.expected_embedding(probs.reshape(B * N, V), W).reshape(B, N, d)

    # a9: stop, lock and the next canvas
    meanH, stop, final, lock = update_canvas(cfg, sc, state, block, step, H, pmax, amax, samp, e_new)

    return StepOutput(logits=logits if keep_logits else None, argmax=amax, sample=samp, entropy=H,
                      pmax=pmax, mean_entropy=meanH, stop=stop, final=final, lock=lock,
                      tokens_in=tokens_in, tokens_out=state.tokens.copy(), sample_margin=s_gap,
                      argmax_margin=a_gap, routing=routing or [], expected_emb=e_new)


def decode_block(cfg: ModelConfig, W: Weights, kv: KVCache, sc: smp.SamplerConfig, block: int,
                 batch: int, keep_logits: bool = False, on_step=None):
    """Generate one block per canvas: initialise, step until every canvas has
    stopped or the budget is spent, then append the block to the context.
    Returns (tokens [B, N], steps taken per canvas [B], list of StepOutput)."""
    N = cfg.canvas
    state = new_state(init_canvas(sc.seed, block, batch, N, cfg.vocab), cfg.d_model)
    steps = np.zeros(batch, np.int64)
    outs = []
    for s in range(sc.max_steps):
        active = ~state.done
        o = denoise_step(cfg, W, kv, state, sc, block, s, keep_logits=keep_logits)
        steps[active] += 1
        outs.append(o)
        if on_step is not None:
            on_step(s, o)
        if state.done.all():
            break
    tokens = state.tokens.copy()
    encode_context(cfg, W, kv, tokens)
    return tokens, steps, outs



def ar_step(cfg: ModelConfig, W: Weights, kv: KVCache, tokens, temperature: float, seed: int):
    """Retained autoregressive mode (the laozijiushiniubi.cn article, section
    七: the same weights still generate one token at a time): tokens [B] are
    appended at position P = kv.length with causal attention (the causal
    encode of one token), and that position's logits give the next token:
    its argmax and its Gumbel-max draw from softmax(l / temperature) (draw
    purpose 5, canvas b, c2 = P, position 0).  Returns (logits [B, V] fp32,
    argmax [B], sample [B], Gumbel-key top-2 gaps [B], logit top-2 gaps [B])."""
    tokens = np.asarray(tokens).reshape(-1)
    B = tokens.size
    P = kv.length
    x = W.emb_rows(tokens).reshape(B, 1, cfg.d_model)
    x = forward_layers(cfg, W, x, kv, causal=True, append=True)
    logits = lm_logits(cfg, W, x.reshape(B, cfg.d_model))
    inv_t = np.float32(1.0 / float(np.float32(temperature)))
    amax = np.empty(B, np.int64)
    samp = np.empty(B, np.int64)
    s_gap = np.empty(B)
    a_gap = np.empty(B)
    for b in range(B):
        amax[b] = int(np.argmax(logits[b]))
        words = gumbel_words(seed, b, 0, P, 0, cfg.vocab, purpose=PURPOSE_AR_GUMBEL)
        samp[b], keys = smp.gumbel_sample(logits[b], inv_t, words)
        s_gap[b] = _top2_gap(keys)
        a_gap[b] = _top2_gap(logits[b])
    return logits, amax, samp, s_gap, a_gap


def denoise_step_append(cfg: ModelConfig, W: Weights, kv: KVCache, state: CanvasState,
                        sc: smp.SamplerConfig, block: int, step: int, append_tokens, **kw) -> StepOutput:
    """A round that first appends a finished block to the context (the
    laozijiushiniubi.cn article, sections 二 and 四: a finished block becomes
    context, encoded causally): the causal encode of append_tokens [B, N],
    then the canvas round over the grown context.  The GPU runs both in one
    pass; this is its definition."""
    encode_context(cfg, W, kv, append_tokens)
    return denoise_step(cfg, W, kv, state, sc, block, step, **kw)
