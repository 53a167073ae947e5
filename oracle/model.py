"""Oracle: the MoE transformer forward pass of one canvas (float64).

What the pages fix (the laozijiushiniubi.cn article "谷歌DeepMind如何将一台
'逐字打稿机'改造成'整段喷墨机'", §二): the network is a Gemma-4 mixture of
experts with 128 experts of which 8 are used per token; the prompt (context)
is encoded with causal attention and the 256-token canvas with bidirectional
attention; a self-conditioning input feeds back the previous round's
prediction.  Everything else below is a stated reading (the pages are silent):
pre-norm RMSNorm (eps 1e-6), rotary position embedding (theta 1e4, rotate
halves), grouped-query attention (q head h uses kv head h // (Hq / Hkv)),
softmax router with top-k by router logit (ties to the lower expert id) and
the k weights renormalised, SwiGLU experts, untied embedding and LM head.

Precision contract (both sides round at these points): bf16 for norm
outputs, q/k (after RoPE), v, the attention output, the SwiGLU product and
the self-conditioning state; fp32 for the residual stream, router logits and
weights, expert outputs and LM-head logits.  Everything between those points
is float64 here.

Pins (tests/test_oracle_model.py): RMSNorm and SwiGLU closed forms; RoPE is
the identity at position 0 and q.k depends only on the position difference;
attention equals a second, independent formulation on tiny shapes, is
permutation-equivariant over canvas rows without a mask, returns the mean of
V for identical keys, and with a causal mask row 0 returns v_0; routing with
k = E equals the dense softmax mixture and E = k = 1 is a plain SwiGLU FFN;
routing weights sum to 1 and ties go to the lower id.  One layer's wiring
(layer_forward) is pinned by closed forms: zero output and down projections
keep the stream; zero query/key weights give uniform attention, whose
residual (grouped-query head mapping, head layout, causal prefix, context
keys) is written out; with one expert the MoE reads the stream after the
attention residual.  The final norm and LM head (lm_logits): identity
vocabulary rows return the bf16 normed stream, vocabulary chunking changes
no logit, and with eps 0 a power-of-two scale of the stream changes none.
The composition of the full random-init model
(forward_layers over many layers) has no closed form: parity unpinned beyond
those pieces.
"""

from dataclasses import dataclass, field

import numpy as np

import synth
from .numerics import bf16_round, f32_round, bf16_bits_to_f64


@dataclass(frozen=True)
class ModelConfig:
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    d_ff: int
    vocab: int
    self_cond: bool = False
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    canvas: int = 256


class Weights:
    """Random-init weights from the seeded generator (synth), materialised
    lazily as float64 (one layer at a time).  `std` maps a tensor kind to its
    init standard deviation (default 0.02 for all)."""

    def __init__(self, cfg: ModelConfig, seed: int = 0, std=None, threads: int = 0,
                 keep_chunks: bool = False):
        self.cfg = cfg
        self.seed = seed
        self.std = dict(std or {})
        self.threads = threads
        self._layer_idx = None
        self._layer = None
        # keep_chunks: remember generated embedding / LM-head row blocks so
        # that a timing run measures the arithmetic, not the input generator
        self._chunks = {} if keep_chunks else None

    def _std(self, kind):
        return self.std.get(kind, synth.WEIGHT_STD)

    def _mat(self, row0, rows, cols, tid, kind):
        bits = synth.bf16_rows(row0, rows, cols, self.seed, tid, self._std(kind), self.threads)
        return bf16_bits_to_f64(bits)

    def layer(self, l: int) -> dict:
        if self._layer_idx != l:
            c = self.cfg
            d, hd, E, f = c.d_model, c.head_dim, c.n_experts, c.d_ff
            t = lambda kind: synth.layer_tid(l, kind)  # noqa: E731
            self._layer = {
                "wq": self._mat(0, c.n_q_heads * hd, d, t(synth.KIND_WQ), synth.KIND_WQ),
                "wk": self._mat(0, c.n_kv_heads * hd, d, t(synth.KIND_WK), synth.KIND_WK),
                "wv": self._mat(0, c.n_kv_heads * hd, d, t(synth.KIND_WV), synth.KIND_WV),
                "wo": self._mat(0, d, c.n_q_heads * hd, t(synth.KIND_WO), synth.KIND_WO),
                "wr": self._mat(0, E, d, t(synth.KIND_WR), synth.KIND_WR),
                # experts stay as bf16 bit patterns; decoded one expert at a time
                "wg": synth.bf16_rows(0, E * f, d, self.seed, t(synth.KIND_WG),
                                      self._std(synth.KIND_WG), self.threads).reshape(E, f, d),
                "wu": synth.bf16_rows(0, E * f, d, self.seed, t(synth.KIND_WU),
                                      self._std(synth.KIND_WU), self.threads).reshape(E, f, d),
                "wd": synth.bf16_rows(0, E * d, f, self.seed, t(synth.KIND_WD),
                                      self._std(synth.KIND_WD), self.threads).reshape(E, d, f),
            }
            self._layer_idx = l
        return self._layer

    def router(self, l: int) -> dict:
        """Layer l's router matrix alone ({"wr": [E, d]}), without generating
        the rest of the layer (the same values as layer(l)["wr"])."""
        if self._layer_idx == l:
            return {"wr": self._layer["wr"]}
        c = self.cfg
        return {"wr": self._mat(0, c.n_experts, c.d_model, synth.layer_tid(l, synth.KIND_WR), synth.KIND_WR)}

    def emb_rows(self, tokens) -> np.ndarray:
        tokens = np.asarray(tokens).reshape(-1)
        d = self.cfg.d_model
        out = np.empty((tokens.size, d))
        for i, tok in enumerate(tokens):
            out[i] = self._mat(int(tok), 1, d, synth.KIND_EMB, synth.KIND_EMB)[0]
        return out

    def _chunk(self, kind, v0, n):
        key = (kind, v0, n)
        if self._chunks is not None and key in self._chunks:
            return self._chunks[key]
        m = self._mat(v0, n, self.cfg.d_model, kind, kind)
        if self._chunks is not None:
            self._chunks[key] = m
        return m

    def emb_chunk(self, v0: int, n: int) -> np.ndarray:
        return self._chunk(synth.KIND_EMB, v0, n)

    def lm_chunk(self, v0: int, n: int) -> np.ndarray:
        return self._chunk(synth.KIND_LM, v0, n)

    def sc(self) -> np.ndarray:
        d = self.cfg.d_model
        return self._mat(0, d, d, synth.KIND_SC, synth.KIND_SC)


@dataclass
class KVCache:
    """Per-layer keys (after RoPE) and values of the causally encoded context,
    bf16 values held in float32 arrays [B, C_max, H_kv, hd]."""
    cfg: ModelConfig
    batch: int
    c_max: int
    length: int = 0
    k: list = field(default_factory=list)
    v: list = field(default_factory=list)

    def __post_init__(self):
        c = self.cfg
        shape = (self.batch, self.c_max, c.n_kv_heads, c.head_dim)
        if not self.k:
            self.k = [np.zeros(shape, np.float32) for _ in range(c.n_layers)]
            self.v = [np.zeros(shape, np.float32) for _ in range(c.n_layers)]


def rmsnorm(x, eps, gain=1.0):
    """x / sqrt(mean(x^2) + eps) * gain over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * gain


def rope(x, positions, theta):
    """Rotary embedding on [n, H, hd]: pairs (i, i + hd/2) rotated by the
    angle position * theta^(-2i/hd)."""
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    half = hd // 2
    inv_freq = theta ** (-2.0 * np.arange(half) / hd)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def attention(q, k, v, q_pos, k_pos, causal):
    """softmax(q k^T / sqrt(hd)) v per query head, q [nq, Hq, hd], k/v
    [nk, Hkv, hd].  With `causal`, query i sees key j only when
    k_pos[j] <= q_pos[i] (context encoding); without it every query sees
    every key (the canvas)."""
    nq, Hq, hd = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    out = np.empty((nq, Hq, hd))
    mask = None
    if causal:
        mask = np.asarray(k_pos)[None, :] > np.asarray(q_pos)[:, None]
    for h in range(Hq):
        g = h // group
        s = (q[:, h, :] @ k[:, g, :].T) / np.sqrt(hd)
        if mask is not None:
            s = np.where(mask, -np.inf, s)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, g, :]
    return out


def route(h, wr, top_k, force_idx=None):
    """Router of the mixture of experts: fp32 logits h W_r^T, the top-k
    experts by logit (ties to the lower expert id; the softmax over all
    experts is monotone in the logit) and their softmax probabilities
    renormalised over the chosen k (the full-softmax denominator cancels).
    Returns (idx [T, k] int64, w [T, k] fp32 values, logits [T, E]).
    With force_idx [T, k] those experts are used instead of the top-k (the
    weights are still the softmax of their own logits): a comparison can run
    this model on another implementation's expert choices.
    route_margin() gives each token's smallest gap between consecutive
    sorted logits among the first k + 1 (how close the choice is to a tie)."""
    logits = f32_round(h @ wr.T)
    T, E = logits.shape
    idx = np.empty((T, top_k), np.int64)
    w = np.empty((T, top_k))
    for t in range(T):
        if force_idx is None:
            order = sorted(range(E), key=lambda e: (-logits[t, e], e))[:top_k]
        else:
            order = [int(e) for e in np.asarray(force_idx).reshape(T, top_k)[t]]
        idx[t] = order
        sel = logits[t, order]
        ex = np.exp(sel - sel.max())
        w[t] = ex / ex.sum()
    return idx, f32_round(w), logits


def route_margin(logits, top_k):
    s = -np.sort(-np.asarray(logits, dtype=np.float64), axis=1)[:, :top_k + 1]
    if s.shape[1] < 2:
        return np.full(s.shape[0], np.inf)
    return np.min(s[:, :-1] - s[:, 1:], axis=1)


def silu(a):
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def expert_ffn(x, wg, wu, wd):
    """SwiGLU expert: bf16(silu(x W_g^T) * (x W_u^T)) W_d^T, output fp32."""
    hh = bf16_round(silu(x @ wg.T) * (x @ wu.T))
    return f32_round(hh @ wd.T)


def moe_ffn(h, layer, top_k, force_idx=None):
    """Mixture-of-experts FFN on bf16 inputs h [T, d]: route (or take the
    experts force_idx names, see route), run each expert on the tokens sent
    to it, and combine sum_k w_k y_k (fp32 result).
    Returns (out, idx, w, routing margin, router logits)."""
    wg, wu, wd = layer["wg"], layer["wu"], layer["wd"]
    E = wg.shape[0]
    idx, w, logits = route(h, layer["wr"], top_k, force_idx)
    T = h.shape[0]
    y = np.zeros((T, top_k, h.shape[1]))
    for e in range(E):
        tok, slot = np.nonzero(idx == e)
        if tok.size == 0:
            continue
        y[tok, slot] = expert_ffn(h[tok], bf16_bits_to_f64(wg[e]), bf16_bits_to_f64(wu[e]),
                                  bf16_bits_to_f64(wd[e]))
    out = f32_round(np.sum(w[:, :, None] * y, axis=1))
    return out, idx, w, route_margin(logits, top_k), logits


def attention_block(cfg: ModelConfig, lw: dict, x, kv_k, kv_v, L0: int, causal: bool, append: bool):
    """The attention half of one transformer layer on the residual stream x
    [B, n, d] (fp32 values) whose tokens sit at positions L0 .. L0 + n - 1:
    RMSNorm, q/k/v projections, RoPE, attention over the cached keys [0, L0)
    of kv_k / kv_v ([B, C_max, H_kv, hd], keys after RoPE) plus the pass's own
    n keys (written to the cache at [L0, L0 + n) when `append`), output
    projection and residual add.  Returns the residual stream after it."""
    c = cfg
    B, n, d = x.shape
    pos = np.arange(L0, L0 + n)
    k_pos = np.arange(0, L0 + n)
    hd, Hq, Hkv = c.head_dim, c.n_q_heads, c.n_kv_heads
    h = bf16_round(rmsnorm(x, c.rms_eps))
    q = h @ lw["wq"].T
    k = h @ lw["wk"].T
    v = bf16_round(h @ lw["wv"].T)
    o = np.empty((B, n, Hq * hd))
    for b in range(B):
        qb = bf16_round(rope(q[b].reshape(n, Hq, hd), pos, c.rope_theta))
        kb = bf16_round(rope(k[b].reshape(n, Hkv, hd), pos, c.rope_theta))
        vb = v[b].reshape(n, Hkv, hd)
        k_all = np.concatenate([kv_k[b, :L0].astype(np.float64), kb], axis=0)
        v_all = np.concatenate([kv_v[b, :L0].astype(np.float64), vb], axis=0)
        o[b] = bf16_round(attention(qb, k_all, v_all, pos, k_pos, causal)).reshape(n, Hq * hd)
        if append:
            kv_k[b, L0:L0 + n] = kb
            kv_v[b, L0:L0 + n] = vb
    return f32_round(np.asarray(x, dtype=np.float64) + f32_round(o @ lw["wo"].T))


def moe_block(cfg: ModelConfig, lw: dict, x, force_idx=None):
    """The mixture-of-experts half of one transformer layer on the residual
    stream x [B, n, d] after the attention half: RMSNorm, router, experts and
    residual add (force_idx [B, n, k]: use these experts, see route).
    Returns the residual stream after the layer and (routing idx, weights,
    routing margin, router logits)."""
    B, n, d = x.shape
    h2 = bf16_round(rmsnorm(x, cfg.rms_eps)).reshape(B * n, d)
    fi = None if force_idx is None else np.asarray(force_idx).reshape(B * n, -1)
    m, idx, w, margin, rlog = moe_ffn(h2, lw, cfg.top_k, fi)
    x = f32_round(np.asarray(x, dtype=np.float64) + m.reshape(B, n, d))
    return x, (idx.reshape(B, n, -1), w.reshape(B, n, -1), margin.reshape(B, n), rlog.reshape(B, n, -1))


def router_block(cfg: ModelConfig, lw: dict, x):
    """The router alone on the residual stream x [B, n, d] after the attention
    half (the first steps of moe_block): routing idx, weights, margin and
    router logits, shaped as moe_block returns them."""
    B, n, d = x.shape
    h2 = bf16_round(rmsnorm(x, cfg.rms_eps)).reshape(B * n, d)
    idx, w, logits = route(h2, lw["wr"], cfg.top_k)
    margin = route_margin(logits, cfg.top_k)
    return idx.reshape(B, n, -1), w.reshape(B, n, -1), margin.reshape(B, n), logits.reshape(B, n, -1)


def layer_forward(cfg: ModelConfig, lw: dict, x, kv_k, kv_v, L0: int, causal: bool, append: bool,
                  force_idx=None):
    """One transformer layer on the residual stream x [B, n, d] (fp32 values)
    whose tokens sit at positions L0 .. L0 + n - 1: attention_block then
    moe_block.  Returns the residual stream after the layer and (routing idx,
    weights, routing margin, router logits).  With force_idx the experts are
    those it names and the returned idx is the router's own top-k choice."""
    x = attention_block(cfg, lw, x, kv_k, kv_v, L0, causal, append)
    if force_idx is None:
        return moe_block(cfg, lw, x)
    own = router_block(cfg, lw, x)[0]
    x, (_, w, margin, rlog) = moe_block(cfg, lw, x, force_idx)
    return x, (own, w, margin, rlog)


def forward_layers(cfg: ModelConfig, W: Weights, x, kv: KVCache, causal: bool, append: bool,
                   record=None, force=None):
    """Run all transformer layers on the residual stream x [B, n, d] (fp32
    values) whose tokens sit at positions kv.length .. kv.length + n - 1.

    Keys are the cached context [0, kv.length) plus this pass's own n keys.
    Context encoding uses causal=True and append=True (its keys are stored and
    kv.length grows); a canvas pass uses causal=False and append=False (the
    canvas attends to the whole context and to itself, and its keys are not
    kept).  Returns the final residual stream.  `record`, if a list, receives
    per layer (routing idx, weights, routing margin, residual stream after the
    layer, router logits).  `force`, if given, maps a layer to the experts
    [B, n, k] its MoE uses (layer_forward's force_idx); the record keeps the
    router's own choice."""
    L0 = kv.length
    n = x.shape[1]
    x = f32_round(x)
    for l in range(cfg.n_layers):
        fi = None if force is None else force(l)
        x, (idx, w, margin, rlog) = layer_forward(cfg, W.layer(l), x, kv.k[l], kv.v[l], L0, causal, append, fi)
        if record is not None:
            record.append((idx, w, margin, x.copy(), rlog))
    if append:
        kv.length = L0 + n
    return x


def lm_logits(cfg: ModelConfig, W: Weights, x, chunk: int = 16384):
    """Final RMSNorm and LM head: fp32 logits [T, V] of x [T, d]."""
    hf = bf16_round(rmsnorm(x, cfg.rms_eps))
    V = cfg.vocab
    out = np.empty((hf.shape[0], V), np.float32)
    for v0 in range(0, V, chunk):
        n = min(chunk, V - v0)
        out[:, v0:v0 + n] = (hf @ W.lm_chunk(v0, n).T).astype(np.float32)
    return out
