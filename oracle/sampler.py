"""Oracle: per-position vocabulary statistics, sampling, locking, stopping
and the self-conditioning expected embedding.

What the pages fix (the laozijiushiniubi.cn article "谷歌DeepMind如何将一台
'逐字打稿机'改造成'整段喷墨机'", §四 "智能采样器"): positions are ordered by
entropy, lowest first, and locked one by one until the cumulative entropy
would exceed 0.1; the rest are re-randomised and revised in the next round
(§一 adds that uncertain positions become any vocabulary token, so even
locked tokens can change later); the temperature falls linearly from 0.8 in
early rounds to 0.4 in late rounds; the block stops early when the mean
entropy is below 0.005 and the most likely sequence is unchanged between two
rounds, within a budget of 48 rounds.  The benchmark configuration adds a
second lock rule (max probability > 0.9) and a mean-entropy stop threshold
of 0.5 nats; both rules and both thresholds are parameters.  §二 and §五
describe the self-conditioning input: the previous round's prediction,
carried here as the expected embedding sum_v p_v E_emb[v].

Readings where the pages are silent: entropy and max probability use the
untempered softmax (T = 1, natural log); the draw of each position's next
token is the Gumbel-max categorical sample argmax_v(l_v / T + g_v) with
g = -ln(-ln u), computed in float32 on both sides; the lock mask is recomputed
every round; the cumulative rule locks the longest prefix whose running sum
stays <= the budget; the linear temperature runs over the step budget.

Pins (tests/test_oracle_sampler.py): sum p = 1 and 0 <= H <= ln V;
uniform logits give H = ln V and pmax = 1/V; a two-level logit vector gives
the closed-form H; Gumbel-max frequencies match softmax(l / T) (chi-square);
the cumulative lock rule matches brute-force enumeration; the stop flag fires
exactly below the threshold; the temperature hits 0.8 and 0.4 at the ends;
the expected embedding of a one-hot distribution is that token's row.
"""

from dataclasses import dataclass

import numpy as np

from .philox import gumbel_u, gumbel_words, method_draw, uniform_token, PURPOSE_RENOISE
from .numerics import bf16_round

LOCK_PROB = "prob"
LOCK_ENTROPY_CUMSUM = "entropy_cumsum"


@dataclass(frozen=True)
class SamplerConfig:
    lock_policy: str = LOCK_PROB
    lock_threshold: float = 0.9
    t_start: float = 0.8
    t_end: float = 0.4
    max_steps: int = 48
    stop_entropy: float = 0.5
    stop_require_stable_argmax: bool = False
    seed: int = 0
    persistent_lock: bool = False   # masked-style variant: a locked position keeps its token
    selfcond_topk: int = 0          # 0: full-vocabulary expected embedding; K: top-K variant


def temperature(step: int, max_steps: int, t_start: float = 0.8, t_end: float = 0.4) -> float:
    """Linear anneal from t_start at step 0 to t_end at the last budgeted step."""
    if max_steps <= 1:
        return float(t_start)
    return t_start + (t_end - t_start) * step / (max_steps - 1)


def inv_temperature_f32(step, max_steps, t_start=0.8, t_end=0.4) -> np.float32:
    """1 / T_s rounded to float32 (the value both sides multiply logits by)."""
    return np.float32(1.0 / temperature(step, max_steps, t_start, t_end))


def position_stats(logits):
    """Untempered softmax statistics of one position's fp32 logits [V]:
    (entropy H = -sum p ln p, pmax = max p, argmax with ties to the lower id,
    p as float64)."""
    l = np.asarray(logits, dtype=np.float64)
    m = l.max()
    e = np.exp(l - m)
    p = e / e.sum()
    with np.errstate(divide="ignore", invalid="ignore"):
        terms = np.where(p > 0, p * np.log(p), 0.0)
    H = float(-terms.sum())
    return H, float(p.max()), int(np.argmax(np.asarray(logits, dtype=np.float32))), p


def gumbel_keys(logits_f32, inv_t_f32, words):
    """float32 keys l_v * (1/T) + g_v with g = -ln(-ln u)."""
    u = gumbel_u(words)
    g = -np.log(-np.log(u))
    l = np.asarray(logits_f32, dtype=np.float32)
    return (l * np.float32(inv_t_f32)).astype(np.float32) + g.astype(np.float32)


def gumbel_sample(logits_f32, inv_t_f32, words):
    """Categorical draw from softmax(l / T) by the Gumbel-max rule (first
    index among equal maxima).  Returns (token, keys)."""
    keys = gumbel_keys(logits_f32, inv_t_f32, words)
    return int(np.argmax(keys)), keys


def position_sample(logits_f32, inv_t_f32, seed, canvas, block, step, position):
    words = gumbel_words(seed, canvas, block, step, position, len(logits_f32))
    return gumbel_sample(logits_f32, inv_t_f32, words)


def lock_mask(H, pmax, policy: str, threshold: float):
    """Which positions keep their sampled token this round.

    LOCK_PROB: pmax > threshold (strict).
    LOCK_ENTROPY_CUMSUM: sort positions by (H, position) ascending and lock
    the longest prefix whose cumulative entropy is <= threshold."""
    H = np.asarray(H, dtype=np.float64)
    n = H.size
    if policy == LOCK_PROB:
        return np.asarray(pmax, dtype=np.float64) > threshold
    if policy == LOCK_ENTROPY_CUMSUM:
        order = np.argsort(H, kind="stable")
        csum = np.cumsum(H[order])
        k = int(np.sum(csum <= threshold)) if n else 0
        # csum is non-decreasing (H >= 0), so the "<= threshold" positions form a prefix
        mask = np.zeros(n, dtype=bool)
        mask[order[:k]] = True
        return mask
    raise ValueError(f"unknown lock policy {policy!r}")


def stop_flag(mean_H, stop_entropy, require_stable, step, argmax, prev_argmax) -> bool:
    """Adaptive stop: mean entropy strictly below the threshold and, if
    required, the argmax sequence identical to the previous round's."""
    stop = mean_H < stop_entropy
    if require_stable:
        stop = stop and step > 0 and prev_argmax is not None and \
            bool(np.array_equal(np.asarray(argmax), np.asarray(prev_argmax)))
    return bool(stop)


def renoise_tokens(seed, canvas, block, step, n_pos, vocab):
    """Uniform replacement tokens for every position of one canvas."""
    w0, _, _, _ = method_draw(seed, PURPOSE_RENOISE, canvas, block, step,
                              np.arange(n_pos, dtype=np.uint64))
    return uniform_token(w0, vocab)


def selfcond_probs(logits_f32):
    """The expected embedding's probabilities of one position (precision
    contract): the logits are stored as bf16 for this use only, so
    p_v = exp(bf16(l_v) - m) / Z with m = max l and Z = sum_v exp(l_v - m) of
    the fp32 logits (the statistics the entropy uses).  float64 result."""
    l = np.asarray(logits_f32, dtype=np.float64)
    m = l.max()
    Z = np.exp(l - m).sum()
    return np.exp(bf16_round(l) - m) / Z


def expected_embedding(probs, W, chunk: int = 16384):
    """bf16(sum_v bf16(p_v) E_emb[v]) for probs [T, V] (float64)."""
    T, V = probs.shape
    acc = np.zeros((T, W.cfg.d_model))
    pb = bf16_round(probs)
    for v0 in range(0, V, chunk):
        n = min(chunk, V - v0)
        acc += pb[:, v0:v0 + n] @ W.emb_chunk(v0, n)
    return bf16_round(acc)


def expected_embedding_topk(logits_f32, W, k: int):
    """The high-batch variant of the self-conditioning input (top-k
    vocabulary truncation, the laozijiushiniubi.cn article, section 九): per
    position, the k ids with the largest bf16-stored logits (ties to the lower
    id), p_v = exp(bf16(l_v) - M) / sum over those k of exp(bf16(l_u) - M) with
    M the largest of them, rounded to bf16, and e = bf16(sum_v p_v E_emb[v])
    over those k rows only.  logits_f32 [T, V]; returns (e [T, d] float64
    bf16 values, ids [T, k] in ascending id order)."""
    lb = bf16_round(np.asarray(logits_f32, dtype=np.float64))
    T, V = lb.shape
    k = int(min(k, V))
    e = np.zeros((T, W.cfg.d_model))
    ids = np.empty((T, k), np.int64)
    for t in range(T):
        order = np.lexsort((np.arange(V), -lb[t]))[:k]   # by value descending, then id ascending
        sel = np.sort(order)
        ids[t] = sel
        M = lb[t, sel].max()
        w = np.exp(lb[t, sel] - M)
        p = bf16_round(w / w.sum())
        rows = np.stack([W.emb_rows([int(v)])[0] for v in sel])
        e[t] = p @ rows
    return bf16_round(e), ids
