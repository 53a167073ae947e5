"""GPU (C ABI) vs oracle parity of the denoising step on seeded synthetic
inputs: context encoding, canvas initialisation, logits, routing, per-position
statistics, samples, lock masks, stop flags, the next canvas and the
self-conditioning state, step by step -- every stage on the GPU's own input
(strict decision gate) and the whole step free-running (tests/parity.py)."""

import pytest

from parity import Case, TINY, LAYER1, run_case

pytestmark = pytest.mark.gpu


def _compared(rep, steps, batch=1):
    """Every step compared every stage at every position, and some positions
    end to end."""
    assert rep.steps == steps, rep
    assert rep.tf_decisions > 0 and rep.tf_positions == steps * 256 * batch, rep
    assert rep.compared_positions > 0 and rep.logit_rel > 0 and rep.tf_logit_rel > 0, rep


def test_tiny_decode_prob_lock():
    """2 layers, d 256, 8 heads x 32, 16 experts top-2, vocab 4096, 64 context
    tokens, one canvas, 4 rounds, lock on max prob > 0.9, Philox seed 1234."""
    rep = run_case(Case(cfg=TINY, ctx_len=64, steps=4))
    _compared(rep, 4)


def test_tiny_self_cond_entropy_cumsum_lock_batch2():
    """Peaked LM head so that positions lock; cumulative-entropy lock rule;
    self-conditioning; two canvases with their own contexts and streams;
    ragged context length (not a multiple of 64)."""
    rep = run_case(Case(cfg=TINY, self_cond=True, ctx_len=77, batch=2, steps=3, lm_std=2.0,
                        sampler=dict(lock_policy="entropy_cumsum", lock_threshold=0.1)))
    _compared(rep, 3, batch=2)


def test_tiny_peaked_prob_lock_and_stop():
    """Locks fire (pmax > 0.9) and the adaptive stop fires at its threshold."""
    rep = run_case(Case(cfg=TINY, ctx_len=300, steps=3, lm_std=2.5,
                        sampler=dict(stop_entropy=3.0, stop_require_stable_argmax=False)))
    _compared(rep, 3)


def test_tiny_persistent_lock_variant():
    """The masked-style variant (persistent lock): a position locked in an
    earlier round keeps its token in every later round; peaked LM head so
    that positions lock, four rounds."""
    rep = run_case(Case(cfg=TINY, ctx_len=48, steps=4, lm_std=2.5,
                        sampler=dict(persistent_lock=True, stop_entropy=0.0)))
    _compared(rep, 4)


@pytest.mark.parametrize("k", [1, 64, 1024])
def test_tiny_self_cond_topk_variant(k):
    """The high-batch variant of the self-conditioning input: the expected
    embedding over each position's K largest logits only (K = 1: the argmax
    embedding; K = 1024: the largest K the kernel takes), three rounds."""
    rep = run_case(Case(cfg=TINY, self_cond=True, ctx_len=40, steps=3, lm_std=1.5,
                        sampler=dict(selfcond_topk=k)))
    _compared(rep, 3)


@pytest.mark.parametrize("split,ctx_len,batch,prefill", [(40, 296, 1, 512), (77, 333, 2, 1024), (40, 296, 2, 0),
                                                        (64, 320, 1, 512), (100, 612, 1, 0)])
def test_tiny_context_encoded_in_two_calls(split, ctx_len, batch, prefill):
    """The context appended in two encode calls, the second starting at a
    ragged position (passes of 256 or of `prefill` tokens), then two rounds."""
    rep = run_case(Case(cfg=TINY, ctx_len=ctx_len, batch=batch, steps=2, ctx_split=split, prefill=prefill))
    _compared(rep, 2, batch=batch)


def test_single_layer_full_width_step():
    """1 layer, d 2816, 16 q / 8 kv heads x 176, 128 experts top-8, ffn 704,
    vocab 262144, 2048 context tokens, one canvas, one round."""
    rep = run_case(Case(cfg=LAYER1, ctx_len=2048, steps=1))
    _compared(rep, 1)


@pytest.mark.parametrize("n_experts,top_k,ctx_len", [(4, 4, 0), (6, 1, 17), (6, 3, 64), (256, 8, 0), (256, 8, 64)])
def test_tiny_degenerate_routing_and_context(n_experts, top_k, ctx_len):
    """Routing edge cases against the oracle: every expert chosen by every
    token (top-k = E, the dense softmax mixture), a single expert per token,
    an expert count that is not a multiple of 4, the largest expert count
    (256: 8 router logits per lane, 256 groups in the grouped products); and
    a canvas with no context at all (attention over the canvas keys only) or a
    ragged one."""
    cfg = dict(TINY, n_experts=n_experts, top_k=top_k)
    rep = run_case(Case(cfg=cfg, ctx_len=ctx_len, steps=2))
    _compared(rep, 2)


def test_tiny_batch8_canvases():
    """Eight canvases in one round (2,048 canvas tokens, 4,096 routed pairs
    over 16 experts): every canvas against the oracle."""
    rep = run_case(Case(cfg=TINY, ctx_len=40, batch=8, steps=2))
    _compared(rep, 2, batch=8)


@pytest.mark.parametrize("shape", [
    dict(d_model=4096, n_q_heads=32, n_kv_heads=8, head_dim=128),   # widest model, head_dim 128
    dict(d_model=512, n_q_heads=8, n_kv_heads=2, head_dim=64),      # 4 query heads per kv head
])
def test_width_and_grouped_query_shapes(shape):
    """One layer at the largest model width (d_model 4096: router split 8,
    one float4 per thread of the 4096-wide rows) and at a wider grouped-query
    ratio (G = 4, head_dim 64), end to end against the oracle."""
    cfg = dict(n_layers=1, n_experts=8, top_k=2, d_ff=256, vocab=4096, **shape)
    rep = run_case(Case(cfg=cfg, ctx_len=70, steps=2))
    _compared(rep, 2)


def test_tiny_largest_batch():
    """The largest batch a context takes (64 canvases, 16,384 canvas tokens
    and 32,768 routed pairs in one round; 111 tokens per routing CTA), one
    round end to end against the oracle."""
    rep = run_case(Case(cfg=TINY, ctx_len=16, batch=64, steps=1))
    _compared(rep, 1, batch=64)
