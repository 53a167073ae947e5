"""Device-memory plumbing around the C ABI: torch tensors for the weights,
workspace, KV cache, canvas state and step outputs, and calls into libdg.so.
No arithmetic of the method happens here."""

import ctypes

import torch

from . import (DG_CANVAS, DG_LOCK_PROB, check, dg_block_stats, dg_canvas, dg_kv, dg_model_config,
               dg_sampler_config, dg_step_args, dg_step_out, lib)


def model_config(n_layers, d_model, n_q_heads, n_kv_heads, head_dim, n_experts, top_k, d_ff, vocab,
                 self_cond=False, rope_theta=10000.0, rms_eps=1e-6) -> dg_model_config:
    return dg_model_config(n_layers, d_model, n_q_heads, n_kv_heads, head_dim, n_experts, top_k, d_ff,
                           vocab, int(bool(self_cond)), rope_theta, rms_eps)


def sampler_config(lock_policy=DG_LOCK_PROB, lock_threshold=0.9, t_start=0.8, t_end=0.4, max_steps=48,
                   stop_entropy=0.5, stop_require_stable_argmax=False, seed=0,
                   persistent_lock=False, selfcond_topk=0) -> dg_sampler_config:
    return dg_sampler_config(lock_policy, lock_threshold, t_start, t_end, max_steps, stop_entropy,
                             int(bool(stop_require_stable_argmax)), seed, int(bool(persistent_lock)),
                             int(selfcond_topk))


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


class KVCache:
    """Per-layer K cache [B, Hkv, c_max, hd] (bf16) and transposed V cache
    [B, Hkv, hd, c_max] (fp16 holding the bf16-rounded values).  The capacity is rounded up to a multiple of 8
    positions (the row pitch of the transposed cache must be 16-byte aligned)."""

    def __init__(self, cfg: dg_model_config, batch: int, c_max: int, device="cuda"):
        c_max = (int(c_max) + 7) // 8 * 8
        n = lib.dg_kv_bytes(ctypes.byref(cfg), batch, c_max)
        if n == 0:
            raise ValueError("bad KV cache size")
        self.k = torch.zeros(n, dtype=torch.uint8, device=device)
        self.v = torch.zeros(n, dtype=torch.uint8, device=device)
        self.s = dg_kv(self.k.data_ptr(), self.v.data_ptr(), batch, c_max, 0)
        self.cfg = cfg

    @property
    def length(self):
        return self.s.length

    def layer_kv(self, layer):
        """(K, V) of one layer as [B, Hkv, c_max, hd] views, K bf16 and V fp16
        (V is a transposed view of the [B, Hkv, hd, c_max] storage)."""
        c = self.cfg
        per = self.k.numel() // 2 // c.n_layers
        k = self.k.view(torch.bfloat16)[layer * per:(layer + 1) * per].view(
            self.s.batch, c.n_kv_heads, self.s.c_max, c.head_dim)
        vt = self.v.view(torch.float16)[layer * per:(layer + 1) * per].view(
            self.s.batch, c.n_kv_heads, c.head_dim, self.s.c_max)
        return k, vt.transpose(-1, -2)


class Canvas:
    def __init__(self, cfg: dg_model_config, batch: int, device="cuda"):
        self.tokens = torch.zeros(batch, DG_CANVAS, dtype=torch.int32, device=device)
        self.sc_state = torch.zeros(batch, DG_CANVAS, cfg.d_model, dtype=torch.bfloat16, device=device)
        self.prev_argmax = torch.full((batch, DG_CANVAS), -1, dtype=torch.int32, device=device)
        self.done = torch.zeros(batch, dtype=torch.uint8, device=device)
        self.locked = torch.zeros(batch, DG_CANVAS, dtype=torch.uint8, device=device)
        self.s = dg_canvas(self.tokens.data_ptr(), self.sc_state.data_ptr(), self.prev_argmax.data_ptr(),
                           self.done.data_ptr(), batch, self.locked.data_ptr())


class StepOutputs:
    """Device buffers a round writes.  The per-position and per-canvas results
    (argmax, sample, entropy, pmax, lock, mean entropy, stop, final round) are
    views of one contiguous block, `packed`, so the host can read them with a
    single copy."""

    def __init__(self, cfg: dg_model_config, batch: int, logits=False, routing=False, hidden=False,
                 device="cuda"):
        T = batch * DG_CANVAS
        parts = [("argmax", torch.int32, (batch, DG_CANVAS)), ("sample", torch.int32, (batch, DG_CANVAS)),
                 ("entropy", torch.float32, (batch, DG_CANVAS)), ("pmax", torch.float32, (batch, DG_CANVAS)),
                 ("lock", torch.uint8, (batch, DG_CANVAS)), ("mean_entropy", torch.float32, (batch,)),
                 ("stop", torch.uint8, (batch,)), ("final_round", torch.uint8, (batch,))]
        offs, total = [], 0
        for _, dt, shape in parts:
            nbytes = torch.empty(0, dtype=dt).element_size()
            for n in shape:
                nbytes *= n
            offs.append(total)
            total += (nbytes + 15) // 16 * 16
        self.packed = torch.zeros(total, dtype=torch.uint8, device=device)
        for (name, dt, shape), o in zip(parts, offs):
            esz = torch.empty(0, dtype=dt).element_size()
            n = 1
            for v in shape:
                n *= v
            setattr(self, name, self.packed[o:o + n * esz].view(dt).view(*shape))
        self.logits = (torch.zeros(batch, DG_CANVAS, cfg.vocab, dtype=torch.float32, device=device)
                       if logits else None)
        self.route_idx = (torch.zeros(cfg.n_layers, T, cfg.top_k, dtype=torch.int32, device=device)
                          if routing else None)
        self.route_w = (torch.zeros(cfg.n_layers, T, cfg.top_k, dtype=torch.float32, device=device)
                        if routing else None)
        self.route_logits = (torch.zeros(cfg.n_layers, T, cfg.n_experts, dtype=torch.float32, device=device)
                             if routing else None)
        self.hidden = (torch.zeros(cfg.n_layers + 1, T, cfg.d_model, dtype=torch.float32, device=device)
                       if hidden else None)
        self.hidden_attn = (torch.zeros(cfg.n_layers, T, cfg.d_model, dtype=torch.float32, device=device)
                            if hidden else None)
        self.s = dg_step_out(*[t.data_ptr() if t is not None else None for t in (
            self.argmax, self.sample, self.entropy, self.pmax, self.lock, self.mean_entropy, self.stop,
            self.final_round, self.logits, self.route_idx, self.route_w, self.route_logits, self.hidden,
            self.hidden_attn)])


class Model:
    """Weights + workspace + context handle for up to `batch` canvases."""

    def __init__(self, cfg: dg_model_config, batch: int, seed: int = 0, kind_std=None, device="cuda",
                 stream=None, weights_of=None, prefill_tokens: int = 0):
        """weights_of: another Model whose weight buffer this one shares (a
        second context, e.g. for a larger batch, on the same weights).
        prefill_tokens: encode passes of up to that many tokens."""
        self.cfg = cfg
        self.batch = batch
        nw = lib.dg_weights_bytes(ctypes.byref(cfg))
        if nw == 0:
            raise ValueError(lib.dg_last_error().decode())
        nws = lib.dg_workspace_bytes_ex(ctypes.byref(cfg), batch, prefill_tokens)
        self.workspace = torch.empty(nws, dtype=torch.uint8, device=device)
        if weights_of is not None:
            assert weights_of.weights.numel() == nw
            self.weights = weights_of.weights
        else:
            self.weights = torch.empty(nw, dtype=torch.uint8, device=device)
            std = None
            if kind_std:
                arr = (ctypes.c_float * 32)()
                for kind, v in kind_std.items():
                    arr[kind] = v
                std = ctypes.cast(arr, ctypes.c_void_p)
                self._std = arr
            check(lib.dg_model_init_random(ctypes.byref(cfg), seed, std, _ptr(self.weights), _stream(stream)))
        ctx = ctypes.c_void_p()
        check(lib.dg_context_create_ex(ctypes.byref(cfg), _ptr(self.weights), _ptr(self.workspace), nws, batch,
                                       prefill_tokens, ctypes.byref(ctx)))
        self.ctx = ctx

    def close(self):
        if getattr(self, "ctx", None):
            lib.dg_context_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def encode(self, kv: KVCache, tokens: torch.Tensor, stream=None):
        assert tokens.dtype == torch.int32 and tokens.is_contiguous()
        check(lib.dg_encode_context(self.ctx, ctypes.byref(kv.s), _ptr(tokens), tokens.shape[1],
                                    _stream(stream)))

    def canvas_init(self, cv: Canvas, block: int, seed: int, stream=None):
        check(lib.dg_canvas_init(self.ctx, ctypes.byref(cv.s), block, seed, _stream(stream)))

    def step(self, kv: KVCache, cv: Canvas, block: int, step: int, sampler: dg_sampler_config,
             out: StepOutputs = None, stream=None, graph: bool = False):
        args = dg_step_args(block, step, sampler)
        fn = lib.dg_denoise_step_graph if graph else lib.dg_denoise_step
        check(fn(self.ctx, ctypes.byref(kv.s), ctypes.byref(cv.s), ctypes.byref(args),
                 ctypes.byref(out.s) if out is not None else None, _stream(stream)))

    def decode_block(self, kv: KVCache, cv: Canvas, block: int, sampler: dg_sampler_config, out_tokens,
                     stream=None, pending=None, defer_append=False):
        """One block (dg_decode_block_ex): `pending` is a finished block not
        yet in the context, appended in this block's first round;
        `defer_append` leaves this block out of the context (the next call's
        pending)."""
        steps = (ctypes.c_int32 * cv.s.batch)()
        distinct = (ctypes.c_float * self.cfg.n_layers)()
        stats = dg_block_stats(steps, 0, 0.0, distinct)
        args = dg_step_args(block, 0, sampler)
        check(lib.dg_decode_block_ex(self.ctx, ctypes.byref(kv.s), ctypes.byref(cv.s), ctypes.byref(args),
                                     _ptr(pending), 1 if defer_append else 0, _ptr(out_tokens), ctypes.byref(stats),
                                     _stream(stream)))
        self.last_block_stats = dict(tokens_per_pass=stats.tokens_per_pass, distinct_experts=list(distinct))
        return list(steps), stats.rounds

    def step_append(self, kv: KVCache, cv: Canvas, block: int, step: int, sampler: dg_sampler_config,
                    append: torch.Tensor, out: StepOutputs = None, stream=None):
        """dg_denoise_step_append: append `append` [B, 256] to the context in
        the same pass as this round."""
        assert append.dtype == torch.int32 and append.is_contiguous()
        args = dg_step_args(block, step, sampler)
        check(lib.dg_denoise_step_append(self.ctx, ctypes.byref(kv.s), ctypes.byref(cv.s), ctypes.byref(args),
                                         _ptr(append), ctypes.byref(out.s) if out is not None else None,
                                         _stream(stream)))

    def check_device(self, stream=None):
        check(lib.dg_check_device_error(self.ctx, _stream(stream)))

    def ar_step(self, kv: KVCache, tokens: torch.Tensor, temperature: float, seed: int, out_argmax: torch.Tensor,
                out_sample: torch.Tensor, out_logits: torch.Tensor = None, stream=None):
        """Autoregressive mode: append tokens [B] (int32) to the context and
        write the next token's argmax and sample [B] (int32)."""
        assert tokens.dtype == torch.int32 and out_argmax.dtype == torch.int32 and out_sample.dtype == torch.int32
        check(lib.dg_ar_step(self.ctx, ctypes.byref(kv.s), _ptr(tokens), float(temperature), int(seed),
                             _ptr(out_argmax), _ptr(out_sample), _ptr(out_logits), _stream(stream)))

    def router_probe(self, layer: int, x: torch.Tensor, out_idx: torch.Tensor, stream=None):
        """Route hidden states x [T, d] (fp32) with layer `layer`'s router into
        out_idx [T, top_k] (int32)."""
        assert x.dtype == torch.float32 and x.is_contiguous() and out_idx.dtype == torch.int32
        check(lib.dg_router_probe(self.ctx, layer, _ptr(x), x.shape[0], _ptr(out_idx), _stream(stream)))
