"""The plain C++ oracle (dg_oracle.cpp) through ctypes: one denoising round
(a1-a9) and the causal context encoding, in double precision with plain
loops, from a second implementation that shares no code with the numpy
oracle of this package.  Test infrastructure only; the library is compiled
with g++ on first use (or by the repository's build step)."""

import ctypes
import os
import subprocess

import numpy as np

import synth

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dg_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libdgoracle.so")

I32, F64, VP = ctypes.c_int32, ctypes.c_double, ctypes.c_void_p

LOCK_POLICIES = {"prob": 0, "entropy_cumsum": 1}


def build(force: bool = False) -> str:
    """Compile libdgoracle.so with g++ (no GPU needed)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off", _SRC, "-o", tmp])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class Config(ctypes.Structure):
    _fields_ = [(n, I32) for n in ("n_layers", "d_model", "n_q_heads", "n_kv_heads", "head_dim", "n_experts",
                                   "top_k", "d_ff", "vocab", "self_cond")] + [("rope_theta", F64), ("rms_eps", F64)]


class Layer(ctypes.Structure):
    _fields_ = [(n, VP) for n in ("wq", "wk", "wv", "wo", "wr", "wg", "wu", "wd")]


class Weights(ctypes.Structure):
    _fields_ = [("emb", VP), ("lm", VP), ("sc", VP), ("layers", ctypes.POINTER(Layer))]


class KV(ctypes.Structure):
    _fields_ = [("k", VP), ("v", VP), ("batch", I32), ("c_max", I32), ("length", I32)]


class Sampler(ctypes.Structure):
    _fields_ = [(n, I32) for n in ("lock_policy", "max_steps", "stop_require_stable", "persistent_lock",
                                   "selfcond_topk", "reserved")] + \
               [(n, F64) for n in ("lock_threshold", "t_start", "t_end", "stop_entropy")] + [("seed", ctypes.c_uint64)]


class State(ctypes.Structure):
    _fields_ = [(n, VP) for n in ("tokens", "sc", "prev_argmax", "done", "locked")]


class Out(ctypes.Structure):
    _fields_ = [(n, VP) for n in ("logits", "argmax", "sample", "entropy", "pmax", "mean_entropy", "stop",
                                  "final_round", "lock", "route_idx")]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.dgo_init_canvas.restype = I32
        _lib.dgo_init_canvas.argtypes = [ctypes.c_uint64, I32, I32, I32, I32, VP]
        _lib.dgo_encode_context.restype = I32
        _lib.dgo_encode_context.argtypes = [VP, VP, VP, VP, I32]
        _lib.dgo_denoise_step.restype = I32
        _lib.dgo_denoise_step.argtypes = [VP, VP, VP, I32, VP, VP, I32, I32, VP]
        _lib.dgo_philox.restype = None
        _lib.dgo_philox.argtypes = [ctypes.c_uint32] * 6 + [VP]
        _lib.dgo_bf16.restype = F64
        _lib.dgo_bf16.argtypes = [F64]
    return _lib


def _p(a):
    return a.ctypes.data if a is not None else None


class Model:
    """A model's shape and its random-init weights from the seeded generator
    (bf16 bit patterns, the tensors and ids the generator's recipe names),
    held for the C++ oracle.  `cfg` has the numpy oracle's ModelConfig
    fields; `std` maps a tensor kind to its init standard deviation."""

    def __init__(self, cfg, seed: int = 0, std=None, threads: int = 0):
        self.cfg = cfg
        std = dict(std or {})
        sd = lambda kind: std.get(kind, synth.WEIGHT_STD)  # noqa: E731
        c = cfg
        d, hd, E, f, V = c.d_model, c.head_dim, c.n_experts, c.d_ff, c.vocab
        gen = lambda rows, cols, tid, kind: np.ascontiguousarray(  # noqa: E731
            synth.bf16_rows(0, rows, cols, seed, tid, sd(kind), threads), dtype=np.uint16)
        self._keep = [gen(V, d, synth.KIND_EMB, synth.KIND_EMB), gen(V, d, synth.KIND_LM, synth.KIND_LM),
                      gen(d, d, synth.KIND_SC, synth.KIND_SC) if c.self_cond else None]
        self._layers = (Layer * c.n_layers)()
        for l in range(c.n_layers):
            t = lambda kind: synth.layer_tid(l, kind)  # noqa: E731
            ws = [gen(c.n_q_heads * hd, d, t(synth.KIND_WQ), synth.KIND_WQ),
                  gen(c.n_kv_heads * hd, d, t(synth.KIND_WK), synth.KIND_WK),
                  gen(c.n_kv_heads * hd, d, t(synth.KIND_WV), synth.KIND_WV),
                  gen(d, c.n_q_heads * hd, t(synth.KIND_WO), synth.KIND_WO),
                  gen(E, d, t(synth.KIND_WR), synth.KIND_WR),
                  gen(E * f, d, t(synth.KIND_WG), synth.KIND_WG),
                  gen(E * f, d, t(synth.KIND_WU), synth.KIND_WU),
                  gen(E * d, f, t(synth.KIND_WD), synth.KIND_WD)]
            self._keep += ws
            self._layers[l] = Layer(*[w.ctypes.data for w in ws])
        self.weights = Weights(self._keep[0].ctypes.data, self._keep[1].ctypes.data,
                               self._keep[2].ctypes.data if c.self_cond else None, self._layers)
        self.config = Config(c.n_layers, d, c.n_q_heads, c.n_kv_heads, hd, E, c.top_k, f, V, int(c.self_cond),
                             float(c.rope_theta), float(c.rms_eps))


class Cache:
    """Per layer keys and values [batch, c_max, Hkv, hd] (float32) and the
    number of valid keys."""

    def __init__(self, cfg, batch: int, c_max: int):
        shape = (batch, c_max, cfg.n_kv_heads, cfg.head_dim)
        self.k = [np.zeros(shape, np.float32) for _ in range(cfg.n_layers)]
        self.v = [np.zeros(shape, np.float32) for _ in range(cfg.n_layers)]
        self._kp = (ctypes.c_void_p * cfg.n_layers)(*[a.ctypes.data for a in self.k])
        self._vp = (ctypes.c_void_p * cfg.n_layers)(*[a.ctypes.data for a in self.v])
        self.kv = KV(ctypes.cast(self._kp, VP), ctypes.cast(self._vp, VP), batch, c_max, 0)

    @property
    def length(self):
        return self.kv.length


def init_canvas(seed: int, block: int, batch: int, n_pos: int, vocab: int) -> np.ndarray:
    out = np.zeros((batch, n_pos), np.int64)
    assert lib().dgo_init_canvas(seed, block, batch, n_pos, vocab, out.ctypes.data) == 0
    return out


def encode_context(model: Model, cache: Cache, tokens) -> None:
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    st = lib().dgo_encode_context(ctypes.byref(model.config), ctypes.byref(model.weights), ctypes.byref(cache.kv),
                                  tokens.ctypes.data, tokens.shape[1])
    assert st == 0, "dgo_encode_context: bad arguments"


def sampler(lock_policy="prob", lock_threshold=0.9, t_start=0.8, t_end=0.4, max_steps=48, stop_entropy=0.5,
            stop_require_stable=False, seed=0, persistent_lock=False, selfcond_topk=0) -> Sampler:
    return Sampler(LOCK_POLICIES[lock_policy], max_steps, int(stop_require_stable), int(persistent_lock),
                   selfcond_topk, 0, lock_threshold, t_start, t_end, stop_entropy, seed)


def denoise_step(model: Model, cache: Cache, state: dict, samp: Sampler, block: int, step: int) -> dict:
    """One round; `state` holds numpy arrays tokens [B, N] int64, sc [B, N, d]
    float64, prev_argmax [B, N] int64, done [B] uint8 and locked [B, N] uint8,
    updated in place.  Returns the round's outputs as numpy arrays."""
    c = model.cfg
    B, N = state["tokens"].shape
    o = {"logits": np.zeros((B, N, c.vocab), np.float32), "argmax": np.zeros((B, N), np.int64),
         "sample": np.zeros((B, N), np.int64), "entropy": np.zeros((B, N)), "pmax": np.zeros((B, N)),
         "mean_entropy": np.zeros(B), "stop": np.zeros(B, np.uint8), "final": np.zeros(B, np.uint8),
         "lock": np.zeros((B, N), np.uint8), "route_idx": np.zeros((c.n_layers, B * N, c.top_k), np.int32)}
    out = Out(*[_p(o[n]) for n in ("logits", "argmax", "sample", "entropy", "pmax", "mean_entropy", "stop",
                                   "final", "lock", "route_idx")])
    for n in ("tokens", "prev_argmax"):
        assert state[n].dtype == np.int64 and state[n].flags.c_contiguous
    st = State(_p(state["tokens"]), _p(state["sc"]), _p(state["prev_argmax"]), _p(state["done"]), _p(state["locked"]))
    r = lib().dgo_denoise_step(ctypes.byref(model.config), ctypes.byref(model.weights), ctypes.byref(cache.kv), N,
                               ctypes.byref(st), ctypes.byref(samp), block, step, ctypes.byref(out))
    assert r == 0, "dgo_denoise_step: bad arguments"
    o["route_idx"] = o["route_idx"].reshape(c.n_layers, B, N, c.top_k)
    return o
