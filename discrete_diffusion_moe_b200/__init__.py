"""Python binding of libdg.so, the sm_100a DiffusionGemma denoising-step library.

Argument marshalling only: every step of the method runs in the library's
CUDA kernels.  PyTorch is used for device memory and streams.  The binding
fails loudly when the compiled library is missing; there is no fallback.

The C ABI is declared in include/dg.h (and the GEMM test hooks in
include/dg_testing.h); the names here are the same.
"""

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdg.so")

DG_CANVAS = 256
DG_OK, DG_ERR_INVALID_ARG, DG_ERR_CUDA, DG_ERR_WORKSPACE, DG_ERR_TIMEOUT, DG_ERR_UNSUPPORTED, \
    DG_ERR_BAD_TOKEN = range(7)
DG_LOCK_PROB, DG_LOCK_ENTROPY_CUMSUM = 0, 1
DG_DECODE_DEFER_APPEND = 1

# size of the library's fixed split-KV scratch array (dg_attention_static_scratch)
DG_ATTN_STATIC_SCRATCH_BYTES = 16 << 20

_STATUS_NAMES = {0: "DG_OK", 1: "DG_ERR_INVALID_ARG", 2: "DG_ERR_CUDA", 3: "DG_ERR_WORKSPACE",
                 4: "DG_ERR_TIMEOUT", 5: "DG_ERR_UNSUPPORTED", 6: "DG_ERR_BAD_TOKEN"}


class DgError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{_STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class dg_model_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("self_cond", ctypes.c_int32), ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float)]


class dg_sampler_config(ctypes.Structure):
    _fields_ = [("lock_policy", ctypes.c_int32), ("lock_threshold", ctypes.c_float),
                ("t_start", ctypes.c_float), ("t_end", ctypes.c_float), ("max_steps", ctypes.c_int32),
                ("stop_entropy", ctypes.c_float), ("stop_require_stable_argmax", ctypes.c_int32),
                ("seed", ctypes.c_uint64), ("persistent_lock", ctypes.c_int32), ("selfcond_topk", ctypes.c_int32)]


class dg_kv(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("c_max", ctypes.c_int32), ("length", ctypes.c_int32)]


class dg_canvas(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_void_p), ("sc_state", ctypes.c_void_p), ("prev_argmax", ctypes.c_void_p),
                ("done", ctypes.c_void_p), ("batch", ctypes.c_int32), ("locked", ctypes.c_void_p)]


class dg_step_args(ctypes.Structure):
    _fields_ = [("block", ctypes.c_int32), ("step", ctypes.c_int32), ("sampler", dg_sampler_config)]


class dg_step_out(ctypes.Structure):
    _fields_ = [("argmax", ctypes.c_void_p), ("sample", ctypes.c_void_p), ("entropy", ctypes.c_void_p),
                ("pmax", ctypes.c_void_p), ("lock", ctypes.c_void_p), ("mean_entropy", ctypes.c_void_p),
                ("stop", ctypes.c_void_p), ("final_round", ctypes.c_void_p), ("logits", ctypes.c_void_p),
                ("route_idx", ctypes.c_void_p), ("route_w", ctypes.c_void_p), ("route_logits", ctypes.c_void_p),
                ("hidden", ctypes.c_void_p), ("hidden_attn", ctypes.c_void_p)]


DG_PROF_EXPERT_GATE_UP, DG_PROF_EXPERT_DOWN, DG_PROF_LM_HEAD, DG_PROF_ATTENTION, DG_PROF_DENSE, \
    DG_PROF_EXPECTED_EMB = range(6)


class dg_profile(ctypes.Structure):
    _fields_ = [("ms", ctypes.c_double * 6), ("launches", ctypes.c_int32 * 6), ("launches_total", ctypes.c_int64)]


class dg_block_stats(ctypes.Structure):
    _fields_ = [("steps_taken", ctypes.POINTER(ctypes.c_int32)), ("rounds", ctypes.c_int32),
                ("tokens_per_pass", ctypes.c_float), ("distinct_experts", ctypes.POINTER(ctypes.c_float))]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python discrete_diffusion_moe_b200/build.py` "
            "(nvcc, sm_100a); this package has no CPU fallback")
    lib = ctypes.CDLL(LIB_PATH)
    P, S, I32, U64, F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint64, ctypes.c_float
    cfgp = ctypes.POINTER(dg_model_config)
    sig = {
        "dg_last_error": (ctypes.c_char_p, []),
        "dg_weights_bytes": (S, [cfgp]),
        "dg_kv_bytes": (S, [cfgp, I32, I32]),
        "dg_workspace_bytes": (S, [cfgp, I32]),
        "dg_workspace_bytes_ex": (S, [cfgp, I32, I32]),
        "dg_context_create_ex": (I32, [cfgp, P, P, S, I32, I32, ctypes.POINTER(P)]),
        "dg_model_init_random": (I32, [cfgp, U64, P, P, P]),
        "dg_context_create": (I32, [cfgp, P, P, S, I32, ctypes.POINTER(P)]),
        "dg_context_destroy": (None, [P]),
        "dg_encode_context": (I32, [P, ctypes.POINTER(dg_kv), P, I32, P]),
        "dg_canvas_init": (I32, [P, ctypes.POINTER(dg_canvas), I32, U64, P]),
        "dg_denoise_step": (I32, [P, ctypes.POINTER(dg_kv), ctypes.POINTER(dg_canvas),
                                  ctypes.POINTER(dg_step_args), ctypes.POINTER(dg_step_out), P]),
        "dg_denoise_step_graph": (I32, [P, ctypes.POINTER(dg_kv), ctypes.POINTER(dg_canvas),
                                        ctypes.POINTER(dg_step_args), ctypes.POINTER(dg_step_out), P]),
        "dg_decode_block": (I32, [P, ctypes.POINTER(dg_kv), ctypes.POINTER(dg_canvas),
                                  ctypes.POINTER(dg_step_args), P, ctypes.POINTER(dg_block_stats), P]),
        "dg_check_device_error": (I32, [P, P]),
        "dg_denoise_step_append": (I32, [P, ctypes.POINTER(dg_kv), ctypes.POINTER(dg_canvas),
                                         ctypes.POINTER(dg_step_args), P, ctypes.POINTER(dg_step_out), P]),
        "dg_decode_block_ex": (I32, [P, ctypes.POINTER(dg_kv), ctypes.POINTER(dg_canvas),
                                     ctypes.POINTER(dg_step_args), P, I32, P, ctypes.POINTER(dg_block_stats), P]),
        "dg_profile_start": (I32, [P]),
        "dg_profile_stop": (I32, [P, ctypes.POINTER(dg_profile)]),
        "dg_test_gemm": (I32, [P, I32, P, I32, I32, P, I32, P]),
        "dg_test_gemm_tiles": (I32, [P, I32, P, I32, I32, P, I32, I32, I32, P]),
        "dg_test_grouped_gemm": (I32, [P, I32, I32, P, I32, I32, P, P, I32, P, P]),
        "dg_test_grouped_schedule": (I32, [I32, I32, I32, P, I32, I32, P, I32, P]),
        "dg_test_dense_schedule": (I32, [I32, I32, I32, I32, I32, I32, I32, P, I32, P]),
        "dg_test_attention": (I32, [P, P, P, P, I32, I32, I32, I32, I32, I32, I32, I32, I32, P, P, P]),
        "dg_test_workspace_buffer": (I32, [P, ctypes.c_char_p, ctypes.POINTER(P), ctypes.POINTER(S)]),
        "dg_test_wait_timeout": (I32, [P, ctypes.c_int64, P]),
        "dg_test_struct_size": (S, [ctypes.c_char_p]),
        "dg_test_expected_embedding_topk": (I32, [P, ctypes.c_int64, I32, P, I32, I32, P, P]),
        "dg_router_probe": (I32, [P, I32, P, I32, P, P]),
        "dg_ar_step": (I32, [P, ctypes.POINTER(dg_kv), P, F, U64, P, P, P, P]),
        "dg_attention_static_scratch": (I32, [P, P, P, P, I32, I32, I32, I32, I32, I32, I32, I32, I32, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def last_error() -> str:
    return lib.dg_last_error().decode(errors="replace")


def check(status: int):
    if status != DG_OK:
        raise DgError(status, last_error())


# ---- thin wrappers with the ABI's names (marshalling only) -------------------

def dg_weights_bytes(cfg: dg_model_config) -> int:
    return lib.dg_weights_bytes(ctypes.byref(cfg))


def dg_kv_bytes(cfg: dg_model_config, batch: int, c_max: int) -> int:
    return lib.dg_kv_bytes(ctypes.byref(cfg), batch, c_max)


def dg_workspace_bytes(cfg: dg_model_config, batch: int) -> int:
    return lib.dg_workspace_bytes(ctypes.byref(cfg), batch)


def dg_model_init_random(cfg, seed, kind_std_ptr, d_weights, stream):
    return lib.dg_model_init_random(ctypes.byref(cfg), seed, kind_std_ptr, d_weights, stream)


def dg_context_create(cfg, d_weights, d_ws, ws_bytes, batch):
    out = ctypes.c_void_p()
    check(lib.dg_context_create(ctypes.byref(cfg), d_weights, d_ws, ws_bytes, batch, ctypes.byref(out)))
    return out


def dg_context_destroy(ctx):
    lib.dg_context_destroy(ctx)


def dg_encode_context(ctx, kv: dg_kv, d_tokens, n, stream):
    return lib.dg_encode_context(ctx, ctypes.byref(kv), d_tokens, n, stream)


def dg_canvas_init(ctx, cv: dg_canvas, block, seed, stream):
    return lib.dg_canvas_init(ctx, ctypes.byref(cv), block, seed, stream)


def dg_denoise_step(ctx, kv: dg_kv, cv: dg_canvas, args: dg_step_args, out, stream):
    return lib.dg_denoise_step(ctx, ctypes.byref(kv), ctypes.byref(cv), ctypes.byref(args),
                               ctypes.byref(out) if out is not None else None, stream)


def dg_denoise_step_graph(ctx, kv: dg_kv, cv: dg_canvas, args: dg_step_args, out, stream):
    return lib.dg_denoise_step_graph(ctx, ctypes.byref(kv), ctypes.byref(cv), ctypes.byref(args),
                                     ctypes.byref(out) if out is not None else None, stream)


def dg_decode_block(ctx, kv: dg_kv, cv: dg_canvas, args: dg_step_args, d_out, stats, stream):
    return lib.dg_decode_block(ctx, ctypes.byref(kv), ctypes.byref(cv), ctypes.byref(args), d_out,
                               ctypes.byref(stats) if stats is not None else None, stream)


def dg_check_device_error(ctx, stream):
    return lib.dg_check_device_error(ctx, stream)


def dg_profile_start(ctx):
    return lib.dg_profile_start(ctx)


def dg_profile_stop(ctx, out: dg_profile):
    return lib.dg_profile_stop(ctx, ctypes.byref(out))


def dg_test_gemm(d_a, M, d_b, N, K, d_d, k_splits, stream):
    return lib.dg_test_gemm(d_a, M, d_b, N, K, d_d, k_splits, stream)


def dg_test_grouped_gemm(d_a, rows_per_group, n_groups, d_b, n_rows, K, d_off, d_d, bn, d_chunk_off, stream):
    return lib.dg_test_grouped_gemm(d_a, rows_per_group, n_groups, d_b, n_rows, K, d_off, d_d, bn, d_chunk_off,
                                    stream)


from .runtime import Model, KVCache, Canvas, StepOutputs, sampler_config, model_config  # noqa: E402,F401
