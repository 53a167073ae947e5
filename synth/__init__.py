"""Seeded synthetic inputs (weights, token ids, hidden states) for both the
CUDA library and the CPU oracle.  See synth.h for the recipe.

This module holds none of the denoising method's arithmetic.  The host
generator is a small C library (libdgsynth.so, built from synth_host.c on
first use); the CUDA library carries the device twin (synth_device.cu).
"""

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdgsynth.so")

KIND_EMB = 1
KIND_LM = 2
KIND_SC = 3
KIND_CTX = 4
KIND_HIDDEN = 5
KIND_WQ = 16
KIND_WK = 17
KIND_WV = 18
KIND_WO = 19
KIND_WR = 20
KIND_WG = 21
KIND_WU = 22
KIND_WD = 23

WEIGHT_STD = 0.02


def layer_tid(layer: int, kind: int) -> int:
    return ((layer + 1) << 5) | kind


def ctx_tid(canvas: int) -> int:
    return KIND_CTX | (canvas << 8)


def build(force: bool = False) -> str:
    """Compile libdgsynth.so with gcc (no GPU needed)."""
    src = os.path.join(_HERE, "synth_host.c")
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(src),
                                                    os.path.getmtime(os.path.join(_HERE, "synth.h")))):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           "-ffp-contract=off", src, "-o", tmp])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        i64, u64, u32, dbl = ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_double
        _lib.synth_fill_bf16_host.argtypes = [ctypes.c_void_p, i64, i64, i64, i64, i64, u64, u32,
                                              dbl, ctypes.c_int]
        _lib.synth_fill_f32_host.argtypes = [ctypes.c_void_p, i64, u64, u32, dbl, ctypes.c_int]
        _lib.synth_fill_tokens_host.argtypes = [ctypes.c_void_p, i64, u64, u32, ctypes.c_int32]
        _lib.synth_philox4x32_10.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        for f in (_lib.synth_fill_bf16_host, _lib.synth_fill_f32_host, _lib.synth_fill_tokens_host):
            f.restype = ctypes.c_int
    return _lib


def bf16_rows(row0: int, nrows: int, cols: int, seed: int, tid: int, std: float = WEIGHT_STD,
              threads: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of rows [row0, row0 + nrows) of a logical
    row-major [*, cols] tensor."""
    out = np.empty((int(nrows), int(cols)), dtype=np.uint16)
    if nrows == 0:
        return out
    rc = lib().synth_fill_bf16_host(out.ctypes.data, int(row0), int(nrows), int(cols), int(cols), 1,
                                    int(seed), int(tid), float(std), int(threads))
    if rc:
        raise RuntimeError("synth_fill_bf16_host failed")
    return out


def bf16_tensor(shape, seed: int, tid: int, std: float = WEIGHT_STD, threads: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of a whole logical tensor, row-major in `shape`."""
    shape = tuple(int(s) for s in shape)
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    return bf16_rows(0, rows, shape[-1], seed, tid, std, threads).reshape(shape)


def f32_tensor(n: int, seed: int, tid: int, std: float = 1.0, threads: int = 0) -> np.ndarray:
    out = np.empty(int(n), dtype=np.float32)
    if lib().synth_fill_f32_host(out.ctypes.data, int(n), seed, tid, std, threads):
        raise RuntimeError("synth_fill_f32_host failed")
    return out


def tokens(n: int, seed: int, tid: int, vocab: int) -> np.ndarray:
    out = np.empty(int(n), dtype=np.int32)
    if lib().synth_fill_tokens_host(out.ctypes.data, int(n), seed, tid, vocab):
        raise RuntimeError("synth_fill_tokens_host failed")
    return out


def context_tokens(batch: int, n: int, seed: int, vocab: int) -> np.ndarray:
    """[B, n] context token ids, canvas b drawn from tensor id ctx_tid(b)."""
    return np.stack([tokens(n, seed, ctx_tid(b), vocab) for b in range(batch)]) if batch else \
        np.zeros((0, n), np.int32)


def philox4x32_10(ctr, key):
    c = (ctypes.c_uint32 * 4)(*[int(v) & 0xFFFFFFFF for v in ctr])
    k = (ctypes.c_uint32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    o = (ctypes.c_uint32 * 4)()
    lib().synth_philox4x32_10(ctypes.addressof(c), ctypes.addressof(k), ctypes.addressof(o))
    return tuple(int(v) for v in o)
