"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

Nothing here computes any part of the decoding method.  The module turns
(seed, stream, index) counters into weights, prompts and window states (see
``synth.c`` for the generator's definition) and describes the workload shapes.
The C source is compiled on first use with the host compiler into
``libwedlm_synth.so`` next to this file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .workloads import CONFIGS, model_dims  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_SO = os.path.join(_HERE, "libwedlm_synth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile synth.c into libwedlm_synth.so (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i64, i32, f64 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
            vp = ctypes.c_void_p
            lib.synth_normal_f32.argtypes = [u64, u64, f64, vp, i64]
            lib.synth_normal_bf16.argtypes = [u64, u64, f64, vp, i64]
            lib.synth_token_ids.argtypes = [u64, u64, i32, i32, vp, i64]
            lib.synth_uniform01.argtypes = [u64, u64, vp, i64]
            lib.synth_raw_u64.argtypes = [u64, u64, vp, i64]
            lib.synth_normal_scale.argtypes = [f64]
            lib.synth_normal_scale.restype = ctypes.c_float
            _lib = lib
    return _lib


def normal(seed: int, stream: int, std: float, shape, dtype: str = "f32") -> np.ndarray:
    """N(0, std^2)-shaped values (Irwin-Hall(4)); dtype 'f32' -> float32, 'bf16' -> uint16 bf16 bits."""
    lib = _load()
    n = int(np.prod(shape))
    if dtype == "f32":
        out = np.empty(shape, dtype=np.float32)
        lib.synth_normal_f32(seed, stream, std, out.ctypes.data, n)
    elif dtype == "bf16":
        out = np.empty(shape, dtype=np.uint16)
        lib.synth_normal_bf16(seed, stream, std, out.ctypes.data, n)
    else:
        raise ValueError(dtype)
    return out


def token_ids(seed: int, stream: int, vocab: int, n: int, exclude: int = -1) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.int32)
    lib.synth_token_ids(seed, stream, vocab, exclude, out.ctypes.data, n)
    return out


def uniform01(seed: int, stream: int, n: int) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.float64)
    lib.synth_uniform01(seed, stream, out.ctypes.data, n)
    return out


def raw_u64(seed: int, stream: int, n: int) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.uint64)
    lib.synth_raw_u64(seed, stream, out.ctypes.data, n)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


# --- model weights ---------------------------------------------------------
# Tensor kinds, matching the C-ABI's tensor enumeration.
T_EMBED, T_LM_HEAD, T_FINAL_NORM, T_ATTN_NORM, T_WQ, T_WK, T_WV, T_WO, T_FFN_NORM, T_WG, T_WU, T_WD = range(12)
_LAYER_STREAM = {T_WQ: 0, T_WK: 1, T_WV: 2, T_WO: 3, T_WG: 4, T_WU: 5, T_WD: 6}
WEIGHT_STD = 0.02


def tensor_shape(dims: dict, kind: int):
    d, hq, hkv, hd, F, V = dims["d"], dims["hq"], dims["hkv"], dims["hd"], dims["F"], dims["V"]
    return {
        T_EMBED: (V, d), T_LM_HEAD: (V, d), T_FINAL_NORM: (d,), T_ATTN_NORM: (d,), T_FFN_NORM: (d,),
        T_WQ: (hq * hd, d), T_WK: (hkv * hd, d), T_WV: (hkv * hd, d), T_WO: (d, hq * hd),
        T_WG: (F, d), T_WU: (F, d), T_WD: (d, F),
    }[kind]


def weight_tensor(dims: dict, kind: int, layer: int, seed: int = 0, dtype: str = "f32") -> np.ndarray:
    """One weight tensor in nn.Linear layout [out_features, in_features].

    RMSNorm gains are all ones (float32).  Matrices are N(0, 0.02^2)-shaped
    draws from stream 1 (embedding), 2 (LM head) or 16 + 16*layer + j (layer
    matrices, j = q,k,v,o,gate,up,down)."""
    shape = tensor_shape(dims, kind)
    if kind in (T_FINAL_NORM, T_ATTN_NORM, T_FFN_NORM):
        return np.ones(shape, dtype=np.float32)
    if kind == T_EMBED:
        stream = 1
    elif kind == T_LM_HEAD:
        stream = 2
    else:
        stream = 16 + 16 * layer + _LAYER_STREAM[kind]
    return normal(seed, stream, WEIGHT_STD, shape, dtype)


def iter_weights(dims: dict, seed: int = 0, dtype: str = "f32"):
    """Yield (kind, layer, array) for every tensor of the model, one at a time."""
    yield T_EMBED, 0, weight_tensor(dims, T_EMBED, 0, seed, dtype)
    yield T_LM_HEAD, 0, weight_tensor(dims, T_LM_HEAD, 0, seed, dtype)
    yield T_FINAL_NORM, 0, weight_tensor(dims, T_FINAL_NORM, 0, seed, dtype)
    for l in range(dims["L"]):
        for kind in (T_ATTN_NORM, T_WQ, T_WK, T_WV, T_WO, T_FFN_NORM, T_WG, T_WU, T_WD):
            yield kind, l, weight_tensor(dims, kind, l, seed, dtype)


def model_weights(dims: dict, seed: int = 0, dtype: str = "f32") -> dict:
    """All weights as a dict keyed like the oracle expects (see oracle.Weights)."""
    w = {"layers": [dict() for _ in range(dims["L"])]}
    names = {T_ATTN_NORM: "attn_norm", T_WQ: "wq", T_WK: "wk", T_WV: "wv", T_WO: "wo",
             T_FFN_NORM: "ffn_norm", T_WG: "wg", T_WU: "wu", T_WD: "wd"}
    for kind, l, arr in iter_weights(dims, seed, dtype):
        if kind == T_EMBED:
            w["embed"] = arr
        elif kind == T_LM_HEAD:
            w["lm_head"] = arr
        elif kind == T_FINAL_NORM:
            w["final_norm"] = arr
        else:
            w["layers"][l][names[kind]] = arr
    w["dtype"] = dtype
    return w


# --- workloads -------------------------------------------------------------
def prompts(cfg: dict, seed: int | None = None):
    """Per-sequence prompts (list of int32 arrays) for a workload config."""
    dims = model_dims(cfg)
    seed = cfg.get("prompt_seed", 1000) if seed is None else seed
    B = cfg["B"]
    P = cfg["P"]
    if isinstance(P, (tuple, list)):
        lo, hi = P
        u = uniform01(seed, 1_000_000, B)
        lens = [int(lo + np.floor(x * (hi - lo + 1))) for x in u]
    else:
        lens = [int(P)] * B
    return [token_ids(seed, b, dims["V"], lens[b], exclude=dims["mask_id"]) for b in range(B)]


def window_state(seed: int, stream: int, n_seq: int, W: int, n_filled: int | None, vocab: int, mask_id: int):
    """Random window states: filled flags [n_seq, W] (uint8) and tokens [n_seq, W] (int32).

    With n_filled=None each slot is filled with probability 1/2; otherwise exactly
    n_filled slots per sequence are filled at random offsets."""
    u = uniform01(seed, stream, n_seq * W).reshape(n_seq, W)
    if n_filled is None:
        filled = (u < 0.5).astype(np.uint8)
    else:
        order = np.argsort(u, axis=1, kind="stable")
        filled = np.zeros((n_seq, W), np.uint8)
        for b in range(n_seq):
            filled[b, order[b, :n_filled]] = 1
    toks = token_ids(seed, stream + 1, vocab, n_seq * W, exclude=mask_id).reshape(n_seq, W)
    toks = np.where(filled == 1, toks, mask_id).astype(np.int32)
    return filled, toks


def paged_kv(seed: int, lengths, hkv: int, hd: int = 128, std: float = 1.0, spare_pages: int = 3):
    """A one-layer paged KV pool with seeded random page tables.

    Returns (pool, page_table): pool holds bf16 bits (uint16) [num_pages][2 (K, V)]
    [hkv][16][hd] of N(0, std^2)-shaped values; page_table [n_seq][pages_per_seq]
    (int32, -1 past a sequence's pages) maps sequence b's 16-token block i to a
    page, the pages being a seeded random permutation of the pool (so a
    sequence's pages are scattered).  Position p of sequence b lives in page
    page_table[b][p // 16], token p % 16."""
    lengths = [int(x) for x in lengths]
    need = [(x + 15) // 16 for x in lengths]
    num_pages = sum(need) + spare_pages
    pps = max(1, max(need) if need else 1)
    order = np.argsort(uniform01(seed, 7_000_001, num_pages), kind="stable").astype(np.int32)
    table = np.full((len(lengths), pps), -1, np.int32)
    k = 0
    for b, m in enumerate(need):
        table[b, :m] = order[k:k + m]
        k += m
    pool = normal(seed, 7_000_002, std, (num_pages, 2, hkv, 16, hd), "bf16")
    return pool, table
