"""Python binding of libwedlm: the C-ABI calls under the same names, with
argument marshalling only.  Every step of the decode path runs in the CUDA
library; this module never computes any part of it.

Host arrays are numpy; device buffers are torch CUDA tensors (PyTorch supplies
device memory and streams)."""
from __future__ import annotations

import ctypes

import numpy as np

from . import _lib
from ._lib import ModelCfg, SeqStats, StepParams, WedlmError

C = _lib.header_constants()
DTYPE = {"f32": C["WEDLM_DTYPE_F32"], "bf16": C["WEDLM_DTYPE_BF16"]}


def _ptr(a) -> int:
    if a is None:
        return 0
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return int(a.data_ptr())  # torch tensor


def _check(st: int, where: str, ctx=None):
    if st != 0:
        detail = _lib.load().wedlm_last_error(ctx).decode() if ctx else ""
        raise WedlmError(st, where, detail)


def step_params(lam: float, tau: float, tau_none: bool = False, logit_scale: float = 1.0, blockwise: bool = False,
                temperature: float = 0.0, seed: int = 0) -> StepParams:
    return StepParams(float(lam), float(tau), 1 if tau_none else 0, float(logit_scale), 1 if blockwise else 0,
                      float(temperature), int(seed))


class Engine:
    """One libwedlm context (one model, a batch of sequence slots)."""

    def __init__(self, dims: dict, max_batch: int, max_window: int, max_ctx: int, dtype: str | None = None,
                 num_pages: int = 0, prefill_chunk: int = 0, stream=None):
        self.lib = _lib.load()
        self.dims = dict(dims)
        dtype = dtype or dims.get("dtype", "f32")
        self.dtype = dtype
        cfg = ModelCfg(dims["L"], dims["d"], dims["hq"], dims["hkv"], dims["hd"], dims["F"], dims["V"],
                       dims["mask_id"], float(dims["theta"]), float(dims["eps"]), DTYPE[dtype], max_batch,
                       max_window, max_ctx, num_pages, prefill_chunk)
        self.max_batch, self.max_window, self.max_ctx = max_batch, max_window, max_ctx
        self.stream = stream
        h = ctypes.c_void_p()
        _check(self.lib.wedlm_create(ctypes.byref(cfg), ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(h)),
               "wedlm_create")
        self.ctx = h

    # -- lifetime ---------------------------------------------------------
    def close(self):
        if getattr(self, "ctx", None):
            self.lib.wedlm_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    # -- weights ------------------------------------------------------------
    def load_weights(self, kind: int, layer: int, src):
        """src: numpy array (host) or torch CUDA tensor (device); float32 or bf16 (uint16 bits / torch.bfloat16)."""
        if isinstance(src, np.ndarray):
            src = np.ascontiguousarray(src)
            dt = C["WEDLM_DTYPE_BF16"] if src.dtype == np.uint16 else C["WEDLM_DTYPE_F32"]
            if src.dtype not in (np.uint16, np.float32):
                raise TypeError(src.dtype)
            mem = C["WEDLM_MEM_HOST"]
        else:
            import torch
            dt = C["WEDLM_DTYPE_BF16"] if src.dtype in (torch.bfloat16, torch.int16) else C["WEDLM_DTYPE_F32"]
            mem = C["WEDLM_MEM_DEVICE"] if src.is_cuda else C["WEDLM_MEM_HOST"]
            src = src.contiguous()
        _check(self.lib.wedlm_load_weights(self.ctx, kind, layer, _ptr(src), dt, mem), "wedlm_load_weights",
               self.ctx)

    def load_model(self, weight_iter):
        for kind, layer, arr in weight_iter:
            self.load_weights(kind, layer, arr)

    # -- sequences -----------------------------------------------------------
    def prefill(self, slot: int, prompt, max_new_tokens: int, window: int):
        p = np.ascontiguousarray(np.asarray(prompt, dtype=np.int32))
        _check(self.lib.wedlm_prefill(self.ctx, slot, p.ctypes.data if len(p) else None, len(p), max_new_tokens,
                                      window), "wedlm_prefill", self.ctx)

    def kv_reset(self, slot: int = -1):
        _check(self.lib.wedlm_kv_reset(self.ctx, slot), "wedlm_kv_reset", self.ctx)

    def stream_step(self, params: StepParams):
        """One decode step: returns (committed tokens per slot, counts, active)."""
        committed = np.zeros((self.max_batch, self.max_window), np.int32)
        counts = np.zeros(self.max_batch, np.int32)
        active = np.zeros(1, np.int32)
        _check(self.lib.wedlm_stream_step(self.ctx, ctypes.byref(params), committed.ctypes.data, counts.ctypes.data,
                                          active.ctypes.data), "wedlm_stream_step", self.ctx)
        return [committed[b, :counts[b]].tolist() for b in range(self.max_batch)], counts, int(active[0])

    def stream_step_into(self, params: StepParams, committed: np.ndarray, counts: np.ndarray, active: np.ndarray):
        """Same as stream_step with caller-provided (e.g. pinned) host buffers."""
        _check(self.lib.wedlm_stream_step(self.ctx, ctypes.byref(params), _ptr(committed), _ptr(counts),
                                          _ptr(active)), "wedlm_stream_step", self.ctx)

    def stream_step_async(self, params: StepParams, n_steps: int = 1):
        _check(self.lib.wedlm_stream_step_async(self.ctx, ctypes.byref(params), n_steps), "wedlm_stream_step_async",
               self.ctx)

    def read_generated(self, slot: int) -> list:
        buf = np.zeros(self.max_ctx, np.int32)
        n = ctypes.c_int32()
        _check(self.lib.wedlm_read_generated(self.ctx, slot, buf.ctypes.data, len(buf), ctypes.byref(n)),
               "wedlm_read_generated", self.ctx)
        return buf[:n.value].tolist()

    def stats(self, slot: int) -> dict:
        s = SeqStats()
        _check(self.lib.wedlm_get_stats(self.ctx, slot, ctypes.byref(s)), "wedlm_get_stats", self.ctx)
        return {f: getattr(s, f) for f, _ in SeqStats._fields_}

    def kernel_launches(self) -> int:
        n = ctypes.c_int64()
        _check(self.lib.wedlm_kernel_launches(self.ctx, ctypes.byref(n)), "wedlm_kernel_launches")
        return n.value

    def autotune(self, enable: bool = True):
        _check(self.lib.wedlm_autotune(self.ctx, 1 if enable else 0), "wedlm_autotune", self.ctx)

    def keep_logits(self, enable: bool = True):
        """Test hook: True writes logits every step (two-pass LM head + entropy)."""
        _check(self.lib.wedlm_debug_keep_logits(self.ctx, 1 if enable else 0), "wedlm_debug_keep_logits", self.ctx)

    def force_fused_entropy(self, enable: bool = True):
        """Test hook: greedy bf16 steps always take the fused LM-head entropy epilogue."""
        _check(self.lib.wedlm_debug_keep_logits(self.ctx, 2 if enable else 0), "wedlm_debug_keep_logits", self.ctx)

    def debug_capture(self, enable: bool = True):
        """Keep the residual stream at every layer boundary of each decode step (test hook)."""
        _check(self.lib.wedlm_debug_capture(self.ctx, 1 if enable else 0), "wedlm_debug_capture", self.ctx)

    def debug_residual(self, layer: int, rows: int) -> np.ndarray:
        """x entering `layer` (layer = L: after the last layer), [rows][d] fp32, of the last step."""
        out = np.empty((rows, self.dims["d"]), np.float32)
        _check(self.lib.wedlm_debug_residual(self.ctx, layer, out.ctypes.data, rows), "wedlm_debug_residual",
               self.ctx)
        return out

    def gemm_plan(self, kind: str, rows: int):
        """(tile_w, tile_n, k_splits, us) recorded for a projection kind ('gemm_qkv', ...) at `rows`, or None."""
        tw, tn, ks, us = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32(), ctypes.c_float()
        st = self.lib.wedlm_gemm_plan(self.ctx, C["WEDLM_PROF_" + kind.upper()], rows, ctypes.byref(tw),
                                      ctypes.byref(tn), ctypes.byref(ks), ctypes.byref(us))
        return (tw.value, tn.value, ks.value, round(us.value, 2)) if st == 0 else None

    def gemm_schedule(self, kind: str, rows: int):
        """Names of the schedule features of the recorded plan (CTA pairs, hybrid or
        cluster K split, ...), or None."""
        sc = ctypes.c_int32()
        st = self.lib.wedlm_gemm_schedule(self.ctx, C["WEDLM_PROF_" + kind.upper()], rows, ctypes.byref(sc))
        if st != 0:
            return None
        names = {1: "cta_pair", 2: "hybrid_split", 4: "cluster_split", 8: "co_resident_fixup",
                 16: "two_weight_subtiles", 32: "bk32"}
        return [n for bit, n in names.items() if sc.value & bit]

    def profile_enable(self, on: bool = True):
        _check(self.lib.wedlm_profile_enable(self.ctx, 1 if on else 0), "wedlm_profile_enable", self.ctx)

    def profile_read(self) -> dict:
        """{kind: (total ms, launches)} for kinds WEDLM_PROF_* since profile_enable."""
        nk = C["WEDLM_PROF_KINDS"]
        ms = np.zeros(nk, np.float64)
        n = np.zeros(nk, np.int64)
        _check(self.lib.wedlm_profile_read(self.ctx, ms.ctypes.data, n.ctypes.data), "wedlm_profile_read", self.ctx)
        names = {v: k[len("WEDLM_PROF_"):].lower() for k, v in C.items()
                 if k.startswith("WEDLM_PROF_") and k != "WEDLM_PROF_KINDS"}
        return {names[i]: (float(ms[i]), int(n[i])) for i in range(nk)}

    # -- test hooks ---------------------------------------------------------
    def debug_read(self, item: str, shape, dtype):
        out = np.zeros(shape, dtype)
        _check(self.lib.wedlm_debug_read(self.ctx, C["WEDLM_DBG_" + item], out.ctypes.data, out.nbytes),
               "wedlm_debug_read", self.ctx)
        return out

    def last_rows(self):
        v = self.debug_read("ROWSTRIDE", 2, np.int32)
        return int(v[0]), int(v[1])

    def debug_kv(self, slot: int, layer: int, pos0: int, n: int):
        hkv, hd = self.dims["hkv"], self.dims["hd"]
        k = np.zeros((n, hkv, hd), np.float32)
        v = np.zeros((n, hkv, hd), np.float32)
        _check(self.lib.wedlm_debug_kv(self.ctx, slot, layer, pos0, n, k.ctypes.data, v.ctypes.data),
               "wedlm_debug_kv", self.ctx)
        return k, v

    def get_window(self, slot: int):
        f = np.zeros(self.max_window, np.uint8)
        t = np.zeros(self.max_window, np.int32)
        n = ctypes.c_int32()
        _check(self.lib.wedlm_debug_get_window(self.ctx, slot, f.ctypes.data, t.ctypes.data, self.max_window,
                                               ctypes.byref(n)), "wedlm_debug_get_window", self.ctx)
        return f[:n.value].copy(), t[:n.value].copy()

    def set_window(self, slot: int, filled, tokens):
        f = np.ascontiguousarray(np.asarray(filled, np.uint8))
        t = np.ascontiguousarray(np.asarray(tokens, np.int32))
        _check(self.lib.wedlm_debug_set_window(self.ctx, slot, f.ctypes.data, t.ctypes.data, len(f)),
               "wedlm_debug_set_window", self.ctx)

    SCHEDULE_BITS = {"cta_pair": 1, "hybrid_split": 2, "cluster_split": 4, "co_resident_fixup": 8,
                     "two_weight_subtiles": 16, "bk32": 32, "fused_entropy": 64}

    def set_plan(self, kind: str, rows: int, tile_n: int, k_splits: int = 1, schedule=()):
        """Test hook: pin the GEMM launch shape of a projection kind at `rows` (see
        wedlm_debug_set_plan); `schedule` is a list of names.  Returns False if the
        shape cannot be built as asked."""
        bits = 0
        for name in schedule:
            bits |= self.SCHEDULE_BITS[name]
        st = self.lib.wedlm_debug_set_plan(self.ctx, C["WEDLM_PROF_" + kind.upper()], rows, tile_n, k_splits, bits)
        if st == C["WEDLM_ERR_INVALID_ARG"]:
            return False
        _check(st, "wedlm_debug_set_plan", self.ctx)
        return True

    def read_weight(self, kind: int, layer: int, nbytes: int) -> np.ndarray:
        """Test hook: the first `nbytes` of a weight tensor's device storage (uint8)."""
        out = np.empty(nbytes, np.uint8)
        _check(self.lib.wedlm_debug_read_weight(self.ctx, kind, layer, out.ctypes.data, nbytes),
               "wedlm_debug_read_weight", self.ctx)
        return out

    def set_page(self, slot: int, index: int, page: int) -> int:
        """Overwrite one device page-table entry, unchecked (fault-injection hook); returns the old entry."""
        old = ctypes.c_int32()
        _check(self.lib.wedlm_debug_set_page(self.ctx, slot, index, page, ctypes.byref(old)),
               "wedlm_debug_set_page", self.ctx)
        return int(old.value)


def _stream_handle(stream) -> int:
    if stream is None:
        return 0
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


# -- stand-alone stage launches (device buffers are torch CUDA tensors) -----
def reorder_window(filled, n, S, stride: int, stream=None):
    import torch
    n_seq = filled.shape[0]
    dev = filled.device
    perm = torch.empty((n_seq, stride), dtype=torch.int32, device=dev)
    pos = torch.empty_like(perm)
    k = torch.empty(n_seq, dtype=torch.int32, device=dev)
    nf = torch.empty_like(k)
    _check(_lib.load().wedlm_reorder_window(_ptr(filled), _ptr(n), _ptr(S), n_seq, stride, _ptr(perm), _ptr(pos),
                                            _ptr(k), _ptr(nf), _stream_handle(stream)), "wedlm_reorder_window")
    return perm, pos, k, nf


def entropy_select(logits, vocab: int, mask_id: int, filled, n, stride: int, params: StepParams, stream=None):
    import torch
    n_seq = filled.shape[0]
    dev = logits.device
    ht = torch.empty((n_seq, stride), dtype=torch.float32, device=dev)
    am = torch.empty((n_seq, stride), dtype=torch.int32, device=dev)
    fill = torch.empty((n_seq, stride), dtype=torch.uint8, device=dev)
    _check(_lib.load().wedlm_entropy_select(_ptr(logits), vocab, mask_id, _ptr(filled), _ptr(n), n_seq, stride,
                                            ctypes.byref(params), _ptr(ht), _ptr(am), _ptr(fill),
                                            _stream_handle(stream)), "wedlm_entropy_select")
    return ht, am, fill


def entropy_select_noalloc(logits, vocab: int, mask_id: int, filled, n, stride: int, params: StepParams,
                           stream=None):
    """entropy_select without any device allocation (scratch in a fixed library array)."""
    import torch
    n_seq = filled.shape[0]
    dev = logits.device
    ht = torch.empty((n_seq, stride), dtype=torch.float32, device=dev)
    am = torch.empty((n_seq, stride), dtype=torch.int32, device=dev)
    fill = torch.empty((n_seq, stride), dtype=torch.uint8, device=dev)
    _check(_lib.load().wedlm_entropy_select_noalloc(_ptr(logits), vocab, mask_id, _ptr(filled), _ptr(n), n_seq,
                                                    stride, ctypes.byref(params), _ptr(ht), _ptr(am), _ptr(fill),
                                                    _stream_handle(stream)), "wedlm_entropy_select_noalloc")
    return ht, am, fill


def entropy_select_async(logits, vocab: int, mask_id: int, filled, n, stride: int, params: StepParams,
                         workspace=None, out=None, stream=None):
    """Asynchronous entropy selection on caller scratch (wedlm_entropy_select_async).
    Returns (htilde, argmax, fill, workspace); the first int32 of the workspace is
    the call's device error word (read it after synchronising)."""
    import torch
    n_seq = filled.shape[0]
    dev = logits.device
    lib = _lib.load()
    if workspace is None:
        nb = ctypes.c_int64()
        _check(lib.wedlm_entropy_select_workspace_bytes(n_seq, stride, ctypes.byref(nb)),
               "wedlm_entropy_select_workspace_bytes")
        workspace = torch.zeros(int(nb.value), dtype=torch.uint8, device=dev)
    if out is None:
        out = (torch.empty((n_seq, stride), dtype=torch.float32, device=dev),
               torch.empty((n_seq, stride), dtype=torch.int32, device=dev),
               torch.empty((n_seq, stride), dtype=torch.uint8, device=dev))
    ht, am, fill = out
    _check(lib.wedlm_entropy_select_async(_ptr(logits), vocab, mask_id, _ptr(filled), _ptr(n), n_seq, stride,
                                          ctypes.byref(params), _ptr(ht), _ptr(am), _ptr(fill), _ptr(workspace),
                                          workspace.numel(), _stream_handle(stream)), "wedlm_entropy_select_async")
    return ht, am, fill, workspace


def attention_workspace(n_seq: int, stride: int, n_heads: int, n_kv_heads: int, max_ctx: int, device="cuda"):
    """A zeroed workspace for attention_bf16 (uint8 CUDA tensor)."""
    import torch
    nb = ctypes.c_int64()
    _check(_lib.load().wedlm_attention_workspace_bytes(n_seq, stride, n_heads, n_kv_heads, max_ctx, ctypes.byref(nb)),
           "wedlm_attention_workspace_bytes")
    return torch.zeros(int(nb.value), dtype=torch.uint8, device=device)


def attention_bf16(q, kv_pool, page_table, S, n, stride: int, n_heads: int, n_kv_heads: int, max_ctx: int,
                   workspace, out=None, stream=None):
    """Asynchronous reordered-causal paged attention (wedlm_attention_bf16).
    q [n_seq*stride, n_heads, 128] bf16; kv_pool [pages, 2, n_kv_heads, 16, 128]
    bf16; page_table [n_seq, pages_per_seq] int32; S, n [n_seq] int32; workspace
    from attention_workspace().  Returns `out`; read attention_error(workspace)
    after synchronising."""
    import torch
    n_seq = page_table.shape[0]
    if out is None:
        out = torch.empty_like(q)
    _check(_lib.load().wedlm_attention_bf16(_ptr(q), _ptr(kv_pool), kv_pool.shape[0], n_heads, n_kv_heads,
                                            _ptr(page_table), page_table.shape[1], _ptr(S), _ptr(n), n_seq, stride,
                                            max_ctx, _ptr(out), _ptr(workspace), workspace.numel(),
                                            _stream_handle(stream)), "wedlm_attention_bf16")
    return out


def attention_error(workspace) -> int:
    """The device error word of an attention workspace (synchronise first)."""
    return int(workspace[:4].view(dtype=__import__("torch").int32)[0].item())


def linear_bf16(X, W, stream=None, tile_n: int = 0, k_splits: int = 0, cta_pair: bool = False,
                hybrid: bool = False, cluster_k: bool = False):
    """Y = X W^T (fp32) on the tcgen05 GEMM; X [M][K], W [N][K] torch.bfloat16 CUDA tensors.
    tile_n / k_splits pin the launch shape (0 = automatic); cta_pair runs CTA-pair
    tiles of 256 weight rows (tile_n 128 or 256); hybrid splits K only for the
    tiles of the last partial round of the persistent grid; cluster_k makes the
    k_splits (2..4) slices of a tile one thread-block cluster reduced through
    distributed shared memory."""
    import torch
    M, K = X.shape
    N = W.shape[0]
    Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    X, W = X.contiguous(), W.contiguous()
    lib = _lib.load()
    if cta_pair or hybrid or cluster_k:
        sched = (1 if cta_pair else 0) | (2 if hybrid else 0) | (4 if cluster_k else 0)
        _check(lib.wedlm_linear_bf16_sched(_ptr(X), _ptr(W), _ptr(Y), M, N, K, tile_n, k_splits, sched,
                                           _stream_handle(stream)), "wedlm_linear_bf16_sched")
    else:
        _check(lib.wedlm_linear_bf16_plan(_ptr(X), _ptr(W), _ptr(Y), M, N, K, tile_n, k_splits,
                                          _stream_handle(stream)), "wedlm_linear_bf16_plan")
    return Y
