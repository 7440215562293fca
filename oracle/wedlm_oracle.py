"""Plain fp64 CPU oracle of WeDLM Streaming Parallel Decoding.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
calls it and shares no code with it; the only thing both sides share is the
seeded input generator in ``synth`` (weights, prompts, window states).

Sources (cited by page and section throughout):
  [Summary/Method]  hyper.ai summary of arXiv 2512.22737, section "Method"
                    (Topological Reordering; Streaming Parallel Decoding;
                    distance-penalised entropy selection).
  [Review/...]      sai.science review "WeDLM: Reconciling Diffusion Language
                    Models with Standard Causal Attention for Fast Inference",
                    sections Summary, Weaknesses, Reproducibility & code,
                    Recommended Changes.
  [Abstract]        arXiv abstract of 2512.22737 (mlsanity.com index page).

Everything is computed in float64 with numpy; weights arrive as float32 or as
bf16 bit patterns (uint16) and are widened exactly.  Readings of points the
pages leave open are marked R1..R16 (the same numbering as the design notes):
  R1  the commit run is the run of slots already filled when the forward starts;
      their K/V come from this forward (Summary/Method: with a causal mask those
      K/V are functions of earlier tokens alone, so they can be cached at once).
  R2  the logits of a mask row predict that row's own slot.
  R3  entropy is Shannon entropy in nats of softmax(logit_scale * logits).
  R4  H~_j = H_j + lambda * j with j the slot's offset from the window start
      (the sign that favours earlier positions, Summary/Method).
  R5  fill {j : H~_j < tau}; if empty (or tau is None) fill the single argmin,
      lowest offset on ties.
  R6  the mask id is never predicted: excluded from entropy and argmax.
  R8  RoPE is rotate-half over pairs (i, i + hd/2), inv_freq = theta^(-2i/hd),
      applied at logical positions.
  R9  greedy fill (argmax, lowest id on ties).
  R12 the window never extends past position P+N-1; decoding ends when the
      committed length reaches P+N.
  R15 prefill commits the whole prompt; the first window is all masks.
  R16 filled tokens are never re-masked.
  R20 sampled fills (the pages decode at temperature 0.1): the fill token of a
      selected slot is argmax_v (logit_scale * z_v / T + G_v), v != mask, with
      Gumbel noise G_v = -log(-log u_v) (the Gumbel-max form of sampling from
      softmax(logit_scale * z / T)); u_v comes from a counter-based generator on
      the SplitMix64 finaliser keyed by (seed, batch slot, the slot's decode
      step, logical position, v).  Slot selection still uses the temperature-1
      entropy (R3).
  R19 block-wise ("stop-and-wait") decoding, the comparison baseline: the same
      step, except that nothing is committed until every slot of the window is
      filled; then the whole window commits and the next window starts
      (Summary/Method: block decoding must finalise the entire block before
      any of it can be cached).
  R18 the bf16 mode's precision contract: fp32 accumulation of operands held
      in bf16 at five points (the normed hidden states entering a projection,
      q/k/v after RoPE (k and v as stored in the cache), the attention output,
      the SwiGLU product, the final normed hidden state).  ``Model(...,
      act_round=round_bf16)`` applies exactly those roundings; the default
      (None) is the exact fp64 definition.
Parity pins for every function live in tests/test_oracle_*.py.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


def _widen(a: np.ndarray) -> np.ndarray:
    """float32 or bf16-bits (uint16) -> float64, exactly."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def round_bf16(x) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even) via float32, returned as
    float64 (R18).  Finite inputs only."""
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


class Model:
    """A causal decoder (RMSNorm, GQA attention with RoPE, SwiGLU FFN, untied LM head).

    ``weights`` is the dict built by ``synth.model_weights``; matrices are in
    nn.Linear layout [out, in].  ``cache_fp64`` keeps widened copies (small
    models); otherwise each matrix is widened when used.  ``act_round`` (R18)
    is applied at the bf16 mode's five rounding points; None = exact."""

    def __init__(self, dims: dict, weights: dict, cache_fp64: bool = True, act_round=None):
        self.L, self.d = dims["L"], dims["d"]
        self.hq, self.hkv, self.hd = dims["hq"], dims["hkv"], dims["hd"]
        self.F, self.V = dims["F"], dims["V"]
        self.theta, self.eps = float(dims["theta"]), float(dims["eps"])
        self.mask_id = int(dims["mask_id"])
        assert self.hq % self.hkv == 0
        self.g = self.hq // self.hkv
        self.w = weights
        self._cache = {} if cache_fp64 else None
        self.act_round = act_round

    def rnd(self, x: np.ndarray) -> np.ndarray:
        return x if self.act_round is None else self.act_round(x)

    def mat(self, name: str, layer: int | None = None) -> np.ndarray:
        key = (name, layer)
        if self._cache is not None and key in self._cache:
            return self._cache[key]
        src = self.w[name] if layer is None else self.w["layers"][layer][name]
        m = _widen(src)
        if self._cache is not None:
            self._cache[key] = m
        return m

    def embed_rows(self, toks) -> np.ndarray:
        return _widen(self.w["embed"][np.asarray(toks, dtype=np.int64)])


# ---------------------------------------------------------------- layers ---
def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotary embedding at (logical) positions ``pos`` (R8; Summary/Method:
    logical position ids are kept through the reordering).

    x: [n, heads, hd]; pair (i, i+hd/2) is rotated by angle pos * theta^(-2i/hd)."""
    n, _, hd = x.shape
    half = hd // 2
    inv_freq = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def window_attention(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                     k_win: np.ndarray, v_win: np.ndarray) -> np.ndarray:
    """Causal attention of window rows in physical order (Summary/Method: a causal
    forward over the reordered window, conditioned on the persistent KV cache).

    q: [n, hq, hd]; k_cache/v_cache: [S, hkv, hd]; k_win/v_win: [n, hkv, hd].
    Physical row r attends to all S cached keys and to window rows 0..r."""
    n, hq, hd = q.shape
    hkv = k_win.shape[1]
    g = hq // hkv
    keys = np.concatenate([k_cache, k_win], axis=0)
    vals = np.concatenate([v_cache, v_win], axis=0)
    S = k_cache.shape[0]
    out = np.empty_like(q)
    scale = 1.0 / math.sqrt(hd)
    for r in range(n):
        kk = keys[: S + r + 1]                      # [T, hkv, hd]
        vv = vals[: S + r + 1]
        qr = q[r].reshape(hkv, g, hd)
        scores = np.einsum("kgd,tkd->kgt", qr, kk) * scale
        scores -= scores.max(axis=-1, keepdims=True)
        p = np.exp(scores)
        p /= p.sum(axis=-1, keepdims=True)
        out[r] = np.einsum("kgt,tkd->kgd", p, vv).reshape(hq, hd)
    return out


@dataclass
class KVCache:
    """Committed K/V of one sequence: per layer a [S, hkv, hd] float64 array."""
    k: list
    v: list

    @staticmethod
    def empty(m: Model) -> "KVCache":
        z = np.zeros((0, m.hkv, m.hd))
        return KVCache([z.copy() for _ in range(m.L)], [z.copy() for _ in range(m.L)])

    @property
    def length(self) -> int:
        return self.k[0].shape[0]

    def append(self, k_rows: list, v_rows: list):
        for l in range(len(self.k)):
            self.k[l] = np.concatenate([self.k[l], k_rows[l]], axis=0)
            self.v[l] = np.concatenate([self.v[l], v_rows[l]], axis=0)


def layer_forward(m: Model, l: int, x: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, pos):
    """Layer l of the decoder on window rows x [n, d] (physical order) at logical
    positions ``pos``, attending to a committed cache (k_cache, v_cache) of that
    layer.  Returns (x after the layer, window K [n,hkv,hd], window V)."""
    n = x.shape[0]
    pos = np.asarray(pos, dtype=np.float64)
    h = m.rnd(rms_norm(x, m.mat("attn_norm", l), m.eps))
    q = (h @ m.mat("wq", l).T).reshape(n, m.hq, m.hd)
    k = (h @ m.mat("wk", l).T).reshape(n, m.hkv, m.hd)
    v = m.rnd((h @ m.mat("wv", l).T).reshape(n, m.hkv, m.hd))
    q = m.rnd(rope(q, pos, m.theta))
    k = m.rnd(rope(k, pos, m.theta))
    a = m.rnd(window_attention(q, k_cache, v_cache, k, v))
    x = x + a.reshape(n, m.hq * m.hd) @ m.mat("wo", l).T
    h = m.rnd(rms_norm(x, m.mat("ffn_norm", l), m.eps))
    x = x + m.rnd(silu(h @ m.mat("wg", l).T) * (h @ m.mat("wu", l).T)) @ m.mat("wd", l).T
    return x, k, v


def final_hidden(m: Model, x: np.ndarray) -> np.ndarray:
    """Final RMSNorm of the residual stream (the LM head's input)."""
    return m.rnd(rms_norm(x, m.mat("final_norm"), m.eps))


def forward_window(m: Model, cache: KVCache, toks, pos):
    """Forward of window rows (physical order) against a committed cache.

    Returns (final-normed hidden [n, d], per-layer window K [n,hkv,hd], window V)."""
    toks = np.asarray(toks)
    x = m.embed_rows(toks)
    wk, wv = [], []
    for l in range(m.L):
        x, k, v = layer_forward(m, l, x, cache.k[l], cache.v[l], pos)
        wk.append(k)
        wv.append(v)
    return final_hidden(m, x), wk, wv


def lm_logits(m: Model, hidden: np.ndarray, logit_scale: float) -> np.ndarray:
    """logit_scale * (hidden @ W_lm^T): [n, V]."""
    return logit_scale * (hidden @ m.mat("lm_head").T)


# ------------------------------------------------------------- selection ---
def entropy_argmax(z: np.ndarray, mask_id: int):
    """Entropy (nats) of softmax(z) and argmax of z over ids != mask_id (R3, R6, R9).

    Entropy by its definition -sum p log p (terms with p = 0 contribute 0);
    argmax is the lowest id among the maxima."""
    z = np.array(z, dtype=np.float64)
    if 0 <= mask_id < z.shape[0]:
        z[mask_id] = -np.inf
    a = int(np.argmax(z))
    e = np.exp(z - z[a])
    p = e / e.sum()
    nz = p > 0
    H = float(-(p[nz] * np.log(p[nz])).sum())
    return H, a


def penalised_entropy(H: float, offset: int, lam: float) -> float:
    """Distance-penalised entropy H~ = H + lambda * offset (R4; Summary/Method:
    the rule prioritises earlier positions; Review/Weaknesses: the formula is
    not printed, sign ambiguous)."""
    return H + lam * offset


def select_fills(Ht: dict, tau: float, tau_none: bool) -> list:
    """Slots to fill this step from {offset: H~} of the masked slots (R5).

    Threshold rule with the at-least-one fallback; tau_none gives one-by-one
    decoding (Review/Reproducibility: threshold None yields one-by-one)."""
    offs = sorted(Ht)
    fills = [] if tau_none else [j for j in offs if Ht[j] < tau]
    if not fills and offs:
        best = offs[0]
        for j in offs[1:]:
            if Ht[j] < Ht[best]:
                best = j
        fills = [best]
    return fills


def reorder(filled) -> list:
    """Topological reordering of a window: filled slots first, then masks, each
    group in ascending slot order (Summary/Method; Abstract)."""
    filled = list(filled)
    return [j for j, f in enumerate(filled) if f] + [j for j, f in enumerate(filled) if not f]


def leading_filled(filled) -> int:
    """Length of the leftmost contiguous run of filled slots (the commit run, R1)."""
    k = 0
    for f in filled:
        if not f:
            break
        k += 1
    return k


# -------------------------------------------------------------- sampling ---
_GOLDEN = np.uint64(0x9E3779B97F4A7C15)


def mix64(z) -> np.ndarray:
    """SplitMix64 output function (Steele, Lea and Flood, "Fast splittable
    pseudorandom number generators", OOPSLA 2014) on uint64 (wrapping):
    z += golden gamma, then two xor-shift-multiply rounds and a final xor-shift."""
    with np.errstate(over="ignore"):
        z = np.asarray(z, dtype=np.uint64) + _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def sampling_uniforms(seed: int, slot: int, step: int, position: int, V: int) -> np.ndarray:
    """u_v in (0, 1) for v = 0..V-1 (R20): h = mix(mix(mix(mix(seed ^ slot) ^ step)
    ^ position) ^ v), u = ((h >> 40) + 1/2) / 2^24."""
    h = mix64(np.uint64(seed) ^ np.uint64(slot))
    h = mix64(h ^ np.uint64(step))
    h = mix64(h ^ np.uint64(position))
    h = mix64(h ^ np.arange(V, dtype=np.uint64))
    return ((h >> np.uint64(40)).astype(np.float64) + 0.5) / float(1 << 24)


def sample_token(z: np.ndarray, mask_id: int, logit_scale: float, temperature: float, u: np.ndarray) -> int:
    """Gumbel-max draw from softmax(logit_scale * z / temperature) over ids != mask_id (R20)."""
    key = np.array(z, dtype=np.float64) * (logit_scale / temperature) - np.log(-np.log(u))
    if 0 <= mask_id < key.shape[0]:
        key[mask_id] = -np.inf
    return int(np.argmax(key))


# ------------------------------------------------------------- decoding ---
@dataclass
class StepTrace:
    S: int
    n: int
    perm: list
    k: int
    committed: list
    masked: list
    H: dict
    Ht: dict
    argmax: dict
    fills: list


@dataclass
class SeqState:
    prompt: np.ndarray
    N: int
    W: int
    cache: KVCache
    S: int
    end: int
    filled: list = field(default_factory=list)
    token: list = field(default_factory=list)
    out: list = field(default_factory=list)
    steps: int = 0
    rows: int = 0
    n_fills: int = 0
    trace: list = field(default_factory=list)

    @property
    def done(self) -> bool:
        return self.S >= self.end


def prefill(m: Model, prompt, N: int, W: int) -> SeqState:
    """Causal forward over the prompt; all of it is committed (R15)."""
    prompt = np.asarray(prompt, dtype=np.int64)
    P = len(prompt)
    cache = KVCache.empty(m)
    if P:
        _, wk, wv = forward_window(m, cache, prompt, np.arange(P))
        cache.append(wk, wv)
    return SeqState(prompt=prompt, N=N, W=W, cache=cache, S=P, end=P + N)


def stream_step(m: Model, st: SeqState, lam: float, tau: float, tau_none: bool,
                logit_scale: float, forward=None, keep_trace: bool = True, choose=None,
                blockwise: bool = False, temperature: float = 0.0, seed: int = 0,
                slot: int = 0) -> StepTrace | None:
    """One Streaming Parallel Decoding step (Summary/Method), in the pages' order:
    refill the window with masks, reorder, causal forward, commit the leftmost
    filled run, then fill selected masks (distance-penalised entropy rule).

    ``forward(m, cache, toks, pos) -> (logits rows [n, V] or None, wk, wv)`` may
    replace the model forward (used by tests with a scripted predictor).
    ``choose(step_index, Ht, fills) -> fills`` lets a test make the oracle follow
    another implementation's fill decision where floating point leaves it open;
    it does not change how anything is computed.  ``blockwise`` selects the
    block-wise baseline (R19): the commit run is the whole window or nothing.
    ``temperature`` > 0 samples the fill tokens (R20) with ``seed``; ``slot``
    is the sequence's batch slot (one of the sampler's counters)."""
    if st.done:
        return None
    # refill: masks appended so the window holds min(W, end - S) slots (R12)
    n = min(st.W, st.end - st.S)
    while len(st.filled) < n:
        st.filled.append(False)
        st.token.append(m.mask_id)
    filled = list(st.filled)
    k = leading_filled(filled)                                  # R1
    if blockwise and k < n:
        k = 0                                                   # R19
    perm = reorder(filled)
    toks = [st.token[j] if filled[j] else m.mask_id for j in perm]
    pos = [st.S + j for j in perm]                              # logical positions
    if forward is None:
        hidden, wk, wv = forward_window(m, st.cache, toks, pos)
        masked_rows = [r for r, j in enumerate(perm) if not filled[j]]
        logits = {perm[r]: lm_logits(m, hidden[r:r + 1], logit_scale)[0] for r in masked_rows}
    else:
        rows_logits, wk, wv = forward(m, st.cache, toks, pos)
        logits = {perm[r]: rows_logits[r] for r in range(n) if not filled[perm[r]]}
    # commit rows 0..k-1 (== slots 0..k-1) into the cache
    st.cache.append([a[:k] for a in wk], [a[:k] for a in wv])
    committed = [st.token[j] for j in range(k)]
    st.out.extend(committed)
    # selection over masked slots
    masked = [j for j in range(n) if not filled[j]]
    H, Ht, amax = {}, {}, {}
    for j in masked:
        H[j], amax[j] = entropy_argmax(logits[j], m.mask_id)
        Ht[j] = penalised_entropy(H[j], j, lam)
    fills = select_fills(Ht, tau, tau_none)
    if choose is not None:
        fills = list(choose(st.steps, Ht, fills))
    for j in fills:
        st.filled[j] = True
        if temperature > 0:
            u = sampling_uniforms(seed, slot, st.steps, st.S + j, len(logits[j]))
            st.token[j] = sample_token(logits[j], m.mask_id, 1.0, temperature, u)
        else:
            st.token[j] = amax[j]
    # slide the window past the committed run
    st.filled = st.filled[k:]
    st.token = st.token[k:]
    st.S += k
    st.steps += 1
    st.rows += n
    st.n_fills += len(fills)
    tr = StepTrace(S=st.S - k, n=n, perm=perm, k=k, committed=committed, masked=masked,
                   H=H, Ht=Ht, argmax=amax, fills=fills)
    if keep_trace:
        st.trace.append(tr)
    return tr


def stream_decode(m: Model, prompt, N: int, W: int, lam: float, tau: float,
                  tau_none: bool = False, logit_scale: float = 1.0, max_steps: int | None = None,
                  forward=None, choose=None, blockwise: bool = False, temperature: float = 0.0,
                  seed: int = 0, slot: int = 0) -> SeqState:
    """Decode N tokens after ``prompt`` with Streaming Parallel Decoding (or,
    with ``blockwise``, the block-wise baseline, R19)."""
    st = prefill(m, prompt, N, W) if forward is None else SeqState(
        prompt=np.asarray(prompt), N=N, W=W, cache=KVCache.empty(m), S=len(prompt), end=len(prompt) + N)
    while not st.done:
        if max_steps is not None and st.steps >= max_steps:
            break
        stream_step(m, st, lam, tau, tau_none, logit_scale, forward=forward, choose=choose, blockwise=blockwise,
                    temperature=temperature, seed=seed, slot=slot)
    return st


def p_cache(st: SeqState) -> float:
    """Prefix cacheability: committed generated tokens / rows processed by decode
    forwards (R14; Review/Summary names the metric, its definition is not printed)."""
    return len(st.out) / st.rows if st.rows else 0.0


def ar_greedy_recompute(m: Model, prompt, N: int, logit_scale: float = 1.0) -> list:
    """Naive greedy decoding without any cache: for every new position, a
    from-scratch causal forward over [committed tokens, MASK] and the argmax of
    the last row (mask id excluded).  Streaming with W=1, lambda=0 must equal
    this (Abstract: the decoder stays compatible with AR prefix caching)."""
    seq = list(np.asarray(prompt, dtype=np.int64))
    out = []
    for _ in range(N):
        toks = seq + [m.mask_id]
        hidden, _, _ = forward_window(m, KVCache.empty(m), toks, np.arange(len(toks)))
        z = lm_logits(m, hidden[-1:], logit_scale)[0]
        _, a = entropy_argmax(z, m.mask_id)
        out.append(a)
        seq.append(a)
    return out


def full_causal_kv(m: Model, tokens):
    """K/V of every layer from one from-scratch causal forward over ``tokens``."""
    toks = np.asarray(tokens, dtype=np.int64)
    _, wk, wv = forward_window(m, KVCache.empty(m), toks, np.arange(len(toks)))
    return wk, wv


def teacher_forced_step_logits(m: Model, prompt, committed_extra, filled, token, logit_scale: float):
    """Logits of the masked rows for a given window state on top of a committed
    sequence (prompt + committed_extra): returns {slot offset: logits}."""
    seq = np.concatenate([np.asarray(prompt, np.int64), np.asarray(committed_extra, np.int64)])
    cache = KVCache.empty(m)
    if len(seq):
        _, wk, wv = forward_window(m, cache, seq, np.arange(len(seq)))
        cache.append(wk, wv)
    S = len(seq)
    perm = reorder(filled)
    toks = [token[j] if filled[j] else m.mask_id for j in perm]
    pos = [S + j for j in perm]
    hidden, _, _ = forward_window(m, cache, toks, pos)
    return {perm[r]: lm_logits(m, hidden[r:r + 1], logit_scale)[0]
            for r in range(len(perm)) if not filled[perm[r]]}
