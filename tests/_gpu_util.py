"""Helpers shared by the GPU parity tests (not collected as tests)."""
from __future__ import annotations

import numpy as np

import synth
from oracle import wedlm_oracle as O

# Decisions compare only where floating point cannot flip them: every candidate
# H~ more than MARGIN nats from tau, and the best two more than MARGIN apart.
MARGIN = 1e-3


def make_engine(dims: dict, max_batch: int, max_window: int, max_ctx: int, seed: int = 0, **kw):
    from streaming_decoding_b200 import Engine
    eng = Engine(dims, max_batch=max_batch, max_window=max_window, max_ctx=max_ctx, **kw)
    eng.load_model(synth.iter_weights(dims, seed=seed, dtype=dims["dtype"]))
    return eng


def oracle_model(dims: dict, seed: int = 0, cache_fp64: bool = True) -> O.Model:
    return O.Model(dims, synth.model_weights(dims, seed=seed, dtype=dims["dtype"]), cache_fp64=cache_fp64)


def comparable(Ht: dict, tau: float, tau_none: bool) -> bool:
    vals = sorted(Ht.values())
    if not vals:
        return True
    if not tau_none and any(abs(v - tau) <= MARGIN for v in vals):
        return False
    if len(vals) > 1 and vals[1] - vals[0] <= MARGIN:
        return False
    return True


def oracle_select(logits_rows: dict, mask_id: int, lam: float, tau: float, tau_none: bool, scale: float):
    """Oracle decisions for {slot: fp32 logits}: (H~, argmax, fills)."""
    Ht, am = {}, {}
    for j, z in logits_rows.items():
        H, a = O.entropy_argmax(scale * np.asarray(z, np.float64), mask_id)
        Ht[j] = O.penalised_entropy(H, j, lam)
        am[j] = a
    return Ht, am, O.select_fills(Ht, tau, tau_none)


def valid_fill_decision(Ht: dict, tau: float, tau_none: bool, fills) -> bool:
    """Is `fills` a decision the rule allows once every H~ may be off by MARGIN?

    Slots with H~ < tau - MARGIN must be filled and slots with H~ > tau + MARGIN
    must not (threshold branch); a single fill is also valid as the fallback if
    no slot is certainly under tau and the slot is within MARGIN of the minimum."""
    fills = sorted(fills)
    if not Ht:
        return fills == []
    under = {j for j, v in Ht.items() if v < tau - MARGIN}
    over = {j for j, v in Ht.items() if v > tau + MARGIN}
    lo = min(Ht.values())
    if len(fills) == 1 and not (under and not tau_none) and Ht.get(fills[0], float("inf")) <= lo + MARGIN:
        return True
    if tau_none or not fills:
        return False
    F = set(fills)
    return F.issubset(Ht) and under.issubset(F) and not (F & over)
