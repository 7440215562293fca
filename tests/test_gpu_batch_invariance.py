"""Batch invariance of the bf16 decode step: a sequence decoded alone and the
same sequence decoded among 15 neighbours.

Summary, section Method: committed K/V depend only on earlier tokens of their
own sequence, so a sequence's results should not depend on what else shares
the batch.  In this library the attention's key chunking is fixed per context
(it depends on the context's capacity, never on which slots are busy), but the
dense projections run over all live rows of a step, and the GEMM launch shape
(tile, K slices, fused or two-pass LM head) is tuned per row count: a batch of
one and a batch of sixteen take different plans, so fp32 accumulation orders
differ and a bf16 rounding may land on the other side.  The documented bound
is the bf16 logit tolerance: the masked rows' logits of the lone sequence and
of the same sequence in the full batch agree within max relative error 2e-2
at every step (teacher forcing is not needed: the windows are compared first
and must be equal while the decisions are), and the committed token streams
are identical as long as every fill decision is comparable (no entropy within
1e-3 nats of tau or of the runner-up)."""
import numpy as np
import pytest

import synth
from _gpu_util import comparable, make_engine, oracle_select

pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

MID = dict(L=2, d=512, hq=8, hkv=2, hd=128, F=1536, V=1000, theta=1e6, eps=1e-6, mask_id=999, dtype="bf16")
B, W, N = 16, 16, 24
TOL = 2e-2


def _run(prompts: dict, steps: int, lam: float, tau: float, scale: float):
    from streaming_decoding_b200 import step_params
    eng = make_engine(MID, max_batch=B, max_window=W, max_ctx=1024, prefill_chunk=128)
    eng.keep_logits(True)
    for b, p in prompts.items():
        eng.prefill(b, p, N, W)
    prm = step_params(lam, tau, False, scale)
    out = []
    for _ in range(steps):
        f, t = eng.get_window(0)
        eng.stream_step(prm)
        stride, rows = eng.last_rows()
        kn = eng.debug_read("KN", (B, 3), np.int32)
        perm = eng.debug_read("PERM", rows, np.int32).reshape(-1, stride)
        z = eng.debug_read("LOGITS", (rows, MID["V"]), np.float32).reshape(-1, stride, MID["V"])
        k, n, nf = (int(v) for v in kn[0])
        out.append(dict(window=(list(f), list(t)), rows={int(perm[0, r]): z[0, r].copy() for r in range(nf, n)},
                        gen=eng.read_generated(0)))
        if n == 0:
            break
    eng.close()
    return out


@pytest.mark.parametrize("lam,tau,scale", [(0.1, 0.3, 1.0), (0.05, 6.0, 16.0)])
def test_sequence_alone_equals_sequence_in_full_batch(lam, tau, scale):
    prompts = {b: synth.token_ids(23, b, MID["V"], 40 + 37 * b, MID["mask_id"]) for b in range(B)}
    alone = _run({0: prompts[0]}, 10, lam, tau, scale)
    full = _run(prompts, 10, lam, tau, scale)
    worst = 0.0
    for sa, sf in zip(alone, full):
        if sa["window"] != sf["window"]:
            break  # an earlier non-comparable decision went the other way
        assert sa["rows"].keys() == sf["rows"].keys()
        for j, za in sa["rows"].items():
            zf = sf["rows"][j]
            err = float(np.abs(za - zf).max() / np.abs(za).max())
            worst = max(worst, err)
            assert err < TOL, (j, err)
        Ht, _, fills = oracle_select(sa["rows"], MID["mask_id"], lam, tau, False, scale)
        if comparable(Ht, tau, False):
            _, _, fills_f = oracle_select(sf["rows"], MID["mask_id"], lam, tau, False, scale)
            assert fills == fills_f
        else:
            break
    else:
        assert alone[-1]["gen"] == full[len(alone) - 1]["gen"]
    print(f"alone vs batch of {B}: worst logits max-rel {worst:.3e}")
