"""Full-size parity, sampled: the Qwen3-8B-shaped bf16 model (36 layers) at
batch 16 and window 16, the launch configuration bench.py times, against the
fp64 oracle.

The whole batch of 16 prompts (U[128, 1024] tokens) is prefilled and decoded
for a few steps on the GPU; the residual stream is captured at every layer
boundary of the last step.  One sequence (the shortest prompt) is sampled and
checked layer by layer, each layer teacher-forced with the GPU's own input to
it and the GPU's own committed cache of that layer:

* each layer's update of the residual stream, x_{l+1} - x_l, agrees with the
  oracle's layer on the same input within 2e-2 (Frobenius-relative; the layer
  keeps four operands in bf16, each rounded to 2^-9 relative);
* the window K/V each layer writes into the cache agree within 2e-2;
* the logits of the masked rows, from the GPU's final residual stream, agree
  within max relative error 2e-2 per row (the bf16 logit tolerance), and the
  fill decisions taken from the GPU's logits equal the oracle's where
  comparable.

End to end (no teacher forcing) bf16 arithmetic itself drifts with depth on
this random-init model: the exact oracle and an oracle that rounds at the bf16
mode's points differ by about 5e-2 in the logits.  The GPU's own end-to-end
deviation is printed and bounded by what it measures with margin: about 5e-2
against the exact oracle and 4e-2 against the oracle with the bf16 rounding
points (runs differ by a few thousandths with the tuned GEMM launch shapes),
guarded at 8e-2 and 6e-2."""
import numpy as np
import pytest

import synth
from oracle import wedlm_oracle as O
from _gpu_util import MARGIN, comparable, oracle_select

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-2


def frob(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_full_size_batch16_per_layer_against_oracle():
    from streaming_decoding_b200 import Engine, step_params
    cfg = synth.CONFIGS["qwen3_8b_b16"]
    dims = cfg["model"]
    B, W, N, L = cfg["B"], cfg["W"], cfg["N"], cfg["model"]["L"]
    prompts = synth.prompts(cfg)
    eng = Engine(dims, max_batch=B, max_window=W, max_ctx=1024 + N, stream=torch.cuda.Stream())
    eng.load_model(synth.iter_weights(dims, seed=0, dtype="bf16"))
    for b, p in enumerate(prompts):
        eng.prefill(b, p, N, W)
    prm = step_params(cfg["lam"], cfg["tau"], False, cfg["logit_scale"])
    eng.stream_step_async(prm, 3)
    plans = {k: (eng.gemm_plan(k, B * W), eng.gemm_schedule(k, B * W))
             for k in ("gemm_qkv", "gemm_o", "gemm_gate_up", "gemm_down", "gemm_lm_head")}
    print("tuned GEMM plans at", B * W, "rows:", plans)
    b = int(np.argmin([len(p) for p in prompts]))
    f0, t0 = eng.get_window(b)
    gen = eng.read_generated(b)
    eng.debug_capture(True)
    eng.keep_logits(True)  # the logits are read back
    eng.stream_step(prm)
    stride, rows = eng.last_rows()
    assert (stride, rows) == (W, B * W)
    kn = eng.debug_read("KN", (B, 3), np.int32)
    k, n, nf = (int(v) for v in kn[b])
    perm = eng.debug_read("PERM", rows, np.int32).reshape(B, W)[b, :n]
    z = eng.debug_read("LOGITS", (rows, dims["V"]), np.float32).reshape(B, W, dims["V"])[b]
    ht = eng.debug_read("HTILDE", (B, W), np.float32)[b]
    fl = eng.debug_read("FILL", (B, W), np.uint8)[b]
    xs = [eng.debug_residual(l, rows)[b * W:b * W + n].astype(np.float64) for l in range(L + 1)]
    seq = list(prompts[b]) + gen
    S = len(seq)
    cache = [eng.debug_kv(b, l, 0, S) for l in range(L)]
    win = [eng.debug_kv(b, l, S, n) for l in range(L)]
    eng.close()

    filled = list(f0) + [0] * (n - len(f0))
    tokens = list(t0) + [dims["mask_id"]] * (n - len(t0))
    assert perm.tolist() == O.reorder(filled) and k == O.leading_filled(filled)
    pos = [S + j for j in perm]
    m = O.Model(dims, synth.model_weights(dims, seed=0, dtype="bf16"), cache_fp64=False)

    # embedding rows entering layer 0
    toks = [tokens[j] if filled[j] else dims["mask_id"] for j in perm]
    assert frob(xs[0], m.embed_rows(toks)) < 1e-6

    upd, kv = [], []
    for l in range(L):
        x1, wk, wv = O.layer_forward(m, l, xs[l], cache[l][0].astype(np.float64), cache[l][1].astype(np.float64), pos)
        upd.append(frob(xs[l + 1] - xs[l], x1 - xs[l]))
        kv.append(max(frob(win[l][0], wk), frob(win[l][1], wv)))
    print(f"per-layer update rel err: max {max(upd):.3e} (layer {int(np.argmax(upd))}), "
          f"window K/V rel err max {max(kv):.3e}")
    assert max(upd) < TOL, upd
    assert max(kv) < TOL, kv

    hidden = O.final_hidden(m, xs[L])
    worst = 0.0
    for r in range(nf, n):
        ref = O.lm_logits(m, hidden[r:r + 1], 1.0)[0]
        worst = max(worst, float(np.abs(z[r] - ref).max() / np.abs(ref).max()))
    print(f"logits from the GPU's final residual stream: worst max-rel err {worst:.3e}")
    assert worst < TOL, worst
    Ht, _, fills = oracle_select({perm[r]: z[r] for r in range(nf, n)}, dims["mask_id"], cfg["lam"], cfg["tau"],
                                 False, cfg["logit_scale"])
    for j, v in Ht.items():
        assert abs(ht[j] - v) < MARGIN
    if comparable(Ht, cfg["tau"], False):
        assert np.nonzero(fl[:n])[0].tolist() == fills

    # end to end (no teacher forcing): the oracle recomputes the sequence from
    # scratch, exactly and with the R18 bf16 rounding points; the GPU's logits
    # are compared with both
    e2e = {}
    m18 = O.Model(dims, synth.model_weights(dims, seed=0, dtype="bf16"), cache_fp64=False, act_round=O.round_bf16)
    for name, mm in (("exact", m), ("r18", m18)):
        ofull = O.KVCache.empty(mm)
        _, ck, cv = O.forward_window(mm, ofull, seq, np.arange(S))
        ofull.append(ck, cv)
        h_e2e, _, _ = O.forward_window(mm, ofull, toks, pos)
        worst_e = 0.0
        for r in range(nf, n):
            ref = O.lm_logits(mm, h_e2e[r:r + 1], 1.0)[0]
            worst_e = max(worst_e, float(np.abs(z[r] - ref).max() / np.abs(ref).max()))
        e2e[name] = worst_e
    print(f"full-size sampled: sequence {b} (P={len(prompts[b])}, S={S}), {n - nf} masked rows; "
          f"end-to-end logits max-rel vs the exact oracle {e2e['exact']:.3e}, vs the R18 oracle {e2e['r18']:.3e}")
    # measured about 5.0e-2 / 3.8e-2; guarded with about 1.5x margin
    assert e2e["exact"] < 0.08 and e2e["r18"] < 0.06, e2e
