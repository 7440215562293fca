"""Every GEMM launch shape the autotuner may pick, under every fused epilogue.

The tuner chooses, per projection and row count, among single-CTA tiles
(64 / 128 / 256 activation rows, one or two 128-row weight sub-tiles, 64- or
32-deep k-blocks), CTA-pair tiles, and K split into slices reduced by the
co-resident slices, by the last slice to finish, only in the last partial
round (hybrid), or through distributed shared memory (cluster).  Each of these
runs each projection's own epilogue (RoPE + K/V page write for QKV, residual
add for O and down, SwiGLU for gate/up, logits or fused entropy partials for
the LM head), and which one the tuner keeps varies with timing noise, so each
combination is pinned here in turn (wedlm_debug_set_plan) on the batch-16,
window-16 step of a two-layer model at the Qwen3-8B width, and the step's
results are compared with those of the cost-model plans: the residual stream
after each layer, the window K/V written into the cache, and the masked rows'
logits (or, with the fused entropy epilogue, H~ and the argmax).  Plans differ
only in fp32 summation order, so the tolerances are tight.  The cost-model step
itself is checked against the oracle once (hyper.ai summary, section Method:
the causal forward over the reordered window against the persistent cache)."""
import numpy as np
import pytest

import synth
from oracle import wedlm_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CFG = synth.CONFIGS["qwen3_8b_b16"]
DIMS = dict(CFG["model"], L=2)
B, W, N = CFG["B"], CFG["W"], 64
ROWS = B * W
KINDS = ("gemm_qkv", "gemm_o", "gemm_gate_up", "gemm_down", "gemm_lm_head")
# (tile_n, schedule names) families and K-split variants, as the tuner builds them
FAMILIES = [(256, ["cta_pair"]), (128, ["cta_pair"]), (256, []), (128, []), (64, []),
            (256, ["two_weight_subtiles"]), (128, ["two_weight_subtiles"]),
            (256, ["two_weight_subtiles", "bk32"]), (128, ["two_weight_subtiles", "bk32"]), (256, ["bk32"])]
SPLITS = [(1, []), (2, ["co_resident_fixup"]), (3, ["co_resident_fixup"]), (2, []), (4, []), (8, []),
          (2, ["hybrid_split"]), (3, ["hybrid_split"]), (2, ["cluster_split"]), (4, ["cluster_split"])]


def frob(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def row_rel(a, b):
    """Largest per-row max |a - b| / max |b| (a wrong row shows up as O(1))."""
    a = a.reshape(a.shape[0], -1).astype(np.float64)
    b = b.reshape(b.shape[0], -1).astype(np.float64)
    return float((np.abs(a - b).max(axis=1) / np.maximum(np.abs(b).max(axis=1), 1e-30)).max())


@pytest.fixture(scope="module")
def engine():
    from streaming_decoding_b200 import Engine
    eng = Engine(DIMS, max_batch=B, max_window=W, max_ctx=1024 + N, stream=torch.cuda.Stream())
    eng.autotune(False)
    eng.load_model(synth.iter_weights(DIMS, seed=0, dtype="bf16"))
    eng.debug_capture(True)
    yield eng
    eng.close()


PROMPTS = [p[:200] for p in synth.prompts(CFG)]
SAMPLE = 3  # the slot whose window K/V are read back


def run_step(eng, fused=False):
    """The first decode step (every slot all masks) from a fresh admission."""
    from streaming_decoding_b200 import step_params
    eng.kv_reset(-1)
    for b, p in enumerate(PROMPTS):
        eng.prefill(b, p, N, W)
    if fused:
        eng.force_fused_entropy(True)
    else:
        eng.keep_logits(True)
    eng.stream_step(step_params(CFG["lam"], CFG["tau"], False, CFG["logit_scale"]))
    out = {"x": [eng.debug_residual(l, ROWS) for l in range(DIMS["L"] + 1)],
           "kv": [eng.debug_kv(SAMPLE, l, len(PROMPTS[SAMPLE]), W) for l in range(DIMS["L"])],
           "ht": eng.debug_read("HTILDE", (B, W), np.float32),
           "am": eng.debug_read("ARGMAX", (B, W), np.int32)}
    if not fused:
        out["z"] = eng.debug_read("LOGITS", (ROWS, DIMS["V"]), np.float32)
    eng.keep_logits(False)
    return out


@pytest.fixture(scope="module")
def reference(engine):
    ref = run_step(engine)
    ref_fused = run_step(engine, fused=True)
    # anchor: the cost-model step against the oracle, layer by layer (sample slot)
    m = O.Model(DIMS, synth.model_weights(DIMS, seed=0, dtype="bf16"), cache_fp64=False)
    S = len(PROMPTS[SAMPLE])
    cache = [engine.debug_kv(SAMPLE, l, 0, S) for l in range(DIMS["L"])]
    rows = slice(SAMPLE * W, SAMPLE * W + W)
    pos = np.arange(S, S + W)
    for l in range(DIMS["L"]):
        xl = ref["x"][l][rows].astype(np.float64)
        x1, wk, wv = O.layer_forward(m, l, xl, cache[l][0].astype(np.float64), cache[l][1].astype(np.float64), pos)
        assert frob(ref["x"][l + 1][rows] - xl, x1 - xl) < 2e-2
        assert frob(ref["kv"][l][0], wk) < 2e-2 and frob(ref["kv"][l][1], wv) < 2e-2
    return ref, ref_fused


def plans_for(kind):
    for tile_n, fam in FAMILIES:
        for splits, extra in SPLITS:
            if kind == "gemm_lm_head" and "cluster_split" in extra:
                continue
            yield tile_n, splits, fam + extra


@pytest.mark.parametrize("kind", KINDS)
def test_every_plan_matches_the_cost_model_plan(engine, reference, kind):
    ref, ref_fused = reference
    tried = 0
    bad = []
    for tile_n, splits, sched in plans_for(kind):
        if not engine.set_plan(kind, ROWS, tile_n, splits, sched):
            continue
        got = run_step(engine)
        tried += 1
        err_x = max(frob(got["x"][l], ref["x"][l]) for l in range(1, DIMS["L"] + 1))
        row_x = max(row_rel(got["x"][l], ref["x"][l]) for l in range(1, DIMS["L"] + 1))
        err_kv = max(row_rel(got["kv"][l][i], ref["kv"][l][i]) for l in range(DIMS["L"]) for i in (0, 1))
        err_z = row_rel(got["z"], ref["z"])
        print(f"  {kind} tile_n={tile_n} splits={splits} {'+'.join(sched) or 'plain'}: x frob {err_x:.1e} "
              f"row {row_x:.1e}, K/V row {err_kv:.1e}, logits row {err_z:.1e}")
        if not (err_x < 1e-2 and row_x < 5e-2 and err_kv < 5e-2 and err_z < 5e-2):
            bad.append((tile_n, splits, sched, err_x, row_x, err_kv, err_z))
    if kind == "gemm_lm_head":
        for tile_n, fam in FAMILIES:
            if not engine.set_plan(kind, ROWS, tile_n, 1, fam + ["fused_entropy"]):
                continue
            got = run_step(engine, fused=True)
            tried += 1
            dh = np.nanmax(np.abs(got["ht"] - ref_fused["ht"]))
            # the argmax may flip only where two logits tie to fp32 summation order
            flips = int(np.sum(got["am"] != ref_fused["am"]))
            if not (dh < 1e-3 and flips <= 1):
                bad.append((tile_n, 1, fam + ["fused_entropy"], float(dh), flips))
    engine.autotune(False)  # clear the pinned plans
    print(f"{kind}: {tried} plans checked")
    assert tried >= 10
    for b in bad:
        print("MISMATCH", kind, b)
    assert not bad, bad
