"""End-to-end parity in fp32 mode on the tiny model: the GPU's decode (every
step, every decision, every committed token) against the CPU oracle."""
import numpy as np
import pytest

import synth
from oracle import wedlm_oracle as O
from _gpu_util import MARGIN, comparable, make_engine, oracle_model, valid_fill_decision

pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TINY = synth.CONFIGS["tiny_f32"]
DIMS = TINY["model"]


@pytest.fixture(scope="module")
def model():
    return oracle_model(DIMS)


def run_gpu_traced(eng, slot_prompts, N, W, lam, tau, tau_none, scale, blockwise=False, temperature=0.0, seed=0):
    """Decode to completion; per step record (k, n, perm, fills, H~) of each slot."""
    from streaming_decoding_b200 import step_params
    for b, p in slot_prompts.items():
        eng.prefill(b, p, N, W[b] if isinstance(W, dict) else W)
    prm = step_params(lam, tau, tau_none, scale, blockwise=blockwise, temperature=temperature, seed=seed)
    traces = {b: [] for b in slot_prompts}
    out = {b: [] for b in slot_prompts}
    active = len(slot_prompts)
    steps = 0
    while active:
        committed, counts, active = eng.stream_step(prm)
        stride, rows = eng.last_rows()
        perm = eng.debug_read("PERM", rows, np.int32).reshape(-1, stride)
        kn = eng.debug_read("KN", (eng.max_batch, 3), np.int32)
        ht = eng.debug_read("HTILDE", (eng.max_batch, eng.max_window), np.float32)
        fl = eng.debug_read("FILL", (eng.max_batch, eng.max_window), np.uint8)
        for b in slot_prompts:
            k, n, nf = kn[b]
            if n == 0:
                continue
            traces[b].append(dict(k=int(k), n=int(n), perm=perm[b, :n].tolist(),
                                  fills=np.nonzero(fl[b, :n])[0].tolist(),
                                  Ht={j: float(ht[b, j]) for j in range(n) if not np.isnan(ht[b, j])}))
            out[b].extend(committed[b])
        steps += 1
        assert steps < 10 * N
    return out, traces


def lockstep_oracle(model, prompt, N, W, lam, tau, tau_none, scale, gtrace, blockwise=False, temperature=0.0,
                    seed=0, slot=0):
    """Run the oracle alongside a recorded GPU trace.  Where the oracle's H~
    leave the decision open within MARGIN, the GPU's decision must be a valid
    one and the oracle then follows it; elsewhere decisions must be equal.
    Returns (oracle state, number of near-tie steps)."""
    near = [0]

    def choose(t, Ht, fills):
        g = gtrace[t]["fills"]
        if comparable(Ht, tau, tau_none):
            assert g == fills, (t, g, fills, Ht)
        else:
            assert valid_fill_decision(Ht, tau, tau_none, g), (t, g, fills, Ht)
            near[0] += 1
        return g

    st = O.stream_decode(model, prompt, N, W, lam, tau, tau_none=tau_none, logit_scale=scale, choose=choose,
                         blockwise=blockwise, temperature=temperature, seed=seed, slot=slot)
    return st, near[0]


def compare_traces(st, gtrace):
    """Per-step equality of the commit run, window size, physical order and H~."""
    assert len(st.trace) == len(gtrace)
    for t_or, t_gpu in zip(st.trace, gtrace):
        assert (t_gpu["k"], t_gpu["n"], t_gpu["perm"]) == (t_or.k, t_or.n, t_or.perm)
        assert set(t_gpu["Ht"]) == set(t_or.Ht)
        for j, v in t_or.Ht.items():
            assert abs(t_gpu["Ht"][j] - v) < MARGIN, (j, t_gpu["Ht"][j], v)
        assert t_gpu["fills"] == t_or.fills
    return len(st.trace)


@pytest.mark.parametrize("cfg_name", ["tiny_f32", "tiny_f32_tau"])
def test_token_stream_and_decisions_match_oracle(model, cfg_name):
    cfg = synth.CONFIGS[cfg_name]
    prompt = synth.prompts(cfg)[0]
    eng = make_engine(DIMS, max_batch=1, max_window=cfg["W"], max_ctx=64)
    out, tr = run_gpu_traced(eng, {0: prompt}, cfg["N"], cfg["W"], cfg["lam"], cfg["tau"], False,
                             cfg["logit_scale"])
    st, near = lockstep_oracle(model, prompt, cfg["N"], cfg["W"], cfg["lam"], cfg["tau"], False,
                               cfg["logit_scale"], tr[0])
    compare_traces(st, tr[0])
    assert near <= 2
    assert out[0] == st.out
    assert eng.read_generated(0) == st.out
    s = eng.stats(0)
    assert (s["steps"], s["forward_rows"], s["committed"], s["active"]) == (st.steps, st.rows, len(st.out), 0)
    assert s["fills"] == st.n_fills


@pytest.mark.parametrize("cfg_name", ["tiny_f32", "tiny_f32_tau"])
def test_blockwise_baseline_matches_oracle(model, cfg_name):
    """The block-wise (stop-and-wait) baseline on the same kernels: every step's
    commit run (whole window or nothing), order, H~ and fills equal the oracle's."""
    cfg = synth.CONFIGS[cfg_name]
    prompt = synth.prompts(cfg)[0]
    eng = make_engine(DIMS, max_batch=1, max_window=cfg["W"], max_ctx=64)
    out, tr = run_gpu_traced(eng, {0: prompt}, cfg["N"], cfg["W"], cfg["lam"], cfg["tau"], False,
                             cfg["logit_scale"], blockwise=True)
    st, near = lockstep_oracle(model, prompt, cfg["N"], cfg["W"], cfg["lam"], cfg["tau"], False,
                               cfg["logit_scale"], tr[0], blockwise=True)
    compare_traces(st, tr[0])
    assert near <= 2
    assert all(t["k"] in (0, t["n"]) for t in tr[0])
    assert out[0] == st.out
    s = eng.stats(0)
    assert (s["steps"], s["forward_rows"], s["committed"]) == (st.steps, st.rows, len(st.out))


@pytest.mark.parametrize("temperature", [0.1, 1.0])
def test_sampled_fills_match_oracle(model, temperature):
    """Seeded Gumbel-max sampling of fill tokens (two slots, so the slot is part
    of the generator's key): token streams and decisions equal the oracle's."""
    cfg = synth.CONFIGS["tiny_f32_tau"]
    prompts = synth.prompts(cfg)
    slot_prompts = {0: prompts[0], 1: prompts[0][::-1].copy()}
    eng = make_engine(DIMS, max_batch=2, max_window=cfg["W"], max_ctx=64)
    out, tr = run_gpu_traced(eng, slot_prompts, cfg["N"], cfg["W"], cfg["lam"], cfg["tau"], False,
                             cfg["logit_scale"], temperature=temperature, seed=20251202)
    greedy = O.stream_decode(model, prompts[0], cfg["N"], cfg["W"], cfg["lam"], cfg["tau"],
                             logit_scale=cfg["logit_scale"]).out
    for b, p in slot_prompts.items():
        st, near = lockstep_oracle(model, p, cfg["N"], cfg["W"], cfg["lam"], cfg["tau"], False, cfg["logit_scale"],
                                   tr[b], temperature=temperature, seed=20251202, slot=b)
        compare_traces(st, tr[b])
        assert near <= 2
        assert out[b] == st.out
    if temperature >= 1.0:
        assert out[0] != greedy  # sampling at T = 1 departs from the greedy stream


def test_window_one_is_greedy_autoregression(model):
    """W=1, lambda=0 on the GPU equals the oracle's naive greedy AR recompute."""
    prompt = synth.prompts(TINY)[0]
    N = 16
    eng = make_engine(DIMS, max_batch=1, max_window=1, max_ctx=64)
    out, tr = run_gpu_traced(eng, {0: prompt}, N, 1, 0.0, 0.5, False, TINY["logit_scale"])
    assert out[0] == O.ar_greedy_recompute(model, prompt, N, logit_scale=TINY["logit_scale"])
    assert len(tr[0]) == 2 * N


def test_first_step_logits_match_oracle(model):
    from streaming_decoding_b200 import step_params
    prompt = synth.prompts(TINY)[0]
    eng = make_engine(DIMS, max_batch=1, max_window=4, max_ctx=64)
    eng.prefill(0, prompt, TINY["N"], 4)
    eng.stream_step(step_params(0.1, 0.5, False, 8.0))
    stride, rows = eng.last_rows()
    z = eng.debug_read("LOGITS", (rows, DIMS["V"]), np.float32)
    hidden, _, _ = O.forward_window(model, O.prefill(model, prompt, TINY["N"], 4).cache, [DIMS["mask_id"]] * 4,
                                    np.arange(16, 20))
    ref = O.lm_logits(model, hidden, 1.0)
    err = np.abs(z[:4] - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


@pytest.mark.parametrize("cfg_name", ["tiny_f32", "tiny_f32_tau"])
def test_committed_kv_equals_recompute(model, cfg_name):
    """Prefix cacheability on the GPU: after decoding, the cache rows equal a
    from-scratch causal forward over the committed sequence."""
    cfg = synth.CONFIGS[cfg_name]
    prompt = synth.prompts(cfg)[0]
    eng = make_engine(DIMS, max_batch=1, max_window=cfg["W"], max_ctx=64)
    out, _ = run_gpu_traced(eng, {0: prompt}, cfg["N"], cfg["W"], cfg["lam"], cfg["tau"], False, cfg["logit_scale"])
    seq = list(prompt) + out[0]
    fk, fv = O.full_causal_kv(model, seq)
    for l in range(DIMS["L"]):
        k, v = eng.debug_kv(0, l, 0, len(seq))
        assert np.abs(k - fk[l]).max() <= 1e-5 * np.abs(fk[l]).max()
        assert np.abs(v - fv[l]).max() <= 1e-5 * np.abs(fv[l]).max()


def test_batch_of_ragged_sequences_matches_independent_decodes(model):
    """Slots decode independently: ragged prompt lengths, windows and ends in one
    batch give each sequence the oracle's own token stream."""
    cfg = synth.CONFIGS["tiny_f32_tau"]
    prompts = {0: synth.token_ids(7, 0, 512, 16, 511), 1: synth.token_ids(7, 1, 512, 3, 511),
               2: synth.token_ids(7, 2, 512, 33, 511)}
    W = {0: 4, 1: 3, 2: 2}
    N = 20
    eng = make_engine(DIMS, max_batch=4, max_window=4, max_ctx=64)
    out, tr = run_gpu_traced(eng, prompts, N, W, cfg["lam"], cfg["tau"], False, cfg["logit_scale"])
    for b, p in prompts.items():
        st, near = lockstep_oracle(model, p, N, W[b], cfg["lam"], cfg["tau"], False, cfg["logit_scale"], tr[b])
        compare_traces(st, tr[b])
        assert near <= 2
        assert out[b] == st.out


def test_reset_refill_and_page_exhaustion():
    from streaming_decoding_b200 import step_params
    from streaming_decoding_b200._lib import WedlmError
    eng = make_engine(DIMS, max_batch=2, max_window=4, max_ctx=64, num_pages=5)
    p = synth.prompts(TINY)[0]
    eng.prefill(0, p, 48, 4)               # 64 positions = 4 pages
    with pytest.raises(WedlmError) as e:
        eng.prefill(1, p, 48, 4)           # 4 more pages: only 1 left
    assert e.value.status == -2
    with pytest.raises(WedlmError):
        eng.prefill(0, p, 4, 4)            # slot in use
    eng.kv_reset(0)
    eng.prefill(1, p, 8, 4)
    _, counts, active = eng.stream_step(step_params(0.1, 0.5, False, 8.0))
    assert active == 1 and counts[0] == 0
    with pytest.raises(WedlmError):
        eng.prefill(0, np.array([600], np.int32), 4, 4)   # token id out of range
    with pytest.raises(WedlmError):
        eng.stream_step(step_params(0.1, 0.5, False, 0.0))  # logit_scale must be > 0


def test_async_steps_match_synchronous_steps(model):
    from streaming_decoding_b200 import step_params
    cfg = synth.CONFIGS["tiny_f32_tau"]
    prompt = synth.prompts(cfg)[0]
    st = O.stream_decode(model, prompt, cfg["N"], cfg["W"], cfg["lam"], cfg["tau"], logit_scale=cfg["logit_scale"])
    eng = make_engine(DIMS, max_batch=1, max_window=4, max_ctx=64)
    eng.prefill(0, prompt, cfg["N"], cfg["W"])
    before = eng.kernel_launches()
    eng.stream_step_async(step_params(cfg["lam"], cfg["tau"], False, cfg["logit_scale"]), st.steps + 3)
    assert eng.read_generated(0) == st.out
    assert eng.stats(0)["steps"] == st.steps
    assert eng.kernel_launches() > before
