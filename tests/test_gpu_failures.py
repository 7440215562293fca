"""Failure paths, injected from the host (nothing here faults or hangs the GPU).

* A corrupted page-table entry: the kernels' own bounds checks refuse the
  access (the attention reads a valid page instead, the QKV epilogue skips the
  write), the step returns WEDLM_ERR_DEVICE_ASSERT and the context stays usable.
* Non-finite logits (a NaN planted in a host buffer or in one LM-head weight
  row): such a masked slot is invalid -- H~ NaN, argmax -1, never filled --
  the window's other slots are decided among themselves, and the call returns
  WEDLM_ERR_NONFINITE.  Without this rule a NaN row would read as zero entropy
  and be filled first."""
import numpy as np
import pytest

import synth
from oracle import wedlm_oracle as O
from _gpu_util import comparable, oracle_select

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DIMS = dict(L=2, d=512, hq=8, hkv=2, hd=128, F=1536, V=1000, theta=1e6, eps=1e-6, mask_id=999, dtype="bf16")


def _status(name):
    from streaming_decoding_b200.api import C
    return C[name]


def _logits_case():
    V, stride, n_seq = 1000, 8, 3
    filled = np.array([[1, 0, 0, 1, 0, 0, 0, 0], [0, 0, 0, 0, 0, 0, 0, 0], [0, 1, 0, 1, 1, 1, 1, 1]], np.uint8)
    n = np.array([8, 6, 8], np.int32)
    z = synth.normal(77, 1, 2.0, (n_seq, stride, V), "f32")
    z[0, 2, 17] = np.nan          # one NaN in slot 2 of window 0
    z[0, 5, 3] = np.inf           # an infinity in slot 5 of window 0
    z[1, :, :] = np.nan           # every slot of window 1
    return V, stride, filled, n, z


def _check_nonfinite_outputs(ht, am, fill, V, stride, filled, n, z, lam, tau):
    ht, am, fill = ht.cpu().numpy(), am.cpu().numpy(), fill.cpu().numpy()
    for j in (2, 5):
        assert np.isnan(ht[0, j]) and am[0, j] == -1 and fill[0, j] == 0
    # window 0: the valid masked slots are decided as the oracle decides them
    rows = {j: z[0, j] for j in range(n[0]) if not filled[0, j] and j not in (2, 5)}
    Ht, amax, fills = oracle_select(rows, V - 1, lam, tau, False, 1.0)
    for j, v in Ht.items():
        assert abs(ht[0, j] - v) < 1e-3 and am[0, j] == amax[j]
    if comparable(Ht, tau, False):
        assert np.nonzero(fill[0])[0].tolist() == fills
    # window 1: nothing valid, nothing filled
    assert not fill[1].any() and np.isnan(ht[1, :n[1]]).all() and (am[1, :n[1]] == -1).all()
    # window 2 (all finite) is unaffected
    rows = {j: z[2, j] for j in range(n[2]) if not filled[2, j]}
    Ht, amax, fills = oracle_select(rows, V - 1, lam, tau, False, 1.0)
    if comparable(Ht, tau, False):
        assert np.nonzero(fill[2])[0].tolist() == fills


@pytest.mark.parametrize("variant", ["sync", "async", "noalloc"])
def test_nonfinite_logits_are_never_filled(variant):
    from streaming_decoding_b200 import (entropy_select, entropy_select_async, entropy_select_noalloc,
                                         step_params)
    from streaming_decoding_b200._lib import WedlmError
    V, stride, filled, n, z = _logits_case()
    lam, tau = 0.1, 4.0
    prm = step_params(lam, tau, False, 1.0)
    zd = torch.from_numpy(z).cuda()
    fd = torch.from_numpy(filled).cuda()
    nd = torch.from_numpy(n).cuda()
    if variant == "async":
        ht, am, fill, ws = entropy_select_async(zd, V, V - 1, fd, nd, stride, prm)
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32)[0].item()) == 3
    else:
        fn = entropy_select if variant == "sync" else entropy_select_noalloc
        out = {}

        def grab(*a):
            return fn(*a)
        with pytest.raises(WedlmError) as ei:
            grab(zd, V, V - 1, fd, nd, stride, prm)
        assert ei.value.status == _status("WEDLM_ERR_NONFINITE")
        # the outputs are written all the same: run the async form for them
        ht, am, fill, _ = entropy_select_async(zd, V, V - 1, fd, nd, stride, prm)
        torch.cuda.synchronize()
    _check_nonfinite_outputs(ht, am, fill, V, stride, filled, n, z, lam, tau)
    # and a clean call afterwards succeeds
    z2 = np.nan_to_num(z, nan=0.0, posinf=0.0)
    ht2, _, _ = entropy_select(torch.from_numpy(z2).cuda(), V, V - 1, fd, nd, stride, prm)
    assert not np.isnan(ht2.cpu().numpy()[1, :n[1]]).any()


def _engine(W=8, keep_logits=False, nan_row=None, autotune=False):
    from streaming_decoding_b200 import Engine
    eng = Engine(DIMS, max_batch=2, max_window=W, max_ctx=160, stream=torch.cuda.Stream())
    if not autotune:
        eng.autotune(False)  # fixed choices: the fused LM-head entropy at these row counts
    for kind, layer, arr in synth.iter_weights(DIMS, seed=0, dtype="bf16"):
        if kind == synth.T_LM_HEAD and nan_row is not None:
            arr = arr.copy()
            arr[nan_row, :] = 0x7FC0  # bf16 quiet NaN
        eng.load_weights(kind, layer, arr)
    for b in range(2):
        eng.prefill(b, synth.token_ids(21, b, DIMS["V"], 40 + 9 * b, DIMS["mask_id"]), 32, W)
    eng.keep_logits(keep_logits)
    return eng


def test_corrupted_page_table_entry_is_caught_and_recoverable():
    from streaming_decoding_b200 import step_params
    from streaming_decoding_b200._lib import WedlmError
    eng = _engine()
    prm = step_params(0.1, 2.0, False, 4.0)
    eng.stream_step(prm)
    old = eng.set_page(1, 1, 1 << 24)  # slot 1's second page: far outside the pool
    with pytest.raises(WedlmError) as ei:
        eng.stream_step(prm)
    assert ei.value.status == _status("WEDLM_ERR_DEVICE_ASSERT")
    eng.set_page(1, 1, old)
    # the context is still usable: a fresh admission decodes normally
    eng.kv_reset(-1)
    for b in range(2):
        eng.prefill(b, synth.token_ids(22, b, DIMS["V"], 30, DIMS["mask_id"]), 16, 8)
    total = 0
    for _ in range(40):
        _, counts, active = eng.stream_step(prm)
        total += int(np.sum(counts))
        if not active:
            break
    assert total == 32 and active == 0
    eng.close()


@pytest.mark.parametrize("keep_logits", [False, True])
def test_nan_lm_head_row_fills_nothing(keep_logits):
    """One LM-head row of NaN makes every logit row non-finite: the step fills
    nothing, reports WEDLM_ERR_NONFINITE, and (fused LM-head entropy or the
    two-pass path) marks every masked slot invalid."""
    from streaming_decoding_b200 import step_params
    from streaming_decoding_b200._lib import WedlmError
    eng = _engine(keep_logits=keep_logits, nan_row=123)
    prm = step_params(0.1, 2.0, False, 4.0)
    with pytest.raises(WedlmError) as ei:
        eng.stream_step(prm)
    assert ei.value.status == _status("WEDLM_ERR_NONFINITE")
    fill = eng.debug_read("FILL", (2, 8), np.uint8)
    ht = eng.debug_read("HTILDE", (2, 8), np.float32)
    am = eng.debug_read("ARGMAX", (2, 8), np.int32)
    assert not fill.any() and np.isnan(ht).all() and (am == -1).all()
    for b in range(2):
        f, _ = eng.get_window(b)
        assert not any(f)
    eng.close()
