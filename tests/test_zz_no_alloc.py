"""The allocation-free entropy selection agrees with the allocating one.

wedlm_entropy_select_noalloc serves callers that cannot allocate device memory
(a runtime that already owns the device through its own pool, or a thread that
must not risk the synchronisation an allocation can cause).  It keeps its
scratch in a fixed array inside the library, so this test calls it twice in a
row with different shapes and checks both results against wedlm_entropy_select
on the same inputs.  The file is named to be collected last and sets up all of
its own state, so it runs the same alone or after the other tests."""
import numpy as np
import pytest

import synth
from _gpu_util import MARGIN

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _inputs(seed, n_seq, stride, V, std):
    mask_id = V - 1
    filled, _ = synth.window_state(seed, 0, n_seq, stride, None, V, mask_id)
    n = (np.arange(n_seq) * 7 % stride + 1).astype(np.int32)
    n[0] = stride
    logits = synth.normal(seed, 77, std, (n_seq, stride, V), "f32")
    dev = lambda a, t: torch.as_tensor(np.ascontiguousarray(a)).to(t).cuda()  # noqa: E731
    return dev(logits, torch.float32), dev(filled, torch.uint8), dev(n, torch.int32), mask_id


def _same(ref, got):
    ht_r, am_r, fl_r = (t.cpu().numpy() for t in ref)
    ht_g, am_g, fl_g = (t.cpu().numpy() for t in got)
    assert np.array_equal(np.isnan(ht_r), np.isnan(ht_g))
    ok = ~np.isnan(ht_r)
    assert np.all(np.abs(ht_r[ok] - ht_g[ok]) < MARGIN)
    assert np.array_equal(am_r, am_g)
    assert np.array_equal(fl_r, fl_g)
    assert ok.sum() > 0 and fl_r.sum() > 0


def test_noalloc_matches_allocating_entry_on_two_calls_in_a_row():
    from streaming_decoding_b200 import entropy_select, entropy_select_noalloc, step_params
    cases = [
        (dict(seed=4101, n_seq=8, stride=16, V=151936, std=4.0), step_params(0.1, 5.0, False, 1.0)),
        (dict(seed=4102, n_seq=3, stride=32, V=1000, std=2.0), step_params(0.05, 0.3, False, 4.0)),
    ]
    for shape, prm in cases:
        logits, filled, n, mask_id = _inputs(**shape)
        stride, V = shape["stride"], shape["V"]
        ref = entropy_select(logits, V, mask_id, filled, n, stride, prm)
        got = entropy_select_noalloc(logits, V, mask_id, filled, n, stride, prm)
        _same(ref, got)


def test_noalloc_rejects_more_rows_than_its_scratch_holds():
    from streaming_decoding_b200 import entropy_select_noalloc, step_params
    from streaming_decoding_b200._lib import WedlmError, header_constants
    C = header_constants()
    stride = 16
    n_seq = C["WEDLM_NOALLOC_MAX_ROWS"] // stride + 1
    logits, filled, n, mask_id = _inputs(seed=4103, n_seq=n_seq, stride=stride, V=64, std=1.0)
    with pytest.raises(WedlmError) as e:
        entropy_select_noalloc(logits, 64, mask_id, filled, n, stride, step_params(0.1, 0.5))
    assert e.value.status == C["WEDLM_ERR_INVALID_ARG"]
