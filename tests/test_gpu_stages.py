"""Single stages of the step on the GPU against the CPU oracle, through the C ABI."""
import numpy as np
import pytest

import synth
from oracle import wedlm_oracle as O
from _gpu_util import MARGIN, comparable, oracle_select

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _dev(a, dtype):
    return torch.as_tensor(np.ascontiguousarray(a)).to(dtype).cuda()


@pytest.mark.parametrize("W", range(1, 9))
def test_reorder_exhaustive_small_windows(W):
    """Topological reordering: bit-exact with the oracle over all 2^W fill patterns."""
    from streaming_decoding_b200 import reorder_window
    pats = np.array([[(b >> j) & 1 for j in range(W)] for b in range(1 << W)], np.uint8)
    n = np.full(len(pats), W, np.int32)
    S = (np.arange(len(pats)) * 7 + 3).astype(np.int32)
    perm, pos, k, nf = reorder_window(_dev(pats, torch.uint8), _dev(n, torch.int32), _dev(S, torch.int32), W)
    perm, pos, k, nf = (t.cpu().numpy() for t in (perm, pos, k, nf))
    for i, f in enumerate(pats):
        want = O.reorder(list(f))
        assert perm[i].tolist() == want
        assert pos[i].tolist() == [int(S[i]) + j for j in want]
        assert k[i] == O.leading_filled(list(f))
        assert nf[i] == int(f.sum())


@pytest.mark.parametrize("stride", [16, 32, 64])
def test_reorder_random_ragged(stride):
    from streaming_decoding_b200 import reorder_window
    rng = np.random.default_rng(stride)
    n_seq = 300
    pats = (rng.random((n_seq, stride)) < rng.random((n_seq, 1))).astype(np.uint8)
    n = rng.integers(0, stride + 1, n_seq).astype(np.int32)
    S = rng.integers(0, 40000, n_seq).astype(np.int32)
    perm, pos, k, nf = reorder_window(_dev(pats, torch.uint8), _dev(n, torch.int32), _dev(S, torch.int32), stride)
    perm, pos, k, nf = (t.cpu().numpy() for t in (perm, pos, k, nf))
    for i in range(n_seq):
        f = list(pats[i, :n[i]])
        want = O.reorder(f)
        assert perm[i, :n[i]].tolist() == want and all(perm[i, n[i]:] == -1)
        assert pos[i, :n[i]].tolist() == [int(S[i]) + j for j in want]
        assert k[i] == O.leading_filled(f) and nf[i] == sum(f)


@pytest.mark.parametrize("V,logit_std,lam,tau,tau_none,scale", [
    (151936, 1.0, 0.1, 0.3, False, 1.0),
    (151936, 4.0, 0.1, 5.0, False, 1.0),
    (151936, 16.0, 0.05, 0.5, False, 1.0),
    (151936, 1.0, 0.2, 0.1, True, 4.0),
    (512, 1.8, 0.1, 5.0, False, 8.0),
    (1000, 2.0, 0.0, 100.0, False, 1.0),
])
def test_entropy_select_matches_oracle(V, logit_std, lam, tau, tau_none, scale):
    """Fed the same fp32 logits, the GPU's entropy, argmax and fill decisions
    equal the oracle's (H~ within 1e-3 nats; decisions exact where comparable)."""
    from streaming_decoding_b200 import entropy_select, step_params
    n_seq, stride = 6, 16
    mask_id = V - 1
    filled, _ = synth.window_state(2000 + V % 97, 0, n_seq, stride, None, V, mask_id)
    n = np.array([16, 16, 9, 1, 13, 16], np.int32)
    logits = synth.normal(2100, int(logit_std * 10), logit_std, (n_seq, stride, V), "f32")
    # an exact tie for the argmax rule in the first masked slot of sequence 0
    j0 = int(np.nonzero(filled[0, :n[0]] == 0)[0][0])
    logits[0, j0, 7] = logits[0, j0, 9] = logits[0, j0].max() + 1.0
    prm = step_params(lam, tau, tau_none, scale)
    ht, am, fill = entropy_select(_dev(logits, torch.float32), V, mask_id, _dev(filled, torch.uint8),
                                  _dev(n, torch.int32), stride, prm)
    ht, am, fill = ht.cpu().numpy(), am.cpu().numpy(), fill.cpu().numpy()
    n_compared = 0
    for b in range(n_seq):
        rows = {j: logits[b, j] for j in range(n[b]) if not filled[b, j]}
        Ht, amax, fills = oracle_select(rows, mask_id, lam, tau, tau_none, scale)
        for j in range(stride):
            if j in rows:
                assert abs(ht[b, j] - Ht[j]) < MARGIN, (b, j, ht[b, j], Ht[j])
                assert am[b, j] == amax[j]
            else:
                assert np.isnan(ht[b, j]) and am[b, j] == -1 and fill[b, j] == 0
        if comparable(Ht, tau, tau_none):
            assert sorted(np.nonzero(fill[b])[0].tolist()) == fills
            n_compared += 1
    assert n_compared >= n_seq - 1
    assert am[0, j0] == 7  # lowest id among tied maxima


@pytest.mark.parametrize("M,N,K", [(16, 6144, 4096), (1, 300, 64), (37, 1000, 520), (128, 4096, 4096),
                                   (256, 4096, 12288), (300, 384, 256), (2048, 512, 3584)])
def test_linear_bf16_matches_fp64_matmul(M, N, K):
    """The tcgen05 GEMM (every projection of the step) against an fp64 matmul of
    the same bf16 inputs: bf16 products are exact in fp32, so only fp32
    accumulation error remains."""
    from streaming_decoding_b200 import linear_bf16
    X = synth.normal(31, M * 7 + K, 1.0, (M, K), "bf16")
    W = synth.normal(32, N * 3 + K, 0.02, (N, K), "bf16")
    Xt = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wt = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    Y = linear_bf16(Xt, Wt).cpu().numpy().astype(np.float64)
    ref = synth.bf16_bits_to_f32(X).astype(np.float64) @ synth.bf16_bits_to_f32(W).astype(np.float64).T
    bound = np.abs(synth.bf16_bits_to_f32(X)).astype(np.float64) @ np.abs(synth.bf16_bits_to_f32(W)).astype(np.float64).T
    err = np.abs(Y - ref)
    assert np.all(err <= 1e-4 * bound + 1e-30), float((err / (bound + 1e-30)).max())


@pytest.mark.parametrize("M,N,K,tile_n,k_splits", [
    (256, 6144, 4096, 256, 1),    # QKV-shaped, whole pair tiles
    (256, 4096, 4096, 256, 3),    # K in slices (last-arriver reduction)
    (200, 1152, 520, 256, 1),     # ragged rows, a half-empty pair tile (N % 256 = 128), ragged K
    (256, 1000, 4096, 128, 2),    # two activation tiles per pair tile, ragged N
    (96, 2048, 1024, 128, 1),     # fewer rows than the tile: the odd CTA's half is padding
    (512, 768, 256, 256, 1),      # several activation tiles
])
def test_linear_bf16_cta_pair_matches_fp64_matmul(M, N, K, tile_n, k_splits):
    """CTA-pair tiles (two-CTA tensor-core MMA, operands split across the pair's
    shared memory) against the same fp64 matmul and bound as above."""
    from streaming_decoding_b200 import linear_bf16
    X = synth.normal(33, M * 5 + K, 1.0, (M, K), "bf16")
    W = synth.normal(34, N * 11 + K, 0.02, (N, K), "bf16")
    Xt = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wt = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    Y = linear_bf16(Xt, Wt, tile_n=tile_n, k_splits=k_splits, cta_pair=True).cpu().numpy().astype(np.float64)
    x64 = synth.bf16_bits_to_f32(X).astype(np.float64)
    w64 = synth.bf16_bits_to_f32(W).astype(np.float64)
    ref = x64 @ w64.T
    bound = np.abs(x64) @ np.abs(w64).T
    err = np.abs(Y - ref)
    assert np.all(err <= 1e-4 * bound + 1e-30), float((err / (bound + 1e-30)).max())
    # the same plan without pairs agrees to accumulation order
    Y1 = linear_bf16(Xt, Wt, tile_n=tile_n, k_splits=k_splits).cpu().numpy().astype(np.float64)
    assert np.all(np.abs(Y - Y1) <= 2e-4 * bound + 1e-30)


@pytest.mark.parametrize("M,N,K,tile_n,k_splits,pair", [
    (256, 10240, 512, 128, 3, False),   # 160 tiles: one full round of 148 CTAs, 12 tiles split
    (256, 20480, 256, 256, 2, True),    # 80 pair tiles: a full round of pairs, the rest split
    (200, 10368, 520, 128, 4, False),   # ragged rows and K, a partial round of split tiles
    (64, 1024, 1024, 128, 3, False),    # fewer tiles than CTAs: every tile split
])
def test_linear_bf16_hybrid_split_matches_fp64_matmul(M, N, K, tile_n, k_splits, pair):
    """Hybrid schedule (whole-K tiles for the full rounds of the persistent grid,
    K slices only for the last partial round) against the fp64 matmul and bound
    as above, and against the plain single-slice plan."""
    from streaming_decoding_b200 import linear_bf16
    X = synth.normal(35, M * 3 + K, 1.0, (M, K), "bf16")
    W = synth.normal(36, N * 7 + K, 0.02, (N, K), "bf16")
    Xt = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wt = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    Y = linear_bf16(Xt, Wt, tile_n=tile_n, k_splits=k_splits, cta_pair=pair, hybrid=True)
    Y = Y.cpu().numpy().astype(np.float64)
    x64 = synth.bf16_bits_to_f32(X).astype(np.float64)
    w64 = synth.bf16_bits_to_f32(W).astype(np.float64)
    ref = x64 @ w64.T
    bound = np.abs(x64) @ np.abs(w64).T
    err = np.abs(Y - ref)
    assert np.all(err <= 1e-4 * bound + 1e-30), float((err / (bound + 1e-30)).max())
    Y1 = linear_bf16(Xt, Wt, tile_n=tile_n, k_splits=1, cta_pair=pair).cpu().numpy().astype(np.float64)
    assert np.all(np.abs(Y - Y1) <= 2e-4 * bound + 1e-30)


@pytest.mark.parametrize("M,N,K,tile_n,k_splits", [
    (256, 4096, 12288, 256, 4),   # the down projection's shape, four slices per cluster
    (256, 4096, 4096, 128, 2),
    (200, 1000, 520, 256, 3),     # ragged rows, N and K (9 k-blocks in 3 slices)
    (96, 2048, 1024, 128, 4),     # fewer rows than the tile
])
def test_linear_bf16_cluster_k_split_matches_fp64_matmul(M, N, K, tile_n, k_splits):
    """K slices of a tile as the CTAs of one cluster, reduced through distributed
    shared memory, against the fp64 matmul and bound as above, and against the
    plain single-slice plan."""
    from streaming_decoding_b200 import linear_bf16
    X = synth.normal(37, M * 13 + K, 1.0, (M, K), "bf16")
    W = synth.normal(38, N * 5 + K, 0.02, (N, K), "bf16")
    Xt = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Wt = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    Y = linear_bf16(Xt, Wt, tile_n=tile_n, k_splits=k_splits, cluster_k=True).cpu().numpy().astype(np.float64)
    x64 = synth.bf16_bits_to_f32(X).astype(np.float64)
    w64 = synth.bf16_bits_to_f32(W).astype(np.float64)
    ref = x64 @ w64.T
    bound = np.abs(x64) @ np.abs(w64).T
    err = np.abs(Y - ref)
    assert np.all(err <= 1e-4 * bound + 1e-30), float((err / (bound + 1e-30)).max())
    Y1 = linear_bf16(Xt, Wt, tile_n=tile_n, k_splits=1).cpu().numpy().astype(np.float64)
    assert np.all(np.abs(Y - Y1) <= 2e-4 * bound + 1e-30)
    # deterministic: the slices are summed in a fixed order
    Y2 = linear_bf16(Xt, Wt, tile_n=tile_n, k_splits=k_splits, cluster_k=True).cpu().numpy().astype(np.float64)
    assert np.array_equal(Y, Y2)
