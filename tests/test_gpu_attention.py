"""The decode attention kernel alone (wedlm_attention_bf16) against the oracle's
reordered-causal attention, at the context lengths and head groupings of the
workloads: committed lengths of 1k to 32k keys on scattered random page tables,
4 and 7 query heads per KV head, windows of 16 and 32 rows, ragged windows, an
empty cache, many sequences (more work items than SMs), and a corrupted page
table entry that the kernel's bounds check must catch without touching memory
outside the pool.

Reference: hyper.ai summary of arXiv 2512.22737, section Method: after
Topological Reordering the window runs a plain causal forward conditioned on
the persistent KV cache, so physical window row r attends to every cached key
and to window rows 0..r."""
import numpy as np
import pytest

import synth
from oracle import wedlm_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-2  # bf16 inputs, bf16 P and output: a few 2^-9 roundings


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def run_case(seed, hq, hkv, stride, S_list, n_list, q_std=1.0, corrupt=None):
    from streaming_decoding_b200 import attention_bf16, attention_error, attention_workspace
    n_seq = len(S_list)
    lengths = [S + n for S, n in zip(S_list, n_list)]
    pool, table = synth.paged_kv(seed, lengths, hkv)
    q = synth.normal(seed, 11, q_std, (n_seq * stride, hq, 128), "bf16")
    max_ctx = max(max(lengths), 1)
    ws = attention_workspace(n_seq, stride, hq, hkv, max_ctx)
    tab = table.copy()
    if corrupt is not None:
        b, i, v = corrupt
        tab[b, i] = v
    qd, pd = _bf16_dev(q), _bf16_dev(pool)
    out = torch.full_like(qd, float("nan"))
    S_d = torch.tensor(S_list, dtype=torch.int32, device="cuda")
    n_d = torch.tensor(n_list, dtype=torch.int32, device="cuda")
    t_d = torch.from_numpy(tab).cuda()
    attention_bf16(qd, pd, t_d, S_d, n_d, stride, hq, hkv, max_ctx, ws, out=out)
    torch.cuda.synchronize()
    err = attention_error(ws)
    got = out.float().cpu().numpy()
    # a second launch on the same workspace gives bit-identical results
    out2 = torch.full_like(qd, float("nan"))
    attention_bf16(qd, pd, t_d, S_d, n_d, stride, hq, hkv, max_ctx, ws, out=out2)
    torch.cuda.synchronize()
    return got, out2.float().cpu().numpy(), err, pool, table, q


def oracle_rows(pool, table, q, b, S, n, stride, hq, hkv):
    kv = synth.bf16_bits_to_f32(pool).astype(np.float64)
    pos = np.arange(S + n)
    pages = table[b, pos // 16]
    K = kv[pages, 0, :, pos % 16, :]   # [S+n, hkv, 128]
    V = kv[pages, 1, :, pos % 16, :]
    qb = synth.bf16_bits_to_f32(q[b * stride:b * stride + n]).astype(np.float64)
    return O.window_attention(qb, K[:S], V[:S], K[S:], V[S:])


def check(got, ref, rows):
    for r in range(rows):
        for h in range(ref.shape[1]):
            scale = np.abs(ref[r, h]).max()
            assert np.abs(got[r, h] - ref[r, h]).max() <= TOL * scale, (r, h)


@pytest.mark.parametrize("hq,hkv,stride,S_list,n_list", [
    (32, 8, 16, [4096, 16389], [16, 9]),     # g = 4, DUAL tiles, ragged window and page
    (28, 4, 32, [4000, 8192], [32, 17]),     # g = 7: two row tiles of 18 / 14 rows (126 and 98 query rows)
    (28, 4, 9, [1024, 3], [9, 5]),           # g = 7 DUAL (63 query rows)
    (32, 8, 16, [32768], [16]),              # the longest committed length of the microbench
    (32, 8, 16, [0, 1, 63, 64, 65], [16, 16, 1, 3, 0]),  # empty cache, single keys, empty window
])
def test_attention_matches_oracle(hq, hkv, stride, S_list, n_list):
    got, again, err, pool, table, q = run_case(5, hq, hkv, stride, S_list, n_list)
    assert err == 0
    assert np.array_equal(np.nan_to_num(got, nan=7.0), np.nan_to_num(again, nan=7.0))
    for b, (S, n) in enumerate(zip(S_list, n_list)):
        if n == 0:
            continue
        ref = oracle_rows(pool, table, q, b, S, n, stride, hq, hkv)
        check(got[b * stride:b * stride + n], ref, n)
        # rows past the window are not written
        assert np.isnan(got[b * stride + n:(b + 1) * stride]).all()


def test_attention_sharp_scores_many_sequences():
    """Scores with a wide spread (the running max moves by more than 2^8 inside
    a chunk, so O is rescaled) and 64 sequences at 1k-2k keys: more work items
    than SMs, several per CTA."""
    rng = np.random.default_rng(3)
    S_list = [int(x) for x in rng.integers(900, 2100, 64)]
    n_list = [int(x) for x in rng.integers(1, 17, 64)]
    got, again, err, pool, table, q = run_case(9, 32, 8, 16, S_list, n_list, q_std=6.0)
    assert err == 0
    assert np.array_equal(np.nan_to_num(got, nan=7.0), np.nan_to_num(again, nan=7.0))
    for b in (0, 17, 42, 63):
        ref = oracle_rows(pool, table, q, b, S_list[b], n_list[b], 16, 32, 8)
        check(got[b * 16:b * 16 + n_list[b]], ref, n_list[b])


def test_corrupted_page_id_is_caught():
    """A page id outside the pool: the kernel records a bounds error (1), reads
    a valid page instead and the GPU stays usable."""
    got, _, err, pool, table, q = run_case(13, 32, 8, 16, [2048, 1000], [16, 16],
                                           corrupt=(1, 10, 1 << 20))
    assert err == 1
    # the other sequence is still right
    ref = oracle_rows(pool, table, q, 0, 2048, 16, 16, 32, 8)
    check(got[:16], ref, 16)
    # and the device is healthy: a clean launch afterwards succeeds
    got2, _, err2, pool, table, q = run_case(13, 32, 8, 16, [2048], [16])
    assert err2 == 0
