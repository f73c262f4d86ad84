"""Pins for the CPU oracle against what the paper and mathematics fix.

Each test checks the oracle against something other than itself: hand-derived
permutations from the paper's description, a brute-force construction, a
library routine (numpy / torch SDPA in fp64), or a closed form.  Together they
are chosen so that a dropped term, a wrong index or a transposed operand in
any oracle step fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from image_dits_b200.workload import random_grid_case

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_perm_cases():
    out = []
    with open(os.path.join(GOLDEN, "permutation_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, rhs = line.split(":")
            T, H, W, wt, wh, ww, sink = map(int, lhs.split())
            out.append(((T, H, W, wt, wh, ww, bool(sink)), [int(v) for v in rhs.split()]))
    return out


@pytest.mark.parametrize("case,expected", _golden_perm_cases())
def test_permutation_golden(case, expected):
    assert oracle.permutation(*case).tolist() == expected


def _window_walk(T, H, W, wt, wh, ww, sink):
    """Brute force: enumerate segments, then windows, then tokens, with loops."""
    frames = [list(range(1, T)), [0]] if (sink and T > 1) else [list(range(T))]
    out = []
    for seg in frames:
        for a0 in range(0, len(seg), wt):
            for h0 in range(0, H, wh):
                for w0 in range(0, W, ww):
                    for tl in range(a0, min(a0 + wt, len(seg))):
                        for h in range(h0, min(h0 + wh, H)):
                            for w in range(w0, min(w0 + ww, W)):
                                out.append((seg[tl] * H + h) * W + w)
    return out


def test_permutation_matches_window_walk():
    rng = np.random.default_rng(1)
    from image_dits_b200.workload import random_grid_case
    for _ in range(200):
        case = random_grid_case(rng, max_tokens=2000)
        assert oracle.permutation(*case).tolist() == _window_walk(*case), case


def test_permutation_identities():
    rng = np.random.default_rng(2)
    for _ in range(50):
        T, H, W = (int(v) for v in rng.integers(1, 9, 3))
        ident = list(range(T * H * W))
        assert oracle.permutation(T, H, W, 1, 1, 1, False).tolist() == ident
        assert oracle.permutation(T, H, W, T, H, W, False).tolist() == ident
        assert oracle.permutation(1, H, W, 1, 1 + H // 2, 2, True).tolist() == \
            oracle.permutation(1, H, W, 1, 1 + H // 2, 2, False).tolist()
        p = oracle.permutation(T, H, W, 2, 3, 2, bool(rng.integers(0, 2)))
        assert sorted(p.tolist()) == ident  # bijection


def test_permute_unpermute_roundtrip():
    rng = np.random.default_rng(3)
    x = rng.integers(0, 2**16, size=(3, 7 * 9 * 5, 16), dtype=np.uint16)
    perm = oracle.permutation(7, 9, 5, 4, 4, 4, True)
    xp = oracle.permute(x, perm)
    assert np.array_equal(xp, x[:, perm])
    assert np.array_equal(oracle.unpermute(xp, perm), x)


def test_geometry_golden():
    with open(os.path.join(GOLDEN, "workload_geometry.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert rows
    for r in rows:
        F, H, W, keep, sink = int(r[1]), int(r[2]), int(r[3]), float(r[4]), bool(int(r[5]))
        N, Tb, n, s0 = int(r[7]), int(r[8]), int(r[9]), int(r[10])
        assert F * H * W == N
        assert oracle.num_blocks(N) == Tb
        assert oracle.keep_count(keep, Tb) == n
        assert oracle.sink_start(F, H, W, sink) == s0


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_block_means_bruteforce():
    g = torch.Generator().manual_seed(4)
    x = _bf16_bits(torch.randn(2, 3, 200, 24, generator=g))   # 200 = 3 full blocks + 8
    m = oracle.block_means(x)
    xf = _bf16_to_f64(x)
    assert m.shape == (2, 3, 4, 24)
    for i in range(4):
        ref = xf[:, :, 64 * i:min(64 * i + 64, 200)].mean(axis=2)
        np.testing.assert_allclose(m[:, :, i], ref, rtol=1e-14, atol=1e-14)


def test_pooled_scores_library():
    rng = np.random.default_rng(5)
    qm, km = rng.standard_normal((3, 17, 32)), rng.standard_normal((3, 17, 32))
    S = oracle.pooled_scores(qm, km)
    np.testing.assert_allclose(S, qm @ np.swapaxes(km, -1, -2) / math.sqrt(32), rtol=1e-12, atol=1e-12)


def _topn_bruteforce(S, n, sink_first):
    Tb = S.shape[-1]
    mask = np.zeros(S.shape, np.uint8)
    for idx in np.ndindex(S.shape[:-1]):
        row = S[idx]
        i = idx[-1]
        if sink_first >= 0 and i >= sink_first:
            mask[idx] = 1
            continue
        order = np.lexsort((np.arange(Tb), -row))  # score desc, then j asc
        mask[idx + (order[:n],)] = 1
        if sink_first >= 0:
            mask[idx + (slice(sink_first, Tb),)] = 1
    return mask


@pytest.mark.parametrize("Tb,n,sink_first", [(16, 8, 12), (16, 8, -1), (37, 5, 30), (9, 9, -1), (20, 1, 0)])
def test_select_bruteforce(Tb, n, sink_first):
    rng = np.random.default_rng(6 + Tb)
    S = rng.standard_normal((2, Tb, Tb))
    S[0, 0, :4] = S[0, 0, 4]      # a tie that crosses the threshold in some rows
    mask, thr = oracle.select_blocks(S, n, sink_first)
    assert np.array_equal(mask, _topn_bruteforce(S, n, sink_first))
    for bh in range(2):
        for i in range(Tb):
            if sink_first >= 0 and i >= sink_first:
                assert mask[bh, i].all() and math.isnan(thr[bh, i])
            else:
                assert thr[bh, i] == np.sort(S[bh, i])[::-1][n - 1]
                n_sink = 0 if sink_first < 0 else Tb - sink_first
                assert n <= mask[bh, i].sum() <= min(Tb, n + n_sink)
                if sink_first >= 0:
                    assert mask[bh, i, sink_first:].all()


def test_select_ties_take_lowest_index():
    S = np.zeros((1, 6, 6))
    S[0, :, 3] = 1.0                   # one clear winner, then all ties at 0
    mask, _ = oracle.select_blocks(S, 3, -1)
    assert mask[0].tolist() == [[1, 1, 0, 1, 0, 0]] * 6


def test_select_keep_all():
    rng = np.random.default_rng(8)
    mask, _ = oracle.select_blocks(rng.standard_normal((1, 11, 11)), 11, -1)
    assert mask.all()


def test_identical_key_blocks_tie():
    """Identical K blocks give identical pooled scores: the lowest j must win."""
    rng = np.random.default_rng(9)
    N, d = 6 * 64, 16
    q = _bf16_bits(torch.from_numpy(rng.standard_normal((1, N, d))))
    kblk = rng.standard_normal((64, d))
    k = _bf16_bits(torch.from_numpy(np.tile(kblk, (6, 1))[None]))
    mask, thr, S = oracle.predict_mask(q, k, 0.5, 1, 6, 64, False)
    assert np.all(S[0] == S[0][:, :1])
    assert mask[0].tolist() == [[1, 1, 1, 0, 0, 0]] * 6


def _sdpa_f64(q, k, v, token_mask=None):
    qt = torch.from_numpy(_bf16_to_f64(q))
    kt = torch.from_numpy(_bf16_to_f64(k))
    vt = torch.from_numpy(_bf16_to_f64(v))
    am = None if token_mask is None else torch.from_numpy(token_mask.astype(bool))
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=am).numpy()


def _rand_qkv(BH, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return tuple(_bf16_bits(torch.randn(BH, N, d, generator=g) * s) for s in (1.0, 1.0, 1.0))


@pytest.mark.parametrize("N,d", [(200, 64), (128, 128), (64, 32), (3, 16)])
def test_dense_attention_matches_sdpa(N, d):
    q, k, v = _rand_qkv(2, N, d, seed=N + d)
    Tb = oracle.num_blocks(N)
    out, lse = oracle.full_attention_output(q, k, v, np.ones((2, Tb, Tb), np.uint8))
    np.testing.assert_allclose(out, _sdpa_f64(q, k, v), rtol=0, atol=1e-12)
    s = np.einsum("bnd,bmd->bnm", _bf16_to_f64(q), _bf16_to_f64(k)) / math.sqrt(d)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(s), -1).numpy(), rtol=0, atol=1e-10)


def test_sparse_attention_matches_masked_sdpa():
    N, d = 5 * 64 + 20, 32
    q, k, v = _rand_qkv(3, N, d, seed=11)
    Tb = oracle.num_blocks(N)
    rng = np.random.default_rng(12)
    mask = (rng.random((3, Tb, Tb)) < 0.4).astype(np.uint8)
    mask[:, np.arange(Tb), rng.integers(0, Tb, Tb)] = 1     # every row keeps something
    tok = np.repeat(np.repeat(mask, 64, axis=1), 64, axis=2)[:, :N, :N]
    out, _ = oracle.full_attention_output(q, k, v, mask)
    np.testing.assert_allclose(out, _sdpa_f64(q, k, v, tok), rtol=0, atol=1e-12)


def test_constant_value_single_block():
    """A row keeping a single key block whose V rows are all equal returns that
    V row (up to the fp64 rounding of sum(p*v)/sum(p))."""
    N, d = 3 * 64, 16
    q, k, _ = _rand_qkv(1, N, d, seed=13)
    vrow = _bf16_bits(torch.randn(d, generator=torch.Generator().manual_seed(14)))
    v = np.tile(vrow, (1, N, 1))
    mask = np.zeros((1, 3, 3), np.uint8)
    mask[0, :, 1] = 1
    out, _ = oracle.full_attention_output(q, k, v, mask)
    np.testing.assert_allclose(out, np.broadcast_to(_bf16_to_f64(vrow), out.shape), rtol=1e-14, atol=0)


def test_single_frame_sink_is_dense():
    """One frame with the sink on: every token is a first-frame token, so every
    query block is a sink row and the mask is full (section 3.4)."""
    q, k, v = _rand_qkv(1, 4 * 64, 16, seed=15)
    mask, _, _ = oracle.predict_mask(q, k, 0.25, 1, 16, 16, True)
    assert mask.all()


def test_sink_rows_and_columns():
    T, H, W = 4, 16, 16
    q, k, _ = _rand_qkv(2, T * H * W, 32, seed=16)
    mask, _, _ = oracle.predict_mask(q, k, 0.25, T, H, W, True)
    s0 = oracle.sink_start(T, H, W, True)
    assert s0 == 12
    assert mask[:, s0:, :].all()
    assert mask[:, :, s0:].all()
    counts = mask[:, :s0].sum(-1)
    assert (counts >= 4).all() and (counts <= 4 + 4).all()


# ---- CDF-threshold selection (section 2, online adaptive patterns) --------------------------


def test_cdf_uniform_scores_closed_form():
    """Equal scores: every block has p = 1/T_b, so m = ceil(tau * T_b) blocks,
    and the tie rule keeps the lowest indices."""
    Tb = 20
    S = np.full((1, Tb, Tb), 0.37)
    for tau, m in ((0.33, 7), (0.52, 11), (0.04, 1), (0.96, 20), (0.051, 2)):   # tau*T_b off the integers
        mask, cum, bnd = oracle.select_cdf(S, tau, -1)
        for i in range(Tb):
            assert np.array_equal(np.nonzero(mask[0, i])[0], np.arange(m)), (tau, m)
            assert cum[0, i, 1] >= tau > cum[0, i, 0]


def test_cdf_two_levels_hand_computed():
    """Three blocks with exp-weight 10, seventeen with weight 1 (total 47):
    cumulative 10/47, 20/47, 30/47, then +1/47 per low block."""
    Tb = 20
    row = np.zeros(Tb)
    hi = [4, 11, 17]
    row[hi] = math.log(10.0)
    S = row[None, None, :].repeat(Tb, 1)
    # tau 0.5: 20/47 = 0.4255 < 0.5 <= 30/47 -> the three high blocks
    mask, cum, _ = oracle.select_cdf(S, 0.5, -1)
    assert np.array_equal(np.nonzero(mask[0, 0])[0], hi)
    assert abs(cum[0, 0, 1] - 30 / 47) < 1e-12 and abs(cum[0, 0, 0] - 20 / 47) < 1e-12
    # tau 0.7: 30/47 + k/47 >= 0.7 -> k = 3 low blocks, the lowest indices (0, 1, 2)
    mask, cum, _ = oracle.select_cdf(S, 0.7, -1)
    assert np.array_equal(np.nonzero(mask[0, 0])[0], sorted(hi + [0, 1, 2]))
    assert abs(cum[0, 0, 1] - 33 / 47) < 1e-12
    # tau tiny: the single best block (lowest j among the equal best)
    mask, _, _ = oracle.select_cdf(S, 1e-9, -1)
    assert np.array_equal(np.nonzero(mask[0, 0])[0], [4])


def test_cdf_random_rows_brute_force():
    """The kept set is the shortest prefix of the (score desc, j asc) order whose
    softmax mass reaches tau (numpy lexsort + cumsum as the independent check)."""
    rng = np.random.default_rng(5)
    for Tb in (1, 2, 7, 33, 100):
        S = rng.normal(0.0, 2.0, size=(2, Tb, Tb))
        S[1, :, : Tb // 3] = S[1, :, :1]                   # ties
        for tau in (0.1, 0.5, 0.9, 0.999):
            mask, cum, bnd = oracle.select_cdf(S, tau, -1)
            for bh in range(2):
                for i in range(Tb):
                    s = S[bh, i]
                    order = np.lexsort((np.arange(Tb), -s))
                    p = np.exp(s - s.max())
                    p /= p.sum()
                    c = np.cumsum(p[order])
                    m = int(np.searchsorted(c >= tau, True)) + 1 if (c >= tau).any() else Tb
                    want = np.zeros(Tb, np.uint8)
                    want[order[:m]] = 1
                    assert np.array_equal(mask[bh, i], want), (Tb, tau, bh, i)
                    assert bnd[bh, i] == s[order[m - 1]]


def test_cdf_tau_one_keeps_everything_and_sink():
    rng = np.random.default_rng(6)
    Tb = 24
    S = rng.normal(size=(1, Tb, Tb))
    mask, _, _ = oracle.select_cdf(S, 1.0, -1)
    assert mask.all()
    mask, cum, _ = oracle.select_cdf(S, 0.3, 20)
    assert mask[0, 20:].all() and np.isnan(cum[0, 20:]).all()       # sink rows full
    assert mask[0, :20, 20:].all()                                    # sink columns kept
    # the CDF runs over every key block, sink columns included: where they carry the
    # mass a row keeps no other block; otherwise its kept non-sink blocks are its best
    s = S[0, :20]
    for i in range(20):
        kept = np.nonzero(mask[0, i, :20])[0]
        if kept.size:
            assert s[i, kept].min() >= np.sort(s[i, :20])[::-1][kept.size - 1]


# ---- text tokens of a joint video-text attention (section 3.4) -------------------------------


def test_text_geometry_golden():
    with open(os.path.join(GOLDEN, "text_geometry.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert rows
    for r in rows:
        F, H, W, text, sink = int(r[0]), int(r[1]), int(r[2]), int(r[3]), bool(int(r[4]))
        N, Tb, s0 = int(r[6]), int(r[7]), int(r[8])
        assert F * H * W + text == N
        assert oracle.num_blocks(N) == Tb
        assert oracle.sink_start(F, H, W, sink, text) == s0


def test_text_tokens_keep_their_place():
    """Text tokens follow the permuted video unmoved; the video part is the
    text-free permutation."""
    rng = np.random.default_rng(9)
    for _ in range(30):
        T, H, W, wt, wh, ww, sink = random_grid_case(rng, 1500)
        text = int(rng.integers(1, 100))
        nv = T * H * W
        perm = oracle.permutation(T, H, W, wt, wh, ww, sink, text)
        assert np.array_equal(perm[:nv], oracle.permutation(T, H, W, wt, wh, ww, sink))
        assert np.array_equal(perm[nv:], np.arange(nv, nv + text))


def test_text_sink_rows_and_columns():
    """With text tokens and the first-frame sink off, the blocks from the first
    text token on are full rows and are kept by every row."""
    rng = np.random.default_rng(10)
    T, H, W, text = 2, 8, 8, 70                         # N = 198, T_b = 4, text from token 128 (block 2)
    s0 = oracle.sink_start(T, H, W, False, text)
    assert s0 == 2
    S = rng.normal(size=(1, 4, 4))
    mask, _ = oracle.select_blocks(S, 1, s0)
    assert mask[0, 2:].all() and mask[0, :, 2:].all()
    # top-1 runs over every key block: a non-sink row keeps its best block when that
    # block is not already a sink column
    for i in range(2):
        best = int(np.argmax(S[0, i]))
        assert mask[0, i, :2].sum() == (1 if best < 2 else 0)
