"""Pins for the CPU oracle: facts fixed by the pages or by mathematics, not by the oracle.

Each test checks the oracle against something other than itself: the keep-ratio
table the pages print, closed forms worked by hand, brute force on tiny inputs,
library routines for the special cases that reduce to textbook operations, and
invariants (relative rotary positions, softmax normalisation).
"""
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_inputs(B, N, H, d, r, seed=0):
    g = _rng(seed)
    q = g.standard_normal((B, N, H, d)).astype(np.float32)
    k = g.standard_normal((B, N, H, d)).astype(np.float32)
    v = g.standard_normal((B, N, H, d)).astype(np.float32)
    Wq = (g.standard_normal((H, d, r)) / math.sqrt(d)).astype(np.float32)
    Wk = (g.standard_normal((H, d, r)) / math.sqrt(d)).astype(np.float32)
    gain = g.uniform(0.1, 1.0, H)
    return q, k, v, Wq, Wk, gain


def _all_blocks(B, H, nb):
    return np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(nb)], np.int32)


# ---------------------------------------------------------------- keep ratio (pages' table)

def _golden_keep_ratio():
    rows = []
    with open(os.path.join(GOLDEN, "keep_ratio.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                t, s = line.split()
                rows.append((float(t), int(s)))
    return rows


def test_keep_ratio_matches_pages():
    rows = _golden_keep_ratio()
    assert len(rows) == 3
    for topk, sparsity in rows:
        # Block counts that are multiples of 100: the sparsity is exactly the printed one.
        for nb in (100, 200, 300, 700, 1000, 2000):
            k = O.keep_count(nb, topk)
            assert k * 100 == (100 - sparsity) * nb, (topk, nb, k)
        # Workload block counts (480P: 512 blocks, 720P: 1182): rounds to the printed value.
        for nb in (512, 1182):
            k = O.keep_count(nb, topk)
            assert round(100 * (1 - k / nb)) == sparsity


def test_keep_count_edges():
    assert O.keep_count(16, 0.25) == 4
    assert O.keep_count(16, 1.0) == 16
    assert O.keep_count(16, 1e-6) == 1        # never fewer than one block
    assert O.keep_count(1, 0.03) == 1
    # 0.07 * 100 is 7.000000000000001 in binary floating point: still 7 blocks.
    assert 0.07 * 100 > 7
    assert O.keep_count(100, 0.07) == 7
    assert O.keep_count(512, 0.10) == 52 and O.keep_count(1182, 0.03) == 36


# ---------------------------------------------------------------- pooling

def test_pool_fp32_token_order_with_ragged_tail():
    B, N, H, d = 2, 200, 3, 8          # nb = 4, last block 8 tokens
    x = _rng(1).standard_normal((B, N, H, d)).astype(np.float32)
    s = O.make_shape(B, H, N, d, 4, 0.5)
    got = O.pool(s, x)
    nb = 4
    assert got.shape == (B, H, nb, d) and got.dtype == np.float32
    for i in range(nb):
        n0, n1 = 64 * i, min(N, 64 * i + 64)
        # np.cumsum on float32 adds in order with one rounding per step.
        tot = np.cumsum(x[:, n0:n1], axis=1, dtype=np.float32)[:, -1]   # [B, H, d]
        want = tot / np.float32(n1 - n0)
        np.testing.assert_array_equal(got[:, :, i], want)
    # exact means on integer data
    xi = _rng(2).integers(-8, 8, (B, N, H, d)).astype(np.float32)
    gi = O.pool(s, xi)
    for i in range(nb):
        n0, n1 = 64 * i, min(N, 64 * i + 64)
        np.testing.assert_allclose(gi[:, :, i], xi[:, n0:n1].astype(np.float64).mean(1), rtol=1e-7)


# ---------------------------------------------------------------- selection

def _brute_topk(scores, k):
    """Full stable ordering by (-score, index); the first k, ascending."""
    nb = scores.shape[-1]
    order = np.lexsort((np.arange(nb), -scores))
    return np.sort(order[:k])


@pytest.mark.parametrize("topk", [0.1, 0.25, 0.5, 1.0])
def test_select_matches_brute_force_with_exact_ties(topk):
    B, H, nb, d = 1, 2, 24, 16
    N = nb * 64 - 40                    # ragged last block (24 tokens)
    g = _rng(3)
    # Small integers: every fp32 fused multiply-add chain is exact, so exact ties are real.
    qbar = g.integers(-3, 4, (B, H, nb, d)).astype(np.float32)
    kbar = g.integers(-3, 4, (B, H, nb, d)).astype(np.float32)
    kbar[:, :, 7] = kbar[:, :, 2]       # duplicated key blocks: exact score ties
    kbar[:, :, 19] = kbar[:, :, 2]
    kbar[:, :, 11] = kbar[:, :, 20]
    qbar[:, :, 5] = 0                   # a row where every score ties at 0
    s = O.make_shape(B, H, N, d, 4, topk)
    col, kth, nxt, amax = O.select(s, qbar, kbar)
    k = O.keep_count(nb, topk)
    assert col.shape == (B, H, nb, k)
    exact = np.einsum("bhid,bhjd->bhij", qbar.astype(np.int64), kbar.astype(np.int64))
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                want = _brute_topk(exact[b, h, i].astype(np.float64), k)
                np.testing.assert_array_equal(col[b, h, i], want)
                srt = np.sort(exact[b, h, i])[::-1]
                assert kth[b, h, i] == srt[k - 1]
                assert amax[b, h, i] == np.abs(exact[b, h, i]).max()
                if k < nb:
                    assert nxt[b, h, i] == srt[k]
    # the all-tie row keeps the lowest indices
    np.testing.assert_array_equal(col[0, 0, 5], np.arange(k))


def test_select_agrees_with_double_scores_away_from_ties():
    B, H, nb, d = 1, 2, 40, 32
    g = _rng(4)
    qbar = g.standard_normal((B, H, nb, d)).astype(np.float32)
    kbar = g.standard_normal((B, H, nb, d)).astype(np.float32)
    s = O.make_shape(B, H, nb * 64, d, 4, 0.2)
    col, *_ = O.select(s, qbar, kbar)
    k = O.keep_count(nb, 0.2)
    sc = np.einsum("bhid,bhjd->bhij", qbar.astype(np.float64), kbar.astype(np.float64))
    checked = 0
    for h in range(H):
        for i in range(nb):
            srt = np.sort(sc[0, h, i])[::-1]
            if srt[k - 1] - srt[k] > 1e-4 * np.abs(srt).max():
                np.testing.assert_array_equal(col[0, h, i], _brute_topk(sc[0, h, i], k))
                checked += 1
    assert checked > nb


# ---------------------------------------------------------------- sparse branch

def _dense_attention(q, k, v, scale):
    """Textbook softmax attention per (b, h) with numpy matmuls."""
    B, N, H, d = q.shape
    out = np.zeros((B, N, H, d))
    for b in range(B):
        for h in range(H):
            a = q[b, :, h].astype(np.float64) @ k[b, :, h].astype(np.float64).T * scale
            a -= a.max(1, keepdims=True)
            p = np.exp(a)
            p /= p.sum(1, keepdims=True)
            out[b, :, h] = p @ v[b, :, h].astype(np.float64)
    return out


def test_dense_limit_equals_softmax_attention():
    """topk = 1 and g = 0: RoLA is plain softmax attention over all keys."""
    B, N, H, d, r = 2, 200, 2, 16, 4
    q, k, v, Wq, Wk, _ = _rand_inputs(B, N, H, d, r, seed=5)
    s = O.make_shape(B, H, N, d, r, 1.0, grid=(2, 4, 25))
    out, col = O.forward(s, q, k, v, Wq, Wk, np.zeros(H))
    np.testing.assert_array_equal(col, np.broadcast_to(np.arange(4), col.shape))
    np.testing.assert_allclose(out, _dense_attention(q, k, v, 1 / math.sqrt(d)), rtol=0, atol=1e-12)


def test_sparse_branch_equals_masked_dense_attention():
    """Any mask: the sparse branch equals dense attention with the dropped blocks at -inf."""
    B, N, H, d, r = 1, 300, 2, 16, 4
    q, k, v, Wq, Wk, gain = _rand_inputs(B, N, H, d, r, seed=6)
    s = O.make_shape(B, H, N, d, r, 0.4, grid=(1, 1, N))
    nb = 5
    qbar, kbar = O.pool(s, q), O.pool(s, k)
    col, *_ = O.select(s, qbar, kbar)
    S, z = O.linear_state(s, k, v, Wk)
    sp, li, out = O.attend_blocks(s, q, k, v, Wq, gain, col, S, z, _all_blocks(B, H, nb))
    scale = 1 / math.sqrt(d)
    t = 0
    for h in range(H):
        a = q[0, :, h].astype(np.float64) @ k[0, :, h].astype(np.float64).T * scale
        keep = np.zeros((N, N), bool)
        for i in range(nb):
            for j in col[0, h, i]:
                keep[64 * i:64 * i + 64, 64 * j:64 * j + 64] = True
        a[~keep] = -np.inf
        a -= a.max(1, keepdims=True)
        p = np.exp(a)
        p /= p.sum(1, keepdims=True)
        want = p @ v[0, :, h].astype(np.float64)
        for i in range(nb):
            n1 = min(N, 64 * i + 64)
            np.testing.assert_allclose(sp[t, :n1 - 64 * i], want[64 * i:n1], atol=1e-12)
            assert np.all(sp[t, n1 - 64 * i:] == 0)
            t += 1


def test_constant_values_give_constant_sparse_output():
    """Softmax weights sum to one: v = c everywhere gives O_sparse = c."""
    B, N, H, d, r = 1, 256, 2, 8, 4
    q, k, v, Wq, Wk, gain = _rand_inputs(B, N, H, d, r, seed=7)
    c = _rng(8).standard_normal(d).astype(np.float32)
    v[:] = c
    s = O.make_shape(B, H, N, d, r, 0.5, grid=(2, 2, 64))
    col, *_ = O.select(s, O.pool(s, q), O.pool(s, k))
    S, z = O.linear_state(s, k, v, Wk)
    sp, li, out = O.attend_blocks(s, q, k, v, Wq, gain, col, S, z, _all_blocks(B, H, 4))
    np.testing.assert_allclose(sp, np.broadcast_to(c, sp.shape), atol=1e-12)


# ---------------------------------------------------------------- linear branch

def _phi(x):
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0)))


def _rotation_matrix(r, angles):
    """R = expm(sum_c angle_c * J_c), J_c the generator of pair (2c, 2c+1)."""
    G = np.zeros((r, r))
    for c, a in enumerate(angles):
        G[2 * c + 1, 2 * c] = a
        G[2 * c, 2 * c + 1] = -a
    return scipy.linalg.expm(G)


def test_linear_branch_closed_form_two_tokens():
    """Hand-worked example: 2 tokens at x = 0, 1; r = d = 4, two rotary pairs on w,
    base 4 so the pair frequencies are 1 and 1/2; Wq = Wk = I."""
    s = O.make_shape(1, 1, 2, 4, 4, 1.0, grid=(1, 1, 2), pairs=(0, 0, 2), rope_base=4.0)
    I = np.eye(4, dtype=np.float32)[None]
    q = np.zeros((1, 2, 1, 4), np.float32)
    k = np.zeros((1, 2, 1, 4), np.float32)
    v = np.zeros((1, 2, 1, 4), np.float32)
    q[0, 1, 0] = [-1, 0, 0, 0]         # u_1 = (e^-1, 1, 1, 1); u_0 = (1, 1, 1, 1)
    k[0, 0, 0] = [1, 0, 0, 0]          # f_0 = (2, 1, 1, 1);    f_1 = (1, 1, 1, 1)
    v[0, 0, 0] = [1, 0, 0, 0]
    v[0, 1, 0] = [0, 1, 0, 0]
    S, z = O.linear_state(s, k, v, I)
    np.testing.assert_allclose(z[0, 0], [3, 2, 2, 2], atol=1e-15)
    col = np.zeros((1, 1, 1, 1), np.int32)
    _, li, _ = O.attend_blocks(s, q, k, v, I, np.ones(1), col, S, z, [(0, 0, 0)])
    e = math.exp(-1)
    c1, s1, c5, s5 = math.cos(1), math.sin(1), math.cos(0.5), math.sin(0.5)
    # query 0: <u0, f0> v0 + <u0, R(+1) f1> v1 over <u0, f0> + <u0, f1>
    want0 = [5 / 9, (2 * c1 + 2 * c5) / 9, 0, 0]
    # query 1: <u1, R(-1) f0> v0 + <u1, f1> v1 over <u1, f0> + <u1, f1>
    den1 = 3 * e + 6
    want1 = [(e * (2 * c1 + s1) + (c1 - 2 * s1) + 2 * c5) / den1, (e + 3) / den1, 0, 0]
    np.testing.assert_allclose(li[0, 0], want0, atol=1e-14)
    np.testing.assert_allclose(li[0, 1], want1, atol=1e-14)


def _explicit_linear(s, q, k, v, Wq, Wk, pos):
    """O_lin from its N x N kernel-matrix form, rotations built as matrix exponentials."""
    B, N, H, d = q.shape
    r = s.r
    pairs = [(0, s.pairs_t)] * s.pairs_t + [(1, s.pairs_h)] * s.pairs_h + [(2, s.pairs_w)] * s.pairs_w
    sub = list(range(s.pairs_t)) + list(range(s.pairs_h)) + list(range(s.pairs_w))
    R = [_rotation_matrix(r, [pos[n, ax] * s.rope_base ** (-cp / cnt)
                              for (ax, cnt), cp in zip(pairs, sub)]) for n in range(N)]
    out = np.zeros((B, N, H, d))
    for b in range(B):
        for h in range(H):
            U = _phi(q[b, :, h].astype(np.float64) @ Wq[h].astype(np.float64))
            F = _phi(k[b, :, h].astype(np.float64) @ Wk[h].astype(np.float64))
            RU = np.stack([R[n] @ U[n] for n in range(N)])
            RF = np.stack([R[n] @ F[n] for n in range(N)])
            A = RU @ RF.T
            D = U @ F.T
            out[b, :, h] = (A @ v[b, :, h].astype(np.float64)) / D.sum(1, keepdims=True)
    return out


def _oracle_lin(s, q, k, v, Wq, Wk, pos):
    B, N, H, d = q.shape
    nb = (N + 63) // 64
    col = np.zeros((B, H, nb, 1), np.int32)
    S, z = O.linear_state(s, k, v, Wk, pos)
    _, li, _ = O.attend_blocks(s, q, k, v, Wq, np.ones(H), col, S, z, _all_blocks(B, H, nb), pos)
    out = np.zeros((B, N, H, d))
    t = 0
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                n1 = min(N, 64 * i + 64)
                out[b, 64 * i:n1, h] = li[t, :n1 - 64 * i]
                t += 1
    return out


@pytest.mark.parametrize("grid,pairs", [((2, 4, 12), None), ((1, 1, 96), None), ((3, 4, 8), (1, 2, 1))])
def test_linear_branch_equals_explicit_kernel_matrix(grid, pairs):
    B, H, d, r = 1, 2, 16, 8
    N = grid[0] * grid[1] * grid[2]
    q, k, v, Wq, Wk, _ = _rand_inputs(B, N, H, d, r, seed=9)
    s = O.make_shape(B, H, N, d, r, 0.5, grid=grid, pairs=pairs)
    pos = O.positions(s)
    np.testing.assert_allclose(_oracle_lin(s, q, k, v, Wq, Wk, pos),
                               _explicit_linear(s, q, k, v, Wq, Wk, pos), rtol=1e-9, atol=1e-10)


def test_grid_positions_flatten_t_h_w():
    s = O.make_shape(1, 1, 24, 4, 4, 1.0, grid=(2, 3, 4))
    pos = O.positions(s)
    n = 1 * 12 + 2 * 4 + 3                  # t=1, y=2, x=3
    np.testing.assert_array_equal(pos[n], [1, 2, 3])
    assert O.default_pairs(32, (21, 30, 52)) == (6, 5, 5)
    assert O.default_pairs(16, (1, 1, 1024)) == (0, 0, 8)


def test_linear_branch_depends_only_on_position_differences():
    B, N, H, d, r = 1, 120, 2, 16, 8
    q, k, v, Wq, Wk, _ = _rand_inputs(B, N, H, d, r, seed=10)
    s = O.make_shape(B, H, N, d, r, 0.5, grid=(2, 6, 10))
    pos = O.positions(s)
    base = _oracle_lin(s, q, k, v, Wq, Wk, pos)
    shifted = _oracle_lin(s, q, k, v, Wq, Wk, pos + np.array([3.0, -2.0, 5.0]))
    np.testing.assert_allclose(shifted, base, rtol=1e-10, atol=1e-12)
    # a shift of one token only must change the result (positions are really used)
    p2 = pos.copy()
    p2[7] += np.array([0.0, 1.0, 0.0])
    assert np.abs(_oracle_lin(s, q, k, v, Wq, Wk, p2) - base).max() > 1e-6


def test_zero_angles_give_textbook_linear_attention():
    B, N, H, d, r = 1, 100, 2, 16, 8
    q, k, v, Wq, Wk, _ = _rand_inputs(B, N, H, d, r, seed=11)
    s = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 1, N))
    pos = np.zeros((N, 3))
    got = _oracle_lin(s, q, k, v, Wq, Wk, pos)
    for h in range(H):
        U = _phi(q[0, :, h].astype(np.float64) @ Wq[h].astype(np.float64))
        F = _phi(k[0, :, h].astype(np.float64) @ Wk[h].astype(np.float64))
        want = (U @ (F.T @ v[0, :, h].astype(np.float64))) / (U @ F.sum(0))[:, None]
        np.testing.assert_allclose(got[0, :, h], want, rtol=1e-11, atol=1e-12)


def test_constant_values_and_zero_angles_give_c_times_one_plus_g():
    B, N, H, d, r = 1, 128, 3, 8, 4
    q, k, v, Wq, Wk, gain = _rand_inputs(B, N, H, d, r, seed=12)
    c = _rng(13).standard_normal(d).astype(np.float32)
    v[:] = c
    s = O.make_shape(B, H, N, d, r, 0.5)
    pos = np.zeros((N, 3))
    col, *_ = O.select(s, O.pool(s, q), O.pool(s, k))
    S, z = O.linear_state(s, k, v, Wk, pos)
    _, _, out = O.attend_blocks(s, q, k, v, Wq, gain, col, S, z, _all_blocks(B, H, 2), pos)
    for t, (b, h, i) in enumerate(_all_blocks(B, H, 2)):
        np.testing.assert_allclose(out[t], np.broadcast_to(c * (1 + gain[h]), (64, d)), atol=1e-12)


def test_zero_gain_gives_sparse_branch_and_gain_is_linear():
    B, N, H, d, r = 1, 192, 2, 16, 8
    q, k, v, Wq, Wk, gain = _rand_inputs(B, N, H, d, r, seed=14)
    s = O.make_shape(B, H, N, d, r, 0.34, grid=(1, 3, 64))
    col, *_ = O.select(s, O.pool(s, q), O.pool(s, k))
    S, z = O.linear_state(s, k, v, Wk)
    blocks = _all_blocks(B, H, 3)
    sp, li, out0 = O.attend_blocks(s, q, k, v, Wq, np.zeros(H), col, S, z, blocks)
    np.testing.assert_array_equal(out0, sp)
    _, _, out = O.attend_blocks(s, q, k, v, Wq, gain, col, S, z, blocks)
    for t, (b, h, i) in enumerate(blocks):
        np.testing.assert_allclose(out[t], sp[t] + gain[h] * li[t], atol=1e-13)


def test_per_token_gate_equal_to_the_head_gain_reproduces_the_per_head_output():
    B, N, H, d, r = 2, 200, 3, 16, 8
    q, k, v, Wq, Wk, gain = _rand_inputs(B, N, H, d, r, seed=21)
    s = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 2, 100))
    st = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 2, 100), gate_per_token=True)
    out_h, col_h = O.forward(s, q, k, v, Wq, Wk, gain)
    g_tok = np.broadcast_to(gain, (B, N, H)).copy()
    out_t, col_t = O.forward(st, q, k, v, Wq, Wk, g_tok)
    np.testing.assert_array_equal(col_t, col_h)
    np.testing.assert_array_equal(out_t, out_h)


def test_per_token_gate_scales_each_tokens_linear_branch_by_its_own_gain():
    # out = O_sparse + g[b, n, h] * O_lin: with random gains, out(g) - out(0) must be
    # g[b, n, h] times out(1) - out(0) for every token of every batch entry and head (a
    # gain read at a transposed index, or per head, fails this).
    B, N, H, d, r = 2, 150, 3, 16, 8
    q, k, v, Wq, Wk, _ = _rand_inputs(B, N, H, d, r, seed=22)
    st = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 3, 50), gate_per_token=True)
    g = _rng(23).uniform(0.0, 1.0, (B, N, H))
    out_g, _ = O.forward(st, q, k, v, Wq, Wk, g)
    out_0, _ = O.forward(st, q, k, v, Wq, Wk, np.zeros((B, N, H)))
    out_1, _ = O.forward(st, q, k, v, Wq, Wk, np.ones((B, N, H)))
    lin = out_1 - out_0
    assert np.abs(lin).max() > 0.1
    np.testing.assert_allclose(out_g - out_0, g[..., None] * lin, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- gate from the query
# (README sparse-finetuning section: gate_proj, gate_bias; the gain is read as
# sigmoid(q . gate_proj_h + gate_bias_h) per token and head)

def _proj_gate(wg, bg):
    """The "proj" gate's parameter buffer: gate_proj [H, d] then gate_bias [H]."""
    return np.concatenate([np.asarray(wg, np.float64).ravel(), np.asarray(bg, np.float64)])


def test_projected_gate_with_zero_weights_is_the_sigmoid_of_the_bias():
    # wg = 0: the gain is sigmoid(bg_h) for every token.  With bg = ln 3 and ln(1/3) the
    # gains are 3/4 and 1/4 (worked by hand: 1 / (1 + 1/3) and 1 / (1 + 3)), so the output
    # equals the per-head-gain output with g = (3/4, 1/4).
    B, N, H, d, r = 1, 200, 2, 16, 8
    q, k, v, Wq, Wk, _ = _rand_inputs(B, N, H, d, r, seed=31)
    s_head = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 2, 100))
    s_proj = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 2, 100), gate="proj")
    g = _proj_gate(np.zeros((H, d)), [math.log(3.0), math.log(1.0 / 3.0)])
    out_p, col_p = O.forward(s_proj, q, k, v, Wq, Wk, g)
    out_h, col_h = O.forward(s_head, q, k, v, Wq, Wk, np.array([0.75, 0.25]))
    np.testing.assert_array_equal(col_p, col_h)
    np.testing.assert_allclose(out_p, out_h, rtol=0, atol=1e-14)


def test_projected_gate_limits_are_the_sparse_branch_and_the_unit_gain():
    B, N, H, d, r = 1, 150, 2, 16, 8
    q, k, v, Wq, Wk, _ = _rand_inputs(B, N, H, d, r, seed=32)
    s_head = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 3, 50))
    s_proj = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 3, 50), gate="proj")
    wg = _rng(33).standard_normal((H, d)) * 0.1
    out_off, _ = O.forward(s_proj, q, k, v, Wq, Wk, _proj_gate(wg, [-60.0, -60.0]))
    out_on, _ = O.forward(s_proj, q, k, v, Wq, Wk, _proj_gate(wg, [60.0, 60.0]))
    out_0, _ = O.forward(s_head, q, k, v, Wq, Wk, np.zeros(H))
    out_1, _ = O.forward(s_head, q, k, v, Wq, Wk, np.ones(H))
    np.testing.assert_allclose(out_off, out_0, rtol=0, atol=1e-12)   # sigmoid(-60) ~ 1e-26
    np.testing.assert_allclose(out_on, out_1, rtol=0, atol=1e-12)


def test_projected_gate_reads_each_heads_own_channel_of_its_own_query():
    # gate_proj_h = alpha_h on one channel c_h (a different channel and weight per head):
    # the gain of token n, head h is sigmoid(alpha_h * q[b, n, h, c_h] + bg_h), one product
    # per token, so the output must equal the per-token-gate output with those gains.  A
    # weight read transposed, from another head or another token fails this.
    B, N, H, d, r = 2, 130, 3, 16, 8
    q, k, v, Wq, Wk, _ = _rand_inputs(B, N, H, d, r, seed=34)
    chans, alpha, bg = [3, 11, 0], [1.5, -0.7, 2.0], [0.2, -0.4, 0.1]
    wg = np.zeros((H, d))
    for h in range(H):
        wg[h, chans[h]] = alpha[h]
    s_proj = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 2, 65), gate="proj")
    s_tok = O.make_shape(B, H, N, d, r, 0.5, grid=(1, 2, 65), gate="token")
    g_tok = np.zeros((B, N, H))
    for h in range(H):
        a = alpha[h] * q[:, :, h, chans[h]].astype(np.float64) + bg[h]
        g_tok[:, :, h] = 1.0 / (1.0 + np.exp(-a))
    out_p, _ = O.forward(s_proj, q, k, v, Wq, Wk, _proj_gate(wg, bg))
    out_t, _ = O.forward(s_tok, q, k, v, Wq, Wk, g_tok)
    np.testing.assert_allclose(out_p, out_t, rtol=0, atol=1e-13)
    assert g_tok.std() > 0.1                       # the gains really differ per token


def test_forward_equals_composed_steps_and_lists_are_valid():
    B, N, H, d, r = 2, 330, 2, 16, 8
    q, k, v, Wq, Wk, gain = _rand_inputs(B, N, H, d, r, seed=15)
    s = O.make_shape(B, H, N, d, r, 0.3, grid=(1, 3, 110))
    out, col = O.forward(s, q, k, v, Wq, Wk, gain)
    nb, kk = 6, O.keep_count(6, 0.3)
    assert col.shape == (B, H, nb, kk)
    assert np.all(np.diff(col, axis=-1) > 0) and col.min() >= 0 and col.max() < nb
    c2, *_ = O.select(s, O.pool(s, q), O.pool(s, k))
    np.testing.assert_array_equal(col, c2)
    S, z = O.linear_state(s, k, v, Wk)
    _, _, ob = O.attend_blocks(s, q, k, v, Wq, gain, col, S, z, _all_blocks(B, H, nb))
    t = 0
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                n1 = min(N, 64 * i + 64)
                np.testing.assert_array_equal(out[b, 64 * i:n1, h], ob[t, :n1 - 64 * i])
                t += 1
    assert np.all(np.isfinite(out))
