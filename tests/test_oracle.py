"""Pins for the CPU fp64 oracle (no GPU).

The oracle is checked against what the pages and the mathematics fix, never
against itself: the pages' worked examples (golden fixtures), closed forms,
the brute-force matrix form, the pages' block algorithm, and invariants
(resets, chaining, D linearity, the rank bound of cross-block sub-matrices).
A final test plants plausible mistakes in the NumPy twin of the recurrence and
checks that every one of them fails at least one pin.
"""
import math

import numpy as np
import pytest

import oracle
from workloads import make_custom


def scalar_inputs(x, a=None, log_a=None, b=1.0, c=1.0):
    """One batch row, one head, N = P = 1."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    X = x.reshape(1, T, 1, 1)
    la = np.full((1, T, 1), math.log(a) if log_a is None else log_a, dtype=np.float64)
    B = np.full((1, T, 1, 1), b)
    C = np.full((1, T, 1, 1), c)
    return X, la, B, C


# --------------------------------------------------------------------------- #
# Worked examples (golden fixtures)
# --------------------------------------------------------------------------- #

def test_worked_example_recurrence(golden):
    g = golden("worked_example_a05.txt")
    X, la, B, C = scalar_inputs(g["x"], a=g["a"][0])
    Y, final = oracle.ssd_reference(X, la, B, C)
    np.testing.assert_allclose(Y.ravel(), g["y"], rtol=0, atol=1e-12)
    assert abs(final.ravel()[0] - g["y"][-1]) < 1e-12  # C = 1: y_T = h_T


def test_worked_example_matrix_form(golden):
    g = golden("worked_example_a05.txt")
    X, la, B, C = scalar_inputs(g["x"], a=g["a"][0])
    Y, M = oracle.dual_matrix(X, la, B, C, return_M=True)
    np.testing.assert_allclose(M[0, 0], np.array(g["M"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(Y.ravel(), g["y"], rtol=0, atol=1e-12)


def test_worked_example_chunk_split(golden):
    """Split after step 2; a fourth zero input pads the second block to length 2."""
    g = golden("worked_example_a05.txt")
    q = int(g["split_after"][0])
    X, la, B, C = scalar_inputs(list(g["x"]) + [0.0], a=g["a"][0])
    Y, parts = oracle.blockwise(X, la, B, C, chunk=q, return_parts=True)
    np.testing.assert_allclose(Y.ravel()[:3], g["y"], atol=1e-12)
    assert abs(parts["local_end"][0, 0, 0].item() - g["first_block_end_state"][0]) < 1e-12
    assert abs(parts["local_out"][0, 0, 1, 0].item() - g["second_block_local_output"][0]) < 1e-12
    assert abs(parts["incoming_out"][0, 0, 1, 0].item() - g["second_block_incoming_output"][0]) < 1e-12
    # the chunk-boundary states of the recurrence agree with the block scan
    inc, loc = oracle.chunk_states(X, la, B, chunk=q)
    assert abs(inc[0, 1].item() - g["first_block_end_state"][0]) < 1e-12
    assert abs(loc[0, 0].item() - g["first_block_end_state"][0]) < 1e-12


def test_rank1_cross_block(golden):
    g = golden("rank1_cross_block.txt")
    T, m = int(g["T"][0]), int(g["split_after"][0])
    X, la, B, C = scalar_inputs(np.zeros(T), a=g["a"][0])
    _, M = oracle.dual_matrix(X, la, B, C, return_M=True)
    M = M[0, 0]
    blk = M[m:, :m]
    np.testing.assert_allclose(blk, np.array(g["cross_block"]), atol=1e-15)
    np.testing.assert_allclose(np.outer(g["left_factor"], g["right_factor"]), blk, atol=1e-15)
    assert abs(np.linalg.det(blk) - g["cross_block_det"][0]) < 1e-15
    assert np.linalg.matrix_rank(blk) == int(g["cross_block_rank"][0])
    assert abs(np.linalg.det(M) - g["full_det"][0]) < 1e-12
    assert np.linalg.matrix_rank(M) == int(g["full_rank"][0])
    # the first block passes h_2 = x_1/2 + x_2: its local end state per unit input
    coeffs = []
    for s in range(m):
        x = np.zeros(T)
        x[s] = 1.0
        X1, la1, B1, C1 = scalar_inputs(x, a=g["a"][0])
        _, loc = oracle.chunk_states(X1, la1, B1, chunk=m)
        coeffs.append(loc[0, 0].item())
    np.testing.assert_allclose(coeffs, g["passed_state_coefficients"], atol=1e-15)


def test_lti_1d_example(golden):
    g = golden("lti_1d_example.txt")
    X, la, B, C = scalar_inputs(g["x"], a=g["a"][0], b=g["B"][0], c=g["C"][0])
    Y, _ = oracle.ssd_reference(X, la, B, C)
    np.testing.assert_allclose(Y.ravel(), g["h"], rtol=0, atol=1e-12)
    assert round(Y.ravel()[-1], 3) == g["h_printed_last"][0]


# --------------------------------------------------------------------------- #
# Closed forms and special cases
# --------------------------------------------------------------------------- #

def _rand(T=12, H=3, P=4, N=5, G=1, seed=0, batch=2, **kw):
    d = make_custom(batch, T, H, P, N, ngroups=G, dtype="f32", seed=seed, **kw)
    return d


def test_no_decay_is_causal_prefix_sum():
    """a = 1: y_t = C_t^T sum_{s<=t} B_s x_s^T (linear attention without decay)."""
    d = _rand(seed=1)
    la = np.zeros_like(d["log_a"])
    Y, _ = oracle.ssd_reference(d["X"], la, d["B"], d["C"])
    X, B, C = (np.asarray(d[k], np.float64) for k in ("X", "B", "C"))
    outer = np.einsum("btgn,bthp->bthnp", B, X)  # G = 1
    Hs = np.cumsum(outer, axis=1)
    ref = np.einsum("btgn,bthnp->bthp", C, Hs)
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-12)


def test_full_decay_is_diagonal():
    """a = 0 (log a = -1000): y_t = (C_t . B_t) x_t + D x_t."""
    d = _rand(seed=2, has_D="normal")
    la = np.full_like(d["log_a"], -1000.0)
    Y, _ = oracle.ssd_reference(d["X"], la, d["B"], d["C"], d["D"])
    X, B, C, D = (np.asarray(d[k], np.float64) for k in ("X", "B", "C", "D"))
    cb = np.einsum("btgn,btgn->bt", C, B)
    ref = cb[:, :, None, None] * X + D[None, None, :, None] * X
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-12)


def test_geometric_series():
    """N = P = 1, B = C = 1, constant a: y_t = sum_{s<=t} a^(t-s) x_s."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal(20)
    a = 0.83
    X, la, B, C = scalar_inputs(x, a=a)
    Y, _ = oracle.ssd_reference(X, la, B, C)
    ref = [sum(a ** (t - s) * x[s] for s in range(t + 1)) for t in range(len(x))]
    np.testing.assert_allclose(Y.ravel(), ref, rtol=1e-12, atol=1e-12)


def test_initial_state_closed_form():
    """Zero input: y_t = (prod_{j<=t} a_j) C_t^T H0 (H0 is decayed by a_0)."""
    d = _rand(seed=4, has_init=True, batch=1)
    X = np.zeros_like(d["X"])
    Y, final = oracle.ssd_reference(X, d["log_a"], d["B"], d["C"], init_states=d["init_states"])
    la, C, H0 = (np.asarray(d[k], np.float64) for k in ("log_a", "C", "init_states"))
    decay = np.exp(np.cumsum(la, axis=1))  # [b, t, h]
    ref = decay[..., None] * np.einsum("btgn,bhnp->bthp", C, H0[:, 0])
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(final[:, 0], decay[:, -1, :, None, None] * H0[:, 0], rtol=1e-12)


def test_D_linearity():
    d = _rand(seed=5, has_D="normal")
    Y1, f1 = oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], d["D"])
    Y0, f0 = oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], None)
    np.testing.assert_allclose(Y1 - Y0, np.asarray(d["D"], np.float64)[None, None, :, None] * d["X"],
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(f1, f0)


# --------------------------------------------------------------------------- #
# Independent evaluators: brute-force matrix form and the block algorithm
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("G,H", [(1, 3), (2, 4)])
@pytest.mark.parametrize("with_init", [False, True])
def test_oracle_matches_dual_matrix(G, H, with_init):
    d = _rand(T=11, H=H, G=G, seed=10 + G, has_D="normal", has_init=with_init)
    Y, _ = oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"])
    Yd = oracle.dual_matrix(d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"])
    np.testing.assert_allclose(Y, Yd, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("Q", [1, 2, 3, 4, 6, 12])
def test_oracle_matches_blockwise(Q):
    d = _rand(T=12, seed=20 + Q, has_D="normal", has_init=True)
    Y, final = oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"])
    Yb, parts = oracle.blockwise(d["X"], d["log_a"], d["B"], d["C"], Q, d["D"], d["init_states"],
                                 return_parts=True)
    np.testing.assert_allclose(Y, Yb, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(final[:, 0], parts["final"], rtol=1e-11, atol=1e-12)
    inc, loc = oracle.chunk_states(d["X"], d["log_a"], d["B"], Q, d["init_states"])
    np.testing.assert_allclose(inc, parts["incoming_state"].transpose(0, 2, 1, 3, 4), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(loc, parts["local_end"].transpose(0, 2, 1, 3, 4), rtol=1e-11, atol=1e-12)


def test_segsum_from_cumsum_matches_products():
    """exp(cs[k] - cs[l]) equals the explicit product of a_j over (l, k]."""
    d = _rand(T=8, seed=30)
    cs = oracle.chunk_cumsum(d["log_a"], 8)  # [b, h, 1, 8]
    a = np.exp(np.asarray(d["log_a"], np.float64))
    for b in range(2):
        for h in range(3):
            for k in range(8):
                for l in range(k + 1):
                    prod = np.prod(a[b, l + 1:k + 1, h])
                    assert abs(math.exp(cs[b, h, 0, k] - cs[b, h, 0, l]) - prod) < 1e-12
    assert np.allclose(cs[..., -1], np.log(np.prod(a.reshape(2, 1, 8, 3), axis=2)).transpose(0, 2, 1))


def test_cross_block_rank_at_most_N():
    """Every past-to-future sub-matrix of M has rank <= N (wq-win 088, section 2.2)."""
    N = 2
    d = _rand(T=10, H=1, P=1, N=N, seed=31, batch=1)
    _, M = oracle.dual_matrix(d["X"], d["log_a"], d["B"], d["C"], return_M=True)
    M = M[0, 0]
    for m in range(1, 10):
        s = np.linalg.svd(M[m:, :m], compute_uv=False)
        assert (s > 1e-12 * s[0]).sum() <= N
    assert np.linalg.matrix_rank(M) == 10  # the whole matrix is not low rank


# --------------------------------------------------------------------------- #
# Sequence boundaries, initial/final states, chaining
# --------------------------------------------------------------------------- #

def test_reset_equals_independent_runs():
    lens = [[5, 1, 9, 7], [22]]
    d = make_custom(2, 22, 3, 4, 5, dtype="f32", seed=40, has_D="normal", has_init=True,
                    lengths=lens, nseq=4)
    Y, final = oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"],
                                    d["seq_idx"], nseq=4)
    Yd = oracle.dual_matrix(d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"], d["seq_idx"])
    np.testing.assert_allclose(Y, Yd, rtol=1e-11, atol=1e-12)
    for b, row in enumerate(lens):
        t0 = 0
        for s, L in enumerate(row):
            sl = slice(t0, t0 + L)
            Ys, fs = oracle.ssd_reference(d["X"][b:b + 1, sl], d["log_a"][b:b + 1, sl], d["B"][b:b + 1, sl],
                                          d["C"][b:b + 1, sl], d["D"], d["init_states"][b:b + 1, s:s + 1])
            np.testing.assert_allclose(Y[b:b + 1, sl], Ys, rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(final[b, s], fs[0, 0], rtol=1e-12, atol=1e-13)
            t0 += L
        # ids that never occur keep their initial state
        for s in range(len(row), 4):
            np.testing.assert_array_equal(final[b, s], d["init_states"][b, s])


def test_chaining_final_to_init():
    d = _rand(T=16, seed=41, has_init=True, has_D="normal")
    Y, final = oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"])
    for t1 in (1, 7, 15):
        a = slice(0, t1)
        b = slice(t1, 16)
        Ya, fa = oracle.ssd_reference(d["X"][:, a], d["log_a"][:, a], d["B"][:, a], d["C"][:, a], d["D"],
                                      d["init_states"])
        Yb, fb = oracle.ssd_reference(d["X"][:, b], d["log_a"][:, b], d["B"][:, b], d["C"][:, b], d["D"], fa)
        np.testing.assert_allclose(np.concatenate([Ya, Yb], axis=1), Y, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(fb, final, rtol=1e-12, atol=1e-13)


def test_chunk_states_with_resets():
    lens = [[3, 9, 1, 3], [8, 8]]
    d = make_custom(2, 16, 2, 3, 4, dtype="f32", seed=42, has_init=True, lengths=lens, nseq=4)
    inc, loc = oracle.chunk_states(d["X"], d["log_a"], d["B"], 4, d["init_states"], d["seq_idx"], nseq=4)
    seq = d["seq_idx"]
    for b in range(2):
        for c in range(4):
            t0 = 4 * c
            s0 = seq[b, t0]
            # incoming: the state just before t0 for the sequence of token t0
            start = t0
            while start > 0 and seq[b, start - 1] == s0:
                start -= 1
            sl = slice(start, t0)
            if t0 > start:
                _, f = oracle.ssd_reference(d["X"][b:b + 1, sl], d["log_a"][b:b + 1, sl], d["B"][b:b + 1, sl],
                                            d["C"][b:b + 1, sl], None, d["init_states"][b:b + 1, s0:s0 + 1])
                np.testing.assert_allclose(inc[b, c], f[0, 0], rtol=1e-12, atol=1e-13)
            else:
                np.testing.assert_array_equal(inc[b, c], d["init_states"][b, s0])
            # local: zero-start run over the chunk's last piece
            s1 = seq[b, t0 + 3]
            p0 = t0 + 3
            while p0 > t0 and seq[b, p0 - 1] == s1:
                p0 -= 1
            sl = slice(p0, t0 + 4)
            _, f = oracle.ssd_reference(d["X"][b:b + 1, sl], d["log_a"][b:b + 1, sl], d["B"][b:b + 1, sl],
                                        d["C"][b:b + 1, sl])
            np.testing.assert_allclose(loc[b, c], f[0, 0], rtol=1e-12, atol=1e-13)


def test_chunk_states_and_block_decay_on_the_chunk_split_example(golden):
    """The page's split after step 2, with no padding: the second block is a
    short last block of one token. Its incoming state is the first block's end
    state, its zero-start local end state is its own output (C = 1, N = P = 1),
    its block decay is the product of its a_t, and decay * incoming + local is
    the last output (the block scan of the same page)."""
    g = golden("worked_example_a05.txt")
    q, a = int(g["split_after"][0]), g["a"][0]
    X, la, B, C = scalar_inputs(g["x"], a=a)
    inc, loc = oracle.chunk_states(X, la, B, chunk=q)
    assert inc.shape[1] == 2  # ceil(3 / 2) blocks, the last one short
    assert inc[0, 0].item() == 0.0
    assert abs(inc[0, 1].item() - g["first_block_end_state"][0]) < 1e-12
    assert abs(loc[0, 0].item() - g["first_block_end_state"][0]) < 1e-12
    assert abs(loc[0, 1].item() - g["second_block_local_output"][0]) < 1e-12
    dec = oracle.segment_decay(la, q)
    assert abs(dec[0, 0, 0] - a * a) < 1e-15          # product of the first block's two a_t
    assert abs(dec[0, 1, 0] - a) < 1e-15              # the short block holds one a_t
    # the carried contribution and the scan step of the page
    assert abs(dec[0, 1, 0] * inc[0, 1].item() - g["second_block_incoming_output"][0]) < 1e-12
    assert abs(dec[0, 1, 0] * inc[0, 1].item() + loc[0, 1].item() - g["y"][-1]) < 1e-12


def _last_piece_start(seq_row, t0, t1):
    """First token of the last sequence piece of the block [t0, t1)."""
    p0 = t1 - 1
    while p0 > t0 and seq_row[p0 - 1] == seq_row[t1 - 1]:
        p0 -= 1
    return p0


RAGGED = [(4, [[3, 9, 1, 3, 3], [19]]), (8, [[5, 6, 2, 6], [10, 9]]), (8, [[19], [17, 1, 1]])]


@pytest.mark.parametrize("Q,lens", RAGGED)
def test_chunk_states_ragged_last_chunk_against_recurrence_on_slices(Q, lens):
    """T = 19 is not a multiple of Q: the last block is short. Every block's
    incoming and local states equal the step recurrence run on row slices: from
    the sequence's start (with its initial state) to the block start, and from
    zero over the block's last sequence piece."""
    nseq = max(len(r) for r in lens)
    d = make_custom(2, 19, 2, 3, 4, dtype="f32", seed=50 + Q, has_init=True, lengths=lens, nseq=nseq)
    inc, loc = oracle.chunk_states(d["X"], d["log_a"], d["B"], Q, d["init_states"], d["seq_idx"], nseq=nseq)
    seq = d["seq_idx"]
    nch = -(-19 // Q)
    assert inc.shape[1] == nch and 19 % Q != 0
    sl_args = lambda b, sl, init=None: (d["X"][b:b + 1, sl], d["log_a"][b:b + 1, sl], d["B"][b:b + 1, sl],
                                        d["C"][b:b + 1, sl], None, init)
    for b in range(2):
        for c in range(nch):
            t0, t1 = c * Q, min(19, (c + 1) * Q)
            s0 = seq[b, t0]
            start = t0
            while start > 0 and seq[b, start - 1] == s0:
                start -= 1
            if t0 > start:
                _, f = oracle.ssd_reference(*sl_args(b, slice(start, t0), d["init_states"][b:b + 1, s0:s0 + 1]))
                np.testing.assert_allclose(inc[b, c], f[0, 0], rtol=1e-12, atol=1e-13)
            else:
                np.testing.assert_array_equal(inc[b, c], d["init_states"][b, s0])
            p0 = _last_piece_start(seq[b], t0, t1)
            _, f = oracle.ssd_reference(*sl_args(b, slice(p0, t1)))
            np.testing.assert_allclose(loc[b, c], f[0, 0], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("Q,lens", RAGGED)
def test_segment_decay_is_the_product_over_the_last_piece(Q, lens):
    """The block decay of the page's block scan for blocks that may hold a
    sequence start and may be short: (a) the explicit product of a_t over the
    block's last sequence piece; (b) the factor the step recurrence applies to
    a state carried into that piece (no input, initial state of ones); and a
    piece start off by one either way fails both."""
    nseq = max(len(r) for r in lens)
    d = make_custom(2, 19, 3, 2, 2, dtype="f32", seed=60 + Q, lengths=lens, nseq=nseq)
    la, seq = d["log_a"].astype(np.float64), d["seq_idx"]
    dec = oracle.segment_decay(la, Q, seq)
    nch = -(-19 // Q)
    assert dec.shape == (2, nch, 3)
    for b in range(2):
        for c in range(nch):
            t0, t1 = c * Q, min(19, (c + 1) * Q)
            p0 = _last_piece_start(seq[b], t0, t1)
            for h in range(3):
                prod = 1.0
                for t in range(p0, t1):
                    prod *= math.exp(la[b, t, h])
                assert abs(dec[b, c, h] - prod) <= 1e-14 * prod
                # off-by-one piece starts give other values
                for q0 in (p0 - 1, p0 + 1):
                    if t0 <= q0 < t1 and q0 != p0:
                        wrong = math.prod(math.exp(la[b, t, h]) for t in range(q0, t1))
                        assert abs(wrong - dec[b, c, h]) > 1e-6 * dec[b, c, h]
            sl = slice(p0, t1)
            zeros = np.zeros_like(d["X"][b:b + 1, sl])
            ones = np.ones((1, 1, 3, 2, 2))
            _, f = oracle.ssd_reference(zeros, la[b:b + 1, sl], d["B"][b:b + 1, sl], d["C"][b:b + 1, sl], None, ones)
            np.testing.assert_allclose(f[0, 0, :, 0, 0], dec[b, c], rtol=1e-12)


def test_groups_with_identical_B_C_equal_one_group():
    d = _rand(T=9, H=4, G=1, seed=43, has_D="normal")
    B2 = np.repeat(d["B"], 2, axis=2)
    C2 = np.repeat(d["C"], 2, axis=2)
    Y1, _ = oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], d["D"])
    Y2, _ = oracle.ssd_reference(d["X"], d["log_a"], B2, C2, d["D"])
    np.testing.assert_array_equal(Y1, Y2)


def test_numpy_twin_agrees_with_c_oracle():
    lens = [[4, 6, 3], [13]]
    d = make_custom(2, 13, 3, 4, 5, dtype="f32", seed=44, has_D="normal", has_init=True, lengths=lens, nseq=3)
    args = (d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"], d["seq_idx"])
    Y, f = oracle.ssd_reference(*args, nseq=3)
    Yn, fn = oracle.recurrence_numpy(*args, nseq=3)
    np.testing.assert_allclose(Y, Yn, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(f, fn, rtol=1e-12, atol=1e-13)


def test_oracle_rejects_bad_arguments():
    d = _rand(T=4, H=3, G=1, seed=45)
    with pytest.raises(ValueError):
        oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], nseq=2)  # nseq > 1 needs seq_idx
    with pytest.raises(ValueError):
        oracle.ssd_reference(d["X"], d["log_a"], np.repeat(d["B"], 2, axis=2),
                             np.repeat(d["C"], 2, axis=2))  # 3 heads, 2 groups


# --------------------------------------------------------------------------- #
# The pins catch planted mistakes (mutations of the NumPy twin, on the CPU)
# --------------------------------------------------------------------------- #

def _pin_battery(fn):
    """Run the pins above against a recurrence implementation; return failures."""
    from conftest import load_golden
    fails = []
    g = load_golden("worked_example_a05.txt")
    X, la, B, C = scalar_inputs(g["x"], a=g["a"][0])
    if not np.allclose(fn(X, la, B, C)[0].ravel(), g["y"], atol=1e-12):
        fails.append("worked_example")
    g = load_golden("lti_1d_example.txt")
    X, la, B, C = scalar_inputs(g["x"], a=g["a"][0], b=g["B"][0], c=g["C"][0])
    if not np.allclose(fn(X, la, B, C)[0].ravel(), g["h"], atol=1e-12):
        fails.append("lti_example")
    # brute-force matrix form with init, D, resets (square N = P so a transposed read-out runs)
    lens = [[4, 7], [11]]
    d = make_custom(2, 11, 2, 4, 4, dtype="f32", seed=50, has_D="normal", has_init=True, lengths=lens, nseq=2)
    args = (d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"], d["seq_idx"])
    if not np.allclose(fn(*args)[0], oracle.dual_matrix(*args), rtol=1e-10, atol=1e-12):
        fails.append("dual_matrix")
    # final states of a reset run equal independent runs
    Y, f = fn(*args)
    _, f0 = fn(d["X"][:1, :4], d["log_a"][:1, :4], d["B"][:1, :4], d["C"][:1, :4], d["D"],
               d["init_states"][:1, :1])
    if not np.allclose(f[0, 0], f0[0, 0], rtol=1e-12, atol=1e-13):
        fails.append("reset_final")
    return fails


def test_pins_pass_on_the_unmutated_twin():
    assert _pin_battery(oracle.recurrence_numpy) == []


@pytest.mark.parametrize("mutation", ["decay_index", "decay_sign", "swap_BC", "undecayed_init",
                                      "drop_D", "no_reset", "transpose_readout"])
def test_pins_catch_planted_mistake(mutation):
    def fn(*a, **k):
        return oracle.recurrence_numpy(*a, _mutation=mutation, **k)
    assert _pin_battery(fn) != [], f"no pin caught the planted mistake {mutation!r}"
