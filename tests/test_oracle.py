"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own loop: each compares it with a printed
worked example, a closed form, a textbook routine (numpy matmul / tril /
power), a structural invariant, or an independently written chunked algorithm.
Pages: "Mamba-2" (docsaid.org), sections "Writing the SSM as one matrix",
"Simplifying A to one number", "Computing with four tokens", "Half of each
route"; "Mamba-2 SSD note" (0h-n0.github.io), table "Unified view of attention
variants" (linear attention, RetNet, SSD masks); "Selective SSM guide"
(auturnal.com), eq. (3), composition of affine maps.
"""
import json
import math
import os

import numpy as np
import pytest

from selective_state_space_17_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "four_token_example.json")


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _rand(rng, Bsz, L, H, P, G, N, dt_const=None, A_const=None):
    x = rng.standard_normal((Bsz, L, H, P))
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), (Bsz, L, H)))
    A = -np.exp(rng.uniform(0, math.log(16), (H,)))
    if dt_const is not None:
        dt = np.full_like(dt, dt_const)
    if A_const is not None:
        A = np.full_like(A, A_const)
    Bm = rng.standard_normal((Bsz, L, G, N)) / math.sqrt(N)
    Cm = rng.standard_normal((Bsz, L, G, N)) / math.sqrt(N)
    D = rng.standard_normal((H,))
    return x, dt, A, Bm, Cm, D


def _group_bc(Bm, Cm, H):
    G = Bm.shape[2]
    idx = np.arange(H) // (H // G)
    return Bm[:, :, idx, :], Cm[:, :, idx, :]


# ---------------------------------------------------------------- worked example

@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_four_token_recurrence_matches_printed_output(oracle, golden):
    inp = golden["inputs"]
    x = np.array(inp["x"])[:, None]
    a = np.array(inp["a"])
    B = np.array(inp["B"], float)
    C = np.array(inp["C"], float)
    y, h = oracle.scan_core(a, np.ones(4), x, B, C)
    tol = golden["print_precision_abs"]
    np.testing.assert_allclose(y[:, 0], golden["printed"]["y_recurrent"], atol=tol, rtol=0)
    np.testing.assert_allclose(h[0], golden["derived_by_hand"]["final_state"], atol=1e-12)


def test_four_token_mask_matches_printed_L(oracle, golden):
    Lm = oracle.mask(np.array(golden["inputs"]["a"]))
    np.testing.assert_allclose(Lm, np.array(golden["printed"]["L"]),
                               atol=golden["print_precision_abs"], rtol=0)


def test_four_token_through_the_layer_interface(oracle, golden):
    """The page's example has no step size. Map it onto the layer's parameters:
    A = -1 and dt_t = -ln a_t give exp(dt_t A) = a_t, and x_t / dt_t undoes the
    dt scaling of the input, so both layer routines must print the same y."""
    inp = golden["inputs"]
    a = np.array(inp["a"])
    dt = -np.log(a)
    x = (np.array(inp["x"]) / dt).reshape(1, 4, 1, 1)
    Bm = np.array(inp["B"], float).reshape(1, 4, 1, 2)
    Cm = np.array(inp["C"], float).reshape(1, 4, 1, 2)
    A = np.array([-1.0])
    y, fs = oracle.forward(x, dt.reshape(1, 4, 1), A, Bm, Cm)
    yq = oracle.quadratic(x, dt.reshape(1, 4, 1), A, Bm, Cm)
    tol = golden["print_precision_abs"]
    np.testing.assert_allclose(y.ravel(), golden["printed"]["y_recurrent"], atol=tol, rtol=0)
    np.testing.assert_allclose(yq.ravel(), golden["printed"]["y_quadratic"], atol=tol, rtol=0)
    np.testing.assert_allclose(fs.ravel(), golden["derived_by_hand"]["final_state"], atol=1e-9)


# ------------------------------------------------------- recurrence == quadratic

@pytest.mark.parametrize("shape", [(2, 37, 4, 3, 2, 5), (1, 64, 2, 8, 1, 8), (2, 9, 6, 4, 3, 16)])
def test_recurrence_equals_bruteforce_quadratic(oracle, shape):
    rng = np.random.default_rng(1)
    x, dt, A, Bm, Cm, D = _rand(rng, *shape)
    y, _ = oracle.forward(x, dt, A, Bm, Cm, D)
    yq = oracle.quadratic(x, dt, A, Bm, Cm, D)
    assert _rel(y, yq) < 1e-12


# --------------------------------------------------------- closed-form special cases

def test_a_equals_one_is_causal_linear_attention(oracle):
    """a = 1 (dt = 1, A = 0): Y = tril(C B^T) X per head, textbook causal
    linear attention without softmax."""
    rng = np.random.default_rng(2)
    x, dt, A, Bm, Cm, D = _rand(rng, 2, 40, 4, 5, 2, 6, dt_const=1.0, A_const=0.0)
    y, _ = oracle.forward(x, dt, A, Bm, Cm, None)
    Bh, Ch = _group_bc(Bm, Cm, 4)
    for b in range(2):
        for h in range(4):
            S = np.tril(Ch[b, :, h] @ Bh[b, :, h].T)
            assert _rel(y[b, :, h], S @ x[b, :, h]) < 1e-12


def test_a_equals_gamma_is_retnet_decay(oracle):
    """a = gamma (dt = 1, A = ln gamma): Y = (Gamma o C B^T) X with
    Gamma_ij = gamma^(i-j) for i >= j."""
    gamma = 0.99
    rng = np.random.default_rng(3)
    x, dt, A, Bm, Cm, D = _rand(rng, 1, 50, 2, 4, 1, 8, dt_const=1.0,
                                A_const=math.log(gamma))
    y, _ = oracle.forward(x, dt, A, Bm, Cm, D)
    i = np.arange(50)
    Gam = np.where(i[:, None] >= i[None, :], gamma ** (i[:, None] - i[None, :]).clip(min=0), 0.0)
    for h in range(2):
        ref = (Gam * (Cm[0, :, 0] @ Bm[0, :, 0].T)) @ x[0, :, h] + D[h] * x[0, :, h]
        assert _rel(y[0, :, h], ref) < 1e-12


def test_a_equals_zero_keeps_only_the_diagonal(oracle):
    """a = 0 (dt A = -1000): y_t = (C_t . B_t) dt_t x_t + D x_t."""
    rng = np.random.default_rng(4)
    x, dt, A, Bm, Cm, D = _rand(rng, 2, 33, 4, 6, 2, 8, dt_const=0.1, A_const=-1e4)
    y, fs = oracle.forward(x, dt, A, Bm, Cm, D)
    Bh, Ch = _group_bc(Bm, Cm, 4)
    cb = np.einsum("blhn,blhn->blh", Ch, Bh)
    ref = (cb * dt)[..., None] * x + D[None, None, :, None] * x
    assert _rel(y, ref) < 1e-13
    # state = contribution of the last token only
    last = dt[:, -1, :, None, None] * x[:, -1, :, :, None] * Bh[:, -1, :, None, :]
    assert _rel(fs, last) < 1e-13


# -------------------------------------------------------------- structural invariants

def _independent_chunked(x, dt, A, Bm, Cm, D, Q):
    """Chunked SSD in fp64, written here from the block decomposition of the
    pages (quadratic form inside a chunk, only chunk-end states carried
    across chunks) and sharing nothing with the oracle."""
    Bsz, L, H, P = x.shape
    Bh, Ch = _group_bc(Bm, Cm, H)
    N = Bm.shape[-1]
    y = np.zeros_like(x)
    fs = np.zeros((Bsz, H, P, N))
    for b in range(Bsz):
        for h in range(H):
            state = np.zeros((P, N))
            for c0 in range(0, L, Q):
                c1 = min(c0 + Q, L)
                la = dt[b, c0:c1, h] * A[h]
                cs = np.cumsum(la)
                seg = cs[:, None] - cs[None, :]
                Lm = np.where(np.tril(np.ones((c1 - c0, c1 - c0), bool)), np.exp(seg), 0.0)
                Cc, Bc, xc = Ch[b, c0:c1, h], Bh[b, c0:c1, h], x[b, c0:c1, h]
                u = dt[b, c0:c1, h, None] * xc
                y[b, c0:c1, h] = (Lm * (Cc @ Bc.T)) @ u + np.exp(cs)[:, None] * (Cc @ state.T)
                y[b, c0:c1, h] += D[h] * xc
                w = np.exp(cs[-1] - cs)[:, None] * u
                state = math.exp(cs[-1]) * state + w.T @ Bc
            fs[b, h] = state
    return y, fs


@pytest.mark.parametrize("Q", [1, 4, 16, 100])
def test_chunked_algorithm_equals_recurrence(oracle, Q):
    rng = np.random.default_rng(5)
    x, dt, A, Bm, Cm, D = _rand(rng, 2, 70, 4, 6, 2, 8)
    y, fs = oracle.forward(x, dt, A, Bm, Cm, D)
    yc, fsc = _independent_chunked(x, dt, A, Bm, Cm, D, Q)
    assert _rel(y, yc) < 1e-12
    assert _rel(fs, fsc) < 1e-12


def test_below_diagonal_blocks_have_rank_at_most_N(oracle):
    """Extract M column by column from the recurrence with unit impulses
    (P = 1, dt folded out) and check that every block strictly below the
    diagonal has numerical rank <= N (semiseparable structure)."""
    rng = np.random.default_rng(6)
    L, N = 24, 3
    _, dt, A, Bm, Cm, _ = _rand(rng, 1, L, 1, 1, 1, N)
    M = np.zeros((L, L))
    for i in range(L):
        x = np.zeros((1, L, 1, 1))
        x[0, i, 0, 0] = 1.0 / dt[0, i, 0]
        y, _ = oracle.forward(x, dt, A, Bm, Cm)
        M[:, i] = y[0, :, 0, 0]
    assert np.allclose(np.triu(M, 1), 0.0)
    for k in range(1, L):
        blk = M[k:, :k]
        s = np.linalg.svd(blk, compute_uv=False)
        rank = int(np.sum(s > 1e-10 * s[0])) if s[0] > 0 else 0
        assert rank <= N, (k, rank)
    # and the full lower triangle is not low-rank (the test can fail)
    s = np.linalg.svd(M, compute_uv=False)
    assert int(np.sum(s > 1e-10 * s[0])) > N


def test_affine_scan_composition_and_initial_state(oracle):
    """(a2, b2) o (a1, b1) = (a2 a1, a2 b1 + b2): the final state of a
    sequence equals the second half's own state plus the second half's total
    decay times the first half's state; running the second half from the first
    half's state reproduces the full outputs."""
    rng = np.random.default_rng(7)
    x, dt, A, Bm, Cm, D = _rand(rng, 2, 60, 4, 5, 2, 7)
    y, fs = oracle.forward(x, dt, A, Bm, Cm, D)
    s1 = slice(0, 27)
    s2 = slice(27, 60)
    y1, f1 = oracle.forward(x[:, s1], dt[:, s1], A, Bm[:, s1], Cm[:, s1], D)
    y2, f2 = oracle.forward(x[:, s2], dt[:, s2], A, Bm[:, s2], Cm[:, s2], D)
    decay2 = np.exp(dt[:, s2].sum(axis=1) * A)  # [B, H]
    assert _rel(fs, decay2[:, :, None, None] * f1 + f2) < 1e-12
    y2c, f2c = oracle.forward(x[:, s2], dt[:, s2], A, Bm[:, s2], Cm[:, s2], D, init_state=f1)
    assert _rel(y[:, s2], y2c) < 1e-12 and _rel(fs, f2c) < 1e-12
    assert _rel(y[:, s1], y1) < 1e-14


def test_linearity_and_skip_term(oracle):
    rng = np.random.default_rng(8)
    x, dt, A, Bm, Cm, D = _rand(rng, 1, 30, 4, 4, 4, 6)
    x2 = rng.standard_normal(x.shape)
    ya, _ = oracle.forward(x, dt, A, Bm, Cm, None)
    yb, _ = oracle.forward(x2, dt, A, Bm, Cm, None)
    yab, _ = oracle.forward(2.0 * x - 3.0 * x2, dt, A, Bm, Cm, None)
    assert _rel(yab, 2.0 * ya - 3.0 * yb) < 1e-12
    yd, _ = oracle.forward(x, dt, A, Bm, Cm, D)
    assert _rel(yd - ya, D[None, None, :, None] * x) < 1e-12


def test_group_broadcast_matches_per_head_copies(oracle):
    """G groups shared by H/G consecutive heads each == G = H with B, C copied."""
    rng = np.random.default_rng(9)
    x, dt, A, Bm, Cm, D = _rand(rng, 2, 20, 6, 3, 2, 5)
    y, fs = oracle.forward(x, dt, A, Bm, Cm, D)
    Bh, Ch = _group_bc(Bm, Cm, 6)
    y2, fs2 = oracle.forward(x, dt, A, np.ascontiguousarray(Bh), np.ascontiguousarray(Ch), D)
    assert _rel(y, y2) < 1e-15 and _rel(fs, fs2) < 1e-15


def test_state_columns_split_into_independent_problems(oracle):
    """Each column n of the state evolves on its own (h_t = a_t h_{t-1} +
    dt_t x_t B_tᵀ acts column by column) and y_t = h_t C_t sums over columns, so
    a run over all N columns equals the sum of runs over two column blocks (D
    counted once) and its final state is their concatenation. The tensor-core
    path takes state dims above 128 this way, in two passes."""
    rng = np.random.default_rng(21)
    x, dt, A, Bm, Cm, D = _rand(rng, 2, 40, 4, 3, 2, 10)
    init = rng.standard_normal((2, 4, 3, 10))
    y, fs = oracle.forward(x, dt, A, Bm, Cm, D, init_state=init)
    lo, hi = slice(0, 6), slice(6, 10)
    c = np.ascontiguousarray
    y1, f1 = oracle.forward(x, dt, A, c(Bm[..., lo]), c(Cm[..., lo]), D, init_state=c(init[..., lo]))
    y2, f2 = oracle.forward(x, dt, A, c(Bm[..., hi]), c(Cm[..., hi]), None, init_state=c(init[..., hi]))
    assert _rel(y1 + y2, y) < 1e-12
    assert _rel(np.concatenate([f1, f2], axis=-1), fs) < 1e-15


def test_wide_head_splits_into_narrower_heads(oracle):
    """Each row p of the state evolves on its own, so a head of P = m q channels
    equals m heads of q channels that share its dt, A and D: x, y [B, L, H, P]
    and the states [B, H, P, N] read as [B, L, H m, q] and [B, H m, q, N]. The
    tensor-core path runs P = 64m this way."""
    rng = np.random.default_rng(22)
    Bsz, L, H, P, G, N, m = 2, 30, 4, 6, 2, 5, 2
    x, dt, A, Bm, Cm, D = _rand(rng, Bsz, L, H, P, G, N)
    init = rng.standard_normal((Bsz, H, P, N))
    y, fs = oracle.forward(x, dt, A, Bm, Cm, D, init_state=init)
    q = P // m
    xs = x.reshape(Bsz, L, H * m, q)
    dts = np.ascontiguousarray(np.repeat(dt, m, axis=2))
    ys, fss = oracle.forward(xs, dts, np.repeat(A, m), Bm, Cm, np.repeat(D, m),
                             init_state=init.reshape(Bsz, H * m, q, N))
    assert _rel(ys.reshape(Bsz, L, H, P), y) < 1e-15
    assert _rel(fss.reshape(Bsz, H, P, N), fs) < 1e-15


# ------------------------------------------------------------------------- decode

def test_step_from_zero_reproduces_forward(oracle):
    rng = np.random.default_rng(10)
    x, dt, A, Bm, Cm, D = _rand(rng, 2, 25, 4, 5, 2, 6)
    y, fs = oracle.forward(x, dt, A, Bm, Cm, D)
    state = np.zeros((2, 4, 5, 6))
    for t in range(25):
        yt, state = oracle.step(x[:, t], dt[:, t], A, Bm[:, t], Cm[:, t], D, state)
        assert _rel(yt, y[:, t]) < 1e-12
    assert _rel(state, fs) < 1e-12


def test_step_does_not_modify_input_state(oracle):
    rng = np.random.default_rng(11)
    st = rng.standard_normal((1, 2, 3, 4))
    keep = st.copy()
    oracle.step(np.ones((1, 2, 3)), np.full((1, 2), 0.01), np.array([-1.0, -2.0]),
                np.ones((1, 1, 4)), np.ones((1, 1, 4)), None, st)
    assert np.array_equal(st, keep)


# ------------------------------------------------------------------ input recipe

def test_bf16_rounding_is_round_to_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -30,
                     -2.5, 3.0e-3, 1.0 - 2 ** -10])
    bits = gen.round_to_bf16_bits(vals)
    back = gen.bf16_bits_to_f32(bits).astype(np.float64)
    # ties to even: 1 + 2^-8 -> 1; 1 + 3*2^-8 -> 1 + 2^-6 (even mantissa)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2 ** -6
    assert back[3] == 1.0 + 2 ** -7  # above the tie rounds up
    assert back[4] == -2.5
    assert abs(back[5] - 3.0e-3) <= 3.0e-3 * 2 ** -8
    assert back[6] == 1.0


def test_input_recipe_distributions():
    inp = gen.make_inputs(2, 256, 8, 16, 2, 32, "f32", seed=0)
    assert inp.dt.min() >= 1e-3 * (1 - 1e-6) and inp.dt.max() <= 1e-1 * (1 + 1e-6)
    assert (inp.A < 0).all() and (inp.A >= -16.0001).all() and (inp.A <= -0.9999).all()
    assert abs(float(inp.Bm.std()) * math.sqrt(32) - 1.0) < 0.05
    again = gen.make_inputs(2, 256, 8, 16, 2, 32, "f32", seed=0)
    assert np.array_equal(inp.x, again.x) and np.array_equal(inp.Cm, again.Cm)
    other = gen.make_inputs(2, 256, 8, 16, 2, 32, "f32", seed=1)
    assert not np.array_equal(inp.x, other.x)
