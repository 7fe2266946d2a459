"""Pins of the CPU oracle against values and identities fixed independently of it.

Paper: "Scaling Embeddings Outperforms Scaling Experts in Language Models",
section 2 (N-gram Embedding): Eq. 1, Eq. 2, Eq. 3 and the parameter-count remark
after Eq. 3; section 4.2 (N-gram Cache) for the decode history.
Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong digit order, a 64-bit wrap, a transposed W, a wrong normaliser, an
off-by-one in the context) fails at least one of them.
"""
import os

import numpy as np
import pytest

import oracle
from synth import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _bigint_index(V0, window_newest_first, V):
    """Eq. 2 with Python integers (arbitrary precision), written independently."""
    return sum(int(t) * V0 ** j for j, t in enumerate(window_newest_first)) % V


# ---------------------------------------------------------------- Eq. 2 (hash)

def test_hand_worked_example():
    V0, N, K, V = 1000, 3, 2, [4099, 5003, 6007, 7001]
    seq = np.array([7, 42, 999, 0, 500], dtype=np.int32)
    win = oracle.context_windows(N, seq, [0, 5])
    idx = oracle.hash_indices(V0, N, K, V, win)
    want = np.array([[int(x) for x in r[1:]] for r in _rows("hash_worked_example.txt")])
    np.testing.assert_array_equal(idx, want)
    assert idx[1, 0] == idx[3, 0]  # the collision the fixture records


def test_exact_not_wrapped_u64():
    for V, ctx, exact, wrapped in _rows("hash_exact_vs_wrapped.txt"):
        ctx = [int(x) for x in ctx.split(",")]
        got = oracle.ngram_index(131072, ctx[::-1], int(V))
        assert got == int(exact)
        if exact != wrapped:
            assert got != int(wrapped)


def test_digit_order_newest_is_least_significant():
    # t_{i-1} = 1, t_i = 2, V0 = 10: X = 2 * 10^0 + 1 * 10^1 = 12 (not 21).
    assert oracle.ngram_index(10, [2, 1], 1000) == 12
    win = oracle.context_windows(2, np.array([1, 2], np.int32), [0, 2])
    assert oracle.hash_indices(10, 2, 1, [1000], win)[1, 0] == 12


@pytest.mark.parametrize("seed", range(6))
def test_bruteforce_all_windows(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(2, 9))
    K = int(rng.integers(1, 4))
    V0 = int(rng.choice([2, 7, 1000, 131072, 2 ** 31 - 1]))
    S = (N - 1) * K
    V = [int(x) for x in rng.integers(1, 2 ** 31 - 1, size=S)]
    lengths = rng.integers(0, 12, size=int(rng.integers(1, 5)))
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    tokens = rng.integers(0, V0, size=int(off[-1])).astype(np.int32)
    if len(tokens):
        tokens[rng.integers(0, len(tokens))] = V0 - 1  # the largest id
    win = oracle.context_windows(N, tokens, off)
    idx = oracle.hash_indices(V0, N, K, V, win)
    for b in range(len(lengths)):
        seq = tokens[off[b]:off[b + 1]].tolist()
        for p in range(len(seq)):
            for n in range(2, N + 1):
                # the n-gram t_{i-n+1..i}, pad 0 before the sequence start, newest first
                window = [seq[p - j] if p - j >= 0 else 0 for j in range(n)]
                for k in range(K):
                    s = (n - 2) * K + k
                    assert idx[off[b] + p, s] == _bigint_index(V0, window, V[s])


def test_pad_equals_explicit_zero_prefix():
    N, K, V0 = 5, 2, 131072
    V = [7274513, 7274537, 7274543, 7274569, 7274591, 7274629, 7274639, 7274651]
    tok = gen.zipf_tokens(3, 40, V0)
    a = oracle.hash_indices(V0, N, K, V, oracle.context_windows(N, tok, [0, 40]))
    pref = np.concatenate([np.zeros(N - 1, np.int32), tok])
    b = oracle.hash_indices(V0, N, K, V, oracle.context_windows(N, pref, [0, len(pref)]))
    np.testing.assert_array_equal(a, b[N - 1:])


def test_context_windows_by_hand():
    tok = np.array([5, 6, 7, 8, 9], np.int32)
    w = oracle.context_windows(3, tok, [0, 2, 5])
    np.testing.assert_array_equal(w, [[5, 0, 0], [6, 5, 0], [7, 0, 0], [8, 7, 0], [9, 8, 7]])
    w = oracle.context_windows(3, tok, [0, 2, 5], histories=[[1, 2, 3], [4]])
    np.testing.assert_array_equal(w, [[5, 3, 2], [6, 5, 3], [7, 4, 0], [8, 7, 4], [9, 8, 7]])


# ---------------------------------------------------------------- Eq. 3 (combine)

def _rand_case(rng, D, N, K, V0=50, T=9, dtype=np.float32):
    S = (N - 1) * K
    d = D // S if S else 0
    V = [int(x) for x in rng.integers(3, 40, size=S)]
    E0 = rng.standard_normal((V0, D)).astype(np.float32)
    E = [rng.standard_normal((V[s], d)).astype(np.float32) for s in range(S)]
    W = rng.standard_normal((D, D)).astype(np.float32)
    tok = rng.integers(0, V0, size=T).astype(np.int32)
    off = np.array([0, 4, T], np.int32)
    return V0, V, E0, E, W, tok, off


def _brute_idx(V0, N, K, V, tok, off):
    S = (N - 1) * K
    idx = np.zeros((len(tok), S), np.int64)
    for b in range(len(off) - 1):
        seq = tok[off[b]:off[b + 1]].tolist()
        for p in range(len(seq)):
            for n in range(2, N + 1):
                w = [seq[p - j] if p - j >= 0 else 0 for j in range(n)]
                for k in range(K):
                    idx[off[b] + p, (n - 2) * K + k] = _bigint_index(V0, w, V[(n - 2) * K + k])
    return idx


@pytest.mark.parametrize("D,N,K", [(12, 3, 2), (16, 2, 1), (24, 4, 2), (8, 1, 1)])
def test_forward_matches_library_matmul(D, N, K):
    """Eq. 3 against numpy's fp64 matmul: e = (E0[t] + concat_s E_s[idx_s] @ W_stacked^T) / (S+1)."""
    rng = np.random.default_rng(D * 100 + N * 10 + K)
    V0, V, E0, E, W, tok, off = _rand_case(rng, D, N, K)
    S = (N - 1) * K
    got = oracle.forward(V0, D, N, K, V, tok, off, E0, E, W)
    idx = _brute_idx(V0, N, K, V, tok, off)
    G = (np.concatenate([E[s][idx[:, s]].astype(np.float64) for s in range(S)], axis=1)
         if S else np.zeros((len(tok), D)))
    want = (E0[tok].astype(np.float64) + G @ W.astype(np.float64).T) / (S + 1)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # A transposed W must fail this pin (guards the test itself).
    if S:
        wrong = (E0[tok].astype(np.float64) + G @ W.astype(np.float64)) / (S + 1)
        assert np.abs(wrong - got).max() > 1e-3


def test_gather_rows_by_hand():
    """The row lookup E_s[idx[i, s]] -> [T, S, d]: tables whose every entry encodes its own
    (table, row, column), so each looked-up value names where it came from. A transposed
    stack axis, a swapped index column or a row/column mix-up fails here."""
    S, d = 3, 4
    V = [5, 7, 6]
    tables = [np.array([[1000 * s + 10 * r + c for c in range(d)] for r in range(V[s])], dtype=np.int64)
              for s in range(S)]
    idx = np.array([[0, 6, 5], [4, 0, 2], [2, 3, 0]], dtype=np.int32)  # T = 3 tokens
    got = oracle.gather_rows(tables, idx)
    assert got.shape == (3, S, d)
    for i in range(3):
        for s in range(S):
            assert got[i, s].tolist() == [1000 * s + 10 * int(idx[i, s]) + c for c in range(d)]
    # token 1's block for sub-table 2 is row 2 of table 2, written out
    assert got[1, 2].tolist() == [2020, 2021, 2022, 2023]
    # concatenated along the feature axis it is G's layout: column s * d + c
    G = got.reshape(3, S * d)
    assert G[2, 1 * d + 3] == 1000 * 1 + 10 * 3 + 3


def test_combine_bf16_exact_conversion():
    rng = np.random.default_rng(1)
    D, S = 8, 2
    e0 = gen.f32_to_bf16_bits(rng.standard_normal((3, D)).astype(np.float32))
    sub = gen.f32_to_bf16_bits(rng.standard_normal((3, S, D // S)).astype(np.float32))
    W = gen.f32_to_bf16_bits(rng.standard_normal((D, D)).astype(np.float32))
    got = oracle.combine(D, S, e0, sub, W)
    f = lambda b: gen.bf16_bits_to_f32(b).astype(np.float64)
    want = (f(e0) + f(sub).reshape(3, D) @ f(W).T) / (S + 1)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-14)


def test_n1_reduces_to_base_embedding():
    rng = np.random.default_rng(2)
    E0 = rng.standard_normal((30, 16)).astype(np.float32)
    tok = rng.integers(0, 30, 11).astype(np.int32)
    out = oracle.forward(30, 16, 1, 1, [], tok, [0, 11], E0, [], None)
    np.testing.assert_array_equal(out, E0[tok].astype(np.float64))


def test_zero_subtables_give_scaled_base():
    rng = np.random.default_rng(3)
    V0, V, E0, E, W, tok, off = _rand_case(rng, 16, 3, 2)
    E = [np.zeros_like(e) for e in E]
    out = oracle.forward(V0, 16, 3, 2, V, tok, off, E0, E, W)
    np.testing.assert_allclose(out, E0[tok].astype(np.float64) / 5, rtol=1e-15)


def test_identity_projection_is_gather_average():
    rng = np.random.default_rng(4)
    D, N, K = 12, 4, 1
    V0, V, E0, E, W, tok, off = _rand_case(rng, D, N, K)
    S = 3
    out = oracle.forward(V0, D, N, K, V, tok, off, E0, E, np.eye(D, dtype=np.float32))
    idx = _brute_idx(V0, N, K, V, tok, off)
    cat = np.concatenate([E[s][idx[:, s]] for s in range(S)], axis=1).astype(np.float64)
    np.testing.assert_allclose(out, (E0[tok].astype(np.float64) + cat) / (S + 1), rtol=1e-15)


def test_eq1_special_case():
    """N=2, K=1, W=I: Eq. 3 reduces to Eq. 1, e = (E_0(t_i) + E_2(H_2)) / 2."""
    rng = np.random.default_rng(5)
    D, V0, V2 = 8, 20, 37
    E0 = rng.standard_normal((V0, D)).astype(np.float32)
    E2 = rng.standard_normal((V2, D)).astype(np.float32)
    tok = rng.integers(0, V0, 10).astype(np.int32)
    out = oracle.forward(V0, D, 2, 1, [V2], tok, [0, 10], E0, [E2], np.eye(D, dtype=np.float32))
    prev = np.concatenate([[0], tok[:-1]])
    h2 = (tok.astype(np.int64) + prev * V0) % V2
    np.testing.assert_allclose(out, (E0[tok].astype(np.float64) + E2[h2].astype(np.float64)) / 2, rtol=1e-15)


def test_linear_in_base_table():
    rng = np.random.default_rng(6)
    V0, V, E0, E, W, tok, off = _rand_case(rng, 12, 3, 2)
    E0b = rng.standard_normal(E0.shape).astype(np.float32)
    f = lambda e0: oracle.forward(V0, 12, 3, 2, V, tok, off, e0, E, W)
    lhs = f(E0 + E0b) - f(E0b)
    rhs = E0[tok].astype(np.float64) / 5
    np.testing.assert_allclose(lhs, rhs, atol=1e-5)  # fp32 rounding of E0 + E0b


@pytest.mark.parametrize("V", [4099, 2162717])
def test_parameter_count_independent_of_N_K(V):
    """After Eq. 3: sub-table width D/((N-1)K) makes the N-gram parameter count
    (all E_{n,k} plus all W_{n,k}) equal V*D + D^2 for every N, K (equal V_{n,k})."""
    from synth.configs import NgramConfig
    D = 2 ** 4 * 3 * 5 * 7  # divisible by many S
    for N in range(2, 9):
        for K in range(1, 5):
            S = (N - 1) * K
            if D % S:
                continue
            cfg = NgramConfig(name="x", V0=100, D=D, N=N, K=K, V_nk=(V,) * S, dtype="bf16")
            params = sum(v * cfg.d for v in cfg.V_nk) + S * D * cfg.d
            assert params == V * D + D * D


# ---------------------------------------------------------------- N-gram cache (history)

def test_ring_commit_paths_agree():
    """append(5) then rollback(4 - a) == append(1 + a) for every accept length a."""
    for a in range(5):
        r1, r2 = oracle.RingOracle(1, 8, 3), oracle.RingOracle(1, 8, 3)
        r1.append(0, [1, 2, 3]); r2.append(0, [1, 2, 3])
        ids = [10, 11, 12, 13, 14]
        assert r1.append(0, ids) and r1.rollback(0, 4 - a)
        assert r2.append(0, ids[:1 + a])
        assert r1.hist == r2.hist


def test_ring_rejections():
    r = oracle.RingOracle(1, 8, 3)
    assert not r.append(0, list(range(9)))      # more than C ids
    assert r.append(0, list(range(8)))
    assert not r.rollback(0, 9)                 # more than committed
    assert r.rollback(0, 6)                     # keeps positions 0, 1 (both held)
    assert r.append(0, list(range(8)))          # len 10, holds 2..9
    assert not r.rollback(0, 7)                 # would need positions 1, 2
    assert r.rollback(0, 6)                     # needs positions 2, 3
    assert r.lengths() == [4]
    assert not r.rollback(0, -1)


def test_history_context_equals_prefill_over_full_history():
    """Decode context from committed history == prefill over history ++ in-step ids."""
    N, K, V0 = 3, 4, 131072
    V = [3342341, 3342371, 3342379, 3342413, 3342419, 3342439, 3342457, 3342473]
    rng = np.random.default_rng(7)
    hist = [rng.integers(0, V0, int(n)).tolist() for n in (0, 1, 2, 7)]
    step = rng.integers(0, V0, 4 * 5).astype(np.int32)
    off = np.arange(0, 21, 5, dtype=np.int32)
    dec = oracle.hash_indices(V0, N, K, V, oracle.context_windows(N, step, off, histories=hist))
    for b in range(4):
        full = np.array(hist[b] + step[off[b]:off[b + 1]].tolist(), np.int32)
        pre = oracle.hash_indices(V0, N, K, V, oracle.context_windows(N, full, [0, len(full)]))
        np.testing.assert_array_equal(dec[off[b]:off[b + 1]], pre[len(hist[b]):])


# ---------------------------------------------------------------- amplification (section 3.2.4)

def test_layernorm_worked_example():
    """[1, 2, 3, 4]: mean 2.5, population variance 1.25, so (x - 2.5) / sqrt(1.25)."""
    got = oracle.layernorm(np.array([[1.0, 2.0, 3.0, 4.0]]))
    want = np.array([[-1.5, -0.5, 0.5, 1.5]]) / np.sqrt(1.25)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    np.testing.assert_allclose(got, [[-1.3416407864998738, -0.4472135954999579, 0.4472135954999579,
                                      1.3416407864998738]], rtol=0, atol=1e-15)


def test_layernorm_invariants_and_affine():
    rng = np.random.default_rng(5)
    x = rng.normal(3.0, 0.02, (7, 96))
    y = oracle.layernorm(x, eps=1e-12)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose((y ** 2).mean(axis=1), 1, atol=1e-6)
    # shift and positive scale of a row leave it unchanged; gamma/beta act per column
    np.testing.assert_allclose(oracle.layernorm(5 * x + 11, eps=0), oracle.layernorm(x, eps=0), atol=1e-10)
    g, b = rng.normal(size=96), rng.normal(size=96)
    np.testing.assert_allclose(oracle.layernorm(x, g, b, eps=1e-12), y * g + b, atol=1e-12)
    # eps bounds the gain of a constant row: output 0, not a division by zero
    np.testing.assert_array_equal(oracle.layernorm(np.full((1, 8), 2.0), eps=1e-5), np.zeros((1, 8)))


def test_amplify_is_a_scalar_on_eq3():
    rng = np.random.default_rng(6)
    e = rng.normal(size=(3, 16))
    np.testing.assert_array_equal(oracle.amplify(e, 1.0), e)
    np.testing.assert_allclose(oracle.amplify(e, np.sqrt(16.0)), 4.0 * e, rtol=1e-15)


# ---------------------------------------------------------------- backward

def test_backward_is_the_exact_directional_derivative():
    """L(params) = <g, e(params)>. e is linear in E_0, in each sub-table (indices fixed) and
    in W, so for any direction X of one parameter, L(p + X) - L(p) = <dL/dp, X> exactly (up
    to fp64 rounding). Both sides from independent code: the left from the C forward
    oracle, the right from the numpy backward."""
    rng = np.random.default_rng(11)
    V0, D, N, K = 200, 48, 3, 2
    V = [101, 103, 107, 109]
    S, d = 4, 12
    lengths = [7, 1, 0, 13]
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(off[-1])
    tok = rng.integers(0, 12, T).astype(np.int32)  # few distinct ids: E_0 rows collide
    # small integers everywhere: every sum and product below is exact in fp32 and fp64,
    # so the identity must hold to the last bit
    ints = lambda shape: rng.integers(-8, 9, shape).astype(np.float32)
    E0 = ints((V0, D))
    E = [ints((V[s], d)) for s in range(S)]
    W = ints((D, D))
    g = ints((T, D)).astype(np.float64)
    scale = 2.5  # c = 2.5 / 5 = 0.5: exact
    L = lambda E0_, E_, W_: float(np.sum(g * scale * oracle.forward(V0, D, N, K, V, tok, off, E0_, E_, W_)))
    dE0, dE, dW = oracle.backward(V0, D, N, K, V, tok, off, E, W, g, scale=scale)
    base = L(E0, E, W)
    X = ints(E0.shape)
    assert L(E0 + X, E, W) - base == np.sum(dE0 * X.astype(np.float64))
    for s in range(S):
        X = ints(E[s].shape)
        E2 = [e.copy() for e in E]
        E2[s] = E[s] + X
        assert L(E0, E2, W) - base == np.sum(dE[s] * X.astype(np.float64))
    X = ints(W.shape)
    assert L(E0, E, W + X) - base == np.sum(dW * X.astype(np.float64))
    # a wrong scale, a transposed dW or a dropped collision would each fail one of the above;
    # negative control: the transpose of dW is not the gradient
    assert L(E0, E, W + X) - base != np.sum(dW.T * X.astype(np.float64))


def test_backward_collisions_add_up():
    """Two tokens with the same id (and so the same context and rows) double the row grad."""
    V0, D, N, K = 50, 16, 2, 1
    V = [53]
    tok = np.array([5, 5], np.int32)
    off = np.array([0, 1, 2], np.int32)  # two one-token sequences: both contexts (0, 5)
    E = [np.ones((53, 16), np.float32)]
    W = np.eye(16, dtype=np.float32)
    g = np.ones((2, 16))
    dE0, dE, dW = oracle.backward(V0, D, N, K, V, tok, off, E, W, g)
    np.testing.assert_array_equal(dE0[5], np.full(16, 2 * 0.5))
    r = oracle.hash_indices(V0, N, K, V, oracle.context_windows(N, tok, off))[0, 0]
    np.testing.assert_array_equal(dE[0][r], np.full(16, 2 * 0.5))
    assert np.count_nonzero(dE[0]) == 16
    np.testing.assert_array_equal(dW, np.full((16, 16), 2 * 0.5))


# ---------------------------------------------------------------- hash statistics (section 3.2.2)

def test_hash_stats_worked_example():
    """[7, 42, 999, 0, 500], V0 = 1000, 2-grams: the golden indices mod 4099 are 7, 2943, 2009,
    2943, 500 (positions 1 and 3 collide): 5 windows, 4 rows, 1 collision; mod V0 the row is
    the newest id (5 rows); a modulus above every X_n loses nothing."""
    tok = np.array([7, 42, 999, 0, 500], np.int32)
    off = np.array([0, 5], np.int32)
    golden = [7, 2943, 2009, 2943, 500]
    assert len(set(golden)) == 4
    assert oracle.hash_stats(1000, 2, tok, off, [4099, 1000, 10 ** 7]) == (5, [4, 5, 5])


def test_hash_stats_multiple_of_v0_closed_form():
    """V = m V0 for 2-grams: X_2 mod m V0 = (t_{i-1} mod m) V0 + t_i, so the rows hit are the
    distinct pairs (t_{i-1} mod m, t_i) — counted here from the pairs, not from X."""
    rng = np.random.default_rng(12)
    V0 = 997
    lengths = [50, 1, 200, 77]
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    tok = rng.integers(0, V0, int(off[-1])).astype(np.int32)
    prev = np.zeros_like(tok)
    for b in range(len(lengths)):
        s, e = off[b], off[b + 1]
        prev[s + 1:e] = tok[s:e - 1]  # pad 0 before each start
    for m in (1, 2, 5, 31):
        want = len({(int(p) % m, int(t)) for p, t in zip(prev, tok)})
        windows, rows = oracle.hash_stats(V0, 2, tok, off, [m * V0])
        assert rows == [want] and windows == len({(int(p), int(t)) for p, t in zip(prev, tok)})
    assert oracle.hash_stats(V0, 2, tok, off, [1])[1] == [1]
