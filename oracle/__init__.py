"""CPU oracle for the hashed N-gram embedding layer — TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py`
may import this package. The CUDA library never calls it and shares no code
with it; the two meet only through the seeded inputs of `synth/`.

Everything here follows "Scaling Embeddings Outperforms Scaling Experts in
Language Models" (LongCat team), section 2 "N-gram Embedding":
  Eq. 2  H_n(t_{i-n+1..i}) = (sum_{j=0}^{n-1} t_{i-j} V0^j) mod V_n
  Eq. 3  e_i = (E_0(t_i) + sum_{n=2..N} sum_{k=1..K} W_{n,k} E_{n,k}(H_{n,k}(...))) / ((N-1)K + 1)
with E_{n,k} in R^{V_{n,k} x D/((N-1)K)} and W_{n,k} in R^{D x D/((N-1)K)}, and
section 4.2 "N-gram Cache" for the decode-side id history (RingOracle).
Conventions where the paper is silent: pad id 0 before a sequence start;
sub-table order s = (n-2)K + (k-1); exact integer sum before the modulus.

The heavy loops live in `ngram_oracle.c` (exact multi-limb hash, fp64
combine); this module marshals numpy arrays and keeps the decode history.
Parity status of each function is stated in its docstring; all of them are
pinned by tests under `tests/test_oracle_*.py`.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None
_P = ctypes.c_void_p


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_ngram_index.argtypes = [ctypes.c_int64, ctypes.c_int, _P, ctypes.c_int64]
        lib.oracle_ngram_index.restype = ctypes.c_int64
        lib.oracle_context_windows.argtypes = [ctypes.c_int, _P, _P, ctypes.c_int32, _P, _P, _P]
        lib.oracle_hash.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _P, _P,
                                    ctypes.c_int64, _P]
        for name in ("oracle_combine_bf16", "oracle_combine_f32"):
            getattr(lib, name).argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, _P, _P, _P, _P]
        lib.oracle_forward.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P,
                                       _P, _P]
        _LIB = lib
    return _LIB


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(_P)


def num_threads() -> int:
    return int(_lib().oracle_num_threads())


def ngram_index(V0: int, window_newest_first, V: int) -> int:
    """Eq. 2 for one n-gram: window_newest_first[j] = t_{i-j}, n = len(window)."""
    w = np.ascontiguousarray(window_newest_first, dtype=np.int32)
    r = _lib().oracle_ngram_index(V0, len(w), _ptr(w), V)
    if r < 0:
        raise ValueError("bad n-gram index arguments")
    return int(r)


def _history_arrays(histories, num_seqs):
    if histories is None:
        return None, None
    lens = np.array([len(h) for h in histories], dtype=np.int64)
    assert len(lens) == num_seqs
    off = np.zeros(num_seqs + 1, dtype=np.int64)
    np.cumsum(lens, out=off[1:])
    flat = (np.concatenate([np.asarray(h, dtype=np.int32) for h in histories])
            if off[-1] else np.zeros(1, dtype=np.int32))
    return np.ascontiguousarray(flat, dtype=np.int32), off


def context_windows(N: int, tokens, seq_offsets, histories=None) -> np.ndarray:
    """[T, N] int32 windows, column j = t_{i-j}; before a sequence start: the sequence's
    committed history (newest last) if given, else pad id 0."""
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    off = np.ascontiguousarray(seq_offsets, dtype=np.int32)
    B = len(off) - 1
    hist, hoff = _history_arrays(histories, B)
    T = int(off[-1])
    win = np.zeros((max(T, 1), N), dtype=np.int32)
    if _lib().oracle_context_windows(N, _ptr(tokens), _ptr(off), B, _ptr(hist), _ptr(hoff),
                                     _ptr(win)) != 0:
        raise ValueError("bad sequence offsets")
    return win[:T]


def hash_indices(V0: int, N: int, K: int, V_nk, windows: np.ndarray) -> np.ndarray:
    """[T, S] int32 sub-table row ids (Eq. 2 for every n = 2..N, k = 1..K)."""
    S = (N - 1) * K
    V = np.ascontiguousarray(V_nk, dtype=np.int64)
    assert len(V) == S
    windows = np.ascontiguousarray(windows, dtype=np.int32)
    T = windows.shape[0]
    idx = np.zeros((max(T, 1), max(S, 1)), dtype=np.int32)
    if S and T:
        if _lib().oracle_hash(V0, N, K, _ptr(V), _ptr(windows), T, _ptr(idx)) != 0:
            raise ValueError("bad hash arguments (token ids must be >= 0, N <= 8, V < 2^31)")
    return idx[:T, :S]


def combine(D: int, S: int, e0rows: np.ndarray, subrows: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Eq. 3 in fp64 for M tokens from their gathered rows.

    e0rows [M, D], subrows [M, S, d], W [D, D] (W_stacked, block s = W_{n,k});
    bf16 inputs as uint16 bit patterns, or float32. Returns [M, D] float64."""
    M = e0rows.shape[0]
    out = np.zeros((max(M, 1), D), dtype=np.float64)
    if M == 0:
        return out[:0]
    if e0rows.dtype == np.uint16:
        fn, dt = _lib().oracle_combine_bf16, np.uint16
    else:
        fn, dt = _lib().oracle_combine_f32, np.float32
    e0 = np.ascontiguousarray(e0rows, dtype=dt)
    sub = np.ascontiguousarray(subrows, dtype=dt) if S else np.zeros(1, dtype=dt)
    w = np.ascontiguousarray(W, dtype=dt) if S else np.zeros(1, dtype=dt)
    if fn(D, S, M, _ptr(e0), _ptr(sub), _ptr(w), _ptr(out)) != 0:
        raise ValueError("bad combine arguments")
    return out


def gather_rows(tables, idx: np.ndarray) -> np.ndarray:
    """Row lookup E_s[idx[:, s]] for every s -> [T, S, d]."""
    return np.stack([tables[s][idx[:, s]] for s in range(idx.shape[1])], axis=1)


def forward(V0: int, D: int, N: int, K: int, V_nk, tokens, seq_offsets, E0, E_nk, W,
            histories=None) -> np.ndarray:
    """The whole layer on host tables -> [T, D] float64 (context, Eq. 2, lookup, Eq. 3)."""
    S = (N - 1) * K
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    off = np.ascontiguousarray(seq_offsets, dtype=np.int32)
    B = len(off) - 1
    T = int(off[-1])
    hist, hoff = _history_arrays(histories, B)
    dt = E0.dtype
    elt = 2 if dt == np.uint16 else 4
    E0 = np.ascontiguousarray(E0)
    tabs = [np.ascontiguousarray(E_nk[s], dtype=dt) for s in range(S)]
    tab_ptrs = (ctypes.c_void_p * max(S, 1))(*[t.ctypes.data for t in tabs])
    Wc = np.ascontiguousarray(W, dtype=dt) if S else np.zeros(1, dtype=dt)
    V = np.ascontiguousarray(V_nk, dtype=np.int64) if S else np.zeros(1, dtype=np.int64)
    out = np.zeros((max(T, 1), D), dtype=np.float64)
    rc = _lib().oracle_forward(elt, V0, D, N, K, _ptr(V), _ptr(tokens), _ptr(off), B, _ptr(hist),
                               _ptr(hoff), _ptr(E0), ctypes.cast(tab_ptrs, _P), _ptr(Wc), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_forward: bad arguments")
    return out[:T]


class RingOracle:
    """Decode-side id history per sequence (section 4.2 "N-gram Cache": ids of recent
    tokens kept per sequence, updated as speculative tokens are accepted or rejected).

    The history is an unbounded list of committed ids per slot. A bounded device ring
    of capacity C keeps the newest C positions; `valid_from` mirrors which positions
    such a ring still holds, so that this model can say which operations a ring of
    capacity C must reject:
      append(m):   m > C is rejected; otherwise positions [len, len+m) are written and
                   valid_from = max(valid_from, len + m - C).
      rollback(r): r < 0, r > len, or a rollback after which the newest N-1 committed
                   positions are no longer all held (max(0, len - r - (N-1)) < valid_from)
                   is rejected; otherwise the newest r ids are dropped.
    A rejected operation leaves the slot unchanged.
    """

    def __init__(self, num_slots: int, capacity: int, N: int):
        self.C, self.N = capacity, N
        self.hist = [[] for _ in range(num_slots)]
        self.valid_from = [0] * num_slots

    def reset(self, slots=None):
        for b in (range(len(self.hist)) if slots is None else slots):
            self.hist[b] = []
            self.valid_from[b] = 0

    def append(self, slot: int, ids) -> bool:
        ids = [int(x) for x in ids]
        if len(ids) > self.C:
            return False
        L = len(self.hist[slot])
        self.hist[slot].extend(ids)
        self.valid_from[slot] = max(self.valid_from[slot], L + len(ids) - self.C)
        return True

    def rollback(self, slot: int, r: int) -> bool:
        L = len(self.hist[slot])
        if r < 0 or r > L or max(0, L - r - (self.N - 1)) < self.valid_from[slot]:
            return False
        del self.hist[slot][L - r:]
        return True

    def lengths(self):
        return [len(h) for h in self.hist]

    def histories(self, slots=None):
        return [list(self.hist[b]) for b in (range(len(self.hist)) if slots is None else slots)]


# ---------------------------------------------------------------- embedding amplification
# Section 3.2.4 ("effective training through embedding amplification"): the N-gram
# embedding output is amplified before it joins the residual stream, by a constant factor
# or by a LayerNorm. Plain definitions in fp64.

def amplify(e: np.ndarray, scale: float) -> np.ndarray:
    """Constant amplification: e * scale."""
    return np.asarray(e, dtype=np.float64) * float(scale)


def layernorm(x: np.ndarray, gamma=None, beta=None, eps: float = 0.0) -> np.ndarray:
    """Row LayerNorm: (x - mean) / sqrt(population variance + eps) * gamma + beta."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)
    if beta is not None:
        y = y + np.asarray(beta, dtype=np.float64)
    return y


# ---------------------------------------------------------------- backward (training)
# Gradients of Eq. 3 (section 2) w.r.t. its parameters, given g = dL/de. The layer is
# linear in E_0, in each E_{n,k} (for fixed indices) and in W, so each gradient is the
# plain definition below, written with numpy fp64 primitives (matmul, scatter-add).

def backward(V0: int, D: int, N: int, K: int, V_nk, tokens, seq_offsets, E_nk, W, g, scale: float = 1.0,
             histories=None):
    """-> (dE0 [V0, D], [dE_s [V_s, d]], dW [D, D]) in float64 for grad_out g [T, D].

    c = scale / ((N-1)K + 1); dE0[t_i] += c g_i; dG = c g W; dE_s[idx_s(i)] += dG[i, s-block];
    dW = c g^T G with G the concatenated looked-up sub-rows. Tables as uint16 bf16 bits or
    float32."""
    S = (N - 1) * K
    d = D // S if S else 0
    c = float(scale) / (S + 1)
    tokens = np.asarray(tokens)
    g64 = _to_f64(g)
    dE0 = np.zeros((V0, D), np.float64)
    np.add.at(dE0, tokens.astype(np.int64), c * g64)
    dE = []
    dW = np.zeros((D, D), np.float64)
    if S:
        idx = hash_indices(V0, N, K, V_nk, context_windows(N, tokens, seq_offsets, histories=histories))
        W64 = _to_f64(W)
        dG = c * (g64 @ W64)
        G = np.concatenate([_to_f64(np.asarray(E_nk[s])[idx[:, s]]) for s in range(S)], axis=1)
        for s in range(S):
            gs = np.zeros((V_nk[s], d), np.float64)
            np.add.at(gs, idx[:, s].astype(np.int64), dG[:, s * d:(s + 1) * d])
            dE.append(gs)
        dW = c * (g64.T @ G)
    return dE0, dE, dW


def _to_f64(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:  # bf16 bit patterns
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# ---------------------------------------------------------------- hash statistics
# Section 3.2.2 (Fig. 3): the vocabulary hit rate (table rows hit at least once by the
# stream) and hash collisions (distinct n-gram windows minus distinct rows they map to).
# Plain definitions: Python sets over the windows of the layer's context rule.

def hash_stats(V0: int, n: int, tokens, seq_offsets, moduli):
    """-> (distinct windows, [distinct rows per modulus]) for the n-gram hash X_n mod V."""
    win = context_windows(n, tokens, seq_offsets)  # [T, n]: column j is t_{i-j}, pad 0
    keys = set()
    xs = []
    for w in win.tolist():
        x = sum(int(t) * int(V0) ** j for j, t in enumerate(w))  # Eq. 2's X_n, exact
        keys.add(x)
        xs.append(x)
    return len(keys), [len({x % int(V) for x in xs}) for V in moduli]
