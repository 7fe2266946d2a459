"""GPU hash statistics (section 3.2.2 and Fig. 3 of "Scaling Embeddings Outperforms Scaling
Experts in Language Models": table hit counts and collisions of the n-gram hash) against the
oracle's Python sets; integer results, so bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from synth import gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ne():
    import hashed_gram_embedding_horner_b200 as m
    return m


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def test_worked_example(ne):
    tok, off = np.array([7, 42, 999, 0, 500], np.int32), np.array([0, 5], np.int32)
    assert ne.ngram_hash_stats(1000, 2, dev_i32(tok), dev_i32(off), [4099, 1000, 10 ** 7]) == (5, [4, 5, 5])


@pytest.mark.parametrize("n", [2, 3, 4, 5])
def test_zipf_stream_matches_oracle(ne, n):
    """100 Zipf(1.1) sequences over V0 = 131072 (n <= 3: exact 64-bit window keys; n >= 4:
    V0^n >= 2^64, windows compared id by id), moduli on and off multiples of V0, a ragged
    length mix."""
    V0 = 131072
    rng = np.random.default_rng(n)
    lengths = rng.integers(0, 700, 100)
    lengths[:3] = [0, 1, 2]
    off = gen.offsets_from_lengths([int(x) for x in lengths])
    tok = gen.zipf_tokens(40 + n, int(off[-1]), V0).astype(np.int32)
    moduli = [30 * V0 - 3, 30 * V0, 30 * V0 + 7, int(31.5 * V0), 32 * V0, 32 * V0 + 1, 33 * V0, 4099, 1]
    got = ne.ngram_hash_stats(V0, n, dev_i32(tok), dev_i32(off), moduli)
    windows, rows = oracle.hash_stats(V0, n, tok, off, moduli)
    assert got[1] == rows
    assert got[0] == windows


def test_eight_gram_windows_over_the_largest_vocabulary(ne):
    """n = 8 with V0 = 2^31 - 1 (all four packed words in use; X_8 < 2^248): distinct windows
    and rows against the oracle's exact integers, including repeated windows."""
    V0 = 2 ** 31 - 1
    rng = np.random.default_rng(8)
    base = rng.integers(0, V0, 300).astype(np.int32)
    tok = np.concatenate([base, base[:120], rng.integers(0, 3, 200).astype(np.int32), base[50:90]])
    off = gen.offsets_from_lengths([300, 120, 200, 40])
    moduli = [7274513, 2 ** 31 - 3, 1]
    got = ne.ngram_hash_stats(V0, 8, dev_i32(tok), dev_i32(off), moduli)
    windows, rows = oracle.hash_stats(V0, 8, tok, off, moduli)
    assert got == (windows, rows)
