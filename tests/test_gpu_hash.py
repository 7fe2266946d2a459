"""GPU parity of the hash stage (Eq. 2, context assembly): bit-exact vs the oracle.

Paper: "Scaling Embeddings Outperforms Scaling Experts in Language Models",
section 2, Eq. 2; pad id 0 before a sequence start; decode context from the
N-gram cache (section 4.2).
"""
import numpy as np
import pytest
import torch

import oracle
from synth import configs, gen, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ne():
    import hashed_gram_embedding_horner_b200 as m
    return m


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def gpu_hash(ne, V0, N, K, V, tokens, offsets, cache=None, slots=None, D=None):
    S = (N - 1) * K
    D = D or 16 * S
    plan = ne.ngram_embed_plan_create(V0, D, N, K, V, ne.NGRAM_BF16)
    T = len(tokens)
    ws = ne.new_workspace(plan, T)
    idx = torch.full((max(T, 1), S), -7, dtype=torch.int32, device="cuda")
    ne.ngram_hash_indices(plan, dev_i32(tokens) if T else torch.zeros(1, dtype=torch.int32, device="cuda")[:0],
                          dev_i32(offsets), idx[:T] if T else idx[:0], ws, cache=cache, cache_slots=slots)
    status = ne.ngram_embed_get_status(ws)
    return idx[:T].cpu().numpy(), status


def oracle_hash(V0, N, K, V, tokens, offsets, histories=None):
    return oracle.hash_indices(V0, N, K, V, oracle.context_windows(N, tokens, offsets, histories=histories))


def _decode_prefill_tokens(cfg):
    ds = workloads.DecodeStream(cfg)
    return ds.step_tokens(0), ds.step_offsets()


@pytest.mark.parametrize("cfg", configs.CONFIGS, ids=lambda c: c.name)
def test_hash_bit_exact_on_workloads(ne, cfg):
    if cfg.decode_steps and not cfg.seq_len:
        tokens, offsets = _decode_prefill_tokens(cfg)
    else:
        tokens, offsets = workloads.prefill_tokens(cfg)
    got, status = gpu_hash(ne, cfg.V0, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, D=cfg.D)
    assert status == 0
    np.testing.assert_array_equal(got, oracle_hash(cfg.V0, cfg.N, cfg.K, cfg.V_nk, tokens, offsets))


def test_hash_extremes_of_the_integer_range(ne):
    """V0 = 2^31 - 1, ids V0 - 1, moduli just below 2^31, n up to 8: every Horner step at its
    largest (h * V0 + t close to 2^62)."""
    V0, N, K = 2 ** 31 - 1, 8, 4
    S = (N - 1) * K
    V = [2 ** 31 - 1 - 2 * s for s in range(S)]  # not all prime; any modulus < 2^31 is valid
    rng = np.random.default_rng(11)
    lengths = [1, 2, 7, 8, 9, 0, 40, 3]
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    tok = rng.integers(V0 - 1000, V0, off[-1]).astype(np.int32)
    tok[::5] = V0 - 1
    tok[1::7] = 0
    got, status = gpu_hash(ne, V0, N, K, V, tok, off, D=S * 16)
    assert status == 0
    np.testing.assert_array_equal(got, oracle_hash(V0, N, K, V, tok, off))


def test_hash_worked_example_and_collision(ne):
    seq = np.array([7, 42, 999, 0, 500], np.int32)
    got, _ = gpu_hash(ne, 1000, 3, 2, [4099, 5003, 6007, 7001], seq, [0, 5], D=64)
    np.testing.assert_array_equal(got, [[7, 7, 7, 7], [2943, 2039, 1035, 41], [2009, 2975, 2795, 6994],
                                        [2943, 3403, 894, 5859], [500, 500, 358, 6807]])


def test_hash_ragged_and_empty_sequences(ne):
    V0, N, K = 131072, 5, 2
    V = configs.FULL_SCALE.V_nk
    lengths = [0, 1, 0, 3, 4, 0, 0, 129, 1, 255, 0]
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    tok = gen.zipf_tokens(5, int(off[-1]), V0)
    got, status = gpu_hash(ne, V0, N, K, V, tok, off, D=4096)
    assert status == 0
    np.testing.assert_array_equal(got, oracle_hash(V0, N, K, V, tok, off))


def test_hash_empty_call(ne):
    got, status = gpu_hash(ne, 1000, 3, 2, [4099, 5003, 6007, 7001], np.zeros(0, np.int32), [0], D=64)
    assert got.shape == (0, 4) and status == 0


def test_bad_token_sets_status_and_reads_pad(ne):
    tok = np.array([5, 1000, 7, -3, 9], np.int32)   # 1000 and -3 are outside [0, 1000)
    got, status = gpu_hash(ne, 1000, 3, 2, [4099, 5003, 6007, 7001], tok, [0, 5], D=64)
    assert "BAD_TOKEN" in ne.status_names(status)
    fixed = np.where((tok < 0) | (tok >= 1000), 0, tok).astype(np.int32)
    np.testing.assert_array_equal(got, oracle_hash(1000, 3, 2, [4099, 5003, 6007, 7001], fixed, [0, 5]))


def test_bad_offsets_set_status(ne):
    tok = np.arange(6, dtype=np.int32)
    _, status = gpu_hash(ne, 1000, 3, 2, [4099, 5003, 6007, 7001], tok, [0, 4, 2, 6], D=64)
    assert "BAD_OFFSETS" in ne.status_names(status)
    _, status = gpu_hash(ne, 1000, 3, 2, [4099, 5003, 6007, 7001], tok, [0, 3, 5], D=64)  # ends before T
    assert "BAD_OFFSETS" in ne.status_names(status)


def test_bounded_wait_times_out_and_context_survives(ne):
    plan = ne.ngram_embed_plan_create(1000, 64, 3, 2, [4099, 5003, 6007, 7001], ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, 16)
    ne.ngram_embed_selftest_wait_timeout(ws, 20_000_000)  # 20 ms
    assert ne.status_names(ne.ngram_embed_get_status(ws)) == ["TIMEOUT"]
    ne.ngram_embed_clear_status(ws)
    assert ne.ngram_embed_get_status(ws) == 0
    # the context is still usable
    got, status = gpu_hash(ne, 1000, 3, 2, [4099, 5003, 6007, 7001], np.array([7, 42], np.int32), [0, 2], D=64)
    assert status == 0 and got[1].tolist() == [2943, 2039, 1035, 41]
