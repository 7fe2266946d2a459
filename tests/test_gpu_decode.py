"""Speculative decode through the N-gram cache ("Scaling Embeddings Outperforms Scaling
Experts in Language Models", section 4.2, "N-gram Cache") at the workloads' full sizes, in
the launch configuration the bench times: every step is one ngram_embed_fwd_step (the commit
of the previous step's accepted ids fused with this step's context hashing, then the
projection), default plan, full workspace.

Two workloads, 1000 steps each, 256 sequences x 5 ids (x0 + 4 drafts) per step, accept
lengths a ~ U{0..4} (1 + a ids committed):
  - the full-scale layer's decode half: D = 4096, N = 5, K = 2, ring capacity 16, on the
    59.6 GB sub-tables;
  - the spec-decode layer: D = 4096, N = 3, K = 4, ring capacity 8.
On every step the indices the projection consumed (the workspace's index buffer) equal the
oracle's Eq. 2 hashes over the committed history, bit for bit; on step 0, every 50th step and
the last, sampled output rows (every 128-token tile) match the fp64 oracle within the stated
tolerance (max|err| <= 2e-2, rel-L2 <= 5e-3).
"""
import gc

import numpy as np
import pytest
import torch

import oracle
from synth import configs, gen, workloads
from tests.helpers import assert_close, device_tables, host_W, oracle_rows, to_host_f64

pytestmark = pytest.mark.gpu

# The workspace: a 33,024-byte head (status word, stream-K arrival counters), then the
# [T x S] int32 indices of the call (the layout ngram_embed_workspace_bytes documents).
WS_HEAD_BYTES = 33024


@pytest.fixture(scope="module")
def ne():
    import hashed_gram_embedding_horner_b200 as m
    return m


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def recent(ref: oracle.RingOracle, N: int):
    """Each sequence's last N - 1 committed ids: all of the history that a window of the next
    step can reach (the windows read at most N - 1 ids before a step's first token)."""
    return [h[-(N - 1):] if N > 1 else [] for h in ref.hist]


def decode_rows(T, tile=128, per=4, seed=0):
    rng = np.random.default_rng(seed)
    picks = [rng.integers(a, min(a + tile, T), per) for a in range(0, T, tile)]
    return np.unique(np.concatenate(picks + [np.array([0, T - 1])]))


@pytest.mark.parametrize("cfg", [configs.FULL_SCALE_DECODE, configs.SPEC_DECODE], ids=lambda c: c.name)
def test_decode_1000_steps_through_the_ring(ne, cfg):
    steps = cfg.decode_steps
    assert steps == 1000
    ds = workloads.DecodeStream(cfg)
    B, P, C = ds.B, ds.P, cfg.ring_capacity
    T = B * P
    assert (B, P) == (256, 5) and C >= cfg.N - 1 + P
    E0, E, W = device_tables(cfg)
    Wh = host_W(cfg)
    plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
    # the spec-decode run takes the step in one launch (commit and hashing inside the one-CTA
    # projection), the full-scale run the default two
    ne.ngram_embed_plan_set_fused_step(plan, cfg is configs.SPEC_DECODE)
    ws = ne.new_workspace(plan, T)
    cache = ne.Cache.empty(B, C)
    ne.ngram_cache_reset(plan, cache, ws)
    ref = oracle.RingOracle(B, C, cfg.N)
    # seeded prompts of 0..16 ids, committed in chunks of at most C ids (as the bench does)
    ids, poff = ds.prompts()
    for start in range(0, cfg.prompt_max + 1, C):
        chunk = [ids[poff[b] + start: min(poff[b + 1], poff[b] + start + C)] for b in range(B)]
        off = gen.offsets_from_lengths([len(c) for c in chunk])
        flat = np.concatenate(chunk).astype(np.int32) if off[-1] else np.zeros(1, np.int32)
        ne.ngram_cache_append(plan, cache, dev_i32(flat), dev_i32(off), ws)
        for b in range(B):
            assert ref.append(b, chunk[b])
    off_h = ds.step_offsets()
    off_d = dev_i32(off_h)
    out = torch.empty((T, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx_view = ws[WS_HEAD_BYTES:WS_HEAD_BYTES + T * cfg.S * 4].view(torch.int32).view(T, cfg.S)
    check_out = set(range(0, steps, 50)) | {steps - 1}
    prev = None
    checked_rows = 0
    for step in range(steps):
        tok = ds.step_tokens(step)
        tok_d = dev_i32(tok)
        ne.ngram_embed_fwd_step(plan, tok_d, off_d, E0, E, W, out, ws, cache,
                                commit_tokens=None if prev is None else prev[0], commit_stride=P,
                                commit_counts=None if prev is None else prev[1])
        hist = recent(ref, cfg.N)  # the ring as this step's commit left it
        want_idx = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk,
                                       oracle.context_windows(cfg.N, tok, off_h, histories=hist))
        np.testing.assert_array_equal(idx_view.cpu().numpy(), want_idx, err_msg=f"{cfg.name} step {step}")
        if step in check_out:
            rows = decode_rows(T, seed=step)
            want = oracle_rows(cfg, tok, off_h, rows, Wh, histories=hist)
            assert_close(to_host_f64(out[torch.from_numpy(rows).cuda()]), want, what=f"{cfg.name} step {step}")
            checked_rows += len(rows)
        # this step's accepted prefix, committed by the next step's call
        cnt = 1 + ds.accept_lengths(step)
        for b in range(B):
            assert ref.append(b, tok[b * P:b * P + cnt[b]])
        prev = (tok_d, dev_i32(cnt))
    assert ne.ngram_embed_get_status(ws) == 0
    assert checked_rows >= 21 * 40
    # the ring holds the committed history of every sequence (its newest N - 1 ids at least)
    ne.ngram_cache_commit(plan, cache, prev[0], P, prev[1], ws)
    torch.cuda.synchronize()
    ln = cache.len.cpu().numpy()
    ring = cache.ring.cpu().numpy()
    for b in range(B):
        h = ref.hist[b]
        assert ln[b] == len(h)
        for pos in range(max(0, len(h) - (cfg.N - 1)), len(h)):
            assert ring[b, pos % C] == h[pos]
    del E0, E, W, out, ws
    gc.collect()
    torch.cuda.empty_cache()
