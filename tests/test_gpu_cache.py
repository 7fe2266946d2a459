"""GPU N-gram cache (section 4.2 "N-gram Cache" of "Scaling Embeddings Outperforms
Scaling Experts in Language Models"): ring updates vs the oracle's history model, and
decode-step hashes read through the ring vs the oracle over the committed history.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import configs, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ne():
    import hashed_gram_embedding_horner_b200 as m
    return m


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def csr(lists):
    off = np.concatenate([[0], np.cumsum([len(x) for x in lists])]).astype(np.int32)
    flat = np.concatenate([np.asarray(x, np.int32) for x in lists]) if off[-1] else np.zeros(0, np.int32)
    return flat, off


def check_ring(ne, cache, ref: oracle.RingOracle):
    ln = cache.len.cpu().numpy()
    vf = cache.valid_from.cpu().numpy()
    ring = cache.ring.cpu().numpy()
    C = ring.shape[1]
    assert ln.tolist() == ref.lengths()
    assert vf.tolist() == ref.valid_from
    for b, h in enumerate(ref.hist):
        for pos in range(max(ref.valid_from[b], 0), len(h)):
            assert ring[b, pos % C] == h[pos], (b, pos)


def test_append_rollback_match_history_model(ne):
    rng = np.random.default_rng(3)
    N, C, B, V0 = 5, 16, 6, 131072
    plan = ne.ngram_embed_plan_create(V0, 4096, N, 2, configs.FULL_SCALE.V_nk, ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, 64)
    cache = ne.Cache.empty(B, C)
    ne.ngram_cache_reset(plan, cache, ws)
    ref = oracle.RingOracle(B, C, N)
    for step in range(40):
        slots = rng.permutation(B)[: rng.integers(1, B + 1)].astype(np.int32)
        if rng.random() < 0.6:
            ids = [rng.integers(0, V0, rng.integers(0, C + 3)).tolist() for _ in slots]
            flat, off = csr(ids)
            ne.ngram_cache_append(plan, cache, dev_i32(flat) if len(flat) else dev_i32([0]), dev_i32(off), ws,
                                  slots=dev_i32(slots))
            want_bad = False
            for s, x in zip(slots, ids):
                want_bad |= not ref.append(int(s), x)
        else:
            counts = rng.integers(-1, 8, len(slots)).astype(np.int32)
            ne.ngram_cache_rollback(plan, cache, dev_i32(counts), ws, slots=dev_i32(slots))
            want_bad = False
            for s, r in zip(slots, counts):
                want_bad |= not ref.rollback(int(s), int(r))
        status = ne.ngram_embed_get_status(ws)
        names = ne.status_names(status)
        assert bool(names) == want_bad, (step, names)
        ne.ngram_embed_clear_status(ws)
        check_ring(ne, cache, ref)


def test_commit_paths_agree_on_device(ne):
    """append(5) + rollback(4 - a) leaves the same committed history as append(1 + a)."""
    N, C, B = 3, 8, 5
    plan = ne.ngram_embed_plan_create(1000, 64, N, 2, [4099, 5003, 6007, 7001], ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, 64)
    c1, c2 = ne.Cache.empty(B, C), ne.Cache.empty(B, C)
    for c in (c1, c2):
        ne.ngram_cache_reset(plan, c, ws)
    step = np.arange(B * 5, dtype=np.int32) % 1000
    off5 = (np.arange(B + 1) * 5).astype(np.int32)
    for rnd in range(4):
        a = np.array([(b + rnd) % 5 for b in range(B)], np.int32)
        ne.ngram_cache_append(plan, c1, dev_i32(step + rnd), dev_i32(off5), ws)
        ne.ngram_cache_rollback(plan, c1, dev_i32(4 - a), ws)
        acc = [list(step[b * 5: b * 5 + 1 + a[b]] + rnd) for b in range(B)]
        flat, off = csr(acc)
        ne.ngram_cache_append(plan, c2, dev_i32(flat), dev_i32(off), ws)
    assert ne.ngram_embed_get_status(ws) == 0
    assert torch.equal(c1.len, c2.len)
    ln = c1.len.cpu().numpy()
    r1, r2 = c1.ring.cpu().numpy(), c2.ring.cpu().numpy()
    for b in range(B):
        for pos in range(int(ln[b]) - (N - 1), int(ln[b])):
            assert r1[b, pos % C] == r2[b, pos % C]


def test_commit_equals_append_then_rollback(ne):
    """ngram_cache_commit(counts) leaves the same committed history as append(all P ids) +
    rollback(P - counts), each matching the history model, and rejects counts above the
    stride or the capacity."""
    N, C, B, P = 3, 8, 6, 5
    plan = ne.ngram_embed_plan_create(1000, 64, N, 2, [4099, 5003, 6007, 7001], ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, 64)
    c1, c2 = ne.Cache.empty(B, C), ne.Cache.empty(B, C)
    ref1, ref2 = oracle.RingOracle(B, C, N), oracle.RingOracle(B, C, N)
    rng = np.random.default_rng(9)
    for rnd in range(5):
        step = rng.integers(0, 1000, B * P).astype(np.int32)
        a = rng.integers(0, P, B).astype(np.int32)
        ne.ngram_cache_commit(plan, c1, dev_i32(step), P, dev_i32(1 + a), ws)
        ne.ngram_cache_append(plan, c2, dev_i32(step), dev_i32(np.arange(B + 1) * P), ws)
        ne.ngram_cache_rollback(plan, c2, dev_i32(P - 1 - a), ws)
        assert ne.ngram_embed_get_status(ws) == 0
        for b in range(B):
            assert ref1.append(b, step[b * P:b * P + 1 + a[b]])
            assert ref2.append(b, step[b * P:(b + 1) * P]) and ref2.rollback(b, int(P - 1 - a[b]))
        check_ring(ne, c1, ref1)
        check_ring(ne, c2, ref2)
        # same committed history; committing only the accepted ids evicts no more than append + rollback
        assert torch.equal(c1.len, c2.len) and bool((c1.valid_from <= c2.valid_from).all())
        ln = c1.len.cpu().numpy()
        r1, r2 = c1.ring.cpu().numpy(), c2.ring.cpu().numpy()
        for b in range(B):
            for pos in range(int(ln[b]) - (N - 1), int(ln[b])):
                assert r1[b, pos % C] == r2[b, pos % C]
    ne.ngram_cache_commit(plan, c1, dev_i32(np.zeros(B * P)), P, dev_i32([P + 1] * B), ws)
    assert ne.status_names(ne.ngram_embed_get_status(ws)) == ["BAD_APPEND"]


def test_decode_hashes_through_ring(ne):
    """Spec-decode workload: per step, hashes of the 5 in-step ids read the ring's
    committed history; equal (bit-exact) to the oracle over the full history."""
    cfg = configs.SPEC_DECODE
    ds = workloads.DecodeStream(cfg, num_seqs=64)
    B, P, C = ds.B, ds.P, cfg.ring_capacity
    plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, B * P)
    cache = ne.Cache.empty(B, C)
    ne.ngram_cache_reset(plan, cache, ws)
    ref = oracle.RingOracle(B, C, cfg.N)
    ids, poff = ds.prompts()
    # prompts longer than C are committed in chunks of at most C ids
    for start in range(0, 17, C):
        chunk = [ids[poff[b] + start: min(poff[b + 1], poff[b] + start + C)] for b in range(B)]
        flat, off = csr(chunk)
        ne.ngram_cache_append(plan, cache, dev_i32(flat) if len(flat) else dev_i32([0]), dev_i32(off), ws)
        for b in range(B):
            ref.append(b, chunk[b])
    off_step = dev_i32(ds.step_offsets())
    idx = torch.empty((B * P, cfg.S), dtype=torch.int32, device="cuda")
    for step in range(12):
        tok = ds.step_tokens(step)
        ne.ngram_hash_indices(plan, dev_i32(tok), off_step, idx, ws, cache=cache)
        want = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk,
                                   oracle.context_windows(cfg.N, tok, ds.step_offsets(), histories=ref.histories()))
        np.testing.assert_array_equal(idx.cpu().numpy(), want)
        a = ds.accept_lengths(step)
        ne.ngram_cache_append(plan, cache, dev_i32(tok), off_step, ws)
        ne.ngram_cache_rollback(plan, cache, dev_i32(P - 1 - a), ws)
        for b in range(B):
            assert ref.append(b, tok[b * P:(b + 1) * P]) and ref.rollback(b, int(P - 1 - a[b]))
        assert ne.ngram_embed_get_status(ws) == 0
    check_ring(ne, cache, ref)


def test_evicted_context_is_flagged(ne):
    N, C = 5, 4  # capacity exactly N-1
    plan = ne.ngram_embed_plan_create(1000, 64, N, 1, [4099, 5003, 6007, 7001], ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, 16)
    cache = ne.Cache.empty(1, C)
    ne.ngram_cache_reset(plan, cache, ws)
    ne.ngram_cache_append(plan, cache, dev_i32([1, 2, 3, 4]), dev_i32([0, 4]), ws)
    ne.ngram_cache_append(plan, cache, dev_i32([5, 6]), dev_i32([0, 2]), ws)  # holds positions 2..5
    idx = torch.empty((1, 4), dtype=torch.int32, device="cuda")
    ne.ngram_hash_indices(plan, dev_i32([9]), dev_i32([0, 1]), idx, ws, cache=cache)
    assert ne.ngram_embed_get_status(ws) == 0
    want = oracle.hash_indices(1000, N, 1, [4099, 5003, 6007, 7001],
                               oracle.context_windows(N, np.array([9], np.int32), [0, 1],
                                                      histories=[[1, 2, 3, 4, 5, 6]]))
    np.testing.assert_array_equal(idx.cpu().numpy(), want)
    # a rollback that would need position 1 again is refused and changes nothing
    ne.ngram_cache_rollback(plan, cache, dev_i32([1]), ws)
    assert ne.status_names(ne.ngram_embed_get_status(ws)) == ["BAD_ROLLBACK"]
    assert cache.len.item() == 6
    ne.ngram_embed_clear_status(ws)
    # a caller that corrupts valid_from makes the context read an evicted position
    cache.valid_from.fill_(5)
    ne.ngram_hash_indices(plan, dev_i32([9]), dev_i32([0, 1]), idx, ws, cache=cache)
    assert ne.status_names(ne.ngram_embed_get_status(ws)) == ["EVICTED"]


@pytest.mark.parametrize("form", ["cta_pair", "cta_pair_dense", "one_cta", "one_cta_stream_k", "one_cta_2_launches"])
def test_fused_commit_and_step_equals_separate_calls(ne, form):
    """ngram_embed_fwd_step (commit of the previous step fused with this step's hashing; with
    the dense-A form also with the sub-row gather into G; with the one-CTA forms hashed inside
    the projection and committed by its last CTA, one launch) gives the same outputs, bit for
    bit, the same indices and the same ring as ngram_cache_commit + ngram_embed_fwd."""
    dense_a = int(form == "cta_pair_dense")
    from tests.helpers import host_tables, to_device
    N, K, D, B, P, C = 3, 2, 512, 24, 5, 8
    V0, V = 3000, [4099, 5003, 6007, 7001]
    cfg = configs.NgramConfig(name="step", V0=V0, D=D, N=N, K=K, V_nk=tuple(V), dtype="bf16", seed=13)
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = ne.ngram_embed_plan_create(V0, D, N, K, V, ne.NGRAM_BF16)
    ne.ngram_embed_plan_set_dense_a(plan, dense_a)
    if form.startswith("one_cta"):
        ne.ngram_embed_plan_set_cta_pair(plan, 0)
        ne.ngram_embed_plan_set_stream_k(plan, 1 if form == "one_cta_stream_k" else 2)
        if form == "one_cta_stream_k":
            ne.ngram_embed_plan_set_sm_count(plan, 6)  # 16 units over 6 CTAs: tiles split
    ne.ngram_embed_plan_set_fused_step(plan, form in ("one_cta", "one_cta_stream_k"))
    assert ne.ngram_embed_plan_kernel_form(plan, B * P) == form.replace("_2_launches", "")
    ws1, ws2 = ne.new_workspace(plan, B * P), ne.new_workspace(plan, B * P)
    c1, c2 = ne.Cache.empty(B, C), ne.Cache.empty(B, C)
    for c, w in ((c1, ws1), (c2, ws2)):
        ne.ngram_cache_reset(plan, c, w)
    rng = np.random.default_rng(21)
    off = dev_i32(np.arange(B + 1) * P)
    prev = None
    for step in range(6):
        tok = dev_i32(rng.integers(0, V0, B * P))
        cnt = dev_i32(1 + rng.integers(0, P, B))
        o1 = torch.empty((B * P, D), dtype=torch.bfloat16, device="cuda")
        o2 = torch.empty_like(o1)
        if prev is not None:
            ne.ngram_cache_commit(plan, c1, prev[0], P, prev[1], ws1)
        ne.ngram_embed_fwd(plan, tok, off, E0, E, W, o1, ws1, cache=c1)
        ne.ngram_embed_fwd_step(plan, tok, off, E0, E, W, o2, ws2, c2,
                                commit_tokens=None if prev is None else prev[0], commit_stride=P,
                                commit_counts=None if prev is None else prev[1])
        assert torch.equal(o1, o2), step
        head = 33024  # the workspace's index buffer follows its head
        assert torch.equal(ws1[head:head + B * P * 16], ws2[head:head + B * P * 16])  # [T x S] int32 indices
        assert torch.equal(c1.ring, c2.ring) and torch.equal(c1.len, c2.len) and torch.equal(c1.valid_from, c2.valid_from)
        prev = (tok, cnt)
    assert ne.ngram_embed_get_status(ws1) == 0 and ne.ngram_embed_get_status(ws2) == 0


@pytest.mark.parametrize("one_cta", [False, True], ids=["commit_hash_kernel", "in_projection"])
def test_fused_step_edge_cases_match_separate_calls(ne, one_cta):
    """The fused step's per-sequence paths (commit_hash_kernel: loads in three rounds; one-CTA
    projection: windows hashed by its gather warps, commit by its last CTA; committed ids taken
    from the commit buffer) against ngram_cache_commit + ngram_embed_fwd where it matters: a sequence
    of 40 ids (more than a warp's lanes: the one-load-at-a-time path), empty sequences,
    nothing to commit, a count above the stride (BAD_APPEND), an id outside the vocabulary
    in the commit buffer (BAD_TOKEN: that entry is not committed), and a history cut by
    valid_from (EVICTED). Outputs, indices, ring, lengths and status bits agree."""
    from tests.helpers import host_tables, to_device
    N, K, D, B, P, C = 4, 1, 384, 6, 6, 8
    V0, V = 3000, [4099, 5003, 6007]
    cfg = configs.NgramConfig(name="edges", V0=V0, D=D, N=N, K=K, V_nk=tuple(V), dtype="bf16", seed=17)
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = ne.ngram_embed_plan_create(V0, D, N, K, V, ne.NGRAM_BF16)
    if one_cta:
        ne.ngram_embed_plan_set_cta_pair(plan, 0)
        ne.ngram_embed_plan_set_stream_k(plan, 1)
        ne.ngram_embed_plan_set_sm_count(plan, 4)  # 18 units over 4 CTAs
        ne.ngram_embed_plan_set_fused_step(plan, True)
        assert ne.ngram_embed_plan_kernel_form(plan, 52) == "one_cta_stream_k"
    lengths = [1, 40, 0, 6, 3, 2]
    off_h = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(off_h[-1])
    off = dev_i32(off_h)
    ws1, ws2 = ne.new_workspace(plan, T), ne.new_workspace(plan, T)
    c1, c2 = ne.Cache.empty(B, C), ne.Cache.empty(B, C)
    for c, w in ((c1, ws1), (c2, ws2)):
        ne.ngram_cache_reset(plan, c, w)
    rng = np.random.default_rng(5)
    prev = None
    for step in range(5):
        tok = dev_i32(rng.integers(0, V0, T))
        commit = rng.integers(0, V0, B * P).astype(np.int32)
        counts = np.array([1, 6, 0, 7 if step == 2 else 3, 2, 6], np.int32)
        if step == 3:
            commit[4 * P + 1] = V0 + 5  # entry 4 holds an id outside the vocabulary
        if step == 4:
            for c in (c1, c2):  # history of sequence 0 cut right below its newest position
                c.valid_from[0] = c.len[0] - 1
        o1 = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
        o2 = torch.empty_like(o1)
        if prev is not None:
            ne.ngram_cache_commit(plan, c1, prev[0], P, prev[1], ws1)
        ne.ngram_embed_fwd(plan, tok, off, E0, E, W, o1, ws1, cache=c1)
        ne.ngram_embed_fwd_step(plan, tok, off, E0, E, W, o2, ws2, c2,
                                commit_tokens=None if prev is None else prev[0], commit_stride=P,
                                commit_counts=None if prev is None else prev[1])
        s1, s2 = ne.ngram_embed_get_status(ws1), ne.ngram_embed_get_status(ws2)
        assert s1 == s2, (step, ne.status_names(s1), ne.status_names(s2))
        assert torch.equal(o1, o2), step
        head = 33024
        assert torch.equal(ws1[head:head + T * 12], ws2[head:head + T * 12])  # [T x S] int32 indices
        assert torch.equal(c1.ring, c2.ring) and torch.equal(c1.len, c2.len) and torch.equal(c1.valid_from, c2.valid_from)
        prev = (dev_i32(commit), dev_i32(counts))
    # the edge cases did occur
    assert set(ne.status_names(ne.ngram_embed_get_status(ws2))) == {"BAD_APPEND", "BAD_TOKEN", "EVICTED"}
