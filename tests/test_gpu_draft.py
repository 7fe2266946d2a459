"""Draft-phase N-gram embedding cache (section 4.2 of "Scaling Embeddings Outperforms
Scaling Experts in Language Models", optimisations for speculative decoding): embeddings
computed while drafting are reused when the step is verified.

Checked per call: the number of cache hits against a model of the keys (a token hits iff
its window equals the one its entry was computed for), hits bit-identical to the rows
stored, every output within the tolerance of the fp64 oracle over the committed history.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import gen
from tests.helpers import assert_close, host_tables, to_device, to_host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ne():
    import hashed_gram_embedding_horner_b200 as m
    return m


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


@pytest.mark.parametrize("pair", [None, 0])  # misses by CTA pairs (automatic), or one CTA per tile
def test_draft_then_verify(ne, pair):
    from synth import configs
    V0, D, N, K = 5000, 1024, 3, 2
    V = [4099, 5003, 6007, 7001]
    cfg = configs.NgramConfig(name="draft", V0=V0, D=D, N=N, K=K, V_nk=tuple(V), dtype="bf16", seed=7)
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    B, P, C = 16, 5, 8
    plan = ne.ngram_embed_plan_create(V0, D, N, K, V, ne.NGRAM_BF16)
    if pair is not None:
        ne.ngram_embed_plan_set_cta_pair(plan, pair)
    ws = ne.new_workspace(plan, B * P)
    dws = ne.new_draft_workspace(plan, B * P)
    cache = ne.Cache.empty(B, C)
    ne.ngram_cache_reset(plan, cache, ws)
    dc = ne.DraftCache.empty(plan, B, P)
    ne.ngram_draft_cache_reset(plan, dc, ws)
    ref = oracle.RingOracle(B, C, N)
    rng = np.random.default_rng(1)
    prompt = [rng.integers(0, V0, rng.integers(0, 6)).tolist() for _ in range(B)]
    off = gen.offsets_from_lengths([len(x) for x in prompt])
    flat = np.concatenate([np.asarray(x, np.int32) for x in prompt]) if off[-1] else np.zeros(1, np.int32)
    ne.ngram_cache_append(plan, cache, dev_i32(flat), dev_i32(off), ws)
    for b in range(B):
        ref.append(b, prompt[b])
    keys = {}  # model: (b, j) -> window the entry holds
    hits = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call(step_tok):  # step_tok: list per sequence of in-step ids
        o = gen.offsets_from_lengths([len(x) for x in step_tok])
        tk = np.concatenate([np.asarray(x, np.int32) for x in step_tok])
        win = oracle.context_windows(N, tk, o, histories=ref.histories())
        want_hits = 0
        for b in range(B):
            for j in range(len(step_tok[b])):
                w = tuple(win[o[b] + j].tolist())
                if keys.get((b, j)) == w:
                    want_hits += 1
                keys[(b, j)] = w
        out = torch.full((len(tk), D), float("nan"), dtype=torch.bfloat16, device="cuda")
        hits.zero_()
        ne.ngram_embed_fwd_draft(plan, dev_i32(tk), dev_i32(o), E0, E, W, out, dws, cache, dc, hits=hits)
        assert ne.ngram_embed_get_status(dws) == 0
        assert hits.item() == want_hits
        want = oracle.forward(V0, D, N, K, V, tk, o, E0h, Eh, Wh, histories=ref.histories())
        assert_close(to_host_f64(out), want, what="draft-cache output")
        return out, o

    for step in range(3):
        x0 = rng.integers(0, V0, B)
        drafts = rng.integers(0, V0, (B, P - 1))
        rows = {}
        for k in range(P):  # draft phase: 1, 2, ..., 5 in-step ids per sequence
            out, o = call([[int(x0[b])] + drafts[b, :k].tolist() for b in range(B)])
            for b in range(B):
                rows[(b, k)] = out[o[b] + k].clone()
        if step == 2:  # the draft model changed its mind for some sequences: those windows miss
            drafts[::3, 2] = (drafts[::3, 2] + 1) % V0
        out, o = call([[int(x0[b])] + drafts[b].tolist() for b in range(B)])  # verify
        for b in range(B):
            for j in range(P):
                if step < 2 or b % 3 or j < 3:
                    assert torch.equal(out[o[b] + j], rows[(b, j)])  # a hit is the stored row, bit for bit
        accept = rng.integers(0, P, B)
        ids = np.concatenate([[x0[b]] + drafts[b].tolist() for b in range(B)]).astype(np.int32)
        ne.ngram_cache_commit(plan, cache, dev_i32(ids), P, dev_i32(1 + accept), ws)
        for b in range(B):
            ref.append(b, ids[b * P:b * P + 1 + accept[b]])
    assert ne.ngram_embed_get_status(ws) == 0
