"""GPU backward of the N-gram embedding layer (Eq. 3 of "Scaling Embeddings Outperforms
Scaling Experts in Language Models", section 2; the pages train the layer from scratch)
against the fp64 oracle's gradients.

The GPU accumulates fp32 (tensor-core GEMMs with bf16 operands, fp32 atomic scatters), the
oracle fp64 on the same bf16 values: the only difference is fp32 summation, about
sqrt(K) x 2^-24 relative for K-term sums. Bound used: rel-L2 <= 1e-4 per gradient and
max|err| <= 1e-3 x max|gradient|.
"""
import gc

import numpy as np
import pytest
import torch

import oracle
from synth import configs, gen, workloads
from tests.helpers import device_tables, host_rows, host_W, to_device

pytestmark = pytest.mark.gpu

REL_L2 = 1e-4
MAX_REL = 1e-3


@pytest.fixture(scope="module")
def ne():
    import hashed_gram_embedding_horner_b200 as m
    return m


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def close(got, want, what):
    got = np.asarray(got, np.float64)
    err = got - want
    scale = float(np.abs(want).max()) or 1.0
    rl = float(np.linalg.norm(err) / max(np.linalg.norm(want), 1e-300))
    assert float(np.abs(err).max()) <= MAX_REL * scale and rl <= REL_L2, \
        f"{what}: max|err| {np.abs(err).max():.3e} (scale {scale:.3e}), rel-L2 {rl:.3e}"


def small_problem(D=1024, N=3, K=2, V=(211, 223, 227, 229), V0=300, lengths=(1, 0, 37, 130, 133), seed=3):
    S = (N - 1) * K
    d = D // S
    rng = np.random.default_rng(seed)
    off = gen.offsets_from_lengths(list(lengths))
    T = int(off[-1])
    tok = gen.zipf_tokens(seed, T, V0).astype(np.int32)  # repeated ids: E_0 rows collide
    E = [gen.table_bf16(seed, gen.TAG_SUBTABLE0 + s, V[s], d, 0.02) for s in range(S)]
    W = gen.table_bf16(seed, gen.TAG_W, D, D, d ** -0.5)
    g = gen.f32_to_bf16_bits(rng.normal(0, 0.01, (T, D)).astype(np.float32))
    return dict(V0=V0, D=D, N=N, K=K, V=list(V), S=S, d=d, tok=tok, off=off, E=E, W=W, g=g, T=T)


def run_bwd(ne, P, scale=1.0, which=("E0", "E", "W"), repeat=1, pair=1, sms=0, streams=True, pdl=False):
    plan = ne.ngram_embed_plan_create(P["V0"], P["D"], P["N"], P["K"], P["V"], ne.NGRAM_BF16)
    ne.ngram_embed_plan_set_backward_pair(plan, pair)
    ne.ngram_embed_plan_set_backward_streams(plan, streams)
    if pdl:
        ne.ngram_embed_plan_set_pdl(plan, 1)
    if sms:
        ne.ngram_embed_plan_set_sm_count(plan, sms)
    if scale != 1.0:
        ne.ngram_embed_plan_set_output_scale(plan, scale)
    ws = ne.new_workspace(plan, P["T"])
    idx = torch.empty((P["T"], P["S"]), dtype=torch.int32, device="cuda")
    ne.ngram_hash_indices(plan, dev_i32(P["tok"]), dev_i32(P["off"]), idx, ws)
    Ed = [to_device(e, torch.bfloat16) for e in P["E"]]
    Wd = to_device(P["W"], torch.bfloat16)
    gd = to_device(P["g"], torch.bfloat16)
    dE0 = torch.zeros((P["V0"], P["D"]), dtype=torch.float32, device="cuda") if "E0" in which else None
    dE = [torch.zeros((v, P["d"]), dtype=torch.float32, device="cuda") for v in P["V"]] if "E" in which else None
    dW = torch.zeros((P["D"], P["D"]), dtype=torch.float32, device="cuda") if "W" in which else None
    bws = ne.new_bwd_workspace(plan, P["T"])
    for _ in range(repeat):
        ne.ngram_embed_bwd(plan, dev_i32(P["tok"]), idx, gd, bws, E_nk=Ed, W_stacked=Wd, dE0=dE0, dE_nk=dE, dW=dW)
    assert ne.ngram_embed_get_status(bws) == 0 and ne.ngram_embed_get_status(ws) == 0
    return (dE0.cpu().numpy() if dE0 is not None else None,
            [t.cpu().numpy() for t in dE] if dE is not None else None,
            dW.cpu().numpy() if dW is not None else None)


@pytest.mark.parametrize("shape", [dict(), dict(D=2048, N=3, K=2, V=(97, 101, 103, 107)),
                                   dict(D=1536, N=4, K=1, V=(331, 337, 347)),
                                   dict(D=384, N=2, K=3, V=(61, 67, 71)),
                                   dict(lengths=(4096,), V=(4099, 5003, 6007, 7001), V0=131072),
                                   dict(D=4096, N=5, K=2, V=(1009, 1013, 1019, 1021, 1031, 1033, 1039, 1049),
                                        lengths=(130, 77))],
                         ids=["D1024_ragged", "D2048_dense_collisions", "D1536_N4", "D384_tile128", "T4096_wide_V",
                              "D4096_N5_K2"])
@pytest.mark.parametrize("form", [dict(pair=1), dict(pair=2), dict(pair=0), dict(pair=2, sms=4),
                                  dict(pair=1, sms=5), dict(pair=1, streams=False), dict(pair=1, pdl=True)],
                         ids=["pairs_256", "pairs_wide", "one_cta", "pairs_wide_2", "pairs_256_odd_sms",
                              "one_stream", "pdl"])
def test_backward_matches_oracle(ne, shape, form):
    """Every GEMM form (pairs with 512-column tiles where D % 512 == 0, pairs with 256- or
    128-column tiles, one CTA); with 2 pairs (4 or 5 SMs) each pair runs many (tile, k range)
    units through its accumulators."""
    P = small_problem(**shape)
    dE0, dE, dW = run_bwd(ne, P, scale=3.0, **form)
    w0, wE, wW = oracle.backward(P["V0"], P["D"], P["N"], P["K"], P["V"], P["tok"], P["off"], P["E"], P["W"],
                                 P["g"], scale=3.0)
    close(dE0, w0, "dE0")
    for s in range(P["S"]):
        close(dE[s], wE[s], f"dE[{s}]")
    close(dW, wW, "dW")
    # rows nothing touched stay exactly zero
    touched = np.zeros(P["V0"], bool)
    touched[P["tok"]] = True
    assert not dE0[~touched].any()


@pytest.mark.parametrize("pair", [1, 2, 0], ids=["pairs_256", "pairs_wide", "one_cta"])
def test_backward_accumulates_and_skips(ne, pair):
    """+= semantics (two calls give twice the gradient) and NULL gradients are skipped; a
    single token (CTA 1 of the pair reads rows past the end only)."""
    P = small_problem(lengths=(64, 65))
    once = run_bwd(ne, P, pair=pair)
    twice = run_bwd(ne, P, repeat=2, pair=pair)
    close(twice[0], 2 * once[0].astype(np.float64), "2 dE0")
    close(twice[2], 2 * once[2].astype(np.float64), "2 dW")
    only_w = run_bwd(ne, P, which=("W",), pair=pair)
    assert only_w[0] is None and only_w[1] is None
    close(only_w[2], once[2].astype(np.float64), "dW alone")
    P1 = small_problem(lengths=(1,))
    dE0, dE, dW = run_bwd(ne, P1, pair=pair)
    w0, wE, wW = oracle.backward(P1["V0"], P1["D"], P1["N"], P1["K"], P1["V"], P1["tok"], P1["off"], P1["E"],
                                 P1["W"], P1["g"])
    close(dE0, w0, "dE0 T=1")
    for s in range(P1["S"]):
        close(dE[s], wE[s], f"dE[{s}] T=1")
    close(dW, wW, "dW T=1")


def test_backward_on_a_side_stream_in_a_cuda_graph(ne):
    """The auxiliary-stream fork and join inside a captured graph: every replay adds the same
    gradients as an eager call (after the warm-up call that creates the stream), on a
    non-default stream, all three gradients and each alone."""
    P = small_problem(lengths=(300, 77, 1))
    plan = ne.ngram_embed_plan_create(P["V0"], P["D"], P["N"], P["K"], P["V"], ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, P["T"])
    idx = torch.empty((P["T"], P["S"]), dtype=torch.int32, device="cuda")
    ne.ngram_hash_indices(plan, dev_i32(P["tok"]), dev_i32(P["off"]), idx, ws)
    Ed = [to_device(e, torch.bfloat16) for e in P["E"]]
    Wd = to_device(P["W"], torch.bfloat16)
    gd = to_device(P["g"], torch.bfloat16)
    tok = dev_i32(P["tok"])
    bws = ne.new_bwd_workspace(plan, P["T"])
    w0, wE, wW = oracle.backward(P["V0"], P["D"], P["N"], P["K"], P["V"], P["tok"], P["off"], P["E"], P["W"], P["g"])
    for which in (("E0", "E", "W"), ("E0", "E"), ("E", "W")):
        dE0 = torch.zeros((P["V0"], P["D"]), dtype=torch.float32, device="cuda") if "E0" in which else None
        dE = [torch.zeros((v, P["d"]), dtype=torch.float32, device="cuda") for v in P["V"]]
        dW = torch.zeros((P["D"], P["D"]), dtype=torch.float32, device="cuda") if "W" in which else None
        s = torch.cuda.Stream()
        call = lambda: ne.ngram_embed_bwd(plan, tok, idx, gd, bws, E_nk=Ed, W_stacked=Wd, dE0=dE0, dE_nk=dE, dW=dW,
                                          stream=s)
        with torch.cuda.stream(s):
            call()  # eager: creates the auxiliary stream
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            call()
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        assert ne.ngram_embed_get_status(bws) == 0
        if dE0 is not None:
            close(dE0.cpu().numpy(), 3 * w0, f"{which} dE0")
        for k in range(P["S"]):
            close(dE[k].cpu().numpy(), 3 * wE[k], f"{which} dE[{k}]")
        if dW is not None:
            close(dW.cpu().numpy(), 3 * wW, f"{which} dW")
        del graph


def test_backward_plan_released_right_after_a_forked_call(ne):
    """Destroying the plan straight after a call whose kernels are still running on its
    auxiliary stream waits for them: the gradients are complete, and a new plan's call
    (with its own auxiliary stream) adds the same again."""
    P = small_problem(lengths=(200, 9))
    w0, wE, wW = oracle.backward(P["V0"], P["D"], P["N"], P["K"], P["V"], P["tok"], P["off"], P["E"], P["W"], P["g"])
    Ed = [to_device(e, torch.bfloat16) for e in P["E"]]
    Wd = to_device(P["W"], torch.bfloat16)
    gd = to_device(P["g"], torch.bfloat16)
    tok = dev_i32(P["tok"])
    dE0 = torch.zeros((P["V0"], P["D"]), dtype=torch.float32, device="cuda")
    dE = [torch.zeros((v, P["d"]), dtype=torch.float32, device="cuda") for v in P["V"]]
    dW = torch.zeros((P["D"], P["D"]), dtype=torch.float32, device="cuda")
    for rep in (1, 2):
        plan = ne.ngram_embed_plan_create(P["V0"], P["D"], P["N"], P["K"], P["V"], ne.NGRAM_BF16)
        ws = ne.new_workspace(plan, P["T"])
        idx = torch.empty((P["T"], P["S"]), dtype=torch.int32, device="cuda")
        ne.ngram_hash_indices(plan, tok, dev_i32(P["off"]), idx, ws)
        bws = ne.new_bwd_workspace(plan, P["T"])
        ne.ngram_embed_bwd(plan, tok, idx, gd, bws, E_nk=Ed, W_stacked=Wd, dE0=dE0, dE_nk=dE, dW=dW)
        del plan  # ngram_embed_plan_destroy: waits for the plan's auxiliary stream
        torch.cuda.synchronize()
        assert ne.ngram_embed_get_status(bws) == 0
        close(dE0.cpu().numpy(), rep * w0, f"dE0 x{rep}")
        for k in range(P["S"]):
            close(dE[k].cpu().numpy(), rep * wE[k], f"dE[{k}] x{rep}")
        close(dW.cpu().numpy(), rep * wW, f"dW x{rep}")


def test_backward_full_tables_sampled(ne):
    """prefill D = 2048 tables (2.16M-row sub-tables, 8.9 GB), 4096 Zipf tokens: sampled rows
    of every gradient against the oracle computed for those rows only."""
    cfg = configs.PREFILL_D2048.with_(num_seqs=2, seq_len=2048)
    tok, off = workloads.prefill_tokens(cfg)
    T, D, S, d = len(tok), cfg.D, cfg.S, cfg.d
    E0, E, W = device_tables(cfg)
    Wh = host_W(cfg)
    rng = np.random.default_rng(5)
    g = gen.f32_to_bf16_bits(rng.normal(0, 0.01, (T, D)).astype(np.float32))
    plan = ne.ngram_embed_plan_create(cfg.V0, D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, T)
    idx_d = torch.empty((T, S), dtype=torch.int32, device="cuda")
    ne.ngram_hash_indices(plan, dev_i32(tok), dev_i32(off), idx_d, ws)
    dE0 = torch.zeros((cfg.V0, D), dtype=torch.float32, device="cuda")
    dE = [torch.zeros((v, d), dtype=torch.float32, device="cuda") for v in cfg.V_nk]
    dW = torch.zeros((D, D), dtype=torch.float32, device="cuda")
    bws = ne.new_bwd_workspace(plan, T)
    ne.ngram_embed_bwd(plan, dev_i32(tok), idx_d, to_device(g, torch.bfloat16), bws, E_nk=E, W_stacked=W,
                       dE0=dE0, dE_nk=dE, dW=dW)
    assert ne.ngram_embed_get_status(bws) == 0
    c = 1.0 / (S + 1)
    g64 = oracle._to_f64(g)
    idx = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk, oracle.context_windows(cfg.N, tok, off))
    # dE0 rows of a few tokens (the most and least frequent among them)
    for t in np.unique(np.concatenate([tok[:3], tok[-2:]])):
        want = c * g64[tok == t].sum(axis=0)
        close(dE0[int(t)].cpu().numpy()[None], want[None], f"dE0[{t}]")
    # sub-table rows: c * sum over the tokens that hit the row of (g W)[s-block]
    W64 = oracle._to_f64(Wh)
    for s in range(S):
        for r in np.unique(idx[rng.integers(0, T, 3), s]):
            hit = np.nonzero(idx[:, s] == r)[0]
            want = c * (g64[hit] @ W64[:, s * d:(s + 1) * d]).sum(axis=0)
            close(dE[s][int(r)].cpu().numpy()[None], want[None], f"dE[{s}][{r}]")
    # dW rows o: c * sum_i g[i, o] G[i, :]
    G = np.concatenate([oracle._to_f64(host_rows(cfg, gen.TAG_SUBTABLE0 + s, idx[:, s], d, cfg.e_std))
                        for s in range(S)], axis=1)
    rows = [0, 1, 777, D - 1]
    close(dW[rows].cpu().numpy(), c * (g64[:, rows].T @ G), "dW rows")
    del E0, E, W, dE0, dE, dW
    gc.collect()
    torch.cuda.empty_cache()


def test_backward_rejects_unsupported(ne):
    plan = ne.ngram_embed_plan_create(1000, 64, 3, 2, [4099, 5003, 6007, 7001], ne.NGRAM_F32)
    bws = ne.new_bwd_workspace(plan, 16)
    g = torch.zeros((16, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(ne.NgramError):
        ne.ngram_embed_bwd(plan, dev_i32(np.zeros(16)), dev_i32(np.zeros((16, 4))), g, bws, dW=torch.zeros(
            (64, 64), dtype=torch.float32, device="cuda"), E_nk=[g] * 4)
