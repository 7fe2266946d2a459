"""GPU parity of the whole layer (Eq. 3 of "Scaling Embeddings Outperforms Scaling
Experts in Language Models", section 2) against the fp64 oracle.

Tolerance (bf16 tables, fp32 accumulation, bf16 output): max|err| <= 2e-2 and
rel-L2 <= 5e-3 vs fp64. Sizes span several 128-token tiles with a ragged tail;
the full-size workloads are checked on sampled rows the oracle computes one by one,
in the launch configuration the bench times.
"""
import gc

import numpy as np
import pytest
import torch

import oracle
from synth import configs, gen, workloads
from tests.helpers import assert_close, device_tables, host_W, oracle_rows, to_device, to_host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ne():
    import hashed_gram_embedding_horner_b200 as m
    return m


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def plan_for(ne, cfg, variant=0, tile_n=None, pair=None):
    plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk,
                                      ne.NGRAM_BF16 if cfg.dtype == "bf16" else ne.NGRAM_F32)
    if variant:
        ne.ngram_embed_plan_set_variant(plan, variant)
    if tile_n:
        ne.ngram_embed_plan_set_tile_n(plan, tile_n)
    if pair is not None:
        ne.ngram_embed_plan_set_cta_pair(plan, pair)
    return plan


def run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W, cache=None):
    T = len(tokens)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    out = torch.full((T, cfg.D), float("nan"), dtype=dt, device="cuda")
    ws = ne.new_workspace(plan, T)
    ne.ngram_embed_fwd(plan, dev_i32(tokens), dev_i32(offsets), E0, E, W, out, ws, cache=cache)
    return out, ne.ngram_embed_get_status(ws)


def small_cfg(V0, D, N, K, seed=1, dtype="bf16"):
    S = (N - 1) * K
    V = tuple(configs.primes_from(1009 + 37 * s * s, 1)[0] for s in range(S))
    return configs.NgramConfig(name=f"D{D}N{N}K{K}", V0=V0, D=D, N=N, K=K, V_nk=V, dtype=dtype, seed=seed)


RAGGED = [1, 0, 37, 130, 133]   # T = 301: three 128-token tiles, the last one ragged


def ragged_tokens(cfg, lengths=RAGGED):
    off = gen.offsets_from_lengths(lengths)
    return gen.zipf_tokens(cfg.seed + 17, int(off[-1]), cfg.V0), off


# ---------------------------------------------------------------- small shapes, every kernel

def test_tiny_fp32_config_full_parity(ne):
    cfg = configs.TINY
    tokens, offsets = workloads.prefill_tokens(cfg)
    E0, E, W = device_tables(cfg, fill_on_device=False)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    plan = plan_for(ne, cfg)
    assert not ne.ngram_embed_plan_uses_tensor_cores(plan)
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    ma, rl = assert_close(to_host_f64(out), want, what="tiny fp32")
    assert rl < 1e-6  # fp32 tables and accumulation: far inside the bf16 tolerance


SHAPES = [(5000, 256, 3, 2), (5000, 512, 5, 2), (3000, 1024, 3, 2), (5000, 384, 2, 3), (4000, 512, 3, 4)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "V0%d_D%d_N%d_K%d" % s)
@pytest.mark.parametrize("variant,tile_n,tma_rows,pair", [
    (1, 256, None, 0), (1, 128, None, 0), (2, 256, 64, 0), (2, 128, 64, 0), (2, 256, 0, 0), (2, 128, 32, 0),
    (2, 256, 96, 0), (2, 256, 0, 1), (2, 128, 0, 1), (2, 256, 64, 1), (1, 256, None, 1), (3, None, None, None)],
    ids=["tc_tma_n256", "tc_tma_n128", "tc_split64_n256", "tc_split64_n128", "tc_cpasync_n256", "tc_split32_n128",
         "tc_split96_n256", "pair_cpasync_n256", "pair_cpasync_n128", "pair_split64_n256", "pair_tma_n256", "simt"])
def test_small_shapes_all_kernels(ne, shape, variant, tile_n, tma_rows, pair):
    cfg = small_cfg(*shape)
    if tile_n == 256 and cfg.D % 256:
        pytest.skip("D not a multiple of 256")
    tokens, offsets = ragged_tokens(cfg)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = plan_for(ne, cfg, variant, tile_n, pair)
    if tma_rows is not None:
        ne.ngram_embed_plan_set_tma_rows(plan, tma_rows)
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    assert_close(to_host_f64(out), want, what=f"{cfg.name} variant {variant}")


@pytest.mark.parametrize("variant,tma_rows,pair", [(1, None, 0), (2, 0, 0), (2, 32, 0), (2, 64, 0), (2, 96, 0),
                                                  (1, None, 1), (2, 0, 1), (2, 64, 1)])
@pytest.mark.parametrize("D,N,K", [(384, 2, 3), (896, 8, 1)])  # S + 1 = 4 or 8: the scale is exact
def test_gather_and_layout_bit_exact(ne, variant, tma_rows, pair, D, N, K):
    """W = I and E_0 = 0: out = concat_s E_s[idx_s] / (S+1) exactly (a product by 1 and a power
    of two), so every gathered element must land in its place bit for bit. Then all E_s = 0:
    out = E_0[t] / (S+1) exactly, which pins the E_0 gather of the epilogue."""
    cfg = small_cfg(7000, D, N, K, seed=3)
    S = cfg.S
    tokens, offsets = ragged_tokens(cfg, [5, 128, 200, 3])
    from tests.helpers import host_tables
    E0h, Eh, _ = host_tables(cfg)
    eye = gen.f32_to_bf16_bits(np.eye(D, dtype=np.float32))
    idx = oracle.hash_indices(cfg.V0, N, K, cfg.V_nk, oracle.context_windows(N, tokens, offsets))
    G = np.concatenate([gen.bf16_bits_to_f32(Eh[s][idx[:, s]]) for s in range(S)], axis=1)
    plan = plan_for(ne, cfg, variant, pair=pair)
    if tma_rows is not None:
        ne.ngram_embed_plan_set_tma_rows(plan, tma_rows)
    zeros0 = torch.zeros((cfg.V0, D), dtype=torch.bfloat16, device="cuda")
    Ed = [to_device(e, torch.bfloat16) for e in Eh]
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, zeros0, Ed, to_device(eye, torch.bfloat16))
    assert status == 0
    got = out.float().cpu().numpy()
    np.testing.assert_array_equal(got, G / (S + 1))
    zeros = [torch.zeros_like(e) for e in Ed]
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, to_device(E0h, torch.bfloat16), zeros,
                          to_device(eye, torch.bfloat16))
    np.testing.assert_array_equal(out.float().cpu().numpy(), gen.bf16_bits_to_f32(E0h[tokens]) / (S + 1))


# ---------------------------------------------------------------- stream-K schedule

SK_SHAPES = [(3000, 1024, 3, 2, 301), (5000, 2048, 3, 2, 301), (4000, 4096, 2, 2, 1000), (5000, 1536, 4, 1, 77)]


@pytest.mark.parametrize("shape", SK_SHAPES, ids=lambda s: "V0%d_D%d_N%d_K%d_T%d" % s)
@pytest.mark.parametrize("tile_n", [256, 128])
@pytest.mark.parametrize("sms", [None, 10], ids=["all_sms", "10_sms"])
def test_stream_k_matches_oracle_and_is_repeatable(ne, shape, tile_n, sms):
    """One-CTA kernel with every SM given an equal run of (tile, k-block) units, so tiles are
    split over up to a dozen CTAs (on 10 SMs over at most two, whose last piece is summed
    from a partial staged in the free rings): parity with the oracle; a second call on the
    same workspace gives the same bits (the fixup order is fixed and the arrival counters are
    left at zero); data-parallel schedule agrees within the tolerance."""
    V0, D, N, K, T = shape
    cfg = small_cfg(V0, D, N, K, seed=5)
    if D % tile_n:
        pytest.skip("D not a multiple of the tile width")
    lengths = [T // 3, 0, T - T // 3 - 5, 5]
    tokens, offsets = ragged_tokens(cfg, lengths)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = plan_for(ne, cfg, 2, tile_n, pair=0)
    ne.ngram_embed_plan_set_tma_rows(plan, 0)
    ne.ngram_embed_plan_set_stream_k(plan, 1)
    if sms:
        ne.ngram_embed_plan_set_sm_count(plan, sms)
    out = torch.full((T, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = ne.new_workspace(plan, T)
    tk, of = dev_i32(tokens), dev_i32(offsets)
    ne.ngram_embed_fwd(plan, tk, of, E0, E, W, out, ws)
    assert ne.ngram_embed_get_status(ws) == 0
    assert not ws[256:256 + 2048 * 16].any()  # every split tile's counters back at zero
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    assert_close(to_host_f64(out), want, what=f"{cfg.name} stream-K n{tile_n}")
    again = torch.full_like(out, float("nan"))
    ne.ngram_embed_fwd(plan, tk, of, E0, E, W, again, ws)
    assert ne.ngram_embed_get_status(ws) == 0 and torch.equal(out, again)
    ne.ngram_embed_plan_set_stream_k(plan, 2)
    dp = torch.full_like(out, float("nan"))
    ne.ngram_embed_fwd(plan, tk, of, E0, E, W, dp, ws)
    assert ne.ngram_embed_get_status(ws) == 0
    assert_close(to_host_f64(dp), want, what=f"{cfg.name} data-parallel n{tile_n}")


@pytest.mark.parametrize("shape", SK_SHAPES, ids=lambda s: "V0%d_D%d_N%d_K%d_T%d" % s)
def test_pair_stream_k_matches_oracle_and_is_repeatable(ne, shape):
    """CTA-pair kernel (256 x 256 tiles) with every pair given an equal run of units: tiles
    split over up to a dozen pairs, each CTA of a pair summing its own 128 rows' pieces;
    parity with the oracle, repeatable bits, counters back at zero, and agreement with the
    pairs' data-parallel schedule."""
    V0, D, N, K, T = shape
    cfg = small_cfg(V0, D, N, K, seed=7)
    lengths = [T // 3, 0, T - T // 3 - 5, 5]
    tokens, offsets = ragged_tokens(cfg, lengths)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = plan_for(ne, cfg, 0, 256, pair=1)
    ne.ngram_embed_plan_set_pair_wide(plan, 0)
    ne.ngram_embed_plan_set_stream_k(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, T) == "cta_pair_stream_k"
    out = torch.full((T, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = ne.new_workspace(plan, T)
    tk, of = dev_i32(tokens), dev_i32(offsets)
    ne.ngram_embed_fwd(plan, tk, of, E0, E, W, out, ws)
    assert ne.ngram_embed_get_status(ws) == 0
    assert not ws[256:256 + 2048 * 16].any()  # every split tile's counters back at zero
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    assert_close(to_host_f64(out), want, what=f"{cfg.name} pair stream-K")
    again = torch.full_like(out, float("nan"))
    ne.ngram_embed_fwd(plan, tk, of, E0, E, W, again, ws)
    assert ne.ngram_embed_get_status(ws) == 0 and torch.equal(out, again)
    ne.ngram_embed_plan_set_stream_k(plan, 2)
    assert ne.ngram_embed_plan_kernel_form(plan, T) == "cta_pair"
    dp = torch.full_like(out, float("nan"))
    ne.ngram_embed_fwd(plan, tk, of, E0, E, W, dp, ws)
    assert ne.ngram_embed_get_status(ws) == 0
    assert_close(to_host_f64(dp), want, what=f"{cfg.name} pair data-parallel")


WSK_SHAPES = [((3000, 1024, 3, 2, 301), 6), ((5000, 2048, 3, 2, 301), 10), ((4000, 4096, 2, 2, 1280), 0),
              ((5000, 1536, 4, 1, 77), 4)]


@pytest.mark.parametrize("shape,sms", WSK_SHAPES, ids=lambda s: "V0%d_D%d_N%d_K%d_T%d" % s if isinstance(s, tuple)
                         else f"sms{s}")
def test_wide_stream_k_matches_oracle_and_is_repeatable(ne, shape, sms):
    """CTA pairs with 512-column tiles under stream-K (pieces of a tile summed per row quarter
    and column group by the last piece, through the epilogue's staging): a plan limited to a
    few SMs splits the small shapes' tiles; the 1280-token D = 4096 shape splits its 40
    tiles over the device's pairs. Parity with the oracle, repeatable bits, counters back at
    zero, and agreement with whole 512-column tiles."""
    V0, D, N, K, T = shape
    cfg = small_cfg(V0, D, N, K, seed=9)
    lengths = [T // 3, 0, T - T // 3 - 5, 5]
    tokens, offsets = ragged_tokens(cfg, lengths)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = plan_for(ne, cfg)
    if sms:
        ne.ngram_embed_plan_set_sm_count(plan, sms)
    ne.ngram_embed_plan_set_pair_wide(plan, 1)
    ne.ngram_embed_plan_set_stream_k(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, T) == "cta_pair_wide_stream_k"
    out = torch.full((T, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = ne.new_workspace(plan, T)
    tk, of = dev_i32(tokens), dev_i32(offsets)
    ne.ngram_embed_fwd(plan, tk, of, E0, E, W, out, ws)
    assert ne.ngram_embed_get_status(ws) == 0
    assert not ws[256:256 + 2048 * 16].any()  # every split tile's counters back at zero
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    assert_close(to_host_f64(out), want, what=f"{cfg.name} wide stream-K")
    again = torch.full_like(out, float("nan"))
    ne.ngram_embed_fwd(plan, tk, of, E0, E, W, again, ws)
    assert ne.ngram_embed_get_status(ws) == 0 and torch.equal(out, again)
    ne.ngram_embed_plan_set_stream_k(plan, 2)
    ne.ngram_embed_plan_set_pair_wide(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, T) == "cta_pair_wide"
    whole = torch.full_like(out, float("nan"))
    ne.ngram_embed_fwd(plan, tk, of, E0, E, W, whole, ws)
    assert ne.ngram_embed_get_status(ws) == 0
    assert_close(to_host_f64(whole), want, what=f"{cfg.name} whole wide tiles")


@pytest.mark.parametrize("pair", [0, 1, 2, 3], ids=["one_cta", "pair", "pair_wide", "one_cta_10_sms"])
def test_stream_k_bit_exact_with_identity_w(ne, pair):
    """W = I and E_0 = 0 under stream-K (one-CTA or CTA-pair form): each output element gets
    one nonzero product, so the fp32 partials of a split tile add zeros to it and the
    result stays exact."""
    # S + 1 = 4: the scale is exact; one-CTA: 27 tiles of 128 x 128; pairs: 9 of 256 x 256
    # (108 units of a k-block on 74 pairs); wide: 9 of 256 x 512 on 3 pairs (72 units each);
    # one-CTA on 10 SMs: 48.6 units per CTA, a tile over at most two CTAs (the last piece's
    # partial staged in the rings)
    one = pair in (0, 3)
    cfg = small_cfg(7000, {0: 1152, 1: 768, 2: 1536, 3: 1152}[pair], 2, 3, seed=3)
    S = cfg.S
    tokens, offsets = ragged_tokens(cfg, [5, 128, 200, 3] if one else [5, 300, 400, 3])
    from tests.helpers import host_tables
    _, Eh, _ = host_tables(cfg)
    eye = gen.f32_to_bf16_bits(np.eye(cfg.D, dtype=np.float32))
    idx = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk, oracle.context_windows(cfg.N, tokens, offsets))
    G = np.concatenate([gen.bf16_bits_to_f32(Eh[s][idx[:, s]]) for s in range(S)], axis=1)
    plan = plan_for(ne, cfg, 2 if one else 0, 128 if one else 256, pair=0 if one else 1)
    if one:
        ne.ngram_embed_plan_set_tma_rows(plan, 0)
    ne.ngram_embed_plan_set_pair_wide(plan, 1 if pair == 2 else 0)
    if pair in (2, 3):
        ne.ngram_embed_plan_set_sm_count(plan, 6 if pair == 2 else 10)
    ne.ngram_embed_plan_set_stream_k(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, len(tokens)) == \
        ("one_cta_stream_k", "cta_pair_stream_k", "cta_pair_wide_stream_k", "one_cta_stream_k")[pair]
    zeros0 = torch.zeros((cfg.V0, cfg.D), dtype=torch.bfloat16, device="cuda")
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, zeros0, [to_device(e, torch.bfloat16) for e in Eh],
                          to_device(eye, torch.bfloat16))
    assert status == 0
    np.testing.assert_array_equal(out.float().cpu().numpy(), G / (S + 1))


def test_n1_is_base_embedding(ne):
    cfg = configs.NgramConfig(name="n1", V0=3000, D=256, N=1, K=1, V_nk=(), dtype="bf16")
    tokens, offsets = ragged_tokens(cfg)
    E0h = gen.table_bf16(0, gen.TAG_E0, cfg.V0, cfg.D, 0.02)
    plan = plan_for(ne, cfg)
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, to_device(E0h, torch.bfloat16), [], None)
    assert status == 0
    np.testing.assert_array_equal(out.float().cpu().numpy(), gen.bf16_bits_to_f32(E0h[tokens]))


def test_gather_api_bit_exact(ne):
    cfg = small_cfg(5000, 512, 5, 2)
    tokens, offsets = ragged_tokens(cfg)
    from tests.helpers import host_tables
    _, Eh, _ = host_tables(cfg)
    idx = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk, oracle.context_windows(cfg.N, tokens, offsets))
    plan = plan_for(ne, cfg)
    ws = ne.new_workspace(plan, len(tokens))
    G = torch.empty((len(tokens), cfg.D), dtype=torch.bfloat16, device="cuda")
    ne.ngram_embed_gather(plan, dev_i32(idx), [to_device(e, torch.bfloat16) for e in Eh], G, ws)
    want = oracle.gather_rows(Eh, idx).reshape(len(tokens), cfg.D)
    np.testing.assert_array_equal(G.view(torch.int16).cpu().numpy().view(np.uint16), want)
    # with the E_0 rows of the tokens as well; one token out of range reads row 0 and is flagged
    E0h = gen.table_bf16(cfg.seed, gen.TAG_E0, cfg.V0, cfg.D, cfg.e_std)
    bad = tokens.copy()
    bad[7] = cfg.V0 + 3
    G2 = torch.empty_like(G)
    R0 = torch.empty((len(tokens), cfg.D), dtype=torch.bfloat16, device="cuda")
    ne.ngram_embed_gather(plan, dev_i32(idx), [to_device(e, torch.bfloat16) for e in Eh], G2, ws,
                          tokens=dev_i32(bad), E0=to_device(E0h, torch.bfloat16), E0_out=R0)
    assert ne.status_names(ne.ngram_embed_get_status(ws)) == ["BAD_TOKEN"]
    assert torch.equal(G, G2)
    want0 = E0h[np.where(bad < cfg.V0, bad, 0)]
    np.testing.assert_array_equal(R0.view(torch.int16).cpu().numpy().view(np.uint16), want0)


def test_gather_stage_at_decode_size_sampled(ne):
    """The gather stage at the spec-decode shape (1280 tokens, 8 sub-tables of 3.3M rows):
    sampled sub-rows and E_0 rows equal the generator's rows bit for bit."""
    cfg = configs.SPEC_DECODE
    ds = workloads.DecodeStream(cfg)
    T = ds.B * ds.P
    E0, E, W = device_tables(cfg)
    tok = ds.step_tokens(3)
    idx = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk,
                              oracle.context_windows(cfg.N, tok, ds.step_offsets()))
    plan = plan_for(ne, cfg)
    ws = ne.new_workspace(plan, T)
    G = torch.empty((T, cfg.D), dtype=torch.bfloat16, device="cuda")
    R0 = torch.empty((T, cfg.D), dtype=torch.bfloat16, device="cuda")
    ne.ngram_embed_gather(plan, dev_i32(idx), E, G, ws, tokens=dev_i32(tok), E0=E0, E0_out=R0)
    assert ne.ngram_embed_get_status(ws) == 0
    rows = np.unique(np.concatenate([[0, 1, T - 1], np.random.default_rng(2).integers(0, T, 40)]))
    from tests.helpers import host_rows
    Gh = G[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    Rh = R0[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    for s in range(cfg.S):
        np.testing.assert_array_equal(Gh[:, s * cfg.d:(s + 1) * cfg.d],
                                      host_rows(cfg, gen.TAG_SUBTABLE0 + s, idx[rows, s], cfg.d, cfg.e_std))
    np.testing.assert_array_equal(Rh, host_rows(cfg, gen.TAG_E0, tok[rows], cfg.D, cfg.e_std))
    del E0, E, W
    gc.collect()
    torch.cuda.empty_cache()


def test_project_api_flags_bad_indices(ne):
    cfg = small_cfg(5000, 256, 3, 2)
    tokens, offsets = ragged_tokens(cfg, [130])
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    idx = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk, oracle.context_windows(cfg.N, tokens, offsets))
    plan = plan_for(ne, cfg)
    ws = ne.new_workspace(plan, len(tokens))
    out = torch.empty((len(tokens), cfg.D), dtype=torch.bfloat16, device="cuda")
    args = (to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16))
    ne.ngram_embed_project(plan, dev_i32(tokens), dev_i32(idx), *args, out, ws)
    assert ne.ngram_embed_get_status(ws) == 0
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    assert_close(to_host_f64(out), want, what="project")
    bad = idx.copy()
    bad[3, 1] = cfg.V_nk[1]      # one past the end of sub-table 1
    ne.ngram_embed_project(plan, dev_i32(tokens), dev_i32(bad), *args, out, ws)
    assert "BAD_TOKEN" in ne.status_names(ne.ngram_embed_get_status(ws))


# ---------------------------------------------------------------- full-size workloads (sampled)

def sample_rows(offsets, T, n=192, seed=0):
    rng = np.random.default_rng(seed)
    edges = []
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        edges += [x for x in (s, s + 1, s + 2, s + 3, e - 1) if s <= x < e]
    rows = np.unique(np.concatenate([np.array(edges, np.int64), rng.integers(0, T, n), [T - 1]]))
    return rows


def tile_rows(offsets, T, tile=256, per=2, seed=0):
    """Rows to check at full size: `per` random rows in every `tile`-token block (every pair
    tile of the projection, the last partial one included), every sequence's first four and
    last rows, and the last token."""
    rng = np.random.default_rng(seed)
    starts = np.arange(0, T, tile)
    ends = np.minimum(starts + tile, T)
    picks = [rng.integers(a, b, per) for a, b in zip(starts, ends)]
    return np.unique(np.concatenate([sample_rows(offsets, T, n=0, seed=seed)] + picks))


@pytest.mark.parametrize("cfg", [configs.PREFILL_D2048, configs.PREFILL_D4096_VARLEN, configs.FULL_SCALE],
                         ids=lambda c: c.name)
def test_full_size_prefill(ne, cfg):
    """The full-size prefill workloads in the launch configuration the bench times (default
    plan, full workspace): every output row of the D = 2048 layer against the oracle, and at
    least two rows of every 256-token tile (plus sequence edges) of the D = 4096 layers.
    Then the other kernel forms at the same size on sampled rows."""
    tokens, offsets = workloads.prefill_tokens(cfg)
    T = len(tokens)
    E0, E, W = device_tables(cfg)
    Wh = host_W(cfg)
    plan = plan_for(ne, cfg)
    assert ne.ngram_embed_plan_uses_tensor_cores(plan)
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    assert not torch.isnan(out).any()
    rows = np.arange(T) if cfg is configs.PREFILL_D2048 else tile_rows(offsets, T)
    for a in range(0, len(rows), 8192):  # in slices: host memory for the fp64 rows stays bounded
        r = rows[a:a + 8192]
        want = oracle_rows(cfg, tokens, offsets, r, Wh)
        assert_close(to_host_f64(out[torch.from_numpy(r).cuda()]), want, what=f"{cfg.name} rows {r[0]}..{r[-1]}")
    rows = sample_rows(offsets, T)
    want = oracle_rows(cfg, tokens, offsets, rows, Wh)
    assert ne.ngram_embed_plan_kernel_form(plan, T).startswith("cta_pair")
    # the other pair tile width (256 or 512 columns) agrees with the oracle too
    wide = ne.ngram_embed_plan_kernel_form(plan, T) == "cta_pair_wide"
    ne.ngram_embed_plan_set_pair_wide(plan, 0 if wide else 1)
    outw, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    assert_close(to_host_f64(outw[torch.from_numpy(rows).cuda()]), want, what=cfg.name + " other pair width")
    del outw
    ne.ngram_embed_plan_set_pair_wide(plan, 0)
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    # other splits of the A rows between TMA and cp.async feed the MMAs the same tiles
    for tr in (64, 128):
        ne.ngram_embed_plan_set_tma_rows(plan, tr)
        out2, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
        assert status == 0 and torch.equal(out, out2), tr
    # the one-CTA kernel form (other tile order and k rotation) agrees with the oracle too
    ne.ngram_embed_plan_set_tma_rows(plan, 0)
    ne.ngram_embed_plan_set_cta_pair(plan, 0)
    out1, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    assert_close(to_host_f64(out1[torch.from_numpy(rows).cuda()]), want, what=cfg.name + " one-CTA")
    del E0, E, W, out, out2, out1
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("shape,lengths", [
    ((5000, 512, 5, 2), RAGGED),                     # one m-block pair of tiles, ragged tail
    ((4000, 512, 3, 4), RAGGED),
    ((3000, 1536, 2, 3), [1, 0, 4096, 3000, 77]),    # 3 column tiles of 512
    ((5000, 1024, 3, 2), [9000, 1, 7000, 5001, 3]),  # 166 tiles: pairs take several tiles each
], ids=["D512N5K2", "D512N3K4", "D1536N2K3", "D1024N3K2_multi"])
def test_pair_wide_matches_oracle(ne, shape, lengths):
    """The pair form's 512-column tiles (two N = 256 MMAs per A stage, TMEM halves drained
    and freed separately) against the oracle on every row, and against the 256-column pair
    form (same products, other k-block rotation)."""
    cfg = small_cfg(*shape)
    tokens, offsets = ragged_tokens(cfg, lengths)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = plan_for(ne, cfg, pair=1)
    ne.ngram_embed_plan_set_pair_wide(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, len(tokens)) == "cta_pair_wide"
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    assert_close(to_host_f64(out), want, what=cfg.name + " wide pair")
    again, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0 and torch.equal(out, again)  # fixed order: repeatable bits
    ne.ngram_embed_plan_set_pair_wide(plan, 0)
    assert ne.ngram_embed_plan_kernel_form(plan, len(tokens)) == "cta_pair"
    narrow, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    assert (out.float() - narrow.float()).abs().max().item() <= 2e-2


@pytest.mark.parametrize("shape,lengths,sms", [
    ((5000, 1024, 3, 2), RAGGED, None),                 # 2 row blocks, 37 pairs each: most hold no columns
    ((4000, 2048, 3, 4), [256] * 5, None),              # 1280 tokens at D = 2048: ranges of 128-160 columns
    ((5000, 4096, 3, 4), [5] * 256, None),              # the decode step's shape: ranges of 256-320 columns
    ((3000, 1536, 2, 3), [300, 1, 399], 6),             # 3 pairs, 3 row blocks: 1536 columns in 3 passes
    ((5000, 512, 5, 2), [1, 480, 19, 333, 167], 4),     # 2 pairs, 4 row blocks: whole blocks per pair
    ((4000, 768, 3, 2), [3, 250, 7], 40),               # D % 512 != 0, one ragged block on 20 pairs
], ids=["D1024_idle_pairs", "D2048_T1280", "D4096_T1280", "D1536_three_passes", "D512_blocks_per_pair",
        "D768_ragged"])
@pytest.mark.parametrize("dense", [0, 1], ids=["fused_rows", "dense_a"])
def test_pair_columns_matches_oracle(ne, shape, lengths, sms, dense):
    """The pair form over column ranges (every pair the full K of a range of columns of one
    256-row block; two MMAs of N = half the range per k-step; wider ranges in several
    passes), with the A rows copied by the kernel or read as dense boxes of G, against the
    oracle on every row, twice for repeatable bits."""
    cfg = small_cfg(*shape)
    tokens, offsets = ragged_tokens(cfg, lengths)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = plan_for(ne, cfg)
    if sms:
        ne.ngram_embed_plan_set_sm_count(plan, sms)
    ne.ngram_embed_plan_set_pair_columns(plan, 1)
    ne.ngram_embed_plan_set_dense_a(plan, dense)
    assert ne.ngram_embed_plan_kernel_form(plan, len(tokens)) == ("cta_pair_columns", "cta_pair_columns_dense")[dense]
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    assert_close(to_host_f64(out), want, what=cfg.name + " column ranges")
    again, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0 and torch.equal(out, again)


@pytest.mark.parametrize("D,N,K,sms", [(768, 2, 3, None), (1024, 2, 1, None), (1024, 2, 1, 6), (768, 2, 3, 12)])
@pytest.mark.parametrize("dense", [0, 1], ids=["fused_rows", "dense_a"])
def test_pair_columns_gather_and_layout_bit_exact(ne, D, N, K, sms, dense):
    """W = I and E_0 = 0 (S + 1 a power of two): every output element is one gathered
    element divided exactly, so each column range must put every column in its place bit for
    bit, whatever the range widths (partial W halves by 16-row boxes, second passes)."""
    cfg = small_cfg(7000, D, N, K, seed=3)
    S = cfg.S
    tokens, offsets = ragged_tokens(cfg, [5, 128, 200, 3, 311])
    from tests.helpers import host_tables
    _, Eh, _ = host_tables(cfg)
    eye = gen.f32_to_bf16_bits(np.eye(cfg.D, dtype=np.float32))
    idx = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk, oracle.context_windows(cfg.N, tokens, offsets))
    G = np.concatenate([gen.bf16_bits_to_f32(Eh[s][idx[:, s]]) for s in range(S)], axis=1)
    plan = plan_for(ne, cfg)
    if sms:
        ne.ngram_embed_plan_set_sm_count(plan, sms)
    ne.ngram_embed_plan_set_pair_columns(plan, 1)
    ne.ngram_embed_plan_set_dense_a(plan, dense)
    assert ne.ngram_embed_plan_kernel_form(plan, len(tokens)) == ("cta_pair_columns", "cta_pair_columns_dense")[dense]
    zeros0 = torch.zeros((cfg.V0, cfg.D), dtype=torch.bfloat16, device="cuda")
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, zeros0, [to_device(e, torch.bfloat16) for e in Eh],
                          to_device(eye, torch.bfloat16))
    assert status == 0
    np.testing.assert_array_equal(out.float().cpu().numpy(), G / (S + 1))


def test_pair_wide_not_for_narrow_tiles(ne):
    """512-column tiles need D % 512 == 0 and 256-column W halves; otherwise the knob leaves
    the 256- or 128-column pair form in place."""
    plan = plan_for(ne, small_cfg(5000, 768, 3, 2), pair=1)
    ne.ngram_embed_plan_set_pair_wide(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, 4096) == "cta_pair"
    plan = plan_for(ne, small_cfg(5000, 1024, 3, 2), tile_n=128, pair=1)
    ne.ngram_embed_plan_set_pair_wide(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, 4096) == "cta_pair"


@pytest.mark.parametrize("sms", [40, 9])
def test_reduced_sm_count_every_form(ne, sms):
    """A plan limited to fewer SMs than the device has (grids, pairs and stream-K shares
    shrink, and so does the workspace): every kernel form still matches the oracle."""
    cfg = small_cfg(5000, 1024, 3, 2, seed=13)
    tokens, offsets = ragged_tokens(cfg, [700, 1, 2000, 301, 3])
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    forms = set()
    for pair, wide, sk, dense in ((None, None, 0, 0), (1, 1, 0, 0), (1, 0, 1, 0), (1, 0, 2, 0), (0, 0, 1, 0),
                                  (0, 0, 2, 0), (None, 0, 1, 1), (None, 0, 2, 1), (None, 1, 2, 1), (None, 1, 1, 0),
                                  (1, 1, 2, 0)):
        plan = plan_for(ne, cfg, pair=pair)
        ne.ngram_embed_plan_set_sm_count(plan, sms)
        ne.ngram_embed_plan_set_pair_wide(plan, wide)
        ne.ngram_embed_plan_set_stream_k(plan, sk)
        ne.ngram_embed_plan_set_dense_a(plan, dense)
        forms.add(ne.ngram_embed_plan_kernel_form(plan, len(tokens)))
        out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
        assert status == 0
        assert_close(to_host_f64(out), want, what=f"{sms} SMs, pair={pair} wide={wide} stream-K={sk} dense={dense}")
    assert {"cta_pair_wide", "cta_pair_stream_k", "cta_pair", "one_cta_stream_k", "one_cta", "cta_pair_dense",
            "cta_pair_dense_stream_k", "cta_pair_wide_dense", "cta_pair_wide_stream_k"} <= forms


def test_automatic_kernel_form(ne):
    """Prefill grids run the CTA-pair form with 512-column tiles; a 1280-token decode step at
    D = 4096 (160 tiles of 128 x 256 on 148 SMs) runs the one-CTA form's stream-K schedule, or
    the pairs over column ranges when asked for;
    a grid of one wave keeps the 256-column pair tiles (more SMs busy). The pairs' stream-K
    schedules are taken only when the pair form (or the 512-column tiles) and stream-K are
    both asked for. With the dense-A form on, the decode step runs it with the pairs'
    stream-K schedule (or over column ranges when asked for)."""
    for cfg in (configs.PREFILL_D2048, configs.PREFILL_D4096_VARLEN):
        plan = plan_for(ne, cfg)
        assert ne.ngram_embed_plan_kernel_form(plan, 32768) == "cta_pair_wide"
    plan = plan_for(ne, configs.SPEC_DECODE)
    assert ne.ngram_embed_plan_kernel_form(plan, 1280) == "one_cta_stream_k"
    ne.ngram_embed_plan_set_pair_columns(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, 1280) == "cta_pair_columns"
    ne.ngram_embed_plan_set_pair_columns(plan, 0)
    assert ne.ngram_embed_plan_kernel_form(plan, 128) == "cta_pair"  # one wave: nothing to balance
    ne.ngram_embed_plan_set_cta_pair(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, 1280) == "cta_pair_wide"
    ne.ngram_embed_plan_set_stream_k(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, 1280) == "cta_pair_stream_k"
    ne.ngram_embed_plan_set_pair_wide(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, 1280) == "cta_pair_wide_stream_k"
    ne.ngram_embed_plan_set_cta_pair(plan, None)
    ne.ngram_embed_plan_set_stream_k(plan, 0)
    ne.ngram_embed_plan_set_pair_wide(plan, None)
    ne.ngram_embed_plan_set_dense_a(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, 1280) == "cta_pair_dense_stream_k"
    assert ne.ngram_embed_plan_kernel_form(plan, 128) == "cta_pair_dense"
    ne.ngram_embed_plan_set_pair_columns(plan, 1)
    assert ne.ngram_embed_plan_kernel_form(plan, 1280) == "cta_pair_columns_dense"
    ne.ngram_embed_plan_set_pair_columns(plan, 0)
    assert ne.ngram_embed_plan_kernel_form(plan_for(ne, configs.TINY), 128) == "cuda_cores"


@pytest.mark.parametrize("shape,lengths", [
    ((5000, 512, 5, 2), RAGGED),                     # one m-block pair, ragged tail
    ((4000, 1024, 3, 4), [1, 0, 1100, 3, 77]),        # several tiles, sequences of 1 and 3
    ((3000, 2048, 3, 2), [640, 640]),                # T = 1280: decode-sized, 2 waves of pairs
], ids=["D512N5K2", "D1024N3K4", "D2048N3K2_T1280"])
@pytest.mark.parametrize("knobs,form", [
    ({"stream_k": 2, "pair_wide": 0}, "cta_pair_dense"),
    ({"stream_k": 1, "sms": 10}, "cta_pair_dense_stream_k"),  # 5 pairs: tiles split into pieces
    ({"stream_k": 1}, None),  # stream-K where the units outnumber the device's pairs
    ({"stream_k": 2, "pair_wide": 1}, "cta_pair_wide_dense"),
], ids=["dense", "dense_stream_k_10sms", "dense_stream_k", "dense_wide"])
def test_dense_a_forms_match_oracle(ne, shape, lengths, knobs, form):
    """The dense-A form (sub-rows gathered into G in the workspace, A by 2-D TMA boxes of G)
    in each of its schedules against the oracle on every row; repeatable bits; and the same
    products as the fused pair form within the tolerance."""
    cfg = small_cfg(*shape)
    tokens, offsets = ragged_tokens(cfg, lengths)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = plan_for(ne, cfg)
    ne.ngram_embed_plan_set_dense_a(plan, 1)
    ne.ngram_embed_plan_set_stream_k(plan, knobs["stream_k"])
    if "pair_wide" in knobs:
        ne.ngram_embed_plan_set_pair_wide(plan, knobs["pair_wide"])
    if "sms" in knobs:
        ne.ngram_embed_plan_set_sm_count(plan, knobs["sms"])
    if form is None:
        units = -(-len(tokens) // 256) * (cfg.D // 256) * (cfg.D // 64)
        pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
        form = "cta_pair_dense_stream_k" if units >= pairs else "cta_pair_dense"
    assert ne.ngram_embed_plan_kernel_form(plan, len(tokens)) == form
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    want = oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh)
    assert_close(to_host_f64(out), want, what=f"{cfg.name} {form}")
    again, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0 and torch.equal(out, again)
    ne.ngram_embed_plan_set_dense_a(plan, 0)
    fused, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    assert (out.float() - fused.float()).abs().max().item() <= 2e-2


@pytest.mark.parametrize("stream_k", [1, 2])
def test_dense_a_gather_and_layout_bit_exact(ne, stream_k):
    """W = I and E_0 = 0 through the dense-A form: out = concat_s E_s[idx_s] / (S + 1)
    exactly, so every sub-row the gather kernel copied into G must reach its place in the
    output bit for bit (stream-K pieces add zeros exactly)."""
    cfg = small_cfg(7000, 768, 2, 3, seed=5)  # S + 1 = 4: the scale is exact
    tokens, offsets = ragged_tokens(cfg, [5, 1300, 900, 3])  # 27 tiles of 256 x 256
    from tests.helpers import host_tables
    _, Eh, _ = host_tables(cfg)
    E0 = torch.zeros((cfg.V0, cfg.D), dtype=torch.bfloat16, device="cuda")
    E = [to_device(e, torch.bfloat16) for e in Eh]
    W = torch.eye(cfg.D, dtype=torch.bfloat16, device="cuda")
    plan = plan_for(ne, cfg)
    ne.ngram_embed_plan_set_dense_a(plan, 1)
    ne.ngram_embed_plan_set_stream_k(plan, stream_k)
    ne.ngram_embed_plan_set_pair_wide(plan, 0)
    assert ne.ngram_embed_plan_kernel_form(plan, len(tokens)) == \
        ("cta_pair_dense_stream_k" if stream_k == 1 else "cta_pair_dense")
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    idx = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk, oracle.context_windows(cfg.N, tokens, offsets))
    G = oracle.gather_rows(Eh, idx).reshape(len(tokens), cfg.D)
    want = gen.f32_to_bf16_bits(gen.bf16_bits_to_f32(G) / np.float32(cfg.S + 1))
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)


def test_spec_decode_forward_through_ring(ne):
    """Spec-decode workload (B = 256, 5 ids per sequence per step): each step's outputs read
    their context from the ring; sampled rows vs the oracle over the committed history."""
    cfg = configs.SPEC_DECODE
    ds = workloads.DecodeStream(cfg)
    B, P, C = ds.B, ds.P, cfg.ring_capacity
    E0, E, W = device_tables(cfg)
    Wh = host_W(cfg)
    plan = plan_for(ne, cfg)
    ws = ne.new_workspace(plan, B * P)
    cache = ne.Cache.empty(B, C)
    ne.ngram_cache_reset(plan, cache, ws)
    ref = oracle.RingOracle(B, C, cfg.N)
    ids, poff = ds.prompts()
    for start in range(0, cfg.prompt_max + 1, C):
        chunk = [ids[poff[b] + start: min(poff[b + 1], poff[b] + start + C)] for b in range(B)]
        off = gen.offsets_from_lengths([len(c) for c in chunk])
        flat = np.concatenate(chunk).astype(np.int32) if off[-1] else np.zeros(1, np.int32)
        ne.ngram_cache_append(plan, cache, dev_i32(flat), dev_i32(off), ws)
        for b in range(B):
            ref.append(b, chunk[b])
    off_step = ds.step_offsets()
    out = torch.empty((B * P, cfg.D), dtype=torch.bfloat16, device="cuda")
    for step in range(4):
        tok = ds.step_tokens(step)
        ne.ngram_embed_fwd(plan, dev_i32(tok), dev_i32(off_step), E0, E, W, out, ws, cache=cache)
        rows = sample_rows(off_step, B * P, n=48, seed=step)
        want = oracle_rows(cfg, tok, off_step, rows, Wh, histories=ref.histories())
        assert_close(to_host_f64(out[torch.from_numpy(rows).cuda()]), want, what=f"decode step {step}")
        a = ds.accept_lengths(step)
        ne.ngram_cache_append(plan, cache, dev_i32(tok), dev_i32(off_step), ws)
        ne.ngram_cache_rollback(plan, cache, dev_i32(P - 1 - a), ws)
        for b in range(B):
            ref.append(b, tok[b * P:(b + 1) * P])
            ref.rollback(b, int(P - 1 - a[b]))
    assert ne.ngram_embed_get_status(ws) == 0
    del E0, E, W
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("pair", [0, 1])
def test_pdl_and_graph_replay_match_plain_launches(ne, pair):
    """Decode-like steps back to back (forward through the ring, then commit the accepted
    ids), with no host sync in between: programmatic dependent launches, eagerly and
    replayed from a CUDA graph, give the same bits and the same ring as plain launches."""
    cfg = small_cfg(5000, 1024, 3, 2, seed=11)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    B, P, steps = 40, 5, 4
    rng = np.random.default_rng(4)
    toks = [dev_i32(rng.integers(0, cfg.V0, B * P)) for _ in range(steps)]
    cnts = [dev_i32(1 + rng.integers(0, P, B)) for _ in range(steps)]
    off = dev_i32(np.arange(B + 1) * P)

    def run(pdl, graph):
        plan = plan_for(ne, cfg, pair=pair)
        ne.ngram_embed_plan_set_pdl(plan, pdl)
        ws = ne.new_workspace(plan, B * P)
        cache = ne.Cache.empty(B, 8)
        ne.ngram_cache_reset(plan, cache, ws)
        outs = [torch.full((B * P, cfg.D), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(steps)]

        def body(st=None):
            for i in range(steps):
                ne.ngram_embed_fwd(plan, toks[i], off, E0, E, W, outs[i], ws, cache=cache, stream=st)
                ne.ngram_cache_commit(plan, cache, toks[i], P, cnts[i], ws, stream=st)

        if graph:
            # first call outside the capture: it sets kernel attributes and encodes tensor maps
            ne.ngram_embed_fwd(plan, toks[0], off, E0, E, W, outs[0], ws, cache=cache)
            torch.cuda.synchronize()
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                body(s)
            g.replay()
            torch.cuda.synchronize()
            del g
        else:
            body()
        assert ne.ngram_embed_get_status(ws) == 0
        return [o.clone() for o in outs], cache.ring.clone(), cache.len.clone()

    ref = run(0, False)
    for pdl, graph in ((1, False), (1, True)):
        got = run(pdl, graph)
        assert all(torch.equal(a, b) for a, b in zip(ref[0], got[0])), (pdl, graph)
        assert torch.equal(ref[1], got[1]) and torch.equal(ref[2], got[2])


@pytest.mark.parametrize("pair,tile_n,stages", [(0, 256, 2), (0, 256, 6), (0, 128, 6), (0, 128, 10)])
@pytest.mark.parametrize("tma_rows", [0, 128])
def test_ring_depths_agree(ne, pair, tile_n, stages, tma_rows):
    """Every A/W ring split of the one-CTA kernel feeds the MMAs the same tiles in the same
    order: bits equal to the default split's."""
    cfg = small_cfg(5000, 1024, 3, 2, seed=21)
    tokens, offsets = ragged_tokens(cfg)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = plan_for(ne, cfg, 2, tile_n, pair)
    ne.ngram_embed_plan_set_tma_rows(plan, tma_rows)
    ne.ngram_embed_plan_set_stream_k(plan, 2)
    ref, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    ne.ngram_embed_plan_set_a_stages(plan, stages)
    got, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0 and torch.equal(ref, got)



# ---------------------------------------------------------------- embedding amplification

@pytest.mark.parametrize("pair", [0, 1])
def test_output_scale_amplifies_the_layer(ne, pair):
    """A constant amplification (here sqrt(D)) folded into the epilogue equals the oracle's
    layer output times that constant."""
    cfg = small_cfg(5000, 1024, 3, 2, seed=41)
    tokens, offsets = ragged_tokens(cfg)
    from tests.helpers import host_tables
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = plan_for(ne, cfg, pair=pair)
    amp = float(np.sqrt(cfg.D))
    ne.ngram_embed_plan_set_output_scale(plan, amp)
    out, status = run_fwd(ne, plan, cfg, tokens, offsets, E0, E, W)
    assert status == 0
    want = oracle.amplify(oracle.forward(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, tokens, offsets, E0h, Eh, Wh), amp)
    assert_close(to_host_f64(out), want, max_abs=2e-2 * amp, what="amplified")


@pytest.mark.parametrize("dtype,D,N,K", [("bf16", 2048, 3, 1), ("bf16", 384, 2, 3), ("fp32", 64, 3, 1),
                                         ("fp32", 36, 2, 3), ("bf16", 4096, 5, 2), ("bf16", 8192, 2, 2)])
def test_layernorm_matches_oracle(ne, dtype, D, N, K):
    """LayerNorm amplification of a layer output (bf16: the prefill widths, an odd width, and
    D = 8192, above the rows kept in registers; fp32 tiny widths incl. one not a multiple of
    8), in place and out of place, with and without gamma/beta."""
    rng = np.random.default_rng(7)
    T = 301
    S = (N - 1) * K
    plan = ne.ngram_embed_plan_create(1000, D, N, K, configs.primes_from(4099, 8)[:S], ne.NGRAM_BF16 if dtype == "bf16" else ne.NGRAM_F32)
    ws = ne.new_workspace(plan, T)
    x32 = rng.normal(0.01, 0.007, (T, D)).astype(np.float32)
    if dtype == "bf16":
        xb = gen.f32_to_bf16_bits(x32)
        x = to_device(xb, torch.bfloat16)
        xin = gen.bf16_bits_to_f32(xb)
        tol = dict(max_abs=2e-2, rel_l2=5e-3)
    else:
        x = torch.from_numpy(x32).cuda()
        xin = x32
        tol = dict(max_abs=1e-4, rel_l2=1e-5)
    g = torch.from_numpy(rng.normal(1, 0.1, D).astype(np.float32)).cuda()
    b = torch.from_numpy(rng.normal(0, 0.1, D).astype(np.float32)).cuda()
    y = torch.empty_like(x)
    ne.ngram_embed_layernorm(plan, x, y, ws, gamma=g, beta=b, eps=1e-5)
    want = oracle.layernorm(xin, g.cpu().numpy(), b.cpu().numpy(), eps=1e-5)
    assert_close(to_host_f64(y), want, what=f"layernorm {dtype} D{D}", **tol)
    ne.ngram_embed_layernorm(plan, x, x, ws, eps=1e-5)  # in place, no affine
    assert_close(to_host_f64(x), oracle.layernorm(xin, eps=1e-5), what="in place", **tol)
    assert ne.ngram_embed_get_status(ws) == 0
