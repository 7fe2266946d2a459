"""The C ABI library: loads, exports every declared symbol, validates on the host.

These run without a GPU: no kernel is launched (every call below is rejected by a
host-side check before any launch, or needs no device).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ngram_embed.h")


@pytest.fixture(scope="module")
def ne():
    import hashed_gram_embedding_horner_b200 as m
    return m


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(ngram_\w+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported(ne):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(ne._lib, n), n
    assert sorted(ne.EXPORTED) == names


def test_no_cpu_fallback_symbols(ne):
    """The library is CUDA-only: it neither links nor names the oracle."""
    so = open(ne.LIB_PATH, "rb").read()
    assert b"oracle_" not in so


def _cfg(ne, V0=131072, D=2048, N=3, K=2, V=(2162717, 2162737, 2162747, 2162803), dtype=0):
    arr = (ctypes.c_int64 * max(len(V), 1))(*V)
    return ne._Config(V0, D, N, K, ctypes.cast(arr, ctypes.POINTER(ctypes.c_int64)), dtype), arr


def _create(ne, **kw):
    cfg, keep = _cfg(ne, **kw)
    h = ctypes.c_void_p()
    rc = ne._lib.ngram_embed_plan_create(ctypes.byref(cfg), ctypes.byref(h))
    return rc, h


@pytest.mark.parametrize("kw,code", [
    (dict(V0=0), -1), (dict(V0=2 ** 31), -1), (dict(D=0), -1), (dict(N=0), -1), (dict(K=0), -1),
    (dict(N=9, K=1, V=(5,) * 8), -2),                 # N above the limit
    (dict(N=5, K=9, V=(5,) * 36), -2),                # S above the limit
    (dict(D=2046), -1),                               # D % S != 0
    (dict(V=(0, 1, 2, 3)), -1), (dict(V=(2 ** 31, 1, 2, 3)), -1),
    (dict(dtype=7), -1),
    (dict(D=20, N=2, K=4, V=(7, 7, 7, 7)), -2),       # d * elt not a multiple of 16 bytes
])
def test_plan_rejects_bad_configs(ne, kw, code):
    rc, h = _create(ne, **kw)
    assert rc == code and not h.value


def test_plan_without_device_validates_then_fails_launch(ne):
    import torch
    rc, h = _create(ne)
    if torch.cuda.is_available():
        assert rc == 0
        ne._lib.ngram_embed_plan_destroy(h)
        return
    # No GPU here: the plan is created for argument checks; anything that would launch
    # reports NGRAM_ERR_CUDA, while bad arguments are still reported first.
    assert rc == 0 and h.value
    lib = ne._lib
    ws_need = lib.ngram_embed_workspace_bytes(h, 1000)
    # head (status word + 2048 x 4 stream-K counters), indices; no SM count without a device
    assert ws_need == 256 + 2048 * 4 * 4 + ((1000 * 4 * 4 + 255) // 256) * 256
    fake = ctypes.c_void_p(0x10000)           # never dereferenced
    odd = ctypes.c_void_p(0x10004)
    tabs = (ctypes.c_void_p * 4)(0x20000, 0x30000, 0x40000, 0x50000)
    P = ctypes.c_void_p
    fwd = lambda ws, wsb, out=fake, T=1000: lib.ngram_embed_fwd(h, fake, fake, 1, T, fake, tabs, fake, None, None,
                                                                 out, ws, wsb, None)
    assert fwd(fake, 10) == -4                 # workspace too small
    assert fwd(odd, ws_need) == -3             # misaligned workspace
    assert fwd(fake, ws_need, out=odd) == -3   # misaligned output
    assert fwd(None, ws_need) == -1
    assert fwd(fake, ws_need, T=0) == 0        # nothing to do, nothing launched
    assert fwd(fake, ws_need) == -5            # would launch: no device
    assert lib.ngram_embed_plan_set_variant(h, 9) == -1
    assert lib.ngram_embed_plan_set_tile_n(h, 64) == -1
    assert lib.ngram_embed_plan_set_stream_k(h, 3) == -1 and lib.ngram_embed_plan_set_stream_k(h, 2) == 0
    assert lib.ngram_embed_plan_set_pdl(h, 2) == -1 and lib.ngram_embed_plan_set_pdl(h, 1) == 0
    assert lib.ngram_embed_plan_set_a_stages(h, 5) == -1 and lib.ngram_embed_plan_set_a_stages(h, 6) == 0
    # no device: the stream-K schedule (it needs the SM count) never applies, so the pair form
    assert lib.ngram_embed_plan_kernel_form(h, 1280) == 3 and lib.ngram_embed_plan_kernel_form(h, -1) == -1
    assert lib.ngram_embed_plan_set_dense_a(h, 2) == -1 and lib.ngram_embed_plan_set_dense_a(h, -1) == -1
    assert lib.ngram_embed_plan_set_cta_pair(h, 0) == 0 and lib.ngram_embed_plan_kernel_form(h, 1280) == 1
    assert lib.ngram_embed_plan_set_dense_a(h, 1) == 0 and lib.ngram_embed_plan_kernel_form(h, 1280) == 1
    assert lib.ngram_embed_plan_set_cta_pair(h, -1) == 0 and lib.ngram_embed_plan_set_cta_pair(h, 2) == -1
    # the dense-A form when asked for: at any size whose G the workspace holds (it grows by T x D x 2)
    assert lib.ngram_embed_plan_kernel_form(h, 1280) == 6 and lib.ngram_embed_plan_kernel_form(h, 32768) == 6
    with_g = lib.ngram_embed_workspace_bytes(h, 32768)
    assert lib.ngram_embed_plan_set_dense_a(h, 0) == 0 and lib.ngram_embed_plan_kernel_form(h, 32768) == 3
    assert with_g - lib.ngram_embed_workspace_bytes(h, 32768) == 32768 * 2048 * 2
    # 512-column pair tiles (D = 2048 here): on when forced, automatic needs the SM count
    assert lib.ngram_embed_plan_set_pair_wide(h, 2) == -1 and lib.ngram_embed_plan_set_pair_wide(h, -2) == -1
    # the backward's GEMM forms (0, 1, 2) and streams (0, 1)
    assert lib.ngram_embed_plan_set_backward_pair(h, 3) == -1 and lib.ngram_embed_plan_set_backward_pair(h, -1) == -1
    assert all(lib.ngram_embed_plan_set_backward_pair(h, m) == 0 for m in (0, 2, 1))
    assert lib.ngram_embed_plan_set_backward_streams(h, 2) == -1 and lib.ngram_embed_plan_set_backward_streams(h, -1) == -1
    assert lib.ngram_embed_plan_set_backward_streams(h, 0) == 0 and lib.ngram_embed_plan_set_backward_streams(h, 1) == 0
    assert lib.ngram_embed_plan_set_backward_pair(None, 1) == -1 and lib.ngram_embed_plan_set_backward_streams(None, 1) == -1
    assert lib.ngram_embed_plan_set_pair_wide(h, 1) == 0 and lib.ngram_embed_plan_kernel_form(h, 1280) == 4
    assert lib.ngram_embed_plan_set_dense_a(h, 1) == 0 and lib.ngram_embed_plan_kernel_form(h, 1280) == 8
    assert lib.ngram_embed_plan_set_tile_n(h, 128) == 0 and lib.ngram_embed_plan_kernel_form(h, 1280) == 3
    assert lib.ngram_embed_plan_set_tile_n(h, 256) == 0 and lib.ngram_embed_plan_set_dense_a(h, 0) == 0
    assert lib.ngram_embed_plan_set_pair_wide(h, -1) == 0 and lib.ngram_embed_plan_kernel_form(h, 1280) == 3
    assert lib.ngram_embed_plan_uses_tensor_cores(h) == 1
    bad_cache = ne._Cache(0, 0, 0, 4, 8)
    assert lib.ngram_cache_rollback(h, ctypes.byref(bad_cache), None, fake, 3, fake, ws_need, None) == -1
    small_cap = ne._Cache(0x1000, 0x2000, 0x3000, 1, 8)  # capacity < N - 1
    assert lib.ngram_cache_append(h, ctypes.byref(small_cap), None, fake, fake, 3, fake, ws_need, None) == -1
    lib.ngram_embed_plan_destroy(h)


def test_fp32_and_small_shapes_use_cuda_cores(ne):
    rc, h = _create(ne, V0=1000, D=64, N=3, K=2, V=(4099, 5003, 6007, 7001), dtype=1)
    assert rc == 0
    assert ne._lib.ngram_embed_plan_uses_tensor_cores(h) == 0
    assert ne._lib.ngram_embed_plan_set_variant(h, 1) == -2
    ne._lib.ngram_embed_plan_destroy(h)
    rc, h = _create(ne, D=384, N=2, K=3, V=(11, 13, 17))  # D % 128 == 0, d = 128
    assert rc == 0 and ne._lib.ngram_embed_plan_uses_tensor_cores(h) == 1
    ne._lib.ngram_embed_plan_destroy(h)


def test_error_strings(ne):
    for c in (0, -1, -2, -3, -4, -5, -99):
        assert ne._lib.ngram_embed_error_string(c)


V25 = (3342341, 3342371, 3342379, 3342413, 3342419, 3342439, 3342457, 3342473)


@pytest.mark.parametrize("kw,T,sms,knobs,form", [
    (dict(), 32768, 148, {}, 4),                                  # prefill D = 2048: 512-column pair tiles
    (dict(D=4096, N=5, K=2, V=V25), 65536, 148, {}, 4),           # varlen prefill D = 4096
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {}, 2),            # decode step: one-CTA stream-K
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"pair_columns": 1}, 10),  # pairs over column ranges
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"pair_columns": 1, "cta_pair": 0}, 2),  # they need pairs
    (dict(), 32768, 148, {"pair_columns": 1}, 10),                # at any size: 128 row blocks on 74 pairs
    (dict(), 32768, 148, {"pair_columns": 1, "tile_n": 128}, 3),  # but not with 128-column W halves
    (dict(D=4096, N=3, K=4, V=V25), 128, 148, {}, 3),             # one wave: 256-column pair tiles
    (dict(D=4096, N=3, K=4, V=V25), 5120, 148, {}, 3),            # 160 wide tiles: a thin third wave
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"pair_wide": 0}, 2),  # without wide tiles: one-CTA stream-K
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"stream_k": 2}, 4),   # no stream-K: whole wide tiles
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"cta_pair": 1}, 4),
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"pair_wide": 1, "stream_k": 1}, 9),  # wide tiles, stream-K
    (dict(D=4096, N=3, K=4, V=V25), 128, 148, {"pair_wide": 1, "stream_k": 1}, 2),   # 8 wide tiles: too few
                                                                                     # to split; one-CTA stream-K
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"cta_pair": 1, "stream_k": 1}, 5),
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"cta_pair": 0, "stream_k": 2}, 1),
    (dict(D=4096, N=3, K=4, V=V25), 1280, 40, {}, 4),             # 20 pairs: 40 wide tiles fill 2 waves
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"dense_a": 1}, 7),  # dense A: the pairs' stream-K
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"dense_a": 1, "pair_columns": 1}, 11),  # or column ranges
    (dict(D=4096, N=3, K=4, V=V25), 128, 148, {"dense_a": 1}, 6),
    (dict(D=4096, N=3, K=4, V=V25), 1280, 40, {"dense_a": 1}, 8),  # 20 pairs: wide tiles fill 2 waves
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"dense_a": 1, "stream_k": 2}, 8),
    (dict(D=4096, N=3, K=4, V=V25), 1280, 148, {"dense_a": 1, "cta_pair": 0}, 2),  # dense A needs pairs
    (dict(), 32768, 148, {"tile_n": 128}, 3),                     # 128-column W halves: never wide
    (dict(), 32768, 148, {"tile_n": 128, "dense_a": 1}, 3),       # ... nor dense A
    (dict(), 32768, 148, {"dense_a": 1}, 8),                      # dense A at prefill: wide tiles
    (dict(D=768, N=2, K=3, V=V25[:3]), 32768, 148, {}, 3),        # D % 512 != 0
])
def test_kernel_form_choice_for_a_device_size(ne, kw, T, sms, knobs, form):
    """The automatic choice between the projection kernels, as a device of `sms` SMs would
    make it: the plan's SM count is set by hand, which is what lets this run without one."""
    lib = ne._lib
    rc, h = _create(ne, **kw)
    assert rc == 0
    assert lib.ngram_embed_plan_set_sm_count(h, sms) == 0  # a B200 has 148: also valid on one
    setters = {"cta_pair": lib.ngram_embed_plan_set_cta_pair, "stream_k": lib.ngram_embed_plan_set_stream_k,
               "tile_n": lib.ngram_embed_plan_set_tile_n, "dense_a": lib.ngram_embed_plan_set_dense_a,
               "pair_wide": lib.ngram_embed_plan_set_pair_wide,
               "pair_columns": lib.ngram_embed_plan_set_pair_columns}
    for k, v in knobs.items():
        assert setters[k](h, v) == 0
    assert lib.ngram_embed_plan_kernel_form(h, T) == form
    lib.ngram_embed_plan_destroy(h)


def test_sm_count_sizes_the_stream_k_workspace(ne):
    """Two fp32 partial tiles per SM the plan uses, of 128 x 512 (the widest tile its
    stream-K schedules split: D = 2048 admits the 512-column pair tiles); 0 restores the
    device's count (none here: no partial tiles, no stream-K, no automatic 512-column
    tiles)."""
    import torch
    lib = ne._lib
    rc, h = _create(ne)
    assert rc == 0
    if torch.cuda.is_available():
        pytest.skip("0 restores the device's own count: checked without a device")
    base = lib.ngram_embed_workspace_bytes(h, 1000)
    assert lib.ngram_embed_plan_set_sm_count(h, 1) == -1 and lib.ngram_embed_plan_set_sm_count(h, -3) == -1
    assert lib.ngram_embed_plan_set_sm_count(h, 148) == 0
    assert lib.ngram_embed_workspace_bytes(h, 1000) == base + 2 * 148 * 128 * 512 * 4
    assert lib.ngram_embed_plan_set_sm_count(h, 40) == 0
    assert lib.ngram_embed_workspace_bytes(h, 1000) == base + 2 * 40 * 128 * 512 * 4
    assert lib.ngram_embed_plan_kernel_form(h, 32768) == 4
    assert lib.ngram_embed_plan_set_sm_count(h, 0) == 0
    assert lib.ngram_embed_workspace_bytes(h, 1000) == base
    assert lib.ngram_embed_plan_kernel_form(h, 32768) == 3
    lib.ngram_embed_plan_destroy(h)


def test_next_row_entry_points_validate_on_the_host(ne):
    """Backward, draft cache, fused decode step, amplification and hash statistics reject
    bad arguments on the host, before any device work (no device is needed to check)."""
    lib = ne._lib
    rc, h = _create(ne)  # bf16, D = 2048, N = 3, K = 2: S = 4
    assert rc == 0
    ws, big = ctypes.c_void_p(0x10000), ctypes.c_size_t(1 << 40)
    odd = ctypes.c_void_p(0x10008)  # 8-byte aligned only
    fake = ctypes.c_void_p(0x20000)
    tabs = (ctypes.c_void_p * 4)(*([0x30000] * 4))
    E_nk = ctypes.cast(tabs, ctypes.c_void_p)
    # amplification factor: finite and non-zero
    for bad in (0.0, float("nan"), float("inf"), -float("inf")):
        assert lib.ngram_embed_plan_set_output_scale(h, bad) == -1
    assert lib.ngram_embed_plan_set_output_scale(h, -1.5) == 0 and lib.ngram_embed_plan_set_output_scale(h, 1.0) == 0
    # LayerNorm: eps in [0, 1], sizes, pointers, alignment; nothing to do for 0 rows
    for eps in (-0.1, 2.0, float("nan")):
        assert lib.ngram_embed_layernorm(h, fake, 8, None, None, eps, fake, ws, big, None) == -1
    assert lib.ngram_embed_layernorm(h, fake, -1, None, None, 1e-5, fake, ws, big, None) == -1
    assert lib.ngram_embed_layernorm(h, None, 8, None, None, 1e-5, fake, ws, big, None) == -1
    assert lib.ngram_embed_layernorm(h, odd, 8, None, None, 1e-5, fake, ws, big, None) == -3
    assert lib.ngram_embed_layernorm(h, None, 0, None, None, 1e-5, None, ws, big, None) == 0
    # backward: sizes, workspace, pointers, alignment; nothing to do without outputs or rows
    need = lib.ngram_embed_bwd_workspace_bytes(h, 1000)
    assert need > 0 and lib.ngram_embed_bwd_workspace_bytes(h, -1) == 0
    assert lib.ngram_embed_bwd(h, fake, fake, -1, E_nk, fake, fake, fake, None, None, ws, big, None) == -1
    assert lib.ngram_embed_bwd(h, fake, fake, 1000, E_nk, fake, fake, fake, None, None, ws, need - 1, None) == -4
    assert lib.ngram_embed_bwd(h, fake, fake, 1000, E_nk, fake, fake, fake, None, None, odd, need, None) == -3
    assert lib.ngram_embed_bwd(h, fake, None, 1000, E_nk, fake, fake, fake, None, None, ws, need, None) == -1
    assert lib.ngram_embed_bwd(h, fake, fake, 1000, E_nk, fake, odd, fake, None, None, ws, need, None) == -3
    assert lib.ngram_embed_bwd(h, fake, fake, 0, E_nk, fake, fake, fake, None, None, ws, need, None) == 0
    assert lib.ngram_embed_bwd(h, fake, fake, 1000, E_nk, fake, fake, None, None, None, ws, need, None) == 0
    rc, h32 = _create(ne, V0=1000, D=64, N=3, K=2, V=(4099, 5003, 6007, 7001), dtype=1)
    assert lib.ngram_embed_bwd(h32, fake, fake, 10, E_nk, fake, fake, fake, None, None, ws, big, None) == -2
    lib.ngram_embed_plan_destroy(h32)
    # draft-phase cache
    cache = ne._Cache(0x40000, 0x50000, 0x60000, 8, 256)
    dc = ne._DraftCache(0x70000, 0x80000, 5, 256)
    dneed = lib.ngram_embed_draft_workspace_bytes(h, 1280)
    assert dneed > 0
    assert lib.ngram_draft_cache_reset(h, None, None, 1, ws, big, None) == -1
    assert lib.ngram_draft_cache_reset(h, ctypes.byref(dc), None, 257, ws, big, None) == -1
    assert lib.ngram_draft_cache_reset(h, ctypes.byref(dc), None, 0, ws, big, None) == 0
    args = lambda d, c, n, w: (h, fake, fake, 256, n, fake, E_nk, fake, ctypes.byref(c), None, ctypes.byref(d), fake,
                               None, ws, w, None)
    assert lib.ngram_embed_fwd_draft(*args(dc, cache, 1280, dneed - 1)) == -4
    assert lib.ngram_embed_fwd_draft(*args(dc, cache, 0, dneed)) == 0
    assert lib.ngram_embed_fwd_draft(*args(ne._DraftCache(0x70000, 0x80000, 0, 256), cache, 1280, dneed)) == -1
    assert lib.ngram_embed_fwd_draft(*args(ne._DraftCache(0x70000, 0x80000, 5, 255), cache, 1280, dneed)) == -1
    assert lib.ngram_embed_fwd_draft(*args(ne._DraftCache(0x70000, 0x80008, 5, 256), cache, 1280, dneed)) == -3
    # fused decode step: sequences, cache, commit arguments
    step = lambda ct, stride, cnt, n_seqs, c: (h, ct, stride, cnt, fake, fake, n_seqs, 1280, fake, E_nk, fake, c, None,
                                              fake, ws, big, None)
    assert lib.ngram_embed_fwd_step(*step(fake, 5, fake, 0, ctypes.byref(cache))) == -1
    assert lib.ngram_embed_fwd_step(*step(fake, 5, fake, 256, None)) == -1
    assert lib.ngram_embed_fwd_step(*step(None, 5, fake, 256, ctypes.byref(cache))) == -1
    assert lib.ngram_embed_fwd_step(*step(fake, 0, fake, 256, ctypes.byref(cache))) == -1
    lib.ngram_embed_plan_destroy(h)
    # hash statistics (no plan): n-gram order, V0, moduli, workspace
    moduli = (ctypes.c_int64 * 2)(1009, 262147)
    hits, distinct = (ctypes.c_int64 * 2)(), ctypes.c_int64()
    sneed = lib.ngram_hash_stats_workspace_bytes(1000, 262147, 2)
    assert sneed > 0 and lib.ngram_hash_stats_workspace_bytes(-1, 10, 1) == 0
    assert lib.ngram_hash_stats_workspace_bytes(10, 0, 1) == 0 and lib.ngram_hash_stats_workspace_bytes(10, 10, 0) == 0
    st = lambda V0, n, mod, nm, w, wb: lib.ngram_hash_stats(V0, n, fake, fake, 4, 1000, mod, nm, hits,
                                                          ctypes.byref(distinct), w, wb, None)
    assert st(0, 2, moduli, 2, ws, sneed) == -1 and st(1 << 31, 2, moduli, 2, ws, sneed) == -1
    assert st(131072, 0, moduli, 2, ws, sneed) == -1 and st(131072, 9, moduli, 2, ws, sneed) == -1
    assert st(131072, 2, moduli, 0, ws, sneed) == -1
    assert st(131072, 2, (ctypes.c_int64 * 2)(1009, 0), 2, ws, sneed) == -1
    assert st(131072, 2, moduli, 2, odd, sneed) == -3 and st(131072, 2, moduli, 2, ws, sneed - 1) == -4
