"""ngram_embed_fwd_static_ws: the forward pass for callers that cannot allocate device
memory (plugin hosts that hand a layer only its inputs and outputs, or loops where
cudaMalloc's device-wide synchronisation is not allowed). Its workspace is a fixed array
inside the library, so the caller passes only inputs and outputs.

Checked through the C ABI against ngram_embed_fwd (caller-provided workspace) on two
calls in a row: the same kernels run on the same inputs, so the bits must be equal (which
also puts them within the tolerance the other parity tests use). Also covered: the stream-K
schedule running inside the fixed array (a plan limited to 8 SMs, whose partial tiles fit),
and the status word that each call clears and reports through status_out. This file is
collected last so that a failure here comes after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

from synth import configs, gen
from synth.tables import host_tables, to_device

pytestmark = pytest.mark.gpu

MAX_ABS_TOL, REL_L2_TOL = 2e-2, 5e-3


@pytest.fixture(scope="module")
def ne():
    import hashed_gram_embedding_horner_b200 as m
    return m


def _close(a: torch.Tensor, b: torch.Tensor):
    a64, b64 = a.double().cpu().numpy(), b.double().cpu().numpy()
    err = a64 - b64
    assert np.abs(err).max() <= MAX_ABS_TOL
    assert np.linalg.norm(err) <= REL_L2_TOL * np.linalg.norm(b64)


def _static_ws_fwd(ne, plan, tokens, offsets, E0, E, W, out, status):
    tabs = (ctypes.c_void_p * len(E))(*[t.data_ptr() for t in E])
    return ne._lib.ngram_embed_fwd_static_ws(
        plan.handle, ctypes.c_void_p(tokens.data_ptr()), ctypes.c_void_p(offsets.data_ptr()),
        offsets.numel() - 1, tokens.numel(), ctypes.c_void_p(E0.data_ptr()), tabs, ctypes.c_void_p(W.data_ptr()),
        None, None, ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_workspace_forward_matches_fwd(ne):
    cfg = configs.NgramConfig(name="noalloc", V0=6000, D=512, N=5, K=2,
                              V_nk=tuple(configs.primes_from(20000, 8)), dtype="bf16", seed=5)
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call, lengths in enumerate(([3, 200, 97], [130, 1, 0, 300])):   # two calls in a row
        off_h = gen.offsets_from_lengths(lengths)
        tokens = torch.from_numpy(gen.zipf_tokens(40 + call, int(off_h[-1]), cfg.V0)).cuda()
        offsets = torch.from_numpy(off_h).cuda()
        want = torch.empty((tokens.numel(), cfg.D), dtype=torch.bfloat16, device="cuda")
        ws = ne.new_workspace(plan, tokens.numel())
        ne.ngram_embed_fwd(plan, tokens, offsets, E0, E, W, want, ws)
        got = torch.full_like(want, float("nan"))
        assert _static_ws_fwd(ne, plan, tokens, offsets, E0, E, W, got, status) == 0
        torch.cuda.synchronize()
        assert status.item() == 0
        assert ne.ngram_embed_get_status(ws) == 0
        _close(got, want)
        assert torch.equal(got, want)


def _noalloc_cfg():
    return configs.NgramConfig(name="noalloc", V0=6000, D=512, N=5, K=2,
                               V_nk=tuple(configs.primes_from(20000, 8)), dtype="bf16", seed=5)


@pytest.mark.parametrize("dense_a,wide,form", [(0, 0, "one_cta_stream_k"), (1, -1, "cta_pair_dense_stream_k"),
                                                (0, 1, "cta_pair_wide_stream_k")])
def test_static_workspace_stream_k_matches_fwd(ne, dense_a, wide, form):
    """With 6 SMs the stream-K partial tiles (2 x 6 x 256 KB) fit the fixed array, so the
    schedules whose arrival counters and partials (and, in the dense-A form, the gathered
    sub-rows) live in it run, with tiles split between CTAs or pairs; two calls in a row
    equal ngram_embed_fwd with its own workspace (same schedule) bit for bit."""
    cfg = _noalloc_cfg()
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
    ne.ngram_embed_plan_set_sm_count(plan, 6)
    ne.ngram_embed_plan_set_stream_k(plan, 1)
    ne.ngram_embed_plan_set_dense_a(plan, dense_a)
    ne.ngram_embed_plan_set_pair_wide(plan, wide)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call, lengths in enumerate(([3, 330, 97], [129, 1, 0, 300])):
        off_h = gen.offsets_from_lengths(lengths)
        T = int(off_h[-1])
        assert ne.ngram_embed_plan_kernel_form(plan, T) == form
        assert ne.ngram_embed_workspace_bytes(plan, T) <= 4 << 20  # everything fits the fixed array
        tokens = torch.from_numpy(gen.zipf_tokens(60 + call, T, cfg.V0)).cuda()
        offsets = torch.from_numpy(off_h).cuda()
        want = torch.empty((T, cfg.D), dtype=torch.bfloat16, device="cuda")
        ws = ne.new_workspace(plan, T)
        ne.ngram_embed_fwd(plan, tokens, offsets, E0, E, W, want, ws)
        got = torch.full_like(want, float("nan"))
        assert _static_ws_fwd(ne, plan, tokens, offsets, E0, E, W, got, status) == 0
        torch.cuda.synchronize()
        assert status.item() == 0 and ne.ngram_embed_get_status(ws) == 0
        assert torch.equal(got, want)


def test_static_workspace_reports_and_clears_device_status(ne):
    """A token id outside [0, V0) sets BAD_TOKEN in the call's status (written to status_out);
    the next, clean call starts from a cleared head and reports 0."""
    cfg = _noalloc_cfg()
    E0h, Eh, Wh = host_tables(cfg)
    E0, E, W = to_device(E0h, torch.bfloat16), [to_device(e, torch.bfloat16) for e in Eh], to_device(Wh, torch.bfloat16)
    plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
    off_h = gen.offsets_from_lengths([40, 90])
    tok_h = gen.zipf_tokens(7, int(off_h[-1]), cfg.V0)
    offsets = torch.from_numpy(off_h).cuda()
    out = torch.empty((len(tok_h), cfg.D), dtype=torch.bfloat16, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    bad = tok_h.copy()
    bad[17] = cfg.V0  # one past the last id
    assert _static_ws_fwd(ne, plan, torch.from_numpy(bad).cuda(), offsets, E0, E, W, out, status) == 0
    torch.cuda.synchronize()
    assert ne.status_names(status.item()) == ["BAD_TOKEN"]
    assert _static_ws_fwd(ne, plan, torch.from_numpy(tok_h).cuda(), offsets, E0, E, W, out, status) == 0
    torch.cuda.synchronize()
    assert status.item() == 0


def test_static_workspace_rejects_calls_above_its_size(ne):
    cfg = configs.PREFILL_D4096_VARLEN  # S = 8: 4 MiB holds about 131000 tokens of indices
    plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    tabs = (ctypes.c_void_p * 8)(*([dummy.data_ptr()] * 8))
    too_many = (4 << 20) // (cfg.S * 4) + 1
    rc = ne._lib.ngram_embed_fwd_static_ws(plan.handle, ctypes.c_void_p(dummy.data_ptr()),
                                           ctypes.c_void_p(dummy.data_ptr()), 1, too_many,
                                           ctypes.c_void_p(dummy.data_ptr()), tabs, ctypes.c_void_p(dummy.data_ptr()),
                                           None, None, ctypes.c_void_p(dummy.data_ptr()), None, None)
    assert rc == -4  # NGRAM_ERR_WORKSPACE, nothing launched
