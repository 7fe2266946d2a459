"""Python binding of libngram_embed.so (the C ABI in include/ngram_embed.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. Tensors are torch CUDA tensors (PyTorch provides device memory and
streams); the binding passes their device pointers and sizes, checks the
return code and raises `NgramError` on failure. Importing this module fails
loudly if the library has not been built (`python -m
hashed_gram_embedding_horner_b200.build`); there is no fallback.

Names follow the C ABI. The layer is the hashed N-gram embedding of
"Scaling Embeddings Outperforms Scaling Experts in Language Models", section 2
(Eq. 2, Eq. 3), with the decode-side N-gram cache of section 4.2.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libngram_embed.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m hashed_gram_embedding_horner_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)
_P = ctypes.c_void_p
_I32, _I64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t

NGRAM_BF16, NGRAM_F32 = 0, 1
STATUS_BITS = {
    0x1: "BAD_TOKEN", 0x2: "BAD_OFFSETS", 0x4: "BAD_SLOT", 0x8: "BAD_APPEND",
    0x10: "BAD_ROLLBACK", 0x20: "EVICTED", 0x40: "TIMEOUT",
}
VARIANT_AUTO, VARIANT_TC_TMA_ROWS, VARIANT_TC_SPLIT_ROWS, VARIANT_SIMT = 0, 1, 2, 3

EXPORTED = [
    "ngram_embed_plan_create", "ngram_embed_plan_destroy", "ngram_embed_workspace_bytes",
    "ngram_embed_fwd", "ngram_hash_indices", "ngram_embed_project", "ngram_embed_gather",
    "ngram_cache_reset", "ngram_cache_append", "ngram_cache_rollback", "ngram_embed_get_status",
    "ngram_embed_clear_status", "ngram_embed_error_string", "ngram_embed_plan_uses_tensor_cores",
    "ngram_embed_plan_set_variant", "ngram_embed_plan_set_tile_n", "ngram_embed_plan_set_tma_rows",
    "ngram_embed_selftest_wait_timeout", "ngram_embed_fwd_static_ws", "ngram_embed_plan_set_cta_pair",
    "ngram_cache_commit", "ngram_embed_plan_set_stream_k", "ngram_embed_plan_set_pdl",
    "ngram_embed_plan_set_a_stages", "ngram_embed_plan_kernel_form", "ngram_embed_plan_set_pair_wide",
    "ngram_embed_plan_set_sm_count",
    "ngram_embed_plan_set_output_scale", "ngram_embed_layernorm",
    "ngram_embed_bwd_workspace_bytes", "ngram_embed_bwd",
    "ngram_hash_stats_workspace_bytes", "ngram_hash_stats",
    "ngram_draft_cache_reset", "ngram_embed_draft_workspace_bytes", "ngram_embed_fwd_draft",
    "ngram_embed_fwd_step", "ngram_embed_plan_set_dense_a", "ngram_embed_plan_set_pair_columns",
    "ngram_embed_plan_set_fused_step", "ngram_embed_plan_set_backward_pair",
    "ngram_embed_plan_set_backward_streams",
]


class _Config(ctypes.Structure):
    _fields_ = [("V0", _I64), ("D", _I32), ("N", _I32), ("K", _I32), ("V_nk", ctypes.POINTER(_I64)),
                ("dtype", _I32)]


class _Cache(ctypes.Structure):
    _fields_ = [("ring", _P), ("len", _P), ("valid_from", _P), ("capacity", _I32), ("max_seqs", _I32)]


class _DraftCache(ctypes.Structure):
    _fields_ = [("keys", _P), ("emb", _P), ("positions", _I32), ("max_seqs", _I32)]


def _sig(name, args, res=ctypes.c_int):
    f = getattr(_lib, name)
    f.argtypes, f.restype = args, res


_sig("ngram_embed_plan_create", [ctypes.POINTER(_Config), ctypes.POINTER(_P)])
_sig("ngram_embed_plan_destroy", [_P])
_sig("ngram_embed_workspace_bytes", [_P, _I64], _SZ)
_sig("ngram_embed_fwd", [_P, _P, _P, _I32, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ, _P])
_sig("ngram_hash_indices", [_P, _P, _P, _I32, _I64, _P, _P, _P, _P, _SZ, _P])
_sig("ngram_embed_project", [_P, _P, _P, _I64, _P, _P, _P, _P, _P, _SZ, _P])
_sig("ngram_embed_gather", [_P, _P, _I64, _P, _P, _P, _P, _P, _P, _SZ, _P])
_sig("ngram_cache_reset", [_P, _P, _P, _I32, _P, _SZ, _P])
_sig("ngram_cache_append", [_P, _P, _P, _P, _P, _I32, _P, _SZ, _P])
_sig("ngram_cache_rollback", [_P, _P, _P, _P, _I32, _P, _SZ, _P])
_sig("ngram_cache_commit", [_P, _P, _P, _P, _I32, _P, _I32, _P, _SZ, _P])
_sig("ngram_embed_get_status", [_P, _P, ctypes.POINTER(_I32)])
_sig("ngram_embed_clear_status", [_P, _P])
_sig("ngram_embed_error_string", [ctypes.c_int], ctypes.c_char_p)
_sig("ngram_embed_plan_uses_tensor_cores", [_P])
_sig("ngram_embed_plan_set_variant", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_tile_n", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_tma_rows", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_cta_pair", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_pair_wide", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_dense_a", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_pair_columns", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_backward_pair", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_backward_streams", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_fused_step", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_sm_count", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_stream_k", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_pdl", [_P, ctypes.c_int])
_sig("ngram_embed_plan_set_a_stages", [_P, ctypes.c_int])
_sig("ngram_embed_plan_kernel_form", [_P, _I64])
_sig("ngram_embed_plan_set_output_scale", [_P, ctypes.c_float])
_sig("ngram_embed_bwd_workspace_bytes", [_P, _I64], _SZ)
_sig("ngram_hash_stats_workspace_bytes", [_I64, _I64, ctypes.c_int], _SZ)
_sig("ngram_draft_cache_reset", [_P, _P, _P, _I32, _P, _SZ, _P])
_sig("ngram_embed_fwd_step", [_P, _P, _I32, _P, _P, _P, _I32, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ, _P])
_sig("ngram_embed_draft_workspace_bytes", [_P, _I64], _SZ)
_sig("ngram_embed_fwd_draft", [_P, _P, _P, _I32, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P])
_sig("ngram_hash_stats", [_I64, ctypes.c_int, _P, _P, _I32, _I64, _P, ctypes.c_int, _P, _P, _P, _SZ, _P])
_sig("ngram_embed_bwd", [_P, _P, _P, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ, _P])
_sig("ngram_embed_layernorm", [_P, _P, _I64, _P, _P, ctypes.c_float, _P, _P, _SZ, _P])
_sig("ngram_embed_selftest_wait_timeout", [_P, _I64, _P])
_sig("ngram_embed_fwd_static_ws", [_P, _P, _P, _I32, _I64, _P, _P, _P, _P, _P, _P, _P, _P])


class NgramError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != 0:
        raise NgramError(f"{what}: {_lib.ngram_embed_error_string(rc).decode()} ({rc})")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _i32(t, name):
    import torch
    if t is not None and (t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous()):
        raise NgramError(f"{name} must be a contiguous int32 CUDA tensor")
    return _ptr(t)


class Plan:
    """Host-side plan for one layer shape (owns the C plan)."""

    def __init__(self, handle, V0, D, N, K, V_nk, dtype):
        self.handle, self.V0, self.D, self.N, self.K = handle, V0, D, N, K
        self.V_nk, self.dtype = tuple(V_nk), dtype
        self.S = (N - 1) * K
        self.d = D // self.S if self.S else 0

    def __del__(self):
        h = getattr(self, "handle", None)
        lib = _lib  # None once the module is torn down at interpreter exit
        if h and lib is not None:
            lib.ngram_embed_plan_destroy(h)
            self.handle = None


class Cache:
    """The N-gram cache arrays (caller-owned torch tensors): ring int32 [max_seqs, C],
    len int64 [max_seqs], valid_from int64 [max_seqs]."""

    def __init__(self, ring, length, valid_from):
        self.ring, self.len, self.valid_from = ring, length, valid_from
        self.struct = _Cache(ring.data_ptr(), length.data_ptr(), valid_from.data_ptr(), ring.shape[1],
                             ring.shape[0])

    @classmethod
    def empty(cls, max_seqs: int, capacity: int, device="cuda"):
        import torch
        return cls(torch.zeros((max_seqs, capacity), dtype=torch.int32, device=device),
                   torch.zeros(max_seqs, dtype=torch.int64, device=device),
                   torch.zeros(max_seqs, dtype=torch.int64, device=device))


class DraftCache:
    """Draft-phase embedding cache (caller-owned torch tensors): keys int32
    [max_seqs, positions, N], emb [max_seqs, positions, D] in the plan's dtype."""

    def __init__(self, keys, emb):
        self.keys, self.emb = keys, emb
        self.struct = _DraftCache(keys.data_ptr(), emb.data_ptr(), keys.shape[1], keys.shape[0])

    @classmethod
    def empty(cls, plan: "Plan", max_seqs: int, positions: int, device="cuda"):
        import torch
        dt = torch.bfloat16 if plan.dtype == NGRAM_BF16 else torch.float32
        return cls(torch.full((max_seqs, positions, plan.N), -1, dtype=torch.int32, device=device),
                   torch.zeros((max_seqs, positions, plan.D), dtype=dt, device=device))


def ngram_embed_fwd_step(plan: "Plan", tokens, seq_offsets, E0, E_nk, W_stacked, out, workspace, cache: "Cache",
                         commit_tokens=None, commit_stride: int = 0, commit_counts=None, cache_slots=None,
                         stream=None):
    """Commit the previous step's accepted ids (if commit_counts is given), then the layer
    for this step's ids through the N-gram cache: two launches."""
    tabs = _tables(E_nk)
    rc = _lib.ngram_embed_fwd_step(plan.handle, _i32(commit_tokens, "commit_tokens"), int(commit_stride),
                                   _i32(commit_counts, "commit_counts"), _i32(tokens, "tokens"),
                                   _i32(seq_offsets, "seq_offsets"), seq_offsets.numel() - 1, tokens.numel(),
                                   _ptr(E0), tabs, _ptr(W_stacked), ctypes.byref(cache.struct),
                                   _i32(cache_slots, "cache_slots"), _ptr(out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_embed_fwd_step")


def ngram_draft_cache_reset(plan: "Plan", dc: DraftCache, workspace, slots=None, stream=None):
    n = slots.numel() if slots is not None else dc.keys.shape[0]
    rc = _lib.ngram_draft_cache_reset(plan.handle, ctypes.byref(dc.struct), _i32(slots, "slots"), n, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_draft_cache_reset")


def new_draft_workspace(plan: "Plan", max_tokens: int, device="cuda"):
    import torch
    return torch.zeros(_lib.ngram_embed_draft_workspace_bytes(plan.handle, int(max_tokens)), dtype=torch.uint8,
                       device=device)


def ngram_embed_fwd_draft(plan: "Plan", tokens, seq_offsets, E0, E_nk, W_stacked, out, workspace, cache: "Cache",
                          dc: DraftCache, hits=None, cache_slots=None, stream=None):
    """The layer through the N-gram cache and the draft-phase embedding cache."""
    tabs = _tables(E_nk)
    rc = _lib.ngram_embed_fwd_draft(plan.handle, _i32(tokens, "tokens"), _i32(seq_offsets, "seq_offsets"),
                                    seq_offsets.numel() - 1, tokens.numel(), _ptr(E0), tabs, _ptr(W_stacked),
                                    ctypes.byref(cache.struct), _i32(cache_slots, "cache_slots"),
                                    ctypes.byref(dc.struct), _ptr(out), _i32(hits, "hits"), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_embed_fwd_draft")


def ngram_embed_plan_create(V0: int, D: int, N: int, K: int, V_nk, dtype: int = NGRAM_BF16) -> Plan:
    S = (N - 1) * K
    arr = (_I64 * max(S, 1))(*[int(v) for v in V_nk])
    cfg = _Config(V0, D, N, K, ctypes.cast(arr, ctypes.POINTER(_I64)), dtype)
    h = _P()
    _check(_lib.ngram_embed_plan_create(ctypes.byref(cfg), ctypes.byref(h)), "ngram_embed_plan_create")
    return Plan(h, V0, D, N, K, V_nk, dtype)


def ngram_embed_plan_set_variant(plan: Plan, variant: int):
    _check(_lib.ngram_embed_plan_set_variant(plan.handle, variant), "ngram_embed_plan_set_variant")


def ngram_embed_plan_set_tile_n(plan: Plan, tile_n: int):
    _check(_lib.ngram_embed_plan_set_tile_n(plan.handle, tile_n), "ngram_embed_plan_set_tile_n")


def ngram_embed_plan_set_tma_rows(plan: Plan, rows: int):
    _check(_lib.ngram_embed_plan_set_tma_rows(plan.handle, rows), "ngram_embed_plan_set_tma_rows")


def ngram_embed_plan_set_cta_pair(plan: Plan, on):
    """True/1: CTA pairs; False/0: one CTA per tile; None/-1: automatic (default)."""
    v = -1 if on is None or on == -1 else int(bool(on))
    _check(_lib.ngram_embed_plan_set_cta_pair(plan.handle, v), "ngram_embed_plan_set_cta_pair")


def ngram_embed_plan_set_pair_wide(plan: Plan, on):
    """True/1: the pair form's 512-column tiles; False/0: 256-column; None/-1: automatic."""
    v = -1 if on is None or on == -1 else int(bool(on))
    _check(_lib.ngram_embed_plan_set_pair_wide(plan.handle, v), "ngram_embed_plan_set_pair_wide")


def ngram_embed_plan_set_fused_step(plan: Plan, on: bool):
    """ngram_embed_fwd_step in one launch where the one-CTA form runs it (default False)."""
    _check(_lib.ngram_embed_plan_set_fused_step(plan.handle, int(bool(on))), "ngram_embed_plan_set_fused_step")


def ngram_embed_plan_set_pair_columns(plan: Plan, on):
    """True/1: the pair form over column ranges whenever possible; False/0: never; None/-1: automatic."""
    v = -1 if on is None or on == -1 else int(bool(on))
    _check(_lib.ngram_embed_plan_set_pair_columns(plan.handle, v), "ngram_embed_plan_set_pair_columns")


def ngram_embed_plan_set_backward_pair(plan: Plan, mode):
    """The backward's GEMMs: True/1 CTA pairs with 256-column tiles (default); 2 pairs with
    512-column tiles where D allows; False/0 one CTA per 128-row tile."""
    _check(_lib.ngram_embed_plan_set_backward_pair(plan.handle, int(mode)), "ngram_embed_plan_set_backward_pair")


def ngram_embed_plan_set_backward_streams(plan: Plan, on: bool):
    """True (default): the backward's memory-bound kernels overlap its dG GEMM on the plan's
    auxiliary stream; False: everything on the caller's stream."""
    _check(_lib.ngram_embed_plan_set_backward_streams(plan.handle, int(bool(on))),
           "ngram_embed_plan_set_backward_streams")


def ngram_embed_plan_set_sm_count(plan: Plan, sms: int):
    """SMs the plan's kernels use: 0 = all of the device's; else 2 .. the device's count."""
    _check(_lib.ngram_embed_plan_set_sm_count(plan.handle, int(sms)), "ngram_embed_plan_set_sm_count")


def ngram_embed_plan_set_stream_k(plan: Plan, mode: int):
    """0 automatic, 1 stream-K whenever the workspace and shape allow it, 2 never."""
    _check(_lib.ngram_embed_plan_set_stream_k(plan.handle, int(mode)), "ngram_embed_plan_set_stream_k")


def ngram_embed_plan_set_a_stages(plan: Plan, stages: int):
    """Depth of the one-CTA kernel's A ring (0 = default); the W ring takes the rest."""
    _check(_lib.ngram_embed_plan_set_a_stages(plan.handle, int(stages)), "ngram_embed_plan_set_a_stages")


def ngram_embed_plan_set_output_scale(plan: Plan, scale: float):
    """Embedding amplification by a constant, folded into the epilogue (default 1)."""
    _check(_lib.ngram_embed_plan_set_output_scale(plan.handle, float(scale)), "ngram_embed_plan_set_output_scale")


def ngram_embed_layernorm(plan: Plan, x, y, workspace, gamma=None, beta=None, eps: float = 1e-5, stream=None):
    """Row LayerNorm of a [T, D] layer output (y may be x)."""
    rc = _lib.ngram_embed_layernorm(plan.handle, _ptr(x), x.shape[0], _ptr(gamma), _ptr(beta), float(eps), _ptr(y),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_embed_layernorm")


def new_bwd_workspace(plan: Plan, max_tokens: int, device="cuda"):
    """A zeroed uint8 workspace tensor of ngram_embed_bwd_workspace_bytes(plan, max_tokens)."""
    import torch
    return torch.zeros(_lib.ngram_embed_bwd_workspace_bytes(plan.handle, int(max_tokens)), dtype=torch.uint8,
                       device=device)


def ngram_embed_bwd(plan: Plan, tokens, idx, grad_out, workspace, E_nk=None, W_stacked=None, dE0=None, dE_nk=None,
                    dW=None, stream=None):
    """Accumulate the layer's parameter gradients (fp32 tensors, += semantics) from
    grad_out = dL/de and the forward's indices. Pass None to skip a gradient."""
    tabs = _tables(E_nk) if E_nk is not None else None
    grads = (ctypes.c_void_p * len(dE_nk))(*[t.data_ptr() for t in dE_nk]) if dE_nk is not None else None
    rc = _lib.ngram_embed_bwd(plan.handle, _i32(tokens, "tokens"), _i32(idx, "idx"), tokens.numel(), tabs,
                              _ptr(W_stacked), _ptr(grad_out), _ptr(dE0), grads, _ptr(dW), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_embed_bwd")


def ngram_hash_stats(V0: int, n: int, tokens, seq_offsets, moduli, workspace=None, stream=None):
    """Hit counts and collisions of the n-gram hash X_n mod V for each V in `moduli`:
    returns (distinct_ngrams, [rows_hit per modulus])."""
    import torch
    mods = (_I64 * len(moduli))(*[int(v) for v in moduli])
    hits = (_I64 * len(moduli))()
    dist = _I64()
    need = _lib.ngram_hash_stats_workspace_bytes(tokens.numel(), max(int(v) for v in moduli), len(moduli))
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=tokens.device)
    rc = _lib.ngram_hash_stats(int(V0), int(n), _i32(tokens, "tokens"), _i32(seq_offsets, "seq_offsets"),
                               seq_offsets.numel() - 1, tokens.numel(), mods, len(moduli), hits, ctypes.byref(dist),
                               _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_hash_stats")
    return (None if dist.value < 0 else int(dist.value)), [int(h) for h in hits]


KERNEL_FORMS = {0: "cuda_cores", 1: "one_cta", 2: "one_cta_stream_k", 3: "cta_pair", 4: "cta_pair_wide",
                5: "cta_pair_stream_k", 6: "cta_pair_dense", 7: "cta_pair_dense_stream_k", 8: "cta_pair_wide_dense",
                9: "cta_pair_wide_stream_k", 10: "cta_pair_columns",
                11: "cta_pair_columns_dense"}


def ngram_embed_plan_set_dense_a(plan: "Plan", mode: int):
    """Dense-A form (sub-rows gathered into G first, A by dense TMA): 1 on, 0 off (default)."""
    _check(_lib.ngram_embed_plan_set_dense_a(plan.handle, int(mode)), "ngram_embed_plan_set_dense_a")


def ngram_embed_plan_kernel_form(plan: Plan, num_tokens: int) -> str:
    """Which projection kernel a call of num_tokens tokens runs (with a full-size workspace)."""
    rc = _lib.ngram_embed_plan_kernel_form(plan.handle, int(num_tokens))
    _check(min(rc, 0), "ngram_embed_plan_kernel_form")
    return KERNEL_FORMS[rc]


def ngram_embed_plan_set_pdl(plan: Plan, on: bool):
    """Launch the plan's kernels as programmatic dependent launches (default off)."""
    _check(_lib.ngram_embed_plan_set_pdl(plan.handle, int(bool(on))), "ngram_embed_plan_set_pdl")


def ngram_embed_plan_uses_tensor_cores(plan: Plan) -> bool:
    return bool(_lib.ngram_embed_plan_uses_tensor_cores(plan.handle))


def ngram_embed_workspace_bytes(plan: Plan, max_tokens: int) -> int:
    return int(_lib.ngram_embed_workspace_bytes(plan.handle, max_tokens))


def _tables(E_nk):
    arr = (_P * max(len(E_nk), 1))(*[t.data_ptr() for t in E_nk])
    return arr


def ngram_embed_fwd(plan: Plan, tokens, seq_offsets, E0, E_nk, W_stacked, out, workspace,
                    cache: Cache | None = None, cache_slots=None, stream=None):
    tabs = _tables(E_nk)
    rc = _lib.ngram_embed_fwd(plan.handle, _i32(tokens, "tokens"), _i32(seq_offsets, "seq_offsets"),
                              seq_offsets.numel() - 1, tokens.numel(), _ptr(E0), tabs, _ptr(W_stacked),
                              ctypes.byref(cache.struct) if cache else None, _i32(cache_slots, "cache_slots"),
                              _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream))
    _check(rc, "ngram_embed_fwd")


def ngram_hash_indices(plan: Plan, tokens, seq_offsets, idx_out, workspace, cache: Cache | None = None,
                       cache_slots=None, stream=None):
    rc = _lib.ngram_hash_indices(plan.handle, _i32(tokens, "tokens"), _i32(seq_offsets, "seq_offsets"),
                                 seq_offsets.numel() - 1, tokens.numel(),
                                 ctypes.byref(cache.struct) if cache else None,
                                 _i32(cache_slots, "cache_slots"), _i32(idx_out, "idx_out"), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_hash_indices")


def ngram_embed_project(plan: Plan, tokens, idx, E0, E_nk, W_stacked, out, workspace, stream=None):
    tabs = _tables(E_nk)
    rc = _lib.ngram_embed_project(plan.handle, _i32(tokens, "tokens"), _i32(idx, "idx"), tokens.numel(),
                                  _ptr(E0), tabs, _ptr(W_stacked), _ptr(out), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_embed_project")


def ngram_embed_gather(plan: Plan, idx, E_nk, G_out, workspace, tokens=None, E0=None, E0_out=None, stream=None):
    """Sub-rows E_s[idx[i, s]] into G_out [T x D]; with E0_out, also E_0[tokens[i]] rows."""
    tabs = _tables(E_nk)
    if E0_out is not None and (tokens is None or E0 is None):
        raise ValueError("E0_out needs tokens and E0")
    rc = _lib.ngram_embed_gather(plan.handle, _i32(idx, "idx"), idx.shape[0], tabs, _ptr(G_out),
                                 None if tokens is None else _i32(tokens, "tokens"),
                                 None if E0 is None else _ptr(E0), None if E0_out is None else _ptr(E0_out),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_embed_gather")


def ngram_cache_reset(plan: Plan, cache: Cache, workspace, slots=None, n=None, stream=None):
    n = cache.struct.max_seqs if slots is None and n is None else (slots.numel() if n is None else n)
    rc = _lib.ngram_cache_reset(plan.handle, ctypes.byref(cache.struct), _i32(slots, "slots"), n,
                                _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_cache_reset")


def ngram_cache_append(plan: Plan, cache: Cache, tokens, tok_offsets, workspace, slots=None, stream=None):
    rc = _lib.ngram_cache_append(plan.handle, ctypes.byref(cache.struct), _i32(slots, "slots"),
                                 _i32(tokens, "tokens"), _i32(tok_offsets, "tok_offsets"), tok_offsets.numel() - 1,
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_cache_append")


def ngram_cache_commit(plan: Plan, cache: Cache, tokens, stride: int, counts, workspace, slots=None, stream=None):
    rc = _lib.ngram_cache_commit(plan.handle, ctypes.byref(cache.struct), _i32(slots, "slots"),
                                 _i32(tokens, "tokens"), stride, _i32(counts, "counts"), counts.numel(),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_cache_commit")


def ngram_cache_rollback(plan: Plan, cache: Cache, counts, workspace, slots=None, stream=None):
    rc = _lib.ngram_cache_rollback(plan.handle, ctypes.byref(cache.struct), _i32(slots, "slots"),
                                   _i32(counts, "counts"), counts.numel(), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ngram_cache_rollback")


def ngram_embed_get_status(workspace, stream=None) -> int:
    v = _I32(0)
    _check(_lib.ngram_embed_get_status(_ptr(workspace), _stream(stream), ctypes.byref(v)), "ngram_embed_get_status")
    return int(v.value)


def ngram_embed_clear_status(workspace, stream=None):
    _check(_lib.ngram_embed_clear_status(_ptr(workspace), _stream(stream)), "ngram_embed_clear_status")


def ngram_embed_selftest_wait_timeout(workspace, limit_ns: int, stream=None):
    _check(_lib.ngram_embed_selftest_wait_timeout(_ptr(workspace), limit_ns, _stream(stream)),
           "ngram_embed_selftest_wait_timeout")


def status_names(status: int):
    return [name for bit, name in STATUS_BITS.items() if status & bit]


def new_workspace(plan: Plan, max_tokens: int, device="cuda"):
    """A zeroed uint8 workspace tensor of ngram_embed_workspace_bytes(plan, max_tokens)."""
    import torch
    n = ngram_embed_workspace_bytes(plan, max_tokens)
    return torch.zeros(n, dtype=torch.uint8, device=device)
