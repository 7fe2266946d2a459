"""Shared test plumbing: oracle expectations for sampled rows and the tolerance check.

Inputs come only from `synth`; expected values come only from `oracle`.
"""
from __future__ import annotations

import numpy as np

import oracle
from synth import gen
from synth.configs import NgramConfig
from synth.tables import device_tables, host_rows, host_tables, host_W, to_device  # noqa: F401

# Output tolerance vs the fp64 oracle (bf16 tables, fp32 accumulation, bf16 output).
MAX_ABS_TOL = 2e-2
REL_L2_TOL = 5e-3


def to_host_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def oracle_rows(cfg: NgramConfig, tokens, seq_offsets, rows, W_host, histories=None):
    """fp64 oracle output for the given token positions only, regenerating just the table
    rows they touch: context -> Eq. 2 indices -> row lookup -> Eq. 3."""
    rows = np.asarray(rows, dtype=np.int64)
    win = oracle.context_windows(cfg.N, tokens, seq_offsets, histories=histories)[rows]
    idx = oracle.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk, win) if cfg.S else np.zeros((len(rows), 0), np.int32)
    e0 = host_rows(cfg, gen.TAG_E0, np.asarray(tokens)[rows], cfg.D, cfg.e_std)
    sub = (np.stack([host_rows(cfg, gen.TAG_SUBTABLE0 + s, idx[:, s], cfg.d, cfg.e_std) for s in range(cfg.S)],
                    axis=1) if cfg.S else np.zeros((len(rows), 0, 0), e0.dtype))
    return oracle.combine(cfg.D, cfg.S, e0, sub, W_host if cfg.S else np.zeros(1, e0.dtype))


def assert_close(got: np.ndarray, want: np.ndarray, max_abs=MAX_ABS_TOL, rel_l2=REL_L2_TOL, what=""):
    err = got.astype(np.float64) - want
    ma = float(np.abs(err).max()) if err.size else 0.0
    denom = float(np.linalg.norm(want))
    rl = float(np.linalg.norm(err) / denom) if denom > 0 else float(np.linalg.norm(err))
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max|err|={ma:.3e} (<= {max_abs}), rel-L2={rl:.3e} (<= {rel_l2})"
    return ma, rl
