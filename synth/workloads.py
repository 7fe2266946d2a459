"""Token streams for the five workloads (host arrays, int32).

Prefill: `prefill_tokens(cfg)` -> (tokens[T], seq_offsets[B + 1]).
Decode:  `DecodeStream(cfg)` yields, per step, 5 in-step ids per sequence
(x0 = the step's first token, then 4 draft ids) and one accept length
a in {0..4}; before the first step each sequence gets a seeded prompt of
0..prompt_max ids so both the pad and the history context paths run.
"""
from __future__ import annotations

import numpy as np

from . import gen
from .configs import NgramConfig


def _draw_tokens(cfg: NgramConfig, n: int, tag: int, offset: int = 0) -> np.ndarray:
    if cfg.token_dist == "uniform":
        return gen.uniform_tokens(cfg.seed, n, cfg.V0, tag=tag, offset=offset)
    return gen.zipf_tokens(cfg.seed, n, cfg.V0, cfg.zipf_alpha, tag=tag, offset=offset)


def prefill_lengths(cfg: NgramConfig) -> np.ndarray:
    if cfg.seq_len:
        return np.full(cfg.num_seqs, cfg.seq_len, dtype=np.int32)
    x = cfg.extras
    # one length-1 and one length-(N-2) sequence, so contexts that are all pad
    # (or all pad but one id) are part of the workload.
    return gen.varlen_lengths(cfg.seed, cfg.num_seqs, x["total_tokens"], x["len_lo"],
                              x["len_hi"], fixed=(1, max(cfg.N - 2, 1)))


def prefill_tokens(cfg: NgramConfig):
    lengths = prefill_lengths(cfg)
    offsets = gen.offsets_from_lengths(lengths)
    tokens = _draw_tokens(cfg, int(offsets[-1]), gen.TAG_TOKENS)
    return tokens, offsets


class DecodeStream:
    """Seeded speculative-decode workload: prompts, per-step ids and accept lengths."""

    def __init__(self, cfg: NgramConfig, num_seqs: int | None = None):
        self.cfg = cfg
        self.B = num_seqs or cfg.num_seqs
        self.P = cfg.tokens_per_step

    def prompts(self):
        """(ids, offsets[B + 1]): a prompt of 0..prompt_max ids per sequence."""
        u = gen.uniform01(self.cfg.seed, gen.TAG_PROMPT_LEN, self.B)
        lens = np.floor(u * (self.cfg.prompt_max + 1)).astype(np.int32)
        off = gen.offsets_from_lengths(lens)
        ids = _draw_tokens(self.cfg, int(off[-1]), gen.TAG_TOKENS + 1)
        return ids, off

    def step_tokens(self, step: int) -> np.ndarray:
        """[B * P] in-step ids, sequence-major (sequence b owns [b * P, (b + 1) * P))."""
        n = self.B * self.P
        return _draw_tokens(self.cfg, n, gen.TAG_TOKENS + 2, offset=step * n)

    def step_offsets(self) -> np.ndarray:
        return (np.arange(self.B + 1, dtype=np.int32) * self.P).astype(np.int32)

    def accept_lengths(self, step: int) -> np.ndarray:
        """[B] accept lengths a in {0 .. P - 1}: the step commits 1 + a ids."""
        u = gen.uniform01(self.cfg.seed, gen.TAG_ACCEPT, self.B, offset=step * self.B)
        return np.floor(u * self.P).astype(np.int32)
