"""Seeded layer tables on the host (numpy) or the device (torch, filled on the GPU).

bf16 tables are uint16 bit patterns on the host and torch.bfloat16 on the device.
E_0 and every E_s draw std e_std; W_stacked draws std 1/sqrt(d) (variance 1/width).
"""
from __future__ import annotations

import numpy as np

from . import gen
from .configs import NgramConfig


def host_rows(cfg: NgramConfig, tag: int, rows, width: int, std: float):
    rows = np.asarray(rows, dtype=np.int64)
    if cfg.dtype == "bf16":
        return gen.table_rows_bf16(cfg.seed, tag, rows, width, std)
    return gen.table_values_f32(cfg.seed, tag, rows, width, std)


def host_tables(cfg: NgramConfig):
    """(E0, [E_s], W) on the host."""
    mk = (lambda tag, rows, width, std: gen.table_bf16(cfg.seed, tag, rows, width, std)) if cfg.dtype == "bf16" \
        else (lambda tag, rows, width, std: gen.table_f32(cfg.seed, tag, rows, width, std))
    E0 = mk(gen.TAG_E0, cfg.V0, cfg.D, cfg.e_std)
    E = [mk(gen.TAG_SUBTABLE0 + s, cfg.V_nk[s], cfg.d, cfg.e_std) for s in range(cfg.S)]
    W = mk(gen.TAG_W, cfg.D, cfg.D, cfg.w_std) if cfg.S else None
    return E0, E, W


def host_W(cfg: NgramConfig):
    if not cfg.S:
        return None
    if cfg.dtype == "bf16":
        return gen.table_bf16(cfg.seed, gen.TAG_W, cfg.D, cfg.D, cfg.w_std)
    return gen.table_f32(cfg.seed, gen.TAG_W, cfg.D, cfg.D, cfg.w_std)


def to_device(a: np.ndarray, dt, device="cuda"):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device, dtype=dt)


def device_tables(cfg: NgramConfig, fill_on_device: bool = True, device="cuda"):
    """(E0, [E_s], W) as torch CUDA tensors, filled by the device generator (default) or
    copied from the host generator."""
    import torch
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    if fill_on_device:
        from . import device as sdev
        E0 = torch.empty((cfg.V0, cfg.D), dtype=dt, device=device)
        sdev.fill_table(E0, cfg.seed, gen.TAG_E0, cfg.e_std)
        E = []
        for s in range(cfg.S):
            t = torch.empty((cfg.V_nk[s], cfg.d), dtype=dt, device=device)
            sdev.fill_table(t, cfg.seed, gen.TAG_SUBTABLE0 + s, cfg.e_std)
            E.append(t)
        W = None
        if cfg.S:
            W = torch.empty((cfg.D, cfg.D), dtype=dt, device=device)
            sdev.fill_table(W, cfg.seed, gen.TAG_W, cfg.w_std)
        return E0, E, W
    E0h, Eh, Wh = host_tables(cfg)
    return (to_device(E0h, dt, device), [to_device(e, dt, device) for e in Eh],
            None if Wh is None else to_device(Wh, dt, device))
