"""Helpers for the GPU tests: place a synthetic workload's adapters in a device
pool, run the CUDA path through the C ABI, and compare with the oracle.

Comparison rule: max |y_gpu - y_ref| <= 4e-3 * max |y_ref| (bf16 inputs, fp32
accumulation, bf16 output), element by element over every compared row.
"""

from __future__ import annotations

from typing import Dict, Iterable, Optional, Sequence

import numpy as np
import torch

import adapter_deltas_b200 as L
import oracle
from synth import Workload

REL_TOL = 4e-3


def to_dev_bf16(bits: np.ndarray, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def scales_of(w: Workload) -> np.ndarray:
    """Per-slot scale alpha / r that the caller passes (0 for empty slots)."""
    r = w.rank.astype(np.float64)
    s = np.zeros(w.n_slots, dtype=np.float64)
    nz = r > 0
    s[nz] = w.alpha[nz] / r[nz]
    return s.astype(np.float32)


class DevicePool:
    """A lora pool over a torch uint8 buffer, filled from a workload."""

    def __init__(self, w: Workload, device, slots: Optional[Iterable[int]] = None,
                 page_bytes: Optional[int] = None, scatter_seed: Optional[int] = None,
                 filler_slots: Iterable[int] = (), n_pages: Optional[int] = None):
        self.w = w
        self.device = torch.device(device)
        pb = w.page_bytes if page_bytes is None else page_bytes
        seed = w.scatter_seed if scatter_seed is None else scatter_seed
        nbytes = L.lora_pool_bytes_required(w.targets, w.r_max, w.n_slots, pb)
        assert nbytes > 0
        if n_pages is not None:
            nbytes = n_pages * (pb if pb else nbytes // w.n_slots)
        self.mem = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.pool = L.lora_pool_create(self.device.index or 0, w.targets, w.r_max, w.n_slots, pb, self.mem, seed)
        self.loaded = []
        slots = list(range(w.n_slots)) if slots is None else list(slots)
        if len(slots) > 64:
            w.prefetch(slots, range(len(w.targets)))
        for s in slots:
            self.load_slot(s)
        filler = None
        for s in filler_slots:
            if filler is None:
                filler = {}
            for t, (d_in, d_out) in enumerate(w.targets):
                key = (d_in, d_out)
                if key not in filler:
                    g = torch.Generator(device=self.device).manual_seed(12345)
                    r = w.r_max
                    filler[key] = (
                        (torch.randn(r, d_in, generator=g, device=self.device) / d_in ** 0.5).to(torch.bfloat16),
                        (torch.randn(d_out, r, generator=g, device=self.device) * 0.14).to(torch.bfloat16))
                A, B = filler[key]
                r = int(w.rank[s])
                L.lora_pool_load(self.pool, s, t, r, A[:r].contiguous(), B[:, :r].contiguous())
        torch.cuda.synchronize(self.device)

    def load_slot(self, s: int) -> None:
        for t in range(len(self.w.targets)):
            r = int(self.w.rank[s])
            if r == 0:
                continue
            A, B = self.w.adapter(s, t)
            L.lora_pool_load(self.pool, s, t, r, to_dev_bf16(A, self.device), to_dev_bf16(B, self.device))
        self.loaded.append(s)

    def close(self) -> None:
        L.lora_pool_destroy(self.pool)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def workspace(pool: DevicePool, T: int) -> torch.Tensor:
    """A workspace good for every target of the pool (the largest size)."""
    n = max(L.lora_workspace_bytes(pool.pool, t, T) for t in range(len(pool.w.targets)))
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=pool.device)


def run_gpu(pool: DevicePool, target: int, x_bits: np.ndarray, y_bits: np.ndarray, ids: np.ndarray,
            scales: Optional[np.ndarray] = None, api: str = "ids") -> np.ndarray:
    """One delta call on the GPU; returns y (bf16 bits)."""
    dev = pool.device
    w = pool.w
    x = to_dev_bf16(x_bits, dev)
    y = to_dev_bf16(y_bits, dev)
    sc = torch.from_numpy(scales_of(w) if scales is None else scales).to(dev)
    ws = workspace(pool, y.shape[0])
    if api == "ids":
        L.lora_apply(pool.pool, target, x, y, torch.from_numpy(ids).to(dev), sc, ws)
    elif api == "segments":
        L.lora_apply_segments(pool.pool, target, x, y, torch.from_numpy(w.seg_offsets).to(dev),
                              torch.from_numpy(w.seg_slot).to(dev), sc, ws)
    elif api == "split":
        d = torch.from_numpy(ids).to(dev)
        v = torch.zeros(y.shape[0], w.r_max, dtype=torch.float32, device=dev)
        L.lora_shrink(pool.pool, target, x, d, v, ws)
        L.lora_expand(pool.pool, target, v, y, d, sc, ws)
    else:
        raise ValueError(api)
    torch.cuda.synchronize(dev)
    return to_host_bits(y)


def oracle_y(w: Workload, target: int, x_bits, y_bits, ids, alpha=None, threads: int = 8):
    slots = [int(s) for s in np.unique(ids[ids >= 0]) if w.rank[s] > 0]
    adapters = {s: w.adapter(s, target) for s in slots}
    a = w.alpha if alpha is None else alpha
    y, bad = oracle.lora_apply(x_bits, y_bits, ids, w.n_slots, adapters, a, threads=threads)
    return y, bad


def max_rel_err(y_gpu_bits: np.ndarray, y_ref: np.ndarray) -> float:
    g = oracle.bf16_to_f64(y_gpu_bits)
    scale = np.abs(y_ref).max()
    if scale == 0:
        return float(np.abs(g).max())
    return float(np.abs(g - y_ref).max() / scale)


def assert_close(y_gpu_bits, y_ref, tol: float = REL_TOL, what: str = "") -> float:
    e = max_rel_err(y_gpu_bits, y_ref)
    assert e <= tol, "%s: max|y_gpu - y_ref| / max|y_ref| = %.3e > %.1e" % (what, e, tol)
    return e
