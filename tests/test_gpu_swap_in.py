"""Swap-in of a whole adapter from host memory (one copy, one scatter kernel,
no host wait).  The pool it produces must be byte-identical to the one
lora_pool_load builds from the same matrices (same pages, A rows as given,
B transposed, rank padding zeroed); deltas computed from it must match the
oracle; it must overwrite a loaded slot completely and may run on a second
stream while deltas run on other slots."""

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import synth
from gpu_harness import DevicePool, assert_close, oracle_y, scales_of, to_dev_bf16, to_host_bits, workspace

pytestmark = pytest.mark.gpu

TARGETS = [(512, 256), (512, 256), (256, 512), (1024, 128)]


def _workload(T=48):
    return synth.custom(77, T, TARGETS, [16, 8, 13, 16, 4, 16], 16, page_bytes=4096, scatter_seed=777)


def _ranks(w, s, zero_target=None):
    r = int(w.rank[s])
    return [0 if t == zero_target else r for t in range(len(w.targets))]


def _packed(w, s, ranks):
    parts = []
    for t, r in enumerate(ranks):
        if r > 0:
            A, B = w.adapter(s, t)
            parts += [np.ascontiguousarray(A).ravel(), np.ascontiguousarray(B).ravel()]
    flat = np.concatenate(parts) if parts else np.zeros(0, np.uint16)
    host = torch.empty(flat.size * 2, dtype=torch.uint8).pin_memory()
    host.numpy()[:] = flat.view(np.uint8)
    return host


def _swap(pool, s, ranks, w, stream=None):
    src = _packed(w, s, ranks)
    assert src.numel() == L.lora_swap_src_bytes(pool.pool, ranks)
    staging = torch.empty(L.lora_swap_staging_bytes(pool.pool, ranks), dtype=torch.uint8, device=pool.device)
    L.lora_pool_swap_in(pool.pool, s, ranks, src, staging, stream)
    return src, staging  # keep both alive until the stream has passed the call


def _load(pool, s, ranks, w):
    for t, r in enumerate(ranks):
        if r > 0:
            A, B = w.adapter(s, t)
            L.lora_pool_load(pool.pool, s, t, r, to_dev_bf16(A, pool.device), to_dev_bf16(B, pool.device))
        else:
            L.lora_pool_load(pool.pool, s, t, 0, None, None)


def test_swap_in_builds_the_same_pool_as_load(cuda_device):
    w = _workload()
    with DevicePool(w, cuda_device, slots=[]) as ref, DevicePool(w, cuda_device, slots=[]) as sw:
        keep = []
        for s in range(w.n_slots):
            ranks = _ranks(w, s, zero_target=2 if s == 3 else None)
            _load(ref, s, ranks, w)
            keep.append(_swap(sw, s, ranks, w))
        torch.cuda.synchronize(cuda_device)
        assert torch.equal(ref.mem, sw.mem)
        n = w.n_slots * L.lora_pool_get_info(sw.pool).pages_per_slot
        pt_ref, pt_sw = (torch.as_tensor(_DevArray(L.lora_pool_page_table(p.pool), n), device=cuda_device).clone()
                         for p in (ref, sw))
        assert torch.equal(pt_ref, pt_sw)
        del keep


class _DevArray:
    """A read-only device int32 array seen through __cuda_array_interface__."""

    def __init__(self, ptr, n):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<i4", "data": (ptr, False), "version": 3}


def test_swapped_pool_gives_oracle_deltas(cuda_device):
    w = _workload()
    with DevicePool(w, cuda_device, slots=[]) as pool:
        keep = [_swap(pool, s, _ranks(w, s), w) for s in range(w.n_slots)]
        torch.cuda.synchronize(cuda_device)
        for t in range(len(w.targets)):
            x, y = w.x(t), w.y_in(t)
            dev = pool.device
            xd, yd = to_dev_bf16(x, dev), to_dev_bf16(y, dev)
            sc = torch.from_numpy(scales_of(w)).to(dev)
            L.lora_apply(pool.pool, t, xd, yd, torch.from_numpy(w.ids).to(dev), sc, workspace(pool, w.T))
            torch.cuda.synchronize(dev)
            ref, _ = oracle_y(w, t, x, y, w.ids)
            assert_close(to_host_bits(yd), ref, what="target %d" % t)
        del keep


def test_swap_in_overwrites_a_loaded_slot(cuda_device):
    w = _workload()
    with DevicePool(w, cuda_device, slots=[]) as ref, DevicePool(w, cuda_device, slots=[]) as sw:
        # slot 0 first holds slot 0's adapter (rank 16), then slot 4's (rank 4)
        _load(ref, 0, _ranks(w, 0), w)
        k1 = _swap(sw, 0, _ranks(w, 0), w)
        torch.cuda.synchronize(cuda_device)
        ranks4 = _ranks(w, 4)
        for t, r in enumerate(ranks4):
            A, B = w.adapter(4, t)
            L.lora_pool_load(ref.pool, 0, t, r, to_dev_bf16(A, cuda_device), to_dev_bf16(B, cuda_device))
        src = _packed(w, 4, ranks4)
        staging = torch.empty(L.lora_swap_staging_bytes(sw.pool, ranks4), dtype=torch.uint8, device=cuda_device)
        L.lora_pool_swap_in(sw.pool, 0, ranks4, src, staging)
        torch.cuda.synchronize(cuda_device)
        assert torch.equal(ref.mem, sw.mem)
        del k1


def test_swap_in_on_a_second_stream_beside_deltas(cuda_device):
    w = _workload(T=64)
    ids = w.ids.copy()
    ids[np.isin(ids, [5])] = -1           # the batch avoids the slot being swapped in
    with DevicePool(w, cuda_device, slots=[0, 1, 2, 3, 4]) as pool:
        dev = pool.device
        s_comp, s_swap = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        x, y = w.x(0), w.y_in(0)
        xd, yd = to_dev_bf16(x, dev), to_dev_bf16(y, dev)
        sc = torch.from_numpy(scales_of(w)).to(dev)
        ws = workspace(pool, w.T)
        d_ids = torch.from_numpy(ids).to(dev)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(s_comp):
            L.lora_apply(pool.pool, 0, xd, yd, d_ids, sc, ws)
        keep = _swap(pool, 5, _ranks(w, 5), w, stream=s_swap)
        torch.cuda.synchronize(dev)
        assert L.lora_get_error(pool.pool) == L.LORA_OK
        ref, _ = oracle_y(w, 0, x, y, ids)
        assert_close(to_host_bits(yd), ref, what="deltas beside a swap-in")
        # the swapped slot now serves a batch of its own
        ids5 = np.full(w.T, 5, np.int32)
        y2 = to_dev_bf16(y, dev)
        L.lora_apply(pool.pool, 0, xd, y2, torch.from_numpy(ids5).to(dev), sc, ws)
        torch.cuda.synchronize(dev)
        ref5, _ = oracle_y(w, 0, x, y, ids5)
        assert_close(to_host_bits(y2), ref5, what="swapped slot")
        del keep


def test_swap_in_argument_errors(cuda_device):
    w = _workload()
    with DevicePool(w, cuda_device, slots=[]) as pool:
        ranks = _ranks(w, 0)
        src = _packed(w, 0, ranks)
        need = L.lora_swap_staging_bytes(pool.pool, ranks)
        staging = torch.empty(need + 256, dtype=torch.uint8, device=cuda_device)
        cases = [
            (lambda: L.lora_pool_swap_in(pool.pool, 0, ranks, src[:-16], staging), L.LORA_ERR_INVALID_ARG),
            (lambda: L.lora_pool_swap_in(pool.pool, 0, ranks, src, staging[:need - 16]), L.LORA_ERR_WORKSPACE),
            (lambda: L.lora_pool_swap_in(pool.pool, 0, ranks, src, staging[16:]), L.LORA_ERR_ALIGNMENT),
            (lambda: L.lora_pool_swap_in(pool.pool, 99, ranks, src, staging), L.LORA_ERR_SLOT),
            (lambda: L.lora_pool_swap_in(pool.pool, 0, [17] * len(ranks), src, staging), L.LORA_ERR_INVALID_ARG),
        ]
        for fn, code in cases:
            with pytest.raises(L.LoraError) as e:
                fn()
            assert e.value.code == code
        assert L.lora_swap_src_bytes(pool.pool, [17] * len(ranks)) == 0
