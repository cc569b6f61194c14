"""GPU tests of the integer parts of the path, all bit-exact: the batch plan
(grouping of rows by adapter) against the oracle's stable grouping, the paged
pool against an independent host walk of its page table, pool bookkeeping
(out of pages, unload and reuse), host-side argument errors, and CUDA-graph
capture of a delta call."""

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import oracle
import synth
from gpu_harness import DevicePool, oracle_y, assert_close, run_gpu, scales_of, to_dev_bf16, to_host_bits, workspace

pytestmark = pytest.mark.gpu


def _plan_arrays(pool, ws, T):
    lay = L.lora_plan_layout_get(pool.pool, T)
    raw = ws.cpu().numpy()

    def arr(off, n, w=1):
        return raw[off:off + 4 * n * w].view(np.int32).reshape(-1, w) if w > 1 else raw[off:off + 4 * n].view(np.int32)

    hdr = arr(lay.header, 8)
    S, A, I = int(hdr[0]), int(hdr[1]), int(hdr[2])
    return (hdr, arr(lay.perm, A), arr(lay.seg_start, S + 1), arr(lay.seg_slot, S), arr(lay.items, I, 4),
            arr(lay.tiles, int(hdr[3]), 4))


def _check_items(items, perm, seg_start, seg_slot, max_rows=16):
    # items tile every segment's rows in order, at most max_rows each
    covered = []
    for slot, p0, m, seg in items.tolist():
        assert 1 <= m <= max_rows and seg_slot[seg] == slot
        assert seg_start[seg] <= p0 and p0 + m <= seg_start[seg + 1]
        covered.extend(range(p0, p0 + m))
    assert sorted(covered) == list(range(len(perm)))


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_plan_ids_bit_exact(cuda_device, cfg):
    w = synth.config(cfg)
    with DevicePool(w, cuda_device) as pool:
        for ids in (w.ids, np.full(w.T, -1, np.int32), np.zeros(w.T, np.int32), w.ids[:1], w.ids[::-1].copy()):
            T = ids.size
            ws = workspace(pool, T)
            L.lora_plan_ids(pool.pool, torch.from_numpy(ids).to(cuda_device), ws)
            torch.cuda.synchronize()
            hdr, perm, seg_start, seg_slot, items, _ = _plan_arrays(pool, ws, T)
            p_ref, s_ref, slot_ref, bad = oracle.group_rows(ids, w.n_slots)
            assert bad == 0
            assert np.array_equal(perm, p_ref)
            assert np.array_equal(seg_start, s_ref)
            assert np.array_equal(seg_slot, slot_ref)
            _check_items(items, perm, seg_start, seg_slot)


def test_plan_ids_large_batch_many_slots(cuda_device):
    # T not a multiple of 32 or of the item size; 1000 slots, some unloaded
    w = synth.config(5)
    small = synth.Workload("plan only", 1, [(64, 64)], 16, 1000, 0, 0, 3001,
                           np.random.default_rng(4).integers(-1, 1000, size=3001).astype(np.int32),
                           np.full(1000, 16, np.int32), np.full(1000, 32.0))
    loaded = [s for s in range(1000) if s % 7 != 3]
    with DevicePool(small, cuda_device, slots=loaded) as pool:
        ids = small.ids
        ws = workspace(pool, ids.size)
        L.lora_plan_ids(pool.pool, torch.from_numpy(ids).to(cuda_device), ws)
        _, perm, seg_start, seg_slot, items, _ = _plan_arrays(pool, ws, ids.size)
        valid = np.zeros(1000, np.uint8)
        valid[loaded] = 1
        p_ref, s_ref, slot_ref, bad = oracle.group_rows(ids, 1000, valid)
        assert bad > 0 and L.lora_get_error(pool.pool) == L.LORA_ERR_NOT_LOADED
        assert np.array_equal(perm, p_ref) and np.array_equal(seg_start, s_ref)
        assert np.array_equal(seg_slot, slot_ref)
        _check_items(items, perm, seg_start, seg_slot)
    del w


def test_plan_segments_bit_exact(cuda_device):
    w = synth.config(3)
    with DevicePool(w, cuda_device) as pool:
        ws = workspace(pool, w.T)
        L.lora_plan_segments(pool.pool, torch.from_numpy(w.seg_offsets).to(cuda_device),
                             torch.from_numpy(w.seg_slot).to(cuda_device), w.T, ws)
        hdr, perm, seg_start, seg_slot, items, tiles = _plan_arrays(pool, ws, w.T)
        assert np.array_equal(perm, np.arange(w.T))
        assert np.array_equal(seg_start, w.seg_offsets)
        assert np.array_equal(seg_slot, w.seg_slot)
        mma = L.lora_mma_min_rows_for(len(w.seg_slot), w.T)
        covered = []
        for slot, r0, m, seg in tiles.tolist():
            assert seg_slot[seg] == slot and seg_start[seg + 1] - seg_start[seg] >= mma
            covered.extend(range(r0, r0 + m))
        for slot, p0, m, seg in items.tolist():
            assert seg_start[seg + 1] - seg_start[seg] < mma
            covered.extend(perm[p0:p0 + m].tolist())
        assert sorted(covered) == list(range(w.T))


def test_plan_segments_rejects_malformed_offsets(cuda_device):
    w = synth.config(1)
    with DevicePool(w, cuda_device) as pool:
        ws = workspace(pool, 16)
        off = torch.tensor([0, 10, 5, 16], dtype=torch.int32, device=cuda_device)
        slot = torch.tensor([0, 1, 2], dtype=torch.int32, device=cuda_device)
        y0 = w.y_in(0)
        x = to_dev_bf16(w.x(0), cuda_device)
        y = to_dev_bf16(y0, cuda_device)
        L.lora_apply_segments(pool.pool, 0, x, y, off, slot, torch.from_numpy(scales_of(w)).to(cuda_device), ws)
        assert L.lora_get_error(pool.pool) == L.LORA_ERR_BAD_ID
        assert np.array_equal(to_host_bits(y), y0)


class _DevArray:
    """Wraps a raw device pointer so torch can view it (read-only use)."""

    def __init__(self, ptr, n):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<i4", "data": (ptr, False), "version": 3}


def _device_int32(ptr, n):
    return torch.as_tensor(_DevArray(ptr, n), device="cuda")


def _reconstruct(pool_mem, pt, slot, layout, pps, page_bytes, slot_bytes):
    a_off, bt_off, total = layout
    logical = np.zeros(pps * page_bytes, dtype=np.uint8)
    for p in range(pps):
        at = oracle.pool_locate(slot, p * page_bytes, pt, pps, page_bytes)
        logical[p * page_bytes:(p + 1) * page_bytes] = pool_mem[at:at + page_bytes]
    return logical[:slot_bytes]


def _untile(block: np.ndarray, r_max: int, width: int) -> np.ndarray:
    """A block [r_max, width] (bf16 bits) from its stored arrangement, as the
    header states it: column tiles of 1024 columns (r_max <= 16), 512 (r_max
    <= 32) or 256, each
    tile the rows one after the other, the 16-byte chunks of each complete
    group of eight in a row stored at chunk ^ (row % 8)."""
    tcc = (1024 if r_max <= 16 else 512 if r_max <= 32 else 256) // 8
    nch = width // 8
    u = block.view(np.uint16)
    out = np.empty((r_max, width), np.uint16)
    base = 0
    for k in range(-(-nch // tcc)):
        tw = min(tcc, nch - k * tcc)
        tile = u[base:base + r_max * tw * 8].reshape(r_max, tw, 8)
        c = np.arange(tw)[None, :]
        j = np.arange(r_max)[:, None]
        pos = np.where((c | 7) < tw, c ^ (j & 7), c)
        out[:, k * tcc * 8:(k * tcc + tw) * 8] = tile[j, pos].reshape(r_max, tw * 8)
        base += r_max * tcc * 8
    return out


@pytest.mark.parametrize("cfg,page", [(1, 4096), (4, 1 << 16), (2, 0)])
def test_pool_reconstruction_bitwise(cuda_device, cfg, page):
    w = synth.config(cfg)
    with DevicePool(w, cuda_device, page_bytes=page, scatter_seed=31337) as pool:
        info = L.lora_pool_get_info(pool.pool)
        layout = oracle.slot_layout(w.targets, w.r_max)
        assert info.slot_bytes == layout[2]
        pps, P = info.pages_per_slot, info.page_bytes
        pt = _device_int32(L.lora_pool_page_table(pool.pool), w.n_slots * pps).cpu()
        pt = pt.cpu().numpy()
        assert sorted(pt.tolist()) == list(range(w.n_slots * pps))  # every page used once
        mem = pool.mem.cpu().numpy()
        for s in range(0, w.n_slots, max(1, w.n_slots // 9)):
            logical = _reconstruct(mem, pt, s, layout, pps, P, info.slot_bytes)
            r = int(w.rank[s])
            for t, (d_in, d_out) in enumerate(w.targets):
                A, B = w.adapter(s, t)
                a0, b0 = int(layout[0][t]), int(layout[1][t])
                Ap = _untile(logical[a0:a0 + w.r_max * d_in * 2], w.r_max, d_in)
                Bt = _untile(logical[b0:b0 + w.r_max * d_out * 2], w.r_max, d_out)
                assert np.array_equal(Ap[:r], A) and not Ap[r:].any()
                assert np.array_equal(Bt[:r], B.T) and not Bt[r:].any()


def test_pool_out_of_pages_unload_and_reuse(cuda_device):
    w = synth.config(1)
    with DevicePool(w, cuda_device, slots=[], page_bytes=4096, n_pages=4) as pool:   # room for 2 slots
        pool.load_slot(0)
        pool.load_slot(1)
        with pytest.raises(L.LoraError) as e:
            pool.load_slot(2)
        assert e.value.code == L.LORA_ERR_NO_PAGES
        L.lora_pool_unload(pool.pool, 0)
        pool.load_slot(2)
        ids = np.array([1, 2, 0, 2, 1, -1], np.int32)
        got = run_gpu(pool, 0, w.x(0)[:6], w.y_in(0)[:6], ids)
        assert L.lora_get_error(pool.pool) == L.LORA_ERR_NOT_LOADED        # slot 0 is gone
        ids_ok = ids.copy()
        ids_ok[ids == 0] = -1
        ref, _ = oracle_y(w, 0, w.x(0)[:6], w.y_in(0)[:6], ids_ok)
        assert_close(got, ref)
        assert np.array_equal(got[2], w.y_in(0)[2])
        with pytest.raises(L.LoraError) as e:
            L.lora_pool_unload(pool.pool, 0)
        assert e.value.code == L.LORA_ERR_NOT_LOADED


def test_host_argument_errors(cuda_device):
    w = synth.config(1)
    dev = cuda_device
    with DevicePool(w, dev) as pool:
        x = to_dev_bf16(w.x(0), dev)
        y = to_dev_bf16(w.y_in(0), dev)
        ids = torch.from_numpy(w.ids).to(dev)
        sc = torch.from_numpy(scales_of(w)).to(dev)
        ws = workspace(pool, w.T)

        def code(fn):
            with pytest.raises(L.LoraError) as e:
                fn()
            return e.value.code

        big = torch.zeros(w.T, 264, dtype=torch.bfloat16, device=dev)
        assert code(lambda: L.lora_apply(pool.pool, 0, big[:, 1:257], y, ids, sc, ws)) == L.LORA_ERR_ALIGNMENT
        assert code(lambda: L.lora_apply(pool.pool, 3, x, y, ids, sc, ws)) == L.LORA_ERR_INVALID_ARG
        assert code(lambda: L.lora_apply(pool.pool, 0, x, y, ids, sc, ws[:64])) == L.LORA_ERR_WORKSPACE
        assert code(lambda: L.lora_apply(pool.pool, 0, x, x, ids, sc, ws)) == L.LORA_ERR_INVALID_ARG
        A = torch.zeros(9, 256, dtype=torch.bfloat16, device=dev)
        B = torch.zeros(256, 9, dtype=torch.bfloat16, device=dev)
        assert code(lambda: L.lora_pool_load(pool.pool, 0, 0, 9, A, B)) == L.LORA_ERR_INVALID_ARG
        assert code(lambda: L.lora_pool_load(pool.pool, 4, 0, 8, A[:8], B[:, :8].contiguous())) == L.LORA_ERR_SLOT
        # nothing above launched a kernel that could have touched y
        assert np.array_equal(to_host_bits(y), w.y_in(0))


def test_graph_capture_replays_identically(cuda_device):
    w = synth.config(2)
    dev = cuda_device
    with DevicePool(w, dev) as pool:
        x = to_dev_bf16(w.x(0), dev)
        y0 = to_dev_bf16(w.y_in(0), dev)
        ids = torch.from_numpy(w.ids).to(dev)
        sc = torch.from_numpy(scales_of(w)).to(dev)
        ws = workspace(pool, w.T)
        eager = y0.clone()
        L.lora_apply(pool.pool, 0, x, eager, ids, sc, ws)
        y = y0.clone()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                L.lora_apply(pool.pool, 0, x, y, ids, sc, ws)
        torch.cuda.current_stream().wait_stream(s)
        for _ in range(3):
            y.copy_(y0)
            g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), eager.view(torch.int16))
