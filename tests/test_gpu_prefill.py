"""GPU parity of the segment (prefill) path: segments on the tensor cores
(tcgen05 MMA, TMA tiles; 128-row tiles, a shrink launch over k-slices and an
expand launch over column groups) -- every segment of a batch of at most 16,
else those of 64 rows or more, the short ones then on the decode kernel --
against the fp64 oracle on the same seeded inputs.

Bound: max |y_gpu - y_ref| <= 4e-3 * max |y_ref|, with the base output and
with y = 0 (delta alone); rows outside every segment and rows of segments
without adapter stay bitwise unchanged."""

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import synth
from gpu_harness import DevicePool, assert_close, oracle_y, scales_of, to_dev_bf16, to_host_bits, workspace

pytestmark = pytest.mark.gpu


def _segments(lengths, slots, gap_rows=()):
    """Contiguous segments; gap_rows inserts rows with no segment after segment i."""
    off = [0]
    seg_slot = []
    for i, (ln, sl) in enumerate(zip(lengths, slots)):
        off.append(off[-1] + ln)
        seg_slot.append(sl)
        if i in gap_rows:
            off.append(off[-1] + 3)
            seg_slot.append(-1)
    return np.array(off, np.int32), np.array(seg_slot, np.int32)


def _ids(off, seg_slot):
    ids = np.full(int(off[-1]), -1, np.int32)
    for s, sl in enumerate(seg_slot):
        ids[off[s]:off[s + 1]] = sl
    return ids


def _run_segments(pool, w, t, x_bits, y_bits, off, seg_slot, scales=None):
    dev = pool.device
    x = to_dev_bf16(x_bits, dev)
    y = to_dev_bf16(y_bits, dev)
    sc = torch.from_numpy(scales_of(w) if scales is None else scales).to(dev)
    ws = workspace(pool, y.shape[0])
    L.lora_apply_segments(pool.pool, t, x, y, torch.from_numpy(off).to(dev), torch.from_numpy(seg_slot).to(dev),
                          sc, ws)
    torch.cuda.synchronize(dev)
    assert L.lora_get_error(pool.pool) == L.LORA_OK
    return to_host_bits(y)


def _make(T, d_in, d_out, ranks, r_max, seed=3):
    return synth.custom(seed, T, [(d_in, d_out)], ranks, r_max)


@pytest.mark.parametrize("shape", [(4096, 4096), (256, 512), (200, 328), (1024, 11008)])
def test_tensor_core_segments_match_oracle(cuda_device, shape):
    d_in, d_out = shape
    lengths = [300, 64, 65, 127, 129, 5, 1, 63, 200]
    slots = [0, 1, 2, 3, 0, 4, 1, 2, 3]
    off, seg_slot = _segments(lengths, slots, gap_rows=(2, 6))
    T = int(off[-1])
    w = _make(T, d_in, d_out, [16, 8, 16, 13, 16], 16)
    ids = _ids(off, seg_slot)
    with DevicePool(w, cuda_device) as pool:
        for zero in (False, True):
            y0 = np.zeros_like(w.y_in(0)) if zero else w.y_in(0)
            got = _run_segments(pool, w, 0, w.x(0), y0, off, seg_slot)
            ref, _ = oracle_y(w, 0, w.x(0), y0, ids)
            assert_close(got, ref, what="segments %s y0=%s" % (shape, zero))
            none = ids < 0
            assert np.array_equal(got[none], y0[none])


def test_prefill_config_uses_tensor_cores_and_matches(cuda_device):
    w = synth.config(3)
    with DevicePool(w, cuda_device) as pool:
        n0 = L.lora_kernel_launches()
        got = _run_segments(pool, w, 0, w.x(0), w.y_in(0), w.seg_offsets, w.seg_slot)
        # 8 segments: every one on the tensor cores, no short-segment decode launch
        assert L.lora_mma_min_rows_for(len(w.seg_slot), w.T) == 1
        assert L.lora_kernel_launches() - n0 == 3  # plan, tensor-core shrink, expand
        ref, _ = oracle_y(w, 0, w.x(0), w.y_in(0), w.ids)
        assert_close(got, ref, what="config 3")
        got0 = _run_segments(pool, w, 0, w.x(0), np.zeros_like(w.y_in(0)), w.seg_offsets, w.seg_slot)
        ref0, _ = oracle_y(w, 0, w.x(0), np.zeros_like(w.y_in(0)), w.ids)
        assert_close(got0, ref0, what="config 3 delta only")


def test_many_segments_split_between_tensor_cores_and_decode(cuda_device):
    # 24 segments: those of 64 rows or more on the tensor cores, the short
    # ones (1 - 63 rows) on the decode kernel, in one apply of four launches
    lengths = [300, 5, 1, 63, 64, 70, 2, 3, 129, 17, 40, 1, 128, 9, 33, 200, 6, 7, 64, 11, 1, 90, 12, 2]
    slots = [i % 5 for i in range(len(lengths))]
    off, seg_slot = _segments(lengths, slots, gap_rows=(4,))
    T = int(off[-1])
    assert L.lora_mma_min_rows_for(len(seg_slot), T) == L.lora_mma_min_rows() == 64
    w = _make(T, 512, 384, [16, 8, 16, 13, 16], 16, seed=5)
    ids = _ids(off, seg_slot)
    with DevicePool(w, cuda_device) as pool:
        n0 = L.lora_kernel_launches()
        got = _run_segments(pool, w, 0, w.x(0), w.y_in(0), off, seg_slot)
        assert L.lora_kernel_launches() - n0 == 4  # plan, decode (short segments), tensor-core shrink, expand
        ref, _ = oracle_y(w, 0, w.x(0), w.y_in(0), ids)
        assert_close(got, ref, what="24 segments")
        none = ids < 0
        assert np.array_equal(got[none], w.y_in(0)[none])


def test_rank_32_and_distinct_scales(cuda_device):
    lengths = [256, 90, 130]
    off, seg_slot = _segments(lengths, [0, 1, 2])
    T = int(off[-1])
    w = _make(T, 512, 768, [32, 24, 17], 32)
    ids = _ids(off, seg_slot)
    alpha = np.array([3.0, 50.0, 0.7]) * w.rank
    scales = (alpha / w.rank).astype(np.float32)
    with DevicePool(w, cuda_device) as pool:
        got = _run_segments(pool, w, 0, w.x(0), np.zeros_like(w.y_in(0)), off, seg_slot, scales=scales)
        ref, _ = oracle_y(w, 0, w.x(0), np.zeros_like(w.y_in(0)), ids, alpha=alpha)
        assert_close(got, ref, what="rank 32")


def test_rank_64_pool_falls_back_to_decode_items(cuda_device):
    # r_max 64 is beyond the tensor-core path: every segment runs on the decode kernel
    lengths = [200, 70, 10]
    off, seg_slot = _segments(lengths, [1, 0, 1])
    T = int(off[-1])
    w = _make(T, 512, 256, [64, 40], 64)
    ids = _ids(off, seg_slot)
    with DevicePool(w, cuda_device) as pool:
        n0 = L.lora_kernel_launches()
        got = _run_segments(pool, w, 0, w.x(0), w.y_in(0), off, seg_slot)
        assert L.lora_kernel_launches() - n0 == 2           # plan + decode only
        ref, _ = oracle_y(w, 0, w.x(0), w.y_in(0), ids)
        assert_close(got, ref, what="rank 64 fallback")


def test_segments_and_ids_paths_agree(cuda_device):
    w = synth.config(3)
    with DevicePool(w, cuda_device) as pool:
        dev = pool.device
        x = to_dev_bf16(w.x(0), dev)
        y1 = to_dev_bf16(np.zeros_like(w.y_in(0)), dev)
        y2 = y1.clone()
        sc = torch.from_numpy(scales_of(w)).to(dev)
        ws = workspace(pool, w.T)
        L.lora_apply_segments(pool.pool, 0, x, y1, torch.from_numpy(w.seg_offsets).to(dev),
                              torch.from_numpy(w.seg_slot).to(dev), sc, ws)
        L.lora_apply(pool.pool, 0, x, y2, torch.from_numpy(w.ids).to(dev), sc, ws)
        torch.cuda.synchronize()
        a = to_host_bits(y1)
        b = to_host_bits(y2)
        ref, _ = oracle_y(w, 0, w.x(0), np.zeros_like(w.y_in(0)), w.ids)
        # each path is within the bound of the oracle, so they agree within twice it
        assert_close(a, ref, what="segments path")
        assert_close(b, ref, what="index-vector path")
        import oracle
        fa, fb = oracle.bf16_to_f64(a), oracle.bf16_to_f64(b)
        assert np.abs(fa - fb).max() <= 2 * 4e-3 * np.abs(ref).max()
