"""Batches of at most 256 rows are grouped inside the decode kernel (one
launch, no plan kernel).  The grouping must give exactly the plan kernel's
items, so the one-launch call and lora_plan_ids + lora_apply_plan must agree
bit for bit, and both must match the fp64 oracle; the sticky status of bad
ids and empty slots must be the same on both paths."""

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import synth
from gpu_harness import DevicePool, assert_close, oracle_y, scales_of, to_dev_bf16, to_host_bits, workspace

pytestmark = pytest.mark.gpu

FUSED_MAX_T = 256


def _both_paths(pool, target, x_bits, y_bits, ids):
    """(one-launch y, status), (plan + apply y, status), launches of the first."""
    dev = pool.device
    w = pool.w
    sc = torch.from_numpy(scales_of(w)).to(dev)
    d_ids = torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32)).to(dev)
    ws = workspace(pool, len(ids))
    x = to_dev_bf16(x_bits, dev)
    y1 = to_dev_bf16(y_bits, dev)
    y2 = y1.clone()
    n0 = L.lora_kernel_launches()
    L.lora_apply(pool.pool, target, x, y1, d_ids, sc, ws)
    launches = L.lora_kernel_launches() - n0
    torch.cuda.synchronize(dev)
    st1 = L.lora_get_error(pool.pool)
    L.lora_plan_ids(pool.pool, d_ids, ws)
    L.lora_apply_plan(pool.pool, target, x, y2, sc, ws)
    torch.cuda.synchronize(dev)
    st2 = L.lora_get_error(pool.pool)
    return (to_host_bits(y1), st1), (to_host_bits(y2), st2), launches


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_one_launch_equals_plan_path_on_configs(cuda_device, cfg):
    w = synth.config(cfg)
    assert w.T <= FUSED_MAX_T
    with DevicePool(w, cuda_device) as pool:
        for t in range(len(w.targets)):
            (a, sa), (b, sb), n = _both_paths(pool, t, w.x(t), w.y_in(t), w.ids)
            assert n == 1
            assert sa == sb == L.LORA_OK
            assert np.array_equal(a, b), "target %d" % t
            ref, _ = oracle_y(w, t, w.x(t), w.y_in(t), w.ids)
            assert_close(a, ref, what="config %d target %d" % (cfg, t))


@pytest.mark.parametrize("T", [1, 17, 255, 256])
def test_one_launch_sizes_and_long_runs(cuda_device, T):
    # few adapters, so segments run past one item (16 rows) and are cut
    rng = np.random.default_rng(T)
    ids = rng.integers(-1, 3, size=T).astype(np.int32)
    w = synth.custom(40 + T, T, [(512, 768)], [8, 16, 13], 16, ids=ids)
    with DevicePool(w, cuda_device) as pool:
        (a, sa), (b, sb), n = _both_paths(pool, 0, w.x(0), w.y_in(0), w.ids)
        assert n == 1 and sa == sb == L.LORA_OK
        assert np.array_equal(a, b)
        ref, _ = oracle_y(w, 0, w.x(0), w.y_in(0), w.ids)
        assert_close(a, ref, what="T=%d" % T)


def test_257_rows_take_the_plan_kernel(cuda_device):
    w = synth.custom(7, 257, [(256, 256)], [8, 8], 8)
    with DevicePool(w, cuda_device) as pool:
        (a, _), (b, _), n = _both_paths(pool, 0, w.x(0), w.y_in(0), w.ids)
        assert n == 2
        assert np.array_equal(a, b)


def test_bad_ids_and_empty_slots_same_status(cuda_device):
    w = synth.custom(9, 64, [(256, 512)], [8, 8, 8, 8], 8)
    ids = w.ids.copy()
    ids[3] = 99       # outside [-1, n_slots)
    ids[10] = -7
    with DevicePool(w, cuda_device) as pool:
        (a, sa), (b, sb), _ = _both_paths(pool, 0, w.x(0), w.y_in(0), ids)
        assert sa == sb == L.LORA_ERR_BAD_ID
        assert np.array_equal(a, b)
        assert np.array_equal(a[[3, 10]], w.y_in(0)[[3, 10]])
    # an empty slot: load only slots 0 and 1
    ids2 = w.ids.copy()
    with DevicePool(w, cuda_device, slots=[0, 1]) as pool:
        (a, sa), (b, sb), _ = _both_paths(pool, 0, w.x(0), w.y_in(0), ids2)
        assert sa == sb == L.LORA_ERR_NOT_LOADED
        assert np.array_equal(a, b)
        empty = (ids2 == 2) | (ids2 == 3)
        assert np.array_equal(a[empty], w.y_in(0)[empty])


def test_one_launch_shrink_expand_match_plan_path(cuda_device):
    w = synth.config(2)
    with DevicePool(w, cuda_device) as pool:
        dev = pool.device
        d_ids = torch.from_numpy(w.ids).to(dev)
        ws = workspace(pool, w.T)
        x = to_dev_bf16(w.x(0), dev)
        v1 = torch.zeros(w.T, w.r_max, dtype=torch.float32, device=dev)
        L.lora_shrink(pool.pool, 0, x, d_ids, v1, ws)
        L.lora_plan_ids(pool.pool, d_ids, ws)
        # the plan path of the shrink: a plan followed by the two-phase apply
        # of the same batch gives the same v; compare through expand
        y1 = to_dev_bf16(w.y_in(0), dev)
        y2 = y1.clone()
        sc = torch.from_numpy(scales_of(w)).to(dev)
        L.lora_expand(pool.pool, 0, v1, y1, d_ids, sc, ws)
        L.lora_apply(pool.pool, 0, x, y2, d_ids, sc, ws)
        torch.cuda.synchronize(dev)
        assert np.array_equal(to_host_bits(y1), to_host_bits(y2))
