"""The no-allocation entry point (lora_apply_noalloc) against lora_apply.

lora_apply_noalloc serves callers that cannot allocate device memory: its plan
lives in a fixed device array inside the library instead of a workspace the
caller passes.  These tests call it through the C ABI twice in a row -- a
batch, then a different one, so the second call runs over the first call's
leftover plan -- and require the same bits as lora_apply with a normal
workspace (the same kernels on the same inputs), and the oracle's values
within the parity tolerance.  Batches of 64 and 23 rows take the one-launch
path; 1000 and 4096 rows take the plan kernel, whose plan lives in the fixed
array.  The tests build their own pools, so they pass alone in a fresh
process and after the other tests.
"""

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import synth
from gpu_harness import DevicePool, assert_close, oracle_y, scales_of, to_dev_bf16, to_host_bits, workspace
import oracle

pytestmark = pytest.mark.gpu


def _both(pool, w, x_bits, y_bits, ids):
    dev = pool.device
    x = to_dev_bf16(x_bits, dev)
    d_ids = torch.from_numpy(ids).to(dev)
    sc = torch.from_numpy(scales_of(w)).to(dev)
    y_ref = to_dev_bf16(y_bits, dev)
    L.lora_apply(pool.pool, 0, x, y_ref, d_ids, sc, workspace(pool, ids.size))
    y_new = to_dev_bf16(y_bits, dev)
    L.lora_apply_noalloc(pool.pool, 0, x, y_new, d_ids, sc)
    torch.cuda.synchronize(dev)
    return to_host_bits(y_ref), to_host_bits(y_new)


def test_noalloc_matches_lora_apply_on_two_calls(cuda_device):
    w = synth.config(2)
    with DevicePool(w, cuda_device) as pool:
        # call 1: the whole 64-token batch
        ref1, got1 = _both(pool, w, w.x(0), w.y_in(0), w.ids)
        # call 2: 23 rows, other adapters, some without adapter
        ids2 = ((w.ids[:23] * 7 + 3) % w.n_slots).astype(np.int32)
        ids2[[2, 9]] = -1
        ref2, got2 = _both(pool, w, w.x(0)[:23], w.y_in(0)[:23], ids2)
        assert L.lora_get_error(pool.pool) == L.LORA_OK
    for ref, got in ((ref1, got1), (ref2, got2)):
        assert np.array_equal(got, ref), "noalloc vs lora_apply"
    # and both against the oracle
    want2, _ = oracle_y(w, 0, w.x(0)[:23], w.y_in(0)[:23], ids2)
    assert_close(got2, want2, what="noalloc vs oracle")
    assert np.array_equal(got2[[2, 9]], w.y_in(0)[[2, 9]])


def _rows(w, T, seed):
    """T rows over the workload's adapters: its x, y and ids cycled, with a
    seeded 10 % of the rows without adapter."""
    reps = -(-T // w.T)
    x = np.tile(w.x(0), (reps, 1))[:T]
    y = np.tile(w.y_in(0), (reps, 1))[:T]
    ids = np.tile(w.ids, reps)[:T].astype(np.int32)
    rng = np.random.default_rng(seed)
    ids[rng.random(T) < 0.1] = -1
    return x, y, ids


@pytest.mark.parametrize("T", [1000, 4096])
def test_noalloc_plan_path_matches_lora_apply(cuda_device, T):
    w = synth.config(2)
    with DevicePool(w, cuda_device) as pool:
        x1, y1, ids1 = _rows(w, T, 11)
        ref1, got1 = _both(pool, w, x1, y1, ids1)
        # a second, different batch over the first one's leftover plan
        x2, y2, ids2 = _rows(w, T - 37, 12)
        ids2 = np.where(ids2 >= 0, (ids2 * 5 + 1) % w.n_slots, -1).astype(np.int32)
        ref2, got2 = _both(pool, w, x2, y2, ids2)
        assert L.lora_get_error(pool.pool) == L.LORA_OK
    assert np.array_equal(got1, ref1), "noalloc vs lora_apply, T=%d" % T
    assert np.array_equal(got2, ref2), "noalloc vs lora_apply, T=%d (second call)" % (T - 37)
    none = ids2 == -1
    assert np.array_equal(got2[none], y2[none])
    # the oracle on a sample of rows (every adapter of the sample, and rows
    # without adapter)
    pick = np.sort(np.random.default_rng(13).choice(T - 37, size=96, replace=False))
    want, _ = oracle_y(w, 0, x2[pick], y2[pick], ids2[pick])
    assert_close(got2[pick], want, what="noalloc vs oracle, T=%d" % (T - 37))


def test_noalloc_rejects_batches_beyond_its_array(cuda_device):
    w = synth.config(1)
    with DevicePool(w, cuda_device) as pool:
        T = L.LORA_NOALLOC_MAX_TOKENS + 1
        x = torch.zeros(T, 256, dtype=torch.bfloat16, device=cuda_device)
        y = torch.zeros(T, 256, dtype=torch.bfloat16, device=cuda_device)
        ids = torch.zeros(T, dtype=torch.int32, device=cuda_device)
        sc = torch.from_numpy(scales_of(w)).to(cuda_device)
        with pytest.raises(L.LoraError) as e:
            L.lora_apply_noalloc(pool.pool, 0, x, y, ids, sc)
        assert e.value.code == L.LORA_ERR_WORKSPACE
        assert not y.any()
