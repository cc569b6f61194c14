"""The decode kernel's bounded waits give up cleanly.

lora_selftest_stalled_apply launches the decode kernel of lora_apply with its
copy warp told to fill no stage, so the compute warps' first wait on the
ring can only run out.  With the wait limit lowered to 2 ms the launch must
complete, the pool's sticky status must read LORA_ERR_TIMEOUT (and read back
LORA_OK once cleared), y must be left exactly as it was, and the CUDA
context must stay usable: a normal lora_apply right after must match the
oracle.  No copy is issued for the stalled phase, so nothing is in flight
when the kernel returns.
"""

import time

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import synth
from gpu_harness import DevicePool, assert_close, oracle_y, scales_of, to_dev_bf16, to_host_bits, workspace

pytestmark = pytest.mark.gpu


def test_stalled_decode_times_out_and_leaves_y(cuda_device):
    w = synth.config(2)
    with DevicePool(w, cuda_device) as pool:
        dev = pool.device
        x = to_dev_bf16(w.x(0), dev)
        y = to_dev_bf16(w.y_in(0), dev)
        ids = torch.from_numpy(w.ids).to(dev)
        sc = torch.from_numpy(scales_of(w)).to(dev)
        assert L.lora_get_error(pool.pool) == L.LORA_OK
        L.lora_set_wait_limit_ns(2_000_000)
        try:
            t0 = time.perf_counter()
            L.lora_selftest_stalled_apply(pool.pool, 0, x, y, ids, sc)
            torch.cuda.synchronize(dev)
            elapsed = time.perf_counter() - t0
        finally:
            L.lora_set_wait_limit_ns(0)
        assert elapsed < 5.0, elapsed  # the waits ran out after about the limit, not never
        assert L.lora_get_error(pool.pool) == L.LORA_ERR_TIMEOUT
        assert L.lora_get_error(pool.pool) == L.LORA_OK  # reading cleared it
        assert np.array_equal(to_host_bits(y), w.y_in(0))
        # the context is usable and the default limit is back: a normal call
        # completes and matches the oracle
        y2 = to_dev_bf16(w.y_in(0), dev)
        L.lora_apply(pool.pool, 0, x, y2, ids, sc, workspace(pool, w.T))
        torch.cuda.synchronize(dev)
        assert L.lora_get_error(pool.pool) == L.LORA_OK
        want, _ = oracle_y(w, 0, w.x(0), w.y_in(0), w.ids)
        assert_close(to_host_bits(y2), want, what="lora_apply after a timed-out launch")


def test_stalled_apply_rejects_plan_sized_batches(cuda_device):
    w = synth.config(2)
    with DevicePool(w, cuda_device) as pool:
        T = 257
        x = torch.zeros(T, 4096, dtype=torch.bfloat16, device=cuda_device)
        y = torch.zeros(T, 4096, dtype=torch.bfloat16, device=cuda_device)
        ids = torch.zeros(T, dtype=torch.int32, device=cuda_device)
        sc = torch.from_numpy(scales_of(w)).to(cuda_device)
        with pytest.raises(L.LoraError) as e:
            L.lora_selftest_stalled_apply(pool.pool, 0, x, y, ids, sc)
        assert e.value.code == L.LORA_ERR_INVALID_ARG
