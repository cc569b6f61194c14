"""The no-allocation entry point (lora_apply_noalloc) against lora_apply.

lora_apply_noalloc serves callers that cannot allocate device memory: its plan
lives in a fixed device array inside the library instead of a workspace the
caller passes.  This test calls it through the C ABI twice in a row -- a full
batch, then a smaller different one, so the second call runs over the first
call's leftover plan -- and checks each result against lora_apply with a
normal workspace, within the parity tolerance.  It builds its own pool, so it
passes alone in a fresh process and after the other tests.
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
        assert_close(got, oracle.bf16_to_f64(ref), what="noalloc vs lora_apply")
    # and both against the oracle
    want2, _ = oracle_y(w, 0, w.x(0)[:23], w.y_in(0)[:23], ids2)
    assert_close(got2, want2, what="noalloc vs oracle")
    assert np.array_equal(got2[[2, 9]], w.y_in(0)[[2, 9]])


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
