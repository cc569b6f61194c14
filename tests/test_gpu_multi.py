"""Several same-shape targets sharing x in one launch (q, k, v of a layer):
lora_apply_multi must equal one lora_apply per target on the column slices of
y bit for bit, match the fp64 oracle per target, leave every other column
untouched, and reject bad geometry."""

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import synth
from gpu_harness import DevicePool, assert_close, oracle_y, scales_of, to_dev_bf16, to_host_bits, workspace

pytestmark = pytest.mark.gpu


def _fused_y(w, n_t, d_out, ld, cols, y_mode_zero=False):
    """y [T, ld] holding each target's y_in in its column slice (rest: a
    fixed pattern that must stay untouched)."""
    y = np.full((w.T, ld), 0x3f80, np.uint16)  # bf16 1.0 outside the slices
    for t in range(n_t):
        y[:, cols[t]:cols[t] + d_out] = 0 if y_mode_zero else w.y_in(t)
    return y


def _run(pool, targets, x_bits, y_bits, cols, ids):
    dev = pool.device
    w = pool.w
    x = to_dev_bf16(x_bits, dev)
    y = to_dev_bf16(y_bits, dev)
    sc = torch.from_numpy(scales_of(w)).to(dev)
    ws = workspace(pool, w.T)
    n0 = L.lora_kernel_launches()
    L.lora_apply_multi(pool.pool, targets, x, y, cols, torch.from_numpy(ids).to(dev), sc, ws)
    torch.cuda.synchronize(dev)
    assert L.lora_get_error(pool.pool) == L.LORA_OK
    return to_host_bits(y), L.lora_kernel_launches() - n0


def _separate(pool, targets, x_bits, y_bits, cols, ids, d_out):
    """The same deltas by one lora_apply per target on its column slice."""
    dev = pool.device
    w = pool.w
    x = to_dev_bf16(x_bits, dev)
    y = to_dev_bf16(y_bits, dev)
    sc = torch.from_numpy(scales_of(w)).to(dev)
    ws = workspace(pool, w.T)
    d_ids = torch.from_numpy(ids).to(dev)
    for t, c in zip(targets, cols):
        L.lora_apply(pool.pool, t, x, y[:, c:c + d_out], d_ids, sc, ws)
    torch.cuda.synchronize(dev)
    return to_host_bits(y)


@pytest.mark.parametrize("T", [64, 300])
def test_qkv_one_launch_matches_separate_and_oracle(cuda_device, T):
    d = 1024
    w = synth.custom(21 + T, T, [(d, d)] * 3, [16] * 24, 16)
    targets, cols, ld = [0, 1, 2], [0, d, 2 * d], 3 * d
    # x is shared: every target's oracle reads the same x
    x = w.x(0)
    with DevicePool(w, cuda_device) as pool:
        for zero in (False, True):
            y0 = _fused_y(w, 3, d, ld, cols, zero)
            got, launches = _run(pool, targets, x, y0, cols, w.ids)
            assert launches == (1 if T <= 256 else 2)
            ref_sep = _separate(pool, targets, x, y0, cols, w.ids, d)
            assert np.array_equal(got, ref_sep)
            for t in targets:
                ref, _ = oracle_y(w, t, x, y0[:, cols[t]:cols[t] + d], w.ids)
                assert_close(got[:, cols[t]:cols[t] + d], ref, what="target %d T=%d" % (t, T))


def test_targets_in_any_order_with_gaps_and_none_rows(cuda_device):
    d_in, d_out = 512, 256
    T = 40
    ids = np.random.default_rng(5).integers(-1, 6, size=T).astype(np.int32)
    w = synth.custom(33, T, [(d_in, d_out)] * 4, [8, 16, 12, 16, 4, 16], 16, ids=ids)
    targets, cols, ld = [3, 1], [8, 8 + d_out + 16], 8 + 2 * d_out + 32
    x = w.x(0)
    with DevicePool(w, cuda_device) as pool:
        y0 = np.full((T, ld), 0x3f80, np.uint16)
        for t, c in zip(targets, cols):
            y0[:, c:c + d_out] = w.y_in(t)
        got, _ = _run(pool, targets, x, y0, cols, ids)
        sep = _separate(pool, targets, x, y0, cols, ids, d_out)
        assert np.array_equal(got, sep)
        # columns outside the two slices and rows without adapter are untouched
        mask = np.ones(ld, bool)
        for c in cols:
            mask[c:c + d_out] = False
        assert np.array_equal(got[:, mask], y0[:, mask])
        assert np.array_equal(got[ids < 0], y0[ids < 0])
        for t, c in zip(targets, cols):
            ref, _ = oracle_y(w, t, x, y0[:, c:c + d_out], ids)
            assert_close(got[:, c:c + d_out], ref, what="target %d" % t)


def test_multi_rejects_bad_geometry(cuda_device):
    w = synth.custom(3, 16, [(256, 256), (256, 256), (256, 512)], [8, 8], 8)
    with DevicePool(w, cuda_device) as pool:
        dev = pool.device
        x = to_dev_bf16(w.x(0), dev)
        y = torch.zeros(16, 1024, dtype=torch.bfloat16, device=dev)
        ids = torch.from_numpy(w.ids).to(dev)
        sc = torch.from_numpy(scales_of(w)).to(dev)
        ws = workspace(pool, 16)
        bad = [
            ([0, 2], [0, 256], L.LORA_ERR_INVALID_ARG),       # d_out differs
            ([0, 1], [0, 128], L.LORA_ERR_INVALID_ARG),       # slices overlap
            ([0, 1], [0, 900], L.LORA_ERR_INVALID_ARG),       # slice past ldy
            ([0, 1], [0, 260], L.LORA_ERR_ALIGNMENT),         # not a multiple of 8
            ([0, 1, 0, 1, 0], [0, 256, 512, 768, 0], L.LORA_ERR_INVALID_ARG),  # more than 4
            ([0, 7], [0, 256], L.LORA_ERR_INVALID_ARG),       # no such target
        ]
        for targets, cols, code in bad:
            with pytest.raises(L.LoraError) as e:
                L.lora_apply_multi(pool.pool, targets, x, y, cols, ids, sc, ws)
            assert e.value.code == code, (targets, cols)
