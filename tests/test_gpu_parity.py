"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs.

Float results: max |y_gpu - y_ref| <= 4e-3 * max |y_ref|, both with the base
output y = xW and with y = 0 (which isolates the delta, so a wrong delta
cannot hide under the base term).  Rows without an adapter: bitwise
unchanged.  Small-integer cases: exact (every fp32 partial sum is an exact
integer, so the only rounding is the final bf16 store).
"""

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import oracle
import synth
from gpu_harness import (DevicePool, assert_close, oracle_y, run_gpu, scales_of, to_dev_bf16,
                         to_host_bits, workspace)

pytestmark = pytest.mark.gpu


def _check_call(pool, w, target, ids, api="ids", scales=None, alpha=None, zero_y=False):
    x = w.x(target)
    y = np.zeros_like(w.y_in(target)) if zero_y else w.y_in(target)
    got = run_gpu(pool, target, x, y, ids, scales=scales, api=api)
    ref, bad = oracle_y(w, target, x, y, ids, alpha=alpha)
    assert bad == 0
    err = assert_close(got, ref, what="%s target %d api %s y0=%s" % (w.name, target, api, zero_y))
    none = ids < 0
    assert np.array_equal(got[none], y[none]), "rows without adapter must be untouched"
    return got, err


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_decode_configs(cuda_device, cfg):
    w = synth.config(cfg)
    with DevicePool(w, cuda_device) as pool:
        for t in range(len(w.targets)):
            _check_call(pool, w, t, w.ids)
            _check_call(pool, w, t, w.ids, zero_y=True)


def test_segmented_prefill_config(cuda_device):
    w = synth.config(3)
    with DevicePool(w, cuda_device) as pool:
        g1, _ = _check_call(pool, w, 0, w.ids, api="segments")
        _check_call(pool, w, 0, w.ids, api="segments", zero_y=True)
        g2, _ = _check_call(pool, w, 0, w.ids, api="ids")
        assert np.abs(oracle.bf16_to_f64(g1) - oracle.bf16_to_f64(g2)).max() <= 4e-3 * np.abs(
            oracle.bf16_to_f64(g2)).max()


def test_split_shrink_expand_is_bit_identical_to_apply(cuda_device):
    for cfg in (2, 4):
        w = synth.config(cfg)
        with DevicePool(w, cuda_device) as pool:
            for t in range(len(w.targets)):
                a = run_gpu(pool, t, w.x(t), w.y_in(t), w.ids, api="ids")
                b = run_gpu(pool, t, w.x(t), w.y_in(t), w.ids, api="split")
                assert np.array_equal(a, b)


def test_shrink_v_matches_oracle(cuda_device):
    w = synth.config(4)
    dev = cuda_device
    with DevicePool(w, dev) as pool:
        for t in range(2):
            x = to_dev_bf16(w.x(t), dev)
            ids = torch.from_numpy(w.ids).to(dev)
            v = torch.full((w.T, w.r_max), 7.0, dtype=torch.float32, device=dev)
            L.lora_shrink(pool.pool, t, x, ids, v, workspace(pool, w.T))
            vg = v.cpu().numpy().astype(np.float64)
            slots = [int(s) for s in w.active_slots]
            _, _, vr = oracle.lora_apply(w.x(t), w.y_in(t), w.ids, w.n_slots,
                                         {s: w.adapter(s, t) for s in slots}, w.alpha, want_v=True)
            act = w.ids >= 0
            assert np.all(vg[~act] == 7.0), "rows without adapter keep v"
            scale = np.abs(vr[act]).max()
            assert np.abs(vg[act] - vr[act][:, :w.r_max]).max() <= 1e-5 * scale
            for row in np.nonzero(act)[0]:
                r = w.rank[w.ids[row]]
                assert np.all(vg[row, r:] == 0.0)


def test_expand_with_given_v_matches_oracle(cuda_device):
    w = synth.config(1)
    dev = cuda_device
    g = np.random.default_rng(5)
    vh = g.standard_normal((w.T, w.r_max)).astype(np.float32)
    with DevicePool(w, dev) as pool:
        y = to_dev_bf16(w.y_in(0), dev)
        L.lora_expand(pool.pool, 0, torch.from_numpy(vh).to(dev), y, torch.from_numpy(w.ids).to(dev),
                      torch.from_numpy(scales_of(w)).to(dev), workspace(pool, w.T))
        got = to_host_bits(y)
    Bs = {s: w.adapter(s, 0)[1] for s in range(w.n_slots)}
    ref, bad = oracle.lora_expand(vh.astype(np.float64), w.y_in(0), w.ids, w.n_slots, Bs, w.alpha)
    assert bad == 0
    assert_close(got, ref, what="expand")


def test_distinct_scales_route_per_slot(cuda_device):
    # every slot its own scale 0.5 + a/8: a routing mistake shows up
    w = synth.config(2)
    alpha = (0.5 + np.arange(w.n_slots) / 8.0) * w.rank
    scales = (alpha / w.rank).astype(np.float32)
    with DevicePool(w, cuda_device) as pool:
        _check_call(pool, w, 0, w.ids, scales=scales, alpha=alpha, zero_y=True)


@pytest.mark.parametrize("case", [
    dict(T=8, d_in=64, d_out=48, ranks=[1, 8, 3, 8], r_max=8, e=[0, 1, -1, 2]),
    dict(T=5, d_in=24, d_out=40, ranks=[2, 5], r_max=8, e=[1, 0]),
    dict(T=37, d_in=520, d_out=264, ranks=[8, 1, 7, 4, 6], r_max=8, e=[0, 0, 1, -2, 3]),
    dict(T=19, d_in=64, d_out=64, ranks=[64, 33, 17, 64], r_max=64, e=[-3, -2, -1, -4]),
])
def test_integer_cases_are_exact(cuda_device, case):
    w = synth.integer_case(7, case["T"], case["d_in"], case["d_out"], case["ranks"], case["r_max"], case["e"])
    with DevicePool(w, cuda_device) as pool:
        for api in ("ids", "split"):
            got = run_gpu(pool, 0, w.x(0), w.y_in(0), w.ids, api=api)
            ref, bad = oracle_y(w, 0, w.x(0), w.y_in(0), w.ids)
            want = synth.f32_to_bf16_bits(ref.astype(np.float32))  # exact value, rounded once
            assert np.array_equal(ref, ref.astype(np.float32).astype(np.float64)), "case must stay exact in fp32"
            assert np.array_equal(got, want), api


def test_paged_scattered_pool_is_bit_identical_to_contiguous(cuda_device):
    w = synth.config(2)
    a = DevicePool(w, cuda_device)
    b = DevicePool(w, cuda_device, page_bytes=4096, scatter_seed=99)
    try:
        info = L.lora_pool_get_info(b.pool)
        assert info.pages_per_slot == 64
        ya = run_gpu(a, 0, w.x(0), w.y_in(0), w.ids)
        yb = run_gpu(b, 0, w.x(0), w.y_in(0), w.ids)
        assert np.array_equal(ya, yb)
    finally:
        a.close()
        b.close()


def test_row_permutation_is_bit_invariant(cuda_device):
    w = synth.config(4)
    p = np.random.default_rng(3).permutation(w.T)
    with DevicePool(w, cuda_device) as pool:
        for t in range(2):
            y1 = run_gpu(pool, t, w.x(t), w.y_in(t), w.ids)
            y2 = run_gpu(pool, t, w.x(t)[p], w.y_in(t)[p], w.ids[p])
            assert np.array_equal(y2, y1[p])


def test_single_adapter_and_all_none_and_tiny(cuda_device):
    w = synth.config(1)
    with DevicePool(w, cuda_device) as pool:
        _check_call(pool, w, 0, np.full(w.T, 2, np.int32))            # one adapter for the whole batch
        y = run_gpu(pool, 0, w.x(0), w.y_in(0), np.full(w.T, -1, np.int32))
        assert np.array_equal(y, w.y_in(0))                             # no adapter at all
        for T in (1, 2, 3):
            ids = np.array([3, 0, 3][:T], np.int32)
            got = run_gpu(pool, 0, w.x(0)[:T], w.y_in(0)[:T], ids)
            ref, _ = oracle_y(w, 0, w.x(0)[:T], w.y_in(0)[:T], ids)
            assert_close(got, ref, what="T=%d" % T)


def test_long_segments_split_into_items(cuda_device):
    # 100 rows of one adapter plus a few others: the long group spans many items
    w = synth.config(2)
    ids = np.concatenate([np.full(100, 5), np.arange(8) % 3, [-1, 7]]).astype(np.int32)
    ids = ids[np.random.default_rng(1).permutation(ids.size)]
    T = ids.size
    x = np.concatenate([w.x(0)] * 2)[:T]
    y = np.concatenate([w.y_in(0)] * 2)[:T]
    with DevicePool(w, cuda_device) as pool:
        got = run_gpu(pool, 0, x, y, ids)
        ref, _ = oracle_y(w, 0, x, y, ids)
        assert_close(got, ref)


def test_bad_ids_leave_rows_and_set_sticky_status(cuda_device):
    w = synth.config(1)
    ids = w.ids.copy()
    ids[[1, 5]] = [7, -4]
    with DevicePool(w, cuda_device) as pool:
        assert L.lora_get_error(pool.pool) == L.LORA_OK
        got = run_gpu(pool, 0, w.x(0), w.y_in(0), ids)
        assert L.lora_get_error(pool.pool) == L.LORA_ERR_BAD_ID
        assert L.lora_get_error(pool.pool) == L.LORA_OK            # read clears it
        assert np.array_equal(got[[1, 5]], w.y_in(0)[[1, 5]])
        good = ids.copy()
        good[[1, 5]] = -1
        ref, _ = oracle_y(w, 0, w.x(0), w.y_in(0), good)
        assert_close(got, ref)


def test_config5_paged_full_step(cuda_device):
    """The paged-pool workload at full size: 1000 slots x 128 matrices in 1 MiB
    scattered pages (31.25 GiB), one 512-token step over all 128 matrices in
    the configuration the benchmark times; sampled matrices checked against the
    oracle on every row."""
    w = synth.config(5)
    dev = cuda_device
    active = [int(s) for s in w.active_slots]
    others = [s for s in range(w.n_slots) if s not in set(active)]
    with DevicePool(w, dev, slots=active, filler_slots=others) as pool:
        info = L.lora_pool_get_info(pool.pool)
        assert info.pages_per_slot == 32 and info.free_pages == 0
        T = w.T
        ids = torch.from_numpy(w.ids).to(dev)
        sc = torch.from_numpy(scales_of(w)).to(dev)
        ws = workspace(pool, T)
        L.lora_plan_ids(pool.pool, ids, ws)
        sample = [0, 1, 37, 90, 127]
        ys = {}
        xs = {}
        for t in range(128):
            xs[t] = to_dev_bf16(w.x(t), dev) if t in sample else torch.randn(T, 4096, device=dev).to(torch.bfloat16)
            ys[t] = to_dev_bf16(w.y_in(t), dev) if t in sample else torch.randn(T, 4096, device=dev).to(torch.bfloat16)
        for t in range(128):
            L.lora_apply_plan(pool.pool, t, xs[t], ys[t], sc, ws)
        torch.cuda.synchronize(dev)
        assert L.lora_get_error(pool.pool) == L.LORA_OK
        for t in sample:
            ref, _ = oracle_y(w, t, w.x(t), w.y_in(t), w.ids)
            assert_close(to_host_bits(ys[t]), ref, what="target %d" % t)
    w.drop()
