"""The projection layer with its delta fused (lora_linear): y = x W^T + each
row's s_a B_a (A_a x), written once.  Compared element by element with the
fp64 oracle's whole layer (oracle.lora_linear), with each term isolated
(W = 0 leaves the delta alone; no adapters leave the base alone), over ragged
shapes that leave partial feature tiles, partial token tiles and a partial
last block of d_in, strided operands, a paged pool, bad ids and empty
slots."""

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import oracle
import synth
from gpu_harness import DevicePool, assert_close, scales_of, to_dev_bf16, to_host_bits

pytestmark = pytest.mark.gpu


def _ws(pool, T):
    n = max(L.lora_linear_workspace_bytes(pool.pool, t, T) for t in range(len(pool.w.targets)))
    return torch.zeros(n, dtype=torch.uint8, device=pool.device)


def _run(pool, target, x_bits, W_bits, ids, pad=(0, 0, 0), y_fill=0x7fc0):
    """lora_linear on the GPU; returns (y bits, launches, status).  pad adds
    columns to the leading dimensions of x, W and y; y starts as y_fill
    (bf16 NaN) so that any element the call fails to write shows."""
    dev = pool.device
    T, d_in = x_bits.shape
    d_out = W_bits.shape[0]
    px, pw, py = pad
    x = torch.zeros(T, d_in + px, dtype=torch.bfloat16, device=dev)
    x[:, :d_in] = to_dev_bf16(x_bits, dev)
    W = torch.zeros(d_out, d_in + pw, dtype=torch.bfloat16, device=dev)
    W[:, :d_in] = to_dev_bf16(W_bits, dev)
    y = torch.full((T, d_out + py), y_fill, dtype=torch.int16, device=dev).view(torch.bfloat16)
    sc = torch.from_numpy(scales_of(pool.w)).to(dev)
    d_ids = torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32)).to(dev)
    ws = _ws(pool, T)
    n0 = L.lora_kernel_launches()
    L.lora_linear(pool.pool, target, x[:, :d_in], W[:, :d_in], y[:, :d_out], d_ids, sc, ws)
    launches = L.lora_kernel_launches() - n0
    torch.cuda.synchronize(dev)
    status = L.lora_get_error(pool.pool)
    out = to_host_bits(y)
    if py:
        # columns past d_out are never written
        assert np.all(out[:, d_out:] == np.uint16(y_fill))
    return out[:, :d_out], launches, status


def _oracle(w, target, x_bits, W_bits, ids, threads=16):
    slots = [int(s) for s in np.unique(ids[ids >= 0]) if s < w.n_slots and w.rank[s] > 0]
    adapters = {s: w.adapter(s, target) for s in slots}
    return oracle.lora_linear(x_bits, W_bits, ids, w.n_slots, adapters, w.alpha, threads=threads)


def _check_both_terms(pool, w, target, ids, what, pad=(0, 0, 0)):
    x, W = w.x(target), w.W(target)
    got, launches, st = _run(pool, target, x, W, ids, pad)
    assert st == L.LORA_OK
    ref, _ = _oracle(w, target, x, W, ids)
    assert_close(got, ref, what=what)
    # the delta alone (W = 0): its own scale, so a wrong delta cannot hide
    # under the base term
    zero = np.zeros_like(W)
    got0, _, _ = _run(pool, target, x, zero, ids, pad)
    slots = [int(s) for s in np.unique(ids[ids >= 0]) if s < w.n_slots and w.rank[s] > 0]
    ref0, _ = oracle.lora_apply(x, np.zeros((x.shape[0], W.shape[0])), ids, w.n_slots,
                                {s: w.adapter(s, target) for s in slots}, w.alpha, threads=16)
    if np.abs(ref0).max() > 0:
        assert_close(got0, ref0, what=what + " (delta alone)")
    return launches


@pytest.mark.parametrize("cfg", [1, 2])
def test_linear_matches_oracle_on_configs(cuda_device, cfg):
    w = synth.config(cfg)
    with DevicePool(w, cuda_device) as pool:
        for t in range(len(w.targets)):
            n = _check_both_terms(pool, w, t, w.ids, "config %d target %d" % (cfg, t))
            assert n == 2


def test_linear_mixed_ranks_up_to_64_mlp_shapes(cuda_device):
    # 4096 -> 11008 and 11008 -> 4096, ranks 8..64 (up to four delta steps
    # of 16 ranks per adapter), 10 % of rows without an adapter
    w = synth.config(4)
    with DevicePool(w, cuda_device) as pool:
        for t in range(len(w.targets)):
            _check_both_terms(pool, w, t, w.ids, "config 4 target %d" % t)


@pytest.mark.parametrize("T", [1, 17, 100, 256, 300, 600])
def test_linear_ragged_shapes(cuda_device, T):
    # d_in 320 (five 64-wide blocks: splits of unequal length), d_out 200
    # (a partial feature tile), ranks 4 / 13 / 16 / 20 (chunks of 16 cut
    # short), rows without adapter
    rng = np.random.default_rng(T)
    ids = rng.integers(-1, 4, size=T).astype(np.int32)
    w = synth.custom(60 + T, T, [(320, 200)], [4, 13, 16, 20], 32, ids=ids)
    with DevicePool(w, cuda_device) as pool:
        n = _check_both_terms(pool, w, 0, ids, "T=%d" % T)
        assert n == (2 if T <= 256 else 3)


def test_linear_without_adapters_is_the_base(cuda_device):
    w = synth.custom(71, 96, [(512, 384)], [8, 16], 16)
    ids = np.full(96, -1, np.int32)
    with DevicePool(w, cuda_device) as pool:
        x, W = w.x(0), w.W(0)
        got, _, st = _run(pool, 0, x, W, ids)
        assert st == L.LORA_OK
        assert_close(got, oracle.linear(x, W, threads=8), what="base alone")


def test_linear_strided_operands_and_paged_pool(cuda_device):
    # leading dimensions past the widths; 4 KiB pages scattered through the
    # pool, so B^T rows of one chunk sit on different pages
    w = synth.custom(72, 48, [(256, 512), (384, 256)], [16, 8, 12, 16, 4, 16], 16, page_bytes=4096,
                     scatter_seed=99)
    with DevicePool(w, cuda_device) as pool:
        for t in range(2):
            _check_both_terms(pool, w, t, w.ids, "strided target %d" % t, pad=(8, 24, 16))


def test_linear_bad_ids_and_empty_slots_get_the_base(cuda_device):
    w = synth.custom(73, 40, [(256, 256)], [8, 8, 8, 8], 8)
    ids = w.ids.copy()
    ids[5] = 99
    ids[9] = -4
    x, W = w.x(0), w.W(0)
    base = oracle.linear(x, W)
    with DevicePool(w, cuda_device) as pool:
        got, _, st = _run(pool, 0, x, W, ids)
        assert st == L.LORA_ERR_BAD_ID
        assert_close(got[[5, 9]], base[[5, 9]], what="bad-id rows")
        good = ids.copy()
        good[[5, 9]] = -1
        ref, _ = _oracle(w, 0, x, W, good)
        assert_close(got, ref, what="the other rows")
    with DevicePool(w, cuda_device, slots=[0, 1]) as pool:
        got, _, st = _run(pool, 0, x, W, w.ids)
        assert st == L.LORA_ERR_NOT_LOADED
        empty = (w.ids == 2) | (w.ids == 3)
        assert_close(got[empty], base[empty], what="empty-slot rows")
        kept = w.ids.copy()
        kept[empty] = -1
        ref, _ = _oracle(w, 0, x, W, kept)
        assert_close(got, ref, what="loaded-slot rows")


def test_linear_rejects_bad_arguments(cuda_device):
    w = synth.custom(74, 16, [(256, 256)], [8, 8], 8)
    with DevicePool(w, cuda_device) as pool:
        dev = pool.device
        x = to_dev_bf16(w.x(0), dev)
        W = to_dev_bf16(w.W(0), dev)
        y = torch.zeros(16, 256, dtype=torch.bfloat16, device=dev)
        ids = torch.from_numpy(w.ids).to(dev)
        sc = torch.from_numpy(scales_of(w)).to(dev)
        ws = _ws(pool, 16)
        cases = [
            (lambda: L.lora_linear(pool.pool, 0, x, W, x, ids, sc, ws), L.LORA_ERR_INVALID_ARG),   # y is x
            (lambda: L.lora_linear(pool.pool, 0, x, W, W[:16], ids, sc, ws), L.LORA_ERR_INVALID_ARG),  # y in W
            (lambda: L.lora_linear(pool.pool, 0, x, W, y, ids, sc, ws[:256]), L.LORA_ERR_WORKSPACE),
            (lambda: L.lora_linear(pool.pool, 3, x, W, y, ids, sc, ws), L.LORA_ERR_INVALID_ARG),
        ]
        for fn, code in cases:
            with pytest.raises(L.LoraError) as e:
                fn()
            assert e.value.code == code


@pytest.mark.parametrize("T", [64, 300])
def test_shrink_then_linear_expand_equals_linear(cuda_device, T):
    w = synth.custom(75 + T, T, [(512, 640)], [16, 8, 12, 16, 4, 16], 16)
    with DevicePool(w, cuda_device) as pool:
        dev = pool.device
        x = to_dev_bf16(w.x(0), dev)
        W = to_dev_bf16(w.W(0), dev)
        ids = torch.from_numpy(w.ids).to(dev)
        sc = torch.from_numpy(scales_of(w)).to(dev)
        ws = _ws(pool, T)
        y1 = torch.empty(T, 640, dtype=torch.bfloat16, device=dev)
        y2 = torch.empty_like(y1)
        L.lora_linear(pool.pool, 0, x, W, y1, ids, sc, ws)
        v = torch.zeros(T, w.r_max + 8, dtype=torch.float32, device=dev)   # ldv past r_max
        L.lora_shrink(pool.pool, 0, x, ids, v, ws)
        n0 = L.lora_kernel_launches()
        L.lora_linear_expand(pool.pool, 0, x, W, v, y2, ids, sc)
        assert L.lora_kernel_launches() - n0 == 1
        torch.cuda.synchronize(dev)
        assert L.lora_get_error(pool.pool) == L.LORA_OK
        assert np.array_equal(to_host_bits(y1), to_host_bits(y2))
