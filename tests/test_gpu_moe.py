"""The delta inside expert routing (lora_apply_moe): every (token, chosen
expert) pair p = t * top_k + j adds the delta of slot
adapter(t) * n_experts + expert(p), computed from the token's x row, to the
pair's own output row.  Compared element by element with the oracle's
moe_lora_apply (with the output rows at zero as well, so the delta is
checked on its own scale), bit for bit with lora_apply on x rows repeated
per pair, for the one-launch path (up to 256 pairs) and the planned path,
with tokens without adapter, bad adapter / expert ids and empty slots."""

import numpy as np
import pytest
import torch

import adapter_deltas_b200 as L
import oracle
import synth
from gpu_harness import DevicePool, assert_close, scales_of, to_dev_bf16, to_host_bits

pytestmark = pytest.mark.gpu


def _routing(seed, T, k, E, n_ad, none_frac=0.15):
    """Each token's adapter (some none) and k distinct experts per token."""
    g = np.random.default_rng(seed)
    lora = g.integers(0, n_ad, size=T).astype(np.int32)
    lora[g.random(T) < none_frac] = -1
    topk = np.stack([g.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    return lora, topk


def _workload(seed, T, k, E, n_ad, d_in, d_out, r_max=16, **kw):
    ranks = [int(r) for r in np.random.default_rng(seed + 1).choice([4, 8, 16], size=n_ad * E)]
    ranks = [min(r, r_max) for r in ranks]
    return synth.custom(seed, T, [(d_in, d_out)], ranks, r_max, **kw)


def _y_pairs(seed, n_pairs, d_out):
    return synth.normal_bf16(np.random.default_rng(seed), (n_pairs, d_out), 1.0)


def _run(pool, x_bits, y_bits, lora, topk, E):
    dev = pool.device
    x = to_dev_bf16(x_bits, dev)
    y = to_dev_bf16(y_bits, dev)
    sc = torch.from_numpy(scales_of(pool.w)).to(dev)
    lo = torch.from_numpy(lora).to(dev)
    tk = torch.from_numpy(np.ascontiguousarray(topk)).to(dev)
    ws = torch.zeros(max(256, L.lora_moe_workspace_bytes(pool.pool, 0, topk.size)), dtype=torch.uint8, device=dev)
    n0 = L.lora_kernel_launches()
    L.lora_apply_moe(pool.pool, 0, x, y, lo, tk, E, sc, ws)
    launches = L.lora_kernel_launches() - n0
    torch.cuda.synchronize(dev)
    return to_host_bits(y), launches, L.lora_get_error(pool.pool)


def _oracle(w, x_bits, y_bits, lora, topk, E):
    slots = oracle.moe_pair_slots(lora, topk, E, w.n_slots)
    used = [int(s) for s in np.unique(slots) if 0 <= s < w.n_slots and w.rank[s] > 0]
    return oracle.moe_lora_apply(x_bits, y_bits, lora, topk, E, w.n_slots,
                                 {s: w.adapter(s, 0) for s in used}, w.alpha, threads=8)


@pytest.mark.parametrize("T,k,E,n_ad", [(64, 2, 8, 4), (32, 4, 32, 2), (1, 1, 4, 3), (200, 2, 8, 4), (150, 4, 16, 3)])
def test_moe_matches_oracle(cuda_device, T, k, E, n_ad):
    d_in, d_out = 1024, 512
    w = _workload(100 + T, T, k, E, n_ad, d_in, d_out)
    lora, topk = _routing(200 + T, T, k, E, n_ad)
    y0 = _y_pairs(300 + T, T * k, d_out)
    with DevicePool(w, cuda_device) as pool:
        got, launches, st = _run(pool, w.x(0), y0, lora, topk, E)
        assert st == L.LORA_OK
        assert launches == (1 if T * k <= 256 else 3)
        ref, bad = _oracle(w, w.x(0), y0, lora, topk, E)
        assert bad == 0
        assert_close(got, ref, what="T=%d k=%d" % (T, k))
        none = np.repeat(lora < 0, k)
        assert np.array_equal(got[none], y0[none])
        # the delta alone
        z = np.zeros_like(y0)
        got0, _, _ = _run(pool, w.x(0), z, lora, topk, E)
        ref0, _ = _oracle(w, w.x(0), z, lora, topk, E)
        assert_close(got0, ref0, what="delta alone T=%d k=%d" % (T, k))


@pytest.mark.parametrize("T,k", [(48, 2), (160, 2)])
def test_moe_equals_lora_apply_on_repeated_rows(cuda_device, T, k):
    E, n_ad, d = 8, 4, 512
    w = _workload(400 + T, T * k, k, E, n_ad, d, d)      # x rows for the repeated form
    lora, topk = _routing(500 + T, T, k, E, n_ad)
    x_tok = w.x(0)[:T]
    y0 = _y_pairs(600 + T, T * k, d)
    with DevicePool(w, cuda_device) as pool:
        got, _, st = _run(pool, x_tok, y0, lora, topk, E)
        assert st == L.LORA_OK
        dev = pool.device
        x_rep = to_dev_bf16(np.repeat(x_tok, k, axis=0), dev)
        y = to_dev_bf16(y0, dev)
        ids = torch.from_numpy(oracle.moe_pair_slots(lora, topk, E, w.n_slots)).to(dev)
        ws = torch.zeros(L.lora_workspace_bytes(pool.pool, 0, T * k), dtype=torch.uint8, device=dev)
        L.lora_apply(pool.pool, 0, x_rep, y, ids, torch.from_numpy(scales_of(w)).to(dev), ws)
        torch.cuda.synchronize(dev)
        assert np.array_equal(got, to_host_bits(y))


def test_moe_bad_ids_and_empty_slots(cuda_device):
    T, k, E, n_ad, d = 24, 2, 4, 3, 256
    w = _workload(700, T, k, E, n_ad, d, d)
    lora, topk = _routing(701, T, k, E, n_ad, none_frac=0.0)
    y0 = _y_pairs(702, T * k, d)
    bad_lora, bad_topk = lora.copy(), topk.copy()
    bad_topk[3, 1] = E            # expert out of range
    bad_lora[5] = -3              # adapter id below -1
    bad_lora[7] = n_ad            # slot past the pool
    with DevicePool(w, cuda_device) as pool:
        got, _, st = _run(pool, w.x(0), y0, bad_lora, bad_topk, E)
        assert st == L.LORA_ERR_BAD_ID
        for p in (3 * k + 1, 5 * k, 5 * k + 1, 7 * k, 7 * k + 1):
            assert np.array_equal(got[p], y0[p])
        ref, bad = _oracle(w, w.x(0), y0, bad_lora, bad_topk, E)
        assert bad == 5
        assert_close(got, ref, what="other pairs")
    # slots of adapter 2 empty
    with DevicePool(w, cuda_device, slots=list(range(2 * E))) as pool:
        got, _, st = _run(pool, w.x(0), y0, lora, topk, E)
        assert st == L.LORA_ERR_NOT_LOADED
        empty = np.repeat(lora == 2, k)
        assert empty.any() and np.array_equal(got[empty], y0[empty])
        kept = lora.copy()
        kept[lora == 2] = -1
        ref, _ = _oracle(w, w.x(0), y0, kept, topk, E)
        assert_close(got, ref, what="loaded slots")
