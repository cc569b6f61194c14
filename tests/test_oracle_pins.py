"""Pins for the CPU oracle: each test checks it against something other than
itself -- a value the pages print, a closed-form identity, a library routine
on a special case, or exact brute force on tiny inputs.  No GPU needed.

Passages (pages on multi-LoRA serving):
  merge form W' = W + BA and the row form y = xW + (x A_i) B_i alpha/r:
    "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU", "Why can't you just
    merge LoRA weights into the base model?"; "Serving Many LoRA Adapters From
    One Base Model", "Going deeper" (merging vs keeping adapters separate).
  shapes and sizing: first page, "How much memory does one LoRA adapter
    actually cost?" and its TL;DR.
  one adapter vs many is the same kernel with another index vector: first page,
    "How does one batch run 30 different adapters at once?".
  adapter=None keeps the base output: second page, worked example.
"""

import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=", 1)
            vals[k] = v
    return vals


def _rand_case(seed, T, d_in, d_out, ranks, alphas, none_frac=0.25):
    g = np.random.default_rng(seed)
    x = g.standard_normal((T, d_in))
    W = g.standard_normal((d_out, d_in)) / np.sqrt(d_in)
    y_in = x @ W.T
    adapters = {}
    for a, r in enumerate(ranks):
        adapters[a] = (g.standard_normal((r, d_in)) / np.sqrt(d_in),
                       g.standard_normal((d_out, r)) * 0.14)
    ids = g.integers(0, len(ranks), size=T).astype(np.int32)
    ids[g.random(T) < none_frac] = -1
    return x, W, y_in, adapters, ids, np.asarray(alphas, dtype=np.float64)


# ---------------------------------------------------------------- sizing


def test_sizing_matches_printed_example():
    g = _golden("lora_sizing.txt")
    h = int(g["hidden"])
    params = oracle.lora_params(((h, h),) * int(g["targets"]), int(g["layers"]), int(g["rank"]))
    nbytes = params * int(g["dtype_bytes"])
    assert f"{params / 1e6:.1f}M params, {nbytes / 2**20:.1f} MiB" == g["printed"]
    # closed form: 16 * 8192 * 4 * 32 = 2^24 parameters, exactly 32 MiB
    assert params == 2 ** 24 and nbytes == 32 * 2 ** 20
    assert nbytes // 10**6 == int(g["approx_fp16_MB"])          # 33.55 MB, "~33 MB"
    assert round(100.0 * params / 7e9, 2) == float(g["share_of_7B_base_percent"])


def test_sizing_scales_with_rank_and_targets():
    att = ((4096, 4096),) * 4
    base = oracle.lora_params(att, 32, 16)
    assert oracle.lora_params(att, 32, 32) == 2 * base           # doubling rank doubles bytes
    assert oracle.lora_params(att * 2, 32, 16) == 2 * base       # twice the matrices
    assert oracle.lora_params(((4096, 4096),), 1, 1) == 8192     # r (d_in + d_out)
    assert oracle.lora_params(((3, 5),), 1, 1) == 8              # A 1 x 3, B 5 x 1
    assert oracle.lora_params(((3, 5),), 7, 2) == 7 * 2 * 8       # linear in layers and rank


def test_sizing_of_the_mlp_projections():
    # The same page adds gate/up/down (d_ff = 11008 on Llama-2-7B): each of
    # those matrices is r (4096 + 11008) parameters.  The page calls the
    # result roughly 4x the attention-only adapter; r (d_in + d_out) gives
    # (4 * 8192 + 3 * 15104) / (4 * 8192) = 2.38x -- the formula decides.
    att = ((4096, 4096),) * 4
    mlp = ((4096, 11008), (4096, 11008), (11008, 4096))
    assert oracle.lora_params(mlp, 1, 16) == 3 * 16 * 15104
    both = oracle.lora_params(att + mlp, 32, 16)
    assert both == 32 * 16 * (4 * 8192 + 3 * 15104)
    assert round(both / oracle.lora_params(att, 32, 16), 2) == 2.38


def test_slot_layout_of_the_paged_geometry_is_the_adapter_size():
    # 32 layers x q/k/v/o at hidden 4096, rank 16: one slot is exactly the
    # printed adapter size, and each target block starts 256 KiB after the last.
    a_off, bt_off, total = oracle.slot_layout([(4096, 4096)] * 128, 16)
    assert total == oracle.lora_params(((4096, 4096),) * 4, 32, 16) * 2
    assert np.array_equal(a_off, np.arange(128) * 256 * 1024)
    assert np.array_equal(bt_off, np.arange(128) * 256 * 1024 + 128 * 1024)


def test_slot_layout_rounds_blocks_to_256_bytes():
    a_off, bt_off, total = oracle.slot_layout([(8, 16), (24, 8)], 1)
    # A 1x8 bf16 = 16 B -> 256; B^T 1x16 = 32 B -> 256; A 1x24 = 48 -> 256; B^T 16 -> 256
    assert list(a_off) == [0, 512] and list(bt_off) == [256, 768] and total == 1024


# ---------------------------------------------------------------- delta math


def test_merge_equivalence():
    # x (W + (alpha/r) B A)^T  ==  x W^T + (alpha/r) B (A x), row by row
    x, W, y_in, adapters, ids, alpha = _rand_case(1, 13, 24, 40, [3, 5, 1], [6.0, 2.5, 7.0])
    y, bad = oracle.lora_apply(x, y_in, ids, 3, adapters, alpha)
    assert bad == 0
    for t in range(x.shape[0]):
        a = ids[t]
        if a < 0:
            ref = x[t] @ W.T
        else:
            A, B = adapters[a]
            Wm = W + (alpha[a] / A.shape[0]) * (B @ A)
            ref = x[t] @ Wm.T
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_none_rows_are_bitwise_unchanged_and_zero_B_is_numerically_unchanged():
    x, W, y_in, adapters, ids, alpha = _rand_case(2, 16, 8, 8, [2, 2], [4.0, 4.0], none_frac=0.5)
    y, _ = oracle.lora_apply(x, y_in, ids, 2, adapters, alpha)
    none = ids == -1
    assert none.any()
    assert np.array_equal(y[none].view(np.uint64), y_in[none].view(np.uint64))
    zeroB = {a: (A, np.zeros_like(B)) for a, (A, B) in adapters.items()}
    y0, _ = oracle.lora_apply(x, y_in, ids, 2, zeroB, alpha)
    assert np.array_equal(y0, y_in)


def test_single_adapter_batch_equals_dense_gemm():
    # one adapter for every row: X (s B A)^T + Y_in by a library matmul
    x, W, y_in, adapters, ids, alpha = _rand_case(3, 32, 48, 20, [6], [12.0], none_frac=0.0)
    y, _ = oracle.lora_apply(x, y_in, np.zeros(32, np.int32), 1, adapters, alpha)
    A, B = adapters[0]
    dW = (alpha[0] / 6) * (B @ A)
    ref = y_in + x @ dW.T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_row_permutation_invariance():
    x, W, y_in, adapters, ids, alpha = _rand_case(4, 21, 16, 12, [4, 2, 3], [1.0, 2.0, 3.0])
    y, _ = oracle.lora_apply(x, y_in, ids, 3, adapters, alpha)
    p = np.random.default_rng(9).permutation(21)
    yp, _ = oracle.lora_apply(x[p], y_in[p], ids[p], 3, adapters, alpha)
    assert np.array_equal(yp, y[p])


def test_linearity_in_scale():
    # with a zero base output the result is the delta alone: doubling alpha
    # (a power of two) doubles every delta exactly
    x, W, y_in, adapters, ids, alpha = _rand_case(5, 9, 16, 16, [4, 4], [3.0, 5.0], none_frac=0.0)
    zero = np.zeros_like(y_in)
    d1, _ = oracle.lora_apply(x, zero, ids, 2, adapters, alpha)
    d2, _ = oracle.lora_apply(x, zero, ids, 2, adapters, 2 * alpha)
    assert np.array_equal(d2, 2 * d1) and np.abs(d1).max() > 0


def test_integer_brute_force_exact():
    # tiny integer case, every value computed with Python fractions
    g = np.random.default_rng(6)
    T, d_in, d_out = 6, 5, 7
    ranks = [1, 3, 2]
    alpha = [2.0, 6.0, 1.0]
    x = g.integers(-3, 4, size=(T, d_in)).astype(np.float64)
    y_in = g.integers(-9, 10, size=(T, d_out)).astype(np.float64)
    adapters = {a: (g.integers(-2, 3, size=(r, d_in)).astype(np.float64),
                    g.integers(-2, 3, size=(d_out, r)).astype(np.float64))
                for a, r in enumerate(ranks)}
    ids = np.array([0, 2, -1, 1, 1, 0], dtype=np.int32)
    y, bad = oracle.lora_apply(x, y_in, ids, 3, adapters, alpha)
    assert bad == 0
    for t in range(T):
        a = ids[t]
        for n in range(d_out):
            ref = Fraction(int(y_in[t, n]))
            if a >= 0:
                A, B = adapters[a]
                r = ranks[a]
                s = Fraction(int(alpha[a]), r)
                acc = Fraction(0)
                for q in range(r):
                    vq = sum(Fraction(int(x[t, k])) * int(A[q, k]) for k in range(d_in))
                    acc += int(B[n, q]) * vq
                ref += s * acc
            assert Fraction(y[t, n]) == ref, (t, n)


# ---------------------------------------------------------------- base term


def test_linear_is_a_library_matmul():
    # the base term xW against numpy's matmul (W stored d_out x d_in)
    g = np.random.default_rng(11)
    x = g.standard_normal((7, 33))
    W = g.standard_normal((19, 33))
    ref = x @ W.T
    got = oracle.linear(x, W, threads=3)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13 * np.abs(ref).max())
    # a transposed operand would give another shape or other values
    assert got.shape == (7, 19)


def test_linear_integer_brute_force_exact():
    g = np.random.default_rng(12)
    x = g.integers(-4, 5, size=(3, 6)).astype(np.float64)
    W = g.integers(-3, 4, size=(5, 6)).astype(np.float64)
    got = oracle.linear(x, W)
    for t in range(3):
        for n in range(5):
            assert got[t, n] == sum(int(x[t, k]) * int(W[n, k]) for k in range(6))


def test_lora_linear_equals_merged_weight_per_row():
    # the whole layer: row t equals x[t] (W + (alpha_a/r_a) B_a A_a)^T, the
    # merged form, and the plain base for rows without an adapter
    x, W, _, adapters, ids, alpha = _rand_case(13, 17, 24, 40, [3, 5, 1], [6.0, 2.5, 7.0])
    y, bad = oracle.lora_linear(x, W, ids, 3, adapters, alpha, threads=2)
    assert bad == 0
    for t in range(x.shape[0]):
        a = ids[t]
        Wm = W
        if a >= 0:
            A, B = adapters[a]
            Wm = W + (alpha[a] / A.shape[0]) * (B @ A)
        ref = x[t] @ Wm.T
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_lora_linear_without_adapters_is_the_base():
    x, W, _, adapters, ids, alpha = _rand_case(14, 9, 16, 8, [2], [4.0])
    none = np.full(9, -1, np.int32)
    y, bad = oracle.lora_linear(x, W, none, 1, adapters, alpha)
    assert bad == 0 and np.array_equal(y, oracle.linear(x, W))


# ---------------------------------------------------------------- MoE pairs


def test_moe_pair_slots_by_hand():
    lora = np.array([1, -1, 0, 3, -2], np.int32)
    topk = np.array([[2, 0], [1, 1], [3, 1], [0, 2], [1, 1]], np.int32)
    got = oracle.moe_pair_slots(lora, topk, n_experts=4, n_slots=12)
    # token 0: adapter 1 -> slots 6, 4; token 1: none; token 2: adapter 0 ->
    # 3, 1; token 3: adapter 3 -> 12, 14 are past the 12 slots (invalid);
    # token 4: adapter id -2 (invalid)
    assert got.tolist() == [6, 4, -1, -1, 3, 1, 12, 12, 12, 12]


def test_moe_integer_brute_force_exact():
    g = np.random.default_rng(21)
    T, k, E, n_ad, d_in, d_out = 5, 2, 3, 2, 4, 6
    ranks = {}
    adapters = {}
    for a in range(n_ad):
        for e in range(E):
            r = int(g.integers(1, 4))
            s = a * E + e
            ranks[s] = r
            adapters[s] = (g.integers(-2, 3, size=(r, d_in)).astype(np.float64),
                           g.integers(-2, 3, size=(d_out, r)).astype(np.float64))
    alpha = [2.0 * ranks[s] for s in range(n_ad * E)]
    x = g.integers(-3, 4, size=(T, d_in)).astype(np.float64)
    y = g.integers(-9, 10, size=(T * k, d_out)).astype(np.float64)
    lora = np.array([0, 1, -1, 1, 0], np.int32)
    topk = np.array([[0, 2], [1, 0], [2, 1], [2, 1], [1, 2]], np.int32)
    got, bad = oracle.moe_lora_apply(x, y, lora, topk, E, n_ad * E, adapters, alpha)
    assert bad == 0
    for t in range(T):
        for j in range(k):
            p = t * k + j
            for n in range(d_out):
                ref = Fraction(int(y[p, n]))
                if lora[t] >= 0:
                    s = int(lora[t]) * E + int(topk[t, j])
                    A, B = adapters[s]
                    r = ranks[s]
                    acc = Fraction(0)
                    for q in range(r):
                        acc += int(B[n, q]) * sum(int(x[t, c]) * int(A[q, c]) for c in range(d_in))
                    ref += Fraction(int(alpha[s]), r) * acc
                assert Fraction(got[p, n]) == ref, (t, j, n)


def test_moe_one_expert_top1_is_the_plain_delta():
    x, W, y_in, adapters, ids, alpha = _rand_case(22, 11, 16, 12, [3, 5], [6.0, 2.5])
    got, bad = oracle.moe_lora_apply(x, y_in, ids, ids.reshape(-1, 1) * 0, 1, 2, adapters, alpha)
    ref, bad2 = oracle.lora_apply(x, y_in, ids, 2, adapters, alpha)
    assert bad == bad2 == 0 and np.array_equal(got, ref)


def test_unit_vector_expand_is_a_column_of_B():
    # v = e_j  ->  delta = (alpha/r) * column j of B
    g = np.random.default_rng(7)
    B = g.standard_normal((11, 4))
    for j in range(4):
        v = np.zeros((1, 4))
        v[0, j] = 1.0
        y, _ = oracle.lora_expand(v, np.zeros((1, 11)), np.zeros(1, np.int32), 1, {0: B}, [8.0])
        assert np.array_equal(y[0], 2.0 * B[:, j])


def test_v_is_A_times_x():
    g = np.random.default_rng(8)
    x = g.integers(-3, 4, size=(3, 10)).astype(np.float64)
    A = g.integers(-2, 3, size=(4, 10)).astype(np.float64)
    B = g.standard_normal((5, 4))
    _, _, v = oracle.lora_apply(x, np.zeros((3, 5)), np.array([0, -1, 0], np.int32), 1,
                                {0: (A, B)}, [4.0], want_v=True)
    assert np.array_equal(v[0], A @ x[0]) and np.array_equal(v[2], A @ x[2])
    assert np.array_equal(v[1], np.zeros(4))


def test_invalid_ids_leave_rows_and_are_counted():
    x, W, y_in, adapters, ids, alpha = _rand_case(10, 6, 8, 8, [2, 2], [2.0, 2.0], none_frac=0.0)
    # 5 and -3 are out of range; slot 2 holds no adapter (rank 0): unchanged, not invalid
    ids = np.array([0, 5, -3, 1, 2, -1], dtype=np.int32)
    y, bad = oracle.lora_apply(x, y_in, ids, 3, adapters, [2.0, 2.0, 2.0])
    assert bad == 2
    for t in (1, 2, 4, 5):
        assert np.array_equal(y[t], y_in[t])


def test_rank_zero_slot_is_not_adapted():
    x, W, y_in, adapters, ids, alpha = _rand_case(11, 4, 8, 8, [2], [2.0], none_frac=0.0)
    y, bad = oracle.lora_apply(x, y_in, np.zeros(4, np.int32), 1,
                               {0: (np.zeros((0, 8)), np.zeros((8, 0)))}, [2.0])
    assert bad == 0 and np.array_equal(y, y_in)


def test_bf16_decode_is_exact():
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0000, 0x8000, 0x7F7F, 0x0001], dtype=np.uint16)
    want = [1.0, -1.0, 3.140625, 0.0, -0.0, 3.3895313892515355e38, 9.183549615799121e-41]
    assert list(oracle.bf16_to_f64(bits)) == want


# ---------------------------------------------------------------- grouping


@pytest.mark.parametrize("seed,T,n_slots", [(0, 1, 1), (1, 37, 5), (2, 512, 64), (3, 256, 128)])
def test_group_rows_is_a_stable_sort(seed, T, n_slots):
    g = np.random.default_rng(seed)
    ids = g.integers(-1, n_slots, size=T).astype(np.int32)
    perm, seg_start, seg_slot, bad = oracle.group_rows(ids, n_slots)
    rows = [t for t in sorted(range(T), key=lambda t: ids[t]) if ids[t] >= 0]
    assert bad == 0
    assert perm.tolist() == rows
    slots = sorted(set(ids[ids >= 0].tolist()))
    assert seg_slot.tolist() == slots
    for s, slot in enumerate(slots):
        seg = perm[seg_start[s]:seg_start[s + 1]]
        assert seg.tolist() == [t for t in range(T) if ids[t] == slot]


def test_group_rows_edge_cases():
    perm, seg_start, seg_slot, bad = oracle.group_rows(np.full(7, -1, np.int32), 4)
    assert perm.size == 0 and seg_slot.size == 0 and seg_start.tolist() == [0] and bad == 0
    ids = np.array([3, 9, -2, 3, 1], dtype=np.int32)
    valid = np.array([1, 0, 1, 1], dtype=np.uint8)
    perm, seg_start, seg_slot, bad = oracle.group_rows(ids, 4, valid)
    assert bad == 3                          # 9, -2 out of range; slot 1 not valid
    assert perm.tolist() == [0, 3] and seg_slot.tolist() == [3]


# ---------------------------------------------------------------- paging


def test_pool_locate_identity_is_closed_form():
    pt = np.arange(10, dtype=np.int32)
    for slot in (0, 3, 9):
        for off in (0, 16, 4096, 999_984):
            assert oracle.pool_locate(slot, off, pt, 1, 1 << 20) == slot * (1 << 20) + off


def test_pool_locate_scattered_round_trip():
    # place every logical page of every slot at its physical page by slicing,
    # then read every 16-byte chunk back through the oracle's translation
    g = np.random.default_rng(12)
    n_slots, pps, P = 5, 4, 64
    pt = g.permutation(n_slots * pps).astype(np.int32)
    logical = g.integers(0, 256, size=(n_slots, pps * P), dtype=np.uint8)
    phys = np.zeros(n_slots * pps * P, dtype=np.uint8)
    for s in range(n_slots):
        for p in range(pps):
            q = pt[s * pps + p]
            phys[q * P:(q + 1) * P] = logical[s, p * P:(p + 1) * P]
    for s in range(n_slots):
        for off in range(0, pps * P, 16):
            at = oracle.pool_locate(s, off, pt, pps, P)
            assert np.array_equal(phys[at:at + 16], logical[s, off:off + 16])
