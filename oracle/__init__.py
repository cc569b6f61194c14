"""CPU oracle for the multi-LoRA delta path (fp64, one loop per row).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this package.  It shares no code with
the CUDA library (``adapter_deltas_b200``) and imports nothing from it.

The arithmetic lives in ``lora_oracle.c`` (plain C, fp64); this module builds
it with gcc, decodes bf16 bit patterns to fp64 (exact: a bf16 value is the top
half of an IEEE binary32) and marshals numpy arrays through ctypes.

Functions and the passages they follow (pages on multi-LoRA serving):

* ``lora_apply``   -- "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU",
  section "Why can't you just merge LoRA weights into the base model?"
  (y = xW + (x A_i) B_i alpha/r) with the shapes of section "How much memory
  does one LoRA adapter actually cost?" (A: r x d_in, B: d_out x r);
  "Serving Many LoRA Adapters From One Base Model", sections "How it works"
  and "Batching across adapters" (per-row correction), worked example
  (adapter=None leaves the base output).
* ``lora_expand``  -- the second factor of the same formula, given v = A x.
* ``linear`` / ``lora_linear`` -- the shared base term xW of the same
  formula (W stored d_out x d_in as in the column form W.x of "Serving Many
  LoRA Adapters From One Base Model", section "How it works"), and the whole
  layer output xW + (x A_i) B_i alpha/r.
* ``moe_lora_apply`` -- the same per-row delta inside expert routing
  ("Multi-LoRA Serving: Sharing One GPU Across Adapters", section "MoE Models
  Raise the Bar": each adapted projection of every expert carries the
  adapter's shrink and expand): every (token, chosen expert) pair takes the
  delta of its own (adapter, expert) matrices.
* ``group_rows``   -- "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU",
  section "How does one batch run 30 different adapters at once?" (index
  vector, segmented gather).
* ``pool_locate`` / ``slot_layout`` -- "Multi-LoRA Serving: Sharing One GPU
  Across Adapters", section "How S-LoRA Proved the Model" (paged adapter pool);
  the slot layout is the one the library header documents.
* ``lora_params``  -- "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU",
  section "How much memory does one LoRA adapter actually cost?".

Every function here is pinned by ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lora_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile lora_oracle.c into liboracle.so (gcc, no fast-math, no FMA
    contraction, so every fp64 operation is the one written)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
           "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.oracle_lora_apply.restype = I
    lib.oracle_lora_apply.argtypes = [I, I, I, P, P, P, I, P, P, P, P, P, P, I, I]
    lib.oracle_lora_expand.restype = I
    lib.oracle_lora_expand.argtypes = [I, I, P, I, P, P, I, P, P, P, P]
    lib.oracle_group_rows.restype = I
    lib.oracle_group_rows.argtypes = [I, P, I, P, P, P, P, P, P]
    lib.oracle_pool_locate.restype = ctypes.c_longlong
    lib.oracle_pool_locate.argtypes = [I, ctypes.c_longlong, P, I, ctypes.c_longlong]
    lib.oracle_slot_layout.restype = ctypes.c_longlong
    lib.oracle_slot_layout.argtypes = [I, P, P, I, P, P]
    lib.oracle_linear.restype = None
    lib.oracle_linear.argtypes = [I, I, I, P, P, P, I]
    lib.oracle_lora_params.restype = ctypes.c_longlong
    lib.oracle_lora_params.argtypes = [I, P, P, ctypes.c_longlong, ctypes.c_longlong]
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact decode of bf16 bit patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _as_f64(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return bf16_to_f64(a)
    return np.ascontiguousarray(a, dtype=np.float64)


Adapters = Dict[int, Tuple[np.ndarray, np.ndarray]]


def _slot_tables(n_slots: int, adapters: Adapters, alpha: Sequence[float]):
    A_keep, B_keep = [], []
    A_ptrs = (ctypes.c_void_p * max(n_slots, 1))()
    B_ptrs = (ctypes.c_void_p * max(n_slots, 1))()
    rank = np.zeros(max(n_slots, 1), dtype=np.int32)
    for slot, (A, B) in adapters.items():
        A64 = _as_f64(A)
        B64 = _as_f64(B)
        r = A64.shape[0]
        assert B64.shape[1] == r, "A is r x d_in and B is d_out x r"
        A_keep.append(A64)
        B_keep.append(B64)
        A_ptrs[slot] = _ptr(A64)
        B_ptrs[slot] = _ptr(B64)
        rank[slot] = r
    alpha64 = np.zeros(max(n_slots, 1), dtype=np.float64)
    alpha64[:n_slots] = np.asarray(alpha, dtype=np.float64)[:n_slots]
    return (A_keep, B_keep), A_ptrs, B_ptrs, rank, alpha64


def lora_apply(x, y_in, ids, n_slots: int, adapters: Adapters,
               alpha: Sequence[float], threads: int = 1,
               want_v: bool = False):
    """y[t] = y_in[t] + (alpha_a / r_a) * B_a (A_a x[t]) with a = ids[t].

    x: [T, d_in], y_in: [T, d_out] (bf16 bit patterns as uint16, or floats);
    ids: int32 [T], -1 = no adapter; adapters: slot -> (A [r, d_in],
    B [d_out, r]) at the adapter's own rank (a rank-0 or absent slot leaves
    its rows unchanged); alpha: per-slot alpha.  Returns (y fp64 [T, d_out],
    number of rows with an invalid id[, v fp64 [T, r_max] when want_v]).
    """
    lib = _load()
    x64 = _as_f64(x)
    y64 = _as_f64(y_in)
    ids32 = np.ascontiguousarray(ids, dtype=np.int32)
    T, d_in = x64.shape
    d_out = y64.shape[1]
    keep, A_ptrs, B_ptrs, rank, alpha64 = _slot_tables(n_slots, adapters, alpha)
    out = np.empty((T, d_out), dtype=np.float64)
    ldv = int(rank.max()) if rank.size else 0
    v = np.zeros((T, max(ldv, 1)), dtype=np.float64) if want_v else None
    bad = lib.oracle_lora_apply(T, d_in, d_out, _ptr(x64), _ptr(y64), _ptr(ids32),
                                n_slots, ctypes.addressof(A_ptrs), ctypes.addressof(B_ptrs),
                                _ptr(rank), _ptr(alpha64), _ptr(out),
                                _ptr(v) if want_v else None, max(ldv, 1), threads)
    del keep
    if want_v:
        return out, bad, v
    return out, bad


def lora_expand(v, y_in, ids, n_slots: int, B_by_slot: Dict[int, np.ndarray],
                alpha: Sequence[float]):
    """y[t] = y_in[t] + (alpha_a / r_a) * B_a v[t][:r_a] for a caller-given v."""
    lib = _load()
    v64 = _as_f64(v)
    y64 = _as_f64(y_in)
    ids32 = np.ascontiguousarray(ids, dtype=np.int32)
    T, d_out = y64.shape
    keep = []
    B_ptrs = (ctypes.c_void_p * max(n_slots, 1))()
    rank = np.zeros(max(n_slots, 1), dtype=np.int32)
    for slot, B in B_by_slot.items():
        B64 = _as_f64(B)
        keep.append(B64)
        B_ptrs[slot] = _ptr(B64)
        rank[slot] = B64.shape[1]
    alpha64 = np.zeros(max(n_slots, 1), dtype=np.float64)
    alpha64[:n_slots] = np.asarray(alpha, dtype=np.float64)[:n_slots]
    out = np.empty((T, d_out), dtype=np.float64)
    bad = lib.oracle_lora_expand(T, d_out, _ptr(v64), v64.shape[1], _ptr(y64), _ptr(ids32),
                                 n_slots, ctypes.addressof(B_ptrs), _ptr(rank),
                                 _ptr(alpha64), _ptr(out))
    del keep
    return out, bad


def linear(x, W, threads: int = 1) -> np.ndarray:
    """out[t] = W x[t] (the base term xW with W stored [d_out, d_in]), fp64."""
    lib = _load()
    x64 = _as_f64(x)
    W64 = _as_f64(W)
    T, d_in = x64.shape
    d_out = W64.shape[0]
    assert W64.shape[1] == d_in, "W is d_out x d_in"
    out = np.empty((T, d_out), dtype=np.float64)
    lib.oracle_linear(T, d_in, d_out, _ptr(x64), _ptr(W64), _ptr(out), threads)
    return out


def lora_linear(x, W, ids, n_slots: int, adapters: Adapters,
                alpha: Sequence[float], threads: int = 1):
    """The whole layer: y[t] = W x[t] + (alpha_a / r_a) B_a (A_a x[t]), a = ids[t]
    (rows without a valid adapter get W x[t] alone).  Returns (y fp64, number
    of rows with an invalid id)."""
    return lora_apply(x, linear(x, W, threads), ids, n_slots, adapters, alpha, threads)


def moe_pair_slots(lora_ids, topk_ids, n_experts: int, n_slots: int):
    """Slot of each (token, chosen expert) pair, pair p = t * top_k + j:
    lora_ids[t] * n_experts + topk_ids[t, j], or -1 when the token has no
    adapter (lora_ids[t] == -1); an adapter id below -1, an expert outside
    [0, n_experts) or a slot outside [0, n_slots) gives the invalid id
    n_slots."""
    lo = np.ascontiguousarray(lora_ids, dtype=np.int64)
    tk = np.asarray(topk_ids, dtype=np.int64)
    T, k = tk.shape
    out = np.empty(T * k, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            a, e = int(lo[t]), int(tk[t, j])
            if a == -1:
                s = -1
            elif a < -1 or e < 0 or e >= n_experts or a * n_experts + e >= n_slots:
                s = n_slots
            else:
                s = a * n_experts + e
            out[t * k + j] = s
    return out.astype(np.int32)


def moe_lora_apply(x, y_pairs, lora_ids, topk_ids, n_experts: int, n_slots: int,
                   adapters: Adapters, alpha: Sequence[float], threads: int = 1):
    """y_pairs[t * top_k + j] += (alpha_s / r_s) B_s (A_s x[t]) with s the
    pair's slot (moe_pair_slots): the token's x row, the pair's own output row.
    Returns (y_pairs fp64 [T * top_k, d_out], number of pairs with an invalid
    id)."""
    tk = np.asarray(topk_ids)
    T, k = tk.shape
    x64 = _as_f64(x)
    x_pairs = np.repeat(x64, k, axis=0)           # row p holds x[p // top_k]
    ids = moe_pair_slots(lora_ids, tk, n_experts, n_slots)
    return lora_apply(x_pairs, y_pairs, ids, n_slots, adapters, alpha, threads)


def group_rows(ids, n_slots: int, valid: Optional[np.ndarray] = None):
    """Stable grouping of rows by adapter id: (perm, seg_start, seg_slot, n_bad)."""
    lib = _load()
    ids32 = np.ascontiguousarray(ids, dtype=np.int32)
    T = ids32.shape[0]
    perm = np.zeros(max(T, 1), dtype=np.int32)
    seg_start = np.zeros(max(T, 1) + 1, dtype=np.int32)
    seg_slot = np.zeros(max(T, 1), dtype=np.int32)
    n_active = np.zeros(1, dtype=np.int32)
    n_bad = np.zeros(1, dtype=np.int32)
    v8 = None
    if valid is not None:
        v8 = np.ascontiguousarray(valid, dtype=np.uint8)
    S = lib.oracle_group_rows(T, _ptr(ids32), n_slots, _ptr(v8) if v8 is not None else None,
                              _ptr(perm), _ptr(seg_start), _ptr(seg_slot),
                              _ptr(n_active), _ptr(n_bad))
    return (perm[: n_active[0]].copy(), seg_start[: S + 1].copy(),
            seg_slot[:S].copy(), int(n_bad[0]))


def pool_locate(slot: int, logical_off: int, page_table: np.ndarray,
                pages_per_slot: int, page_bytes: int) -> int:
    """Physical byte offset of a slot's logical byte through the page table."""
    lib = _load()
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    return int(lib.oracle_pool_locate(slot, logical_off, _ptr(pt), pages_per_slot, page_bytes))


def slot_layout(targets: Sequence[Tuple[int, int]], r_max: int):
    """(a_off[t], bt_off[t], slot_bytes) of the documented slot layout."""
    lib = _load()
    d_in = np.array([t[0] for t in targets], dtype=np.int32)
    d_out = np.array([t[1] for t in targets], dtype=np.int32)
    a_off = np.zeros(len(targets), dtype=np.int64)
    bt_off = np.zeros(len(targets), dtype=np.int64)
    total = lib.oracle_slot_layout(len(targets), _ptr(d_in), _ptr(d_out), r_max,
                                   _ptr(a_off), _ptr(bt_off))
    return a_off, bt_off, int(total)


ATTENTION_4096 = ((4096, 4096),) * 4   # q, k, v, o projections of Llama-2-7B (d_in, d_out)


def lora_params(shapes=ATTENTION_4096, layers: int = 32, rank: int = 16) -> int:
    """Parameters of a rank-`rank` adapter on the matrices `shapes` ((d_in,
    d_out) per adapted matrix of one layer) in each of `layers` layers: A is
    r x d_in and B is d_out x r for each matrix."""
    lib = _load()
    d_in = np.array([s[0] for s in shapes], dtype=np.int64)
    d_out = np.array([s[1] for s in shapes], dtype=np.int64)
    return int(lib.oracle_lora_params(len(shapes), _ptr(d_in), _ptr(d_out), layers, rank))
