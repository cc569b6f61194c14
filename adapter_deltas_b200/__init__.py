"""Thin Python binding of the B200 multi-LoRA delta library (liblora_b200.so).

Every function here has the name of the C entry point it calls (see
``include/lora.h``) and only marshals arguments: torch tensors become device
pointers, the current CUDA stream becomes the stream argument, and a non-zero
status raises ``LoraError``.  All arithmetic runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback: importing this package fails if
the library has not been built (``python adapter_deltas_b200/_build.py``).

Tensors: x and y are bf16 [T, ld] (row-major, ld >= d and a multiple of 8),
ids int32 [T], scales fp32 [n_slots], workspace uint8; all on the pool's device.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
# LORA_B200_DEBUG=1 selects the bounds-checking build (LORA_DEBUG)
DEBUG_BUILD = os.environ.get("LORA_B200_DEBUG") == "1"
LIB_PATH = os.path.join(_HERE, "liblora_b200_debug.so" if DEBUG_BUILD else "liblora_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "%s is not built; run `python adapter_deltas_b200/_build.py%s` "
        "(the delta path has no fallback)" % (os.path.basename(LIB_PATH), " --debug" if DEBUG_BUILD else ""))

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_Z = ctypes.c_size_t

LORA_OK = 0
LORA_ERR_INVALID_ARG = 1
LORA_ERR_ALIGNMENT = 2
LORA_ERR_NO_PAGES = 3
LORA_ERR_SLOT = 4
LORA_ERR_NOT_LOADED = 5
LORA_ERR_CUDA = 6
LORA_ERR_BAD_ID = 7
LORA_ERR_TIMEOUT = 8
LORA_ERR_WORKSPACE = 9
LORA_ERR_BOUNDS = 10


class lora_target(ctypes.Structure):
    _fields_ = [("d_in", _I), ("d_out", _I)]


class lora_pool_info(ctypes.Structure):
    _fields_ = [("slot_bytes", _Z), ("page_bytes", _Z), ("pages_per_slot", _I), ("n_pages", _I),
                ("free_pages", _I), ("n_slots", _I), ("n_targets", _I), ("r_max", _I),
                ("decode_ctas", _I)]


class lora_plan_layout(ctypes.Structure):
    _fields_ = [("header", _Z), ("perm", _Z), ("seg_start", _Z), ("seg_slot", _Z), ("items", _Z),
                ("tiles", _Z), ("total", _Z), ("s_max", _I), ("i_max", _I), ("j_max", _I)]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("lora_status_string", ctypes.c_char_p, [_I])
_sig("lora_pool_bytes_required", _Z, [_P, _I, _I, _I, _Z])
_sig("lora_pool_create", _I, [ctypes.POINTER(_P), _I, _P, _I, _I, _I, _Z, _P, _Z, ctypes.c_uint64])
_sig("lora_pool_load", _I, [_P, _I, _I, _I, _P, _P, _I, _P])
_sig("lora_pool_unload", _I, [_P, _I])
_sig("lora_pool_swap_in", _I, [_P, _I, _P, _P, _Z, _P, _Z, _P])
_sig("lora_swap_src_bytes", _Z, [_P, _P])
_sig("lora_swap_staging_bytes", _Z, [_P, _P])
_sig("lora_pool_destroy", _I, [_P])
_sig("lora_pool_page_table", _P, [_P])
_sig("lora_pool_get_info", _I, [_P, ctypes.POINTER(lora_pool_info)])
_sig("lora_pool_target_offsets", _I, [_P, _I, ctypes.POINTER(_Z), ctypes.POINTER(_Z)])
_sig("lora_workspace_bytes", _Z, [_P, _I, _I])
_sig("lora_linear_workspace_bytes", _Z, [_P, _I, _I])
_sig("lora_plan_layout_get", _I, [_P, _I, ctypes.POINTER(lora_plan_layout)])
_sig("lora_plan_ids", _I, [_P, _P, _I, _P, _Z, _P])
_sig("lora_plan_segments", _I, [_P, _P, _P, _I, _I, _P, _Z, _P])
_sig("lora_mma_min_rows", _I, [])
_sig("lora_mma_min_rows_for", _I, [_I, _I])
_sig("lora_apply_plan", _I, [_P, _I, _P, _I, _P, _I, _P, _I, _P, _Z, _P])
_sig("lora_apply", _I, [_P, _I, _P, _I, _P, _I, _P, _P, _I, _P, _Z, _P])
_sig("lora_apply_segments", _I, [_P, _I, _P, _I, _P, _I, _P, _P, _I, _P, _I, _P, _Z, _P])
_sig("lora_apply_multi", _I, [_P, _I, _P, _P, _I, _P, _I, _P, _P, _P, _I, _P, _Z, _P])
_sig("lora_linear", _I, [_P, _I, _P, _I, _P, _I, _P, _I, _P, _P, _I, _P, _Z, _P])
_sig("lora_linear_expand", _I, [_P, _I, _P, _I, _P, _I, _P, _I, _P, _I, _P, _P, _I, _P])
_sig("lora_apply_moe", _I, [_P, _I, _P, _I, _P, _I, _P, _P, _I, _I, _I, _P, _P, _Z, _P])
_sig("lora_moe_workspace_bytes", _Z, [_P, _I, _I])
_sig("lora_shrink", _I, [_P, _I, _P, _I, _P, _I, _P, _I, _P, _Z, _P])
_sig("lora_expand", _I, [_P, _I, _P, _I, _P, _I, _P, _P, _I, _P, _Z, _P])
_sig("lora_apply_noalloc", _I, [_P, _I, _P, _I, _P, _I, _P, _P, _I, _P])
_sig("lora_get_error", _I, [_P, ctypes.POINTER(_I), _P])
_sig("lora_kernel_launches", ctypes.c_uint64, [])
_sig("lora_set_wait_limit_ns", None, [ctypes.c_uint64])
_sig("lora_selftest_stalled_apply", _I, [_P, _I, _P, _I, _P, _I, _P, _P, _I, _P])


class LoraError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s" % (where, lora_status_string(code)))


def _check(code: int, where: str) -> None:
    if code != LORA_OK:
        raise LoraError(code, where)


def lora_status_string(code: int) -> str:
    return _lib.lora_status_string(code).decode()


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ld(t) -> int:
    return int(t.stride(0)) if t is not None and t.dim() == 2 else 0


def _targets(targets: Sequence[Tuple[int, int]]):
    arr = (lora_target * len(targets))()
    for i, (d_in, d_out) in enumerate(targets):
        arr[i].d_in = int(d_in)
        arr[i].d_out = int(d_out)
    return arr


class PoolHandle:
    """The opaque pool pointer plus the Python objects it must outlive."""

    def __init__(self, ptr: int, device: int, mem, targets, r_max: int, n_slots: int):
        self.ptr = ptr
        self.device = device
        self.mem = mem
        self.targets = list(targets)
        self.r_max = r_max
        self.n_slots = n_slots

    @property
    def _as_parameter_(self):
        return self.ptr


# ---------------------------------------------------------------- pool


def lora_pool_bytes_required(targets, r_max: int, n_slots: int, page_bytes: int = 0) -> int:
    arr = _targets(targets)
    return int(_lib.lora_pool_bytes_required(arr, len(arr), r_max, n_slots, page_bytes))


def lora_pool_create(device: int, targets, r_max: int, n_slots: int, page_bytes: int, pool_mem,
                     scatter_seed: int = 0) -> PoolHandle:
    arr = _targets(targets)
    out = _P()
    nbytes = pool_mem.numel() * pool_mem.element_size()
    _check(_lib.lora_pool_create(ctypes.byref(out), device, arr, len(arr), r_max, n_slots, page_bytes,
                                 _ptr(pool_mem), nbytes, scatter_seed), "lora_pool_create")
    return PoolHandle(out.value, device, pool_mem, targets, r_max, n_slots)


def lora_pool_load(pool: PoolHandle, slot: int, target: int, rank: int, A, B, stream=None) -> None:
    """A: bf16 [rank, d_in], B: bf16 [d_out, rank]; torch tensors on the pool's
    device or on the host (contiguous)."""
    on_dev = 1 if (A is not None and A.is_cuda) else 0
    if A is not None:
        assert A.is_contiguous() and B.is_contiguous()
    _check(_lib.lora_pool_load(pool, slot, target, rank, _ptr(A), _ptr(B), on_dev, _stream(stream)),
           "lora_pool_load")


def _int_array(values):
    values = [int(v) for v in values]
    return (ctypes.c_int * len(values))(*values)


def lora_swap_src_bytes(pool: PoolHandle, ranks) -> int:
    return int(_lib.lora_swap_src_bytes(pool, _int_array(ranks)))


def lora_swap_staging_bytes(pool: PoolHandle, ranks) -> int:
    return int(_lib.lora_swap_staging_bytes(pool, _int_array(ranks)))


def lora_pool_swap_in(pool: PoolHandle, slot: int, ranks, src, staging, stream=None) -> None:
    """One adapter, all targets, from host memory `src` (a CPU tensor, pinned
    for an asynchronous copy) through the device tensor `staging`."""
    nbytes = src.numel() * src.element_size()
    _check(_lib.lora_pool_swap_in(pool, slot, _int_array(ranks), _ptr(src), nbytes, _ptr(staging),
                                  staging.numel() * staging.element_size(), _stream(stream)), "lora_pool_swap_in")


def lora_pool_unload(pool: PoolHandle, slot: int) -> None:
    _check(_lib.lora_pool_unload(pool, slot), "lora_pool_unload")


def lora_pool_destroy(pool: PoolHandle) -> None:
    if pool.ptr:
        _check(_lib.lora_pool_destroy(pool), "lora_pool_destroy")
        pool.ptr = 0


def lora_pool_page_table(pool: PoolHandle) -> int:
    return int(_lib.lora_pool_page_table(pool) or 0)


def lora_pool_get_info(pool: PoolHandle) -> lora_pool_info:
    info = lora_pool_info()
    _check(_lib.lora_pool_get_info(pool, ctypes.byref(info)), "lora_pool_get_info")
    return info


def lora_pool_target_offsets(pool: PoolHandle, target: int) -> Tuple[int, int]:
    a, b = _Z(), _Z()
    _check(_lib.lora_pool_target_offsets(pool, target, ctypes.byref(a), ctypes.byref(b)),
           "lora_pool_target_offsets")
    return int(a.value), int(b.value)


# ---------------------------------------------------------------- plans


def lora_workspace_bytes(pool: PoolHandle, target: int, max_tokens: int) -> int:
    return int(_lib.lora_workspace_bytes(pool, target, max_tokens))


def lora_plan_layout_get(pool: PoolHandle, T: int) -> lora_plan_layout:
    out = lora_plan_layout()
    _check(_lib.lora_plan_layout_get(pool, T, ctypes.byref(out)), "lora_plan_layout_get")
    return out


def lora_mma_min_rows() -> int:
    return int(_lib.lora_mma_min_rows())


def lora_mma_min_rows_for(n_segments: int, T: int) -> int:
    """Segment length from which a segment plan of this batch uses the tensor cores."""
    return int(_lib.lora_mma_min_rows_for(n_segments, T))


def lora_plan_ids(pool: PoolHandle, ids, ws, stream=None) -> None:
    _check(_lib.lora_plan_ids(pool, _ptr(ids), ids.shape[0], _ptr(ws), ws.numel(), _stream(stream)),
           "lora_plan_ids")


def lora_plan_segments(pool: PoolHandle, seg_offsets, seg_slot, T: int, ws, stream=None) -> None:
    _check(_lib.lora_plan_segments(pool, _ptr(seg_offsets), _ptr(seg_slot), seg_slot.shape[0], T, _ptr(ws),
                                   ws.numel(), _stream(stream)), "lora_plan_segments")


# ---------------------------------------------------------------- compute


def lora_apply_plan(pool: PoolHandle, target: int, x, y, scales, ws, stream=None) -> None:
    _check(_lib.lora_apply_plan(pool, target, _ptr(x), _ld(x), _ptr(y), _ld(y), _ptr(scales), y.shape[0],
                                _ptr(ws), ws.numel(), _stream(stream)), "lora_apply_plan")


def lora_apply(pool: PoolHandle, target: int, x, y, ids, scales, ws, stream=None) -> None:
    _check(_lib.lora_apply(pool, target, _ptr(x), _ld(x), _ptr(y), _ld(y), _ptr(ids), _ptr(scales),
                           y.shape[0], _ptr(ws), ws.numel(), _stream(stream)), "lora_apply")


def lora_apply_multi(pool: PoolHandle, targets, x, y, y_cols, ids, scales, ws, stream=None) -> None:
    """Several same-shape targets sharing x in one call; target i adds its
    delta to columns y_cols[i] .. y_cols[i] + d_out - 1 of y."""
    n = len(targets)
    t_arr = (ctypes.c_int * n)(*[int(t) for t in targets])
    c_arr = (ctypes.c_int * n)(*[int(c) for c in y_cols])
    _check(_lib.lora_apply_multi(pool, n, t_arr, _ptr(x), _ld(x), _ptr(y), _ld(y), c_arr, _ptr(ids), _ptr(scales),
                                 y.shape[0], _ptr(ws), ws.numel(), _stream(stream)), "lora_apply_multi")


def lora_apply_segments(pool: PoolHandle, target: int, x, y, seg_offsets, seg_slot, scales, ws,
                        stream=None) -> None:
    _check(_lib.lora_apply_segments(pool, target, _ptr(x), _ld(x), _ptr(y), _ld(y), _ptr(seg_offsets),
                                    _ptr(seg_slot), seg_slot.shape[0], _ptr(scales), y.shape[0], _ptr(ws),
                                    ws.numel(), _stream(stream)), "lora_apply_segments")


def lora_linear_workspace_bytes(pool: PoolHandle, target: int, max_tokens: int) -> int:
    return int(_lib.lora_linear_workspace_bytes(pool, target, max_tokens))


def lora_linear(pool: PoolHandle, target: int, x, W, y, ids, scales, ws, stream=None) -> None:
    """y = x W^T + each row's delta, written once (W: [d_out, d_in] row-major)."""
    _check(_lib.lora_linear(pool, target, _ptr(x), _ld(x), _ptr(W), _ld(W), _ptr(y), _ld(y), _ptr(ids),
                            _ptr(scales), y.shape[0], _ptr(ws), ws.numel(), _stream(stream)), "lora_linear")


def lora_linear_expand(pool: PoolHandle, target: int, x, W, v, y, ids, scales, stream=None) -> None:
    """y = x W^T + each row's s_a B_a v[t] (v from lora_shrink), written once."""
    _check(_lib.lora_linear_expand(pool, target, _ptr(x), _ld(x), _ptr(W), _ld(W), _ptr(v), _ld(v), _ptr(y),
                                   _ld(y), _ptr(ids), _ptr(scales), y.shape[0], _stream(stream)),
           "lora_linear_expand")


def lora_moe_workspace_bytes(pool: PoolHandle, target: int, max_pairs: int) -> int:
    return int(_lib.lora_moe_workspace_bytes(pool, target, max_pairs))


def lora_apply_moe(pool: PoolHandle, target: int, x, y, lora_ids, topk_ids, n_experts: int, scales, ws,
                   stream=None) -> None:
    """Routed expert pairs: y[t * k + j] += s B_s (A_s x[t]), s = lora_ids[t] * n_experts + topk_ids[t, j];
    x [T, d_in], y [T * k, d_out], topk_ids [T, k]."""
    T, k = int(topk_ids.shape[0]), int(topk_ids.shape[1])
    _check(_lib.lora_apply_moe(pool, target, _ptr(x), _ld(x), _ptr(y), _ld(y), _ptr(lora_ids), _ptr(topk_ids), T,
                               k, n_experts, _ptr(scales), _ptr(ws), ws.numel(), _stream(stream)),
           "lora_apply_moe")


def lora_shrink(pool: PoolHandle, target: int, x, ids, v, ws, stream=None) -> None:
    _check(_lib.lora_shrink(pool, target, _ptr(x), _ld(x), _ptr(ids), ids.shape[0], _ptr(v), _ld(v), _ptr(ws),
                            ws.numel(), _stream(stream)), "lora_shrink")


def lora_expand(pool: PoolHandle, target: int, v, y, ids, scales, ws, stream=None) -> None:
    _check(_lib.lora_expand(pool, target, _ptr(v), _ld(v), _ptr(y), _ld(y), _ptr(ids), _ptr(scales),
                            ids.shape[0], _ptr(ws), ws.numel(), _stream(stream)), "lora_expand")


LORA_NOALLOC_MAX_TOKENS = 4096


def lora_apply_noalloc(pool: PoolHandle, target: int, x, y, ids, scales, stream=None) -> None:
    """lora_apply without a workspace argument: the workspace lives in a fixed
    device array inside the library (for callers that cannot allocate).
    Calls that overlap on the GPU share that array and must be serialised."""
    _check(_lib.lora_apply_noalloc(pool, target, _ptr(x), _ld(x), _ptr(y), _ld(y), _ptr(ids), _ptr(scales),
                                   y.shape[0], _stream(stream)), "lora_apply_noalloc")


def lora_get_error(pool: PoolHandle, stream=None) -> int:
    st = _I(0)
    _check(_lib.lora_get_error(pool, ctypes.byref(st), _stream(stream)), "lora_get_error")
    return int(st.value)


def lora_kernel_launches() -> int:
    return int(_lib.lora_kernel_launches())


def lora_set_wait_limit_ns(ns: int) -> None:
    """Wall-clock limit of the decode kernel's bounded waits (0: one second)."""
    _lib.lora_set_wait_limit_ns(int(ns))


def lora_selftest_stalled_apply(pool: PoolHandle, target: int, x, y, ids, scales, stream=None) -> None:
    """Test only: the decode launch of lora_apply with no stage ever filled,
    so that its waits run out (LORA_ERR_TIMEOUT in the sticky status)."""
    _check(_lib.lora_selftest_stalled_apply(pool, target, _ptr(x), _ld(x), _ptr(y), _ld(y), _ptr(ids),
                                            _ptr(scales), y.shape[0], _stream(stream)),
           "lora_selftest_stalled_apply")
