"""The LORA_DEBUG build (liblora_b200_debug.so): the same results with the
index and page checks compiled in, and a corrupted plan turned into
LORA_ERR_BOUNDS instead of a bad access.

The checks run in a child process that loads the debug library
(LORA_B200_DEBUG=1): a one-launch decode batch, the plan path over a
scattered 4 KiB-page pool, shrink + expand, and a segment batch on the tensor
cores, each against the fp64 oracle with a clean status.  Then one plan item
is given 17 rows (items hold at most 16): the debug kernel must drop that
item, report LORA_ERR_BOUNDS, leave its rows untouched and still compute the
others.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys
import numpy as np
import torch
sys.path.insert(0, os.path.join(ROOT, "tests"))
import adapter_deltas_b200 as L
assert L.DEBUG_BUILD and L.LIB_PATH.endswith("liblora_b200_debug.so"), L.LIB_PATH
import oracle, synth
from gpu_harness import DevicePool, assert_close, oracle_y, scales_of, to_dev_bf16, to_host_bits, workspace
dev = torch.device("cuda:0")

# (1) one-launch decode (q_proj shape)
w = synth.config(2)
with DevicePool(w, dev) as pool:
    x = to_dev_bf16(w.x(0), dev); y = to_dev_bf16(w.y_in(0), dev)
    ids = torch.from_numpy(w.ids).to(dev); sc = torch.from_numpy(scales_of(w)).to(dev)
    L.lora_apply(pool.pool, 0, x, y, ids, sc, workspace(pool, w.T))
    torch.cuda.synchronize()
    assert L.lora_get_error(pool.pool) == L.LORA_OK
    want, _ = oracle_y(w, 0, w.x(0), w.y_in(0), w.ids)
    assert_close(to_host_bits(y), want, what="debug build, one launch")

# (2) plan path over a scattered paged pool, and shrink + expand
w = synth.config(1)
with DevicePool(w, dev, page_bytes=4096, scatter_seed=5) as pool:
    x = to_dev_bf16(w.x(0), dev)
    ids = torch.from_numpy(w.ids).to(dev); sc = torch.from_numpy(scales_of(w)).to(dev)
    ws = workspace(pool, w.T)
    y = to_dev_bf16(w.y_in(0), dev)
    L.lora_plan_ids(pool.pool, ids, ws)
    L.lora_apply_plan(pool.pool, 0, x, y, sc, ws)
    v = torch.zeros(w.T, w.r_max, dtype=torch.float32, device=dev)
    y2 = to_dev_bf16(w.y_in(0), dev)
    L.lora_shrink(pool.pool, 0, x, ids, v, ws)
    L.lora_expand(pool.pool, 0, v, y2, ids, sc, ws)
    torch.cuda.synchronize()
    assert L.lora_get_error(pool.pool) == L.LORA_OK
    want, _ = oracle_y(w, 0, w.x(0), w.y_in(0), w.ids)
    assert_close(to_host_bits(y), want, what="debug build, plan path")
    assert np.array_equal(to_host_bits(y2), to_host_bits(y))

    # (4) a corrupted plan: item 0 claims 17 rows
    lay = L.lora_plan_layout_get(pool.pool, w.T)
    raw = ws.cpu().numpy().copy()
    items = raw[lay.items:lay.items + 16 * 4].view(np.int32).reshape(-1, 4)
    perm = raw[lay.perm:lay.perm + 4 * w.T].view(np.int32)
    slot0, first0, m0 = (int(v_) for v_ in items[0, :3])
    rows0 = perm[first0:first0 + m0].copy()
    items[0, 2] = 17
    ws.copy_(torch.from_numpy(raw).to(dev))
    y3 = to_dev_bf16(w.y_in(0), dev)
    L.lora_apply_plan(pool.pool, 0, x, y3, sc, ws)
    torch.cuda.synchronize()
    assert L.lora_get_error(pool.pool) == L.LORA_ERR_BOUNDS
    got = to_host_bits(y3)
    assert np.array_equal(got[rows0], w.y_in(0)[rows0])           # the dropped item's rows
    rest = np.setdiff1d(np.arange(w.T), rows0)
    assert np.array_equal(got[rest], to_host_bits(y)[rest])        # every other row as before

# (3) a segment batch on the tensor cores
off = np.array([0, 150, 155, 300], np.int32); seg_slot = np.array([0, 1, 2], np.int32)
row_ids = np.repeat(seg_slot, np.diff(off)).astype(np.int32)
wp = synth.custom(21, 300, [(512, 384)], [16, 8, 13], 16, ids=row_ids)
with DevicePool(wp, dev) as pool:
    x = to_dev_bf16(wp.x(0), dev); y = to_dev_bf16(wp.y_in(0), dev)
    sc = torch.from_numpy(scales_of(wp)).to(dev)
    L.lora_apply_segments(pool.pool, 0, x, y, torch.from_numpy(off).to(dev), torch.from_numpy(seg_slot).to(dev),
                          sc, workspace(pool, wp.T))
    torch.cuda.synchronize()
    assert L.lora_get_error(pool.pool) == L.LORA_OK
    want, _ = oracle_y(wp, 0, wp.x(0), wp.y_in(0), row_ids)
    assert_close(to_host_bits(y), want, what="debug build, segments")
print("debug build ok")
'''


def test_debug_build_matches_and_reports_bounds(cuda_device):
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("_lora_build", os.path.join(ROOT, "adapter_deltas_b200", "_build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build(debug=True)  # (no-op when liblora_b200_debug.so is current)
    env = dict(os.environ, LORA_B200_DEBUG="1", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], env=env, cwd=ROOT,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-4000:]
    assert "debug build ok" in out.stdout
