"""Host-side helpers of bench.py: the ncu traffic figure is read from a
profile summary only while its source hash matches the kernel source, and the
algorithmic bytes follow the definition (distinct adapters at their own rank,
x of the adapted rows, y of the adapted rows read and written), and the routed
workload draws valid routing."""

import hashlib
import os

import numpy as np

import bench
import synth


def _write_profile(root, kernel, workload, sha, traffic):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", "%s_%s.txt" % (kernel, workload)), "w") as f:
        f.write("a summary\nsource_sha256: %s\ntraffic_bytes_per_launch: %d  (a note)\n" % (sha, traffic))


def test_traffic_only_while_the_source_matches(tmp_path, monkeypatch):
    root = str(tmp_path)
    src_dir = os.path.join(root, "adapter_deltas_b200", "csrc")
    os.makedirs(src_dir)
    src = b"__global__ void k() {}\n"
    with open(os.path.join(src_dir, "k.cu"), "wb") as f:
        f.write(src)
    monkeypatch.setattr(bench, "ROOT", root)
    _write_profile(root, "k_kernel", "wl", hashlib.sha256(src).hexdigest(), 12345)
    assert bench.traffic_from_profile("k_kernel", "k.cu", "wl") == 12345
    _write_profile(root, "k_kernel", "wl", "0" * 64, 12345)
    assert bench.traffic_from_profile("k_kernel", "k.cu", "wl") is None
    assert bench.traffic_from_profile("other", "k.cu", "wl") is None


def test_algorithmic_bytes_definition():
    w = synth.custom(5, 6, [(64, 32)], [8, 16, 0], 16, ids=[0, 1, 1, -1, 2, 0])
    # adapted rows: ids 0, 1, 1, 0 (slot 2 has rank 0: not adapted)
    want = (8 + 16) * (64 + 32) * 2 + 4 * 64 * 2 + 4 * 32 * 4
    assert bench.algorithmic_bytes(w, 0, np.asarray(w.ids)) == want


def test_moe_workload_routing():
    # every token picks top_k distinct experts; 10 % of tokens carry no
    # adapter; the pool has one slot per (adapter, expert); output rows per pair
    m = bench.MOE_SHAPE
    w, lora, topk, y = bench.moe_workload(4000)
    assert w.n_slots == m["n_ad"] * m["E"] and w.targets == [(m["d"], m["d"])]
    assert w.x(0).shape == (m["T"], m["d"])
    assert topk.shape == (m["T"], m["k"]) and y.shape == (m["T"] * m["k"], m["d"])
    assert all(len(set(row)) == m["k"] for row in topk.tolist())
    assert topk.min() >= 0 and topk.max() < m["E"]
    assert (lora == -1).sum() == round(0.1 * m["T"])
    assert lora.max() < m["n_ad"] and lora.min() >= -1
    # seeded: the same seed gives the same routing
    _, lora2, topk2, _ = bench.moe_workload(4000)
    assert np.array_equal(lora, lora2) and np.array_equal(topk, topk2)
