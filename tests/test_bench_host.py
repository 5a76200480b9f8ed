"""Host logic of bench.py that needs no GPU: the algorithmic work counts the
roofline divides by, the roofline itself, and the lookup of committed ncu
DRAM traffic, which must turn null once a kernel's sources change."""
import json
import os
import shutil

import pytest

import bench
import synth


def _attended_brute(T, m, N, K, W):
    total = 0
    for t in range(T):
        total += min(min((t + 1) // m, N), K) + min(W, t + 1)
    return total


@pytest.mark.parametrize("T,m,N,K,W", [(1, 4, 0, 16, 32), (37, 4, 9, 3, 5), (200, 4, 50, 16, 32),
                                       (300, 128, 2, 512, 128)])
def test_sum_attended_matches_brute_force(T, m, N, K, W):
    assert bench.sum_attended(T, m, N, K, W) == _attended_brute(T, m, N, K, W)
    assert bench.sum_visible(T, m, N) == sum(min((t + 1) // m, N) for t in range(T))


def test_prefill_attention_work():
    """128K prefill: 83,353,152 attended (query, item) pairs, 4 * 64 * 512 FLOP each."""
    wl = synth.WORKLOADS["csa_prefill_128k"]
    att = bench.sum_attended(wl.T, wl.m, wl.N, wl.K, wl.W)
    assert att == 83_353_152
    assert bench.op_work(wl)["attend"]["flops"] == 4.0 * att * 64 * 512


def test_roofline_bound_and_fraction():
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}
    pf = synth.WORKLOADS["csa_prefill_128k"]
    r = bench.roofline("attend", {"bytes": 1e9, "flops": 1.6e12}, 2.0, peaks, "measured", pf)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(800.0) and r["frac"] == pytest.approx(0.5)
    dec = synth.WORKLOADS["csa_decode_64k"]
    r = bench.roofline("attend", {"bytes": 6.5e6, "flops": 1e9}, 0.002, peaks, "measured", dec)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(3250.0) and r["frac"] == pytest.approx(0.5)


def test_traffic_follows_each_kernels_sources(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "compressed_sparse_attention_16_b200", "csrc")
    dst = tmp_path / "compressed_sparse_attention_16_b200" / "csrc"
    shutil.copytree(src, dst)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {
        "wl": {
            "attend": {"dram_bytes": 123, "kernel": "attend_tc_kernel",
                       "source_sha": bench.source_sha("attend_tc_kernel")},
            "index_topk": {"dram_bytes": 456, "kernel": "index_decode_kernel<4>",
                           "source_sha": bench.source_sha("index_decode_kernel<4>")},
        }
    }
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.kernel_traffic("attend", "wl") == 123
    assert bench.kernel_traffic("index_topk", "wl") == 456
    assert bench.kernel_traffic("attend", "other") is None
    # another kernel's file changes: this record stays valid
    with open(dst / "attend_prefill.cu", "a") as f:
        f.write("\n// edited\n")
    assert bench.kernel_traffic("attend", "wl") == 123
    # the kernel's own file changes: null
    with open(dst / "attend_tc.cu", "a") as f:
        f.write("\n// edited\n")
    assert bench.kernel_traffic("attend", "wl") is None
    assert bench.kernel_traffic("index_topk", "wl") == 456
    # a shared header changes: every record turns null
    with open(dst / "tc.cuh", "a") as f:
        f.write("\n// edited\n")
    assert bench.kernel_traffic("index_topk", "wl") is None



@pytest.mark.parametrize("name", ["tiny_prefill", "csa_decode_64k"])
def test_reference_arm_line(name, monkeypatch):
    """`bench.py --impl reference`: the oracle timed on the host cores, one
    JSON line with the contract's keys (rank 0 only)."""
    import types
    monkeypatch.setenv("RANK", "0")
    line = bench.reference_arm(types.SimpleNamespace(steps=1, warmup=0), synth.WORKLOADS[name])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == ("queries/s" if name == "tiny_prefill" else "tokens/s")
    assert line["config"]["workload"] == name
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    json.dumps(line)
    monkeypatch.setenv("RANK", "1")
    assert bench.reference_arm(types.SimpleNamespace(steps=1, warmup=0), synth.WORKLOADS[name]) is None
