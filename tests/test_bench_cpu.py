"""bench.py bookkeeping that needs no GPU: which ncu traffic figure a bench line may carry,
and the whole-job aggregate."""

import importlib.util
import os
import re
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_code_hash_ignores_comments_and_layout(bench):
    a = "int f(int x) {  // doubles x\n  return 2 * x; /* a block\n comment */ }\n"
    b = "/* header */\nint f(int x) {\n  return 2 * x;\n}  // trailing\n"
    c = "int f(int x) { return 3 * x; }"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    # PTX inside asm strings is code and survives
    assert "tcgen05.commit" in bench._code_only('asm volatile("tcgen05.commit.b64 [%0];" ::"r"(b)); // x')


def _copy_tree(tmp_path):
    for d in ("profiles", os.path.join("paged_mla_decode_11_b200", "csrc")):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d)
    return tmp_path


@pytest.mark.parametrize("workload,kernel,source", [
    ("memory_bound", "decode_mma16_kernel", "decode_mma.cu"),
    ("compute_bound", "decode_wide_kernel", "decode_wide.cu"),
])
def test_traffic_follows_the_kernel_code(bench, monkeypatch, tmp_path, workload, kernel, source):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    path = root / "profiles" / f"decode_{workload}_ncu.md"
    text = path.read_text()
    recorded = float(re.search(r"traffic_bytes_per_launch:\s*(\S+)", text).group(1))
    # stamp the summary with the copied sources' hash: the figure is reported
    stamped = re.sub(r"kernel_source_hash: \S+", "kernel_source_hash: " + bench.kernel_source_hash(kernel), text)
    path.write_text(stamped)
    assert bench.recorded_traffic(workload, kernel) == recorded
    # a comment-only edit keeps it
    src = root / "paged_mla_decode_11_b200" / "csrc" / source
    src.write_text(src.read_text() + "\n// a note\n")
    assert bench.recorded_traffic(workload, kernel) == recorded
    # a code edit drops it
    src.write_text(src.read_text() + "\nstatic int unused_marker_for_the_test;\n")
    assert bench.recorded_traffic(workload, kernel) is None
    # no summary, no figure
    path.unlink()
    assert bench.recorded_traffic(workload, kernel) is None


def test_absorb_traffic_follows_the_kernel_code(bench, monkeypatch, tmp_path):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    path = root / "profiles" / "absorb_ncu.md"
    text = path.read_text()
    recorded = float(re.search(r"traffic_bytes_per_launch:\s*(\S+)", text).group(1))
    stamped = re.sub(r"kernel_source_hash: \S+",
                     "kernel_source_hash: " + bench.kernel_source_hash("absorb_gemm_kernel"), text)
    path.write_text(stamped)
    assert bench.recorded_traffic("absorb", "absorb_gemm_kernel", "absorb_ncu.md") == recorded
    src = root / "paged_mla_decode_11_b200" / "csrc" / "absorb.cu"
    src.write_text(src.read_text() + "\nstatic int unused_marker_for_the_test;\n")
    assert bench.recorded_traffic("absorb", "absorb_gemm_kernel", "absorb_ncu.md") is None


def test_committed_absorb_traffic_is_the_algorithmic_reads(bench):
    # the two products read every weight and activation byte once (their 23 MB of results
    # stay in L2 while they run, so the capture counts reads only)
    T, H = bench.ABSORB_TOKENS, bench.ABSORB_HEADS
    text = open(os.path.join(ROOT, "profiles", "absorb_ncu.md")).read()
    traffic = float(re.search(r"traffic_bytes_per_launch:\s*(\S+)", text).group(1))
    reads = 2 * (T * H * 128 + T * H * 64 + H * 128 * 512 + T * H * 512 + H * 128 * 512)
    assert 0.999 <= traffic / reads <= 1.01


@pytest.mark.parametrize("workload,lo,hi", [("memory_bound", 0.99, 1.05), ("compute_bound", 0.99, 1.10)])
def test_committed_traffic_is_close_to_the_algorithmic_bytes(bench, workload, lo, hi):
    # whatever kernel version it was taken on, a committed figure far from the algorithmic
    # bytes of its workload would mean a wrong capture (another workload, re-reads)
    import torch

    from paged_mla_decode_11_b200 import workloads as W
    text = open(os.path.join(ROOT, "profiles", f"decode_{workload}_ncu.md")).read()
    traffic = float(re.search(r"traffic_bytes_per_launch:\s*(\S+)", text).group(1))
    w = W.WORKLOADS[workload]
    # the lengths are the generator's first draw for seed 0 (the bench's inputs)
    lens = W._draw_seqlens(w, torch.Generator().manual_seed(0)).tolist()
    nbytes, _ = W.algorithmic_work(lens, w.s_q, w.h_q, w.h_kv, w.causal)
    assert lo <= traffic / nbytes <= hi


def test_decode_kernel_choice_follows_rows(bench):
    assert bench.decode_kernel_for(16) == "decode_mma16_kernel"
    assert bench.decode_kernel_for(17) == "decode_wide_kernel"
    assert bench.decode_kernel_for(256) == "decode_wide_kernel"          # g unknown
    # whole 128-row blocks whose g is a multiple or divisor of 64: the CTA-pair kernel
    assert bench.decode_kernel_for(128, 128) == "decode_pair_kernel"
    assert bench.decode_kernel_for(256, 128) == "decode_pair_kernel"
    assert bench.decode_kernel_for(128, 32) == "decode_pair_kernel"
    assert bench.decode_kernel_for(64, 64) == "decode_wide_kernel"      # skewed: one 64-row block
    assert bench.decode_kernel_for(192, 96) == "decode_wide_kernel"


def test_whole_job_aggregate_is_weak_scaling(bench):
    # each rank decodes its own batch: N ranks do N times the units in the slowest rank's time
    assert bench.aggregate_throughput(100.0, 1, 2.0) == 50.0
    assert bench.aggregate_throughput(100.0, 8, 2.0) == 400.0
