"""bench.py host logic that needs no GPU: the code-only source hash that gates the profiled DRAM
traffic, and the whole-job throughput arithmetic."""
import bench


def test_code_only_ignores_comments_and_whitespace_but_not_code():
    a = "int x = 1; // note\n/* block\n comment */ int y =  2;\n"
    b = "int x = 1;\nint y = 2; // another note\n"
    c = "int x = 1; int y = 3;"
    assert bench._code_only(a) == bench._code_only(b) == "int x = 1; int y = 2;"
    assert bench._code_only(c) != bench._code_only(a)


def test_source_hash_covers_the_split_kernel_files():
    """The hash covers decode_sm100.cu and every local header it includes, transitively."""
    import os
    import re
    csrc = os.path.join(os.path.dirname(bench.__file__), "mla_decode_attention_14_b200", "csrc")
    need, todo = set(), ["decode_sm100.cu"]
    while todo:
        name = todo.pop()
        if name in need:
            continue
        need.add(name)
        with open(os.path.join(csrc, name)) as f:
            todo += [m for m in re.findall(r'#include "([^"/]+)"', f.read())]
    assert need <= set(bench.SPLIT_KERNEL_SOURCES), sorted(need - set(bench.SPLIT_KERNEL_SOURCES))
    h = bench.kernel_source_hash()
    assert len(h) == 16 and h == bench.kernel_source_hash()


def test_job_throughput_counts_every_rank():
    # 1 GB per rank, 4 ranks, 2 ms per step -> 2 TB/s
    assert abs(bench.job_throughput(10 ** 9, 4, 2.0) - 2.0) < 1e-12


def test_roofline_fractions_against_both_peaks():
    peaks = (6535.7, 1638.2, 1368.0, "measured")
    # 1 GB and 1 TFLOP in 1 ms: 1000 GB/s and 1000 TFLOP/s
    r = bench.roofline_fracs(10 ** 9, 10 ** 12, 1e-3, peaks)
    assert abs(r["hbm_frac"] - 1000 / 6535.7) < 1e-12
    assert abs(r["tensor_frac"] - 1000 / 1638.2) < 1e-12
    assert abs(r["hbm_frac_spec"] - 1000 / bench.SPEC_HBM_GBS) < 1e-12
    assert abs(r["tensor_frac_spec"] - 1000 / bench.SPEC_BF16_TFLOPS) < 1e-12
    assert r["bound"] == "tensor"  # 1000 flop/B is above the ridge (~251)
    assert bench.roofline_fracs(10 ** 9, 10 ** 10, 1e-3, peaks)["bound"] == "hbm"


def test_config_set_names_known_workloads():
    from mla_decode_attention_14_b200 import workloads as W
    keys = set()
    for name, kv, topk in bench.CONFIG_SET:
        assert name in W.NAMES and kv in ("bf16", "fp8")
        assert topk is None or (kv == "bf16" and topk > 0)
        keys.add((name, kv, topk))
    assert len(keys) == len(bench.CONFIG_SET)
    # every workload appears in both cache formats, apart from tiny (bf16 only)
    assert {n for n, k, t in bench.CONFIG_SET if k == "fp8"} == set(W.NAMES) - {"tiny"}
