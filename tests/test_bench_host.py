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
