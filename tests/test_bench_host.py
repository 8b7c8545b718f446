"""Host logic of bench.py that needs no GPU: the code hash that ties a committed ncu
summary to the kernel sources, and the reading of those summaries."""
import os

import bench


def test_code_hash_ignores_comments_and_blank_lines():
    a = "int f(int x) {  // the identity\n    return x;   /* plain */\n}\n"
    b = "/* header\n   text */\nint f(int x) {\n\n    return x;\n}  // end\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(a.replace("return x", "return x + 1"))


def test_kernel_hash_follows_code_not_comments():
    rel = bench.KERNEL_SOURCES["bf16"][0]
    with open(os.path.join(bench.ROOT, rel)) as f:
        text = f.read()

    def read(extra):
        return lambda r: (text + extra) if r == rel else open(os.path.join(bench.ROOT, r)).read()

    base = bench.kernel_sha("bf16")
    assert bench.kernel_sha("bf16", read("\n// a comment added\n")) == base
    assert bench.kernel_sha("bf16", read("\nint an_added_symbol;\n")) != base


def test_committed_summaries_name_a_traffic_for_each_timed_format():
    for workload, dtype in (("full_prefill", "bf16"), ("fp8_prefill", "fp8"),
                            ("int8_uniform", "int8"), ("nvfp4_prefill", "nvfp4")):
        path = os.path.join(bench.ROOT, "profiles", "gather_%s.txt" % workload)
        kv = dict(l.split(":", 1) for l in open(path) if ":" in l and not l.startswith(" "))
        assert int(kv["traffic_bytes_per_launch"]) > 0
        assert len(kv["kernel_sha"].split()[0]) == 16
