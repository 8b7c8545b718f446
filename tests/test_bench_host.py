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


def test_committed_summaries_hold_the_small_case_figures():
    """Every workload whose traffic the bench estimates has a committed small-case summary
    with the figures profiled_traffic reads."""
    for workload, name in bench.PROFILE_FOR.items():
        path = os.path.join(bench.ROOT, "profiles", name + ".txt")
        kv = dict(l.split(":", 1) for l in open(path) if ":" in l and not l.startswith(" "))
        assert float(kv["small_dram_bytes_per_launch"].split()[0]) > 0, name
        assert float(kv["small_distinct_bytes_per_launch"].split()[0]) > 0, name
        assert int(kv["small_tokens"].split()[0]) == bench.gen.WORKLOADS[kv["small_workload"].split()[0]].N
        assert kv["scaling"].split()[0] in ("per_token", "distinct_ratio"), name
        assert len(kv["kernel_sha"].split()[0]) == 16, name


def _summary(tmp_path, scaling):
    (tmp_path / "profiles").mkdir(exist_ok=True)
    (tmp_path / "profiles" / "gather_bf16_prefill.txt").write_text(
        "kernel_sha: 0123456789abcdef  (comments stripped)\nsmall_workload: profile_prefill\n"
        "small_tokens: 100\nscaling: %s\nsmall_dram_bytes_per_launch: 1200\n"
        "small_distinct_bytes_per_launch: 1000  (U x rb + ...)\n" % scaling)


def test_profiled_traffic_scales_the_small_case(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_sha", lambda dtype="bf16", read=None: "0123456789abcdef")
    _summary(tmp_path, "distinct_ratio")
    t, src = bench.profiled_traffic("full_prefill", "bf16", 5000, 400)
    assert t == 6000 and "1.2000" in src
    _summary(tmp_path, "per_token")
    t, src = bench.profiled_traffic("full_prefill", "bf16", 5000, 400)
    assert t == 4800 and "12 per token" in src
    monkeypatch.setattr(bench, "kernel_sha", lambda dtype="bf16", read=None: "fedcba9876543210")
    t, src = bench.profiled_traffic("full_prefill", "bf16", 5000, 400)
    assert t is None and "other kernel code" in src
    assert bench.profiled_traffic("mid", "bf16", 5000, 400)[0] is None


def test_distinct_bytes_and_the_resolved_launch_in_both_arms():
    import argparse
    w = bench.gen.WORKLOADS["full_prefill"]
    # every distinct row once, residual + out per token, token ids, the gate
    assert bench.distinct_bytes(w, 10) == 10 * 5120 + w.N * (4 * 2560 + 4) + 4 * 2560
    args = argparse.Namespace(launch="auto", variant="default", batches=2, gpus=1)
    assert bench.config_for(w, args)["launch"] == "eager"
    assert bench.config_for(bench.gen.WORKLOADS["full_decode_256"], args)["launch"] == "graph"


def test_decode_batches_span_twice_the_l2():
    for name in ("full_decode_1", "full_decode_16", "full_decode_64", "full_decode_256", "full_prefill"):
        w = bench.gen.WORKLOADS[name]
        nb = bench.batches_for(w)
        assert nb >= 2 and nb * w.N * 16 * bench.row_bytes(w) >= 2 * bench.L2_BYTES
        assert (nb - 1) * w.N * 16 * bench.row_bytes(w) < 2 * bench.L2_BYTES or nb == 2
