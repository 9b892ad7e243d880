"""Host-side pieces of bench.py that need no GPU: the algorithmic byte
counts the roofline divides by, the source digest that ties a committed
profile to the code it was taken on, and the CPU baseline legs."""
import bench
import workloads


def test_step_bytes_match_the_method_counts():
    # each source row read once, each destination written once (prefill:
    # T=4096, H=7168, k=8); the figures are the hand products
    T, H, k, E, R = 4096, 7168, 8, 256, 8
    b = bench.step_bytes(T, H, k, E, R)
    N = T * k
    assert b["dispatch_bf16"] == T * H * 2 + N * H * 2 == 528_482_304
    assert b["dispatch_fp8"] == T * H * 2 + N * H + N * (H // 128) * 4 == 300_941_312
    assert b["combine"] == N * H * 2 + T * H * 2 == 528_482_304
    # the layout reads the ids and writes its arrays: well under 1 MB here
    assert 0 < b["layout"] < 1 << 20


def test_source_digest_ignores_comments():
    code = "int f(int a) { return a + 1; }\n"
    assert bench._code_only("// note\n" + code + "/* block\n comment */\n") == \
        bench._code_only(code)
    assert bench._code_only(code) != bench._code_only(code.replace("+ 1", "+ 2"))


def test_cpu_baseline_reports_both_legs():
    cfg = workloads.CONFIGS["prefill"]
    batch = workloads.make_batch(cfg, seed=0, T=64, H=256)
    res = bench.cpu_baseline(cfg, batch, seconds=0.2)
    assert res["kind"] == "oracle" and res["cores"] == 1 and res["value"] > 0
    assert "whole 64-token" in res["sample"]
    allc = res["all_cores"]
    assert allc["kind"] == "oracle" and allc["cores"] >= 1 and allc["value"] > 0
    assert "threads" in allc["sample"]


def test_profiled_traffic_only_while_the_sources_match(tmp_path, monkeypatch):
    # the roofline's traffic figure is read back only for the code it was
    # captured on: a recorded digest that differs from the current sources'
    # (or a missing entry, or no file) gives None
    import json
    f = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.profiled_traffic("combine") is None
    rec = {"combine": {"traffic_bytes_per_launch": 123456,
                       "source_sha256": bench.kernel_source_digest("combine")},
           "dispatch_bf16": {"traffic_bytes_per_launch": 7,
                             "source_sha256": "0" * 64}}
    f.write_text(json.dumps(rec))
    assert bench.profiled_traffic("combine") == 123456.0
    assert bench.profiled_traffic("dispatch_bf16") is None
    assert bench.profiled_traffic("layout") is None


def test_kernel_digests_cover_distinct_sources():
    # every kernel named in the roofline has a digest over its own files;
    # kernels built from the same files share one
    d = {k: bench.kernel_source_digest(k) for k in bench.KERNEL_SOURCES}
    assert all(len(v) == 64 for v in d.values())
    assert d["combine"] == d["combine_fp8"]
    assert len({d["layout"], d["dispatch_bf16"], d["dispatch_fp8"], d["combine"]}) == 4


def test_workload_config_names_the_step_and_its_bytes():
    cfg = workloads.CONFIGS["prefill"]
    c = bench.workload_config(cfg, 1)
    assert c["workload"].startswith("prefill")
    assert (c["T"], c["H"], c["E"], c["R"], c["k"]) == (4096, 7168, 256, 8, 8)
    assert c["bytes_per_step"] == sum(bench.step_bytes(4096, 7168, 8, 256, 8).values())
    assert "flushed" in c["l2"]
    assert "model" not in c
