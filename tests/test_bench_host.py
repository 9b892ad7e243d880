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
