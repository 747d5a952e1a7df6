"""Host-side arithmetic of bench.py (no GPU): algorithmic bytes of the
quantize kernels and the weak-scaling aggregate."""
import bench
from synth import WORKLOADS


def test_quant_bytes_fp8_is_read_write_and_row_scales():
    layer = WORKLOADS["flux_qkv_fp8"].layers[0]          # 4608 x 3072
    assert bench.quant_bytes(layer) == 4608 * 3072 * 2 + 4608 * 3072 + 4608 * 4


def test_quant_bytes_nvfp4_counts_the_amax_pass():
    layer = WORKLOADS["flux2k_swiglu_nvfp4"].layers[0]   # 16896 x 3072
    mk = 16896 * 3072
    assert bench.quant_bytes(layer) == 2 * mk + 2 * mk + mk // 2 + mk // 16 + 16


def test_weak_scaling_counts_every_rank_over_the_slowest():
    # 2 ranks x 10 steps x 1e12 FLOP in 4 s (the max over ranks) = 5 TFLOP/s
    assert abs(bench.weak_scaling_tflops(1e12, 2, 10, 4000.0) - 5.0) < 1e-12


def test_cpu_baseline_runs_for_every_format_and_epilogue():
    # the oracle leg of the benchmark handles each layer format (and the QKV
    # epilogue's extra inputs); token counts shrunk so it runs in seconds
    for name in ("tiny_fp8", "flux2k_swiglu_nvfp4", "flux_qkv_w8a16", "flux_qkv_normrope_fp8"):
        wl = bench.with_tokens(WORKLOADS[name], 8)
        tflops, rows, dt, cores = bench.cpu_baseline(wl, 0.01)
        assert tflops > 0 and 1 <= rows <= 8 and cores >= 1


def test_kernel_fingerprint_follows_code_not_comments():
    # the recorded DRAM traffic is reported only while the kernel's code is
    # the one that was profiled: comment edits keep the fingerprint, code
    # edits change it
    src = "int a; // note\n/* block\n comment */ int b;\n\n"
    assert bench.strip_comments(src) == bench.strip_comments("int a;   \n int b; // other\n")
    assert bench.strip_comments(src) != bench.strip_comments("int a; int c;\n")
    assert len(bench.gemm_source_sha()) == 16


def _bench(args, env_extra=None):
    import json
    import os
    import subprocess
    import sys
    env = dict(os.environ)
    env.update(env_extra or {})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], env=env,
                       capture_output=True, text=True, timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_prints_the_contract_line():
    # the reference arm is the oracle timed on the host cores, on the same
    # metric and workload as the GPU arm
    (line,) = _bench(["--impl", "reference", "--steps", "2", "--warmup", "1",
                      "--workload", "tiny_fp8"])
    assert line["impl"] == "reference"
    assert line["metric"] == "quantized DiT linear TFLOP/s at FLUX shapes"
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 1 and line["value"] > 0
    assert line["config"]["workload"] == "tiny_fp8"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_runs_on_rank_zero_only():
    # under a multi-rank launch the other ranks exit cleanly without work
    assert _bench(["--impl", "reference", "--steps", "1", "--warmup", "0",
                   "--workload", "tiny_fp8"],
                  {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"}) == []


def test_recorded_traffic_matches_the_algorithmic_bytes_it_was_scaled_by():
    # profiles/traffic.json records, beside each capture, the algorithmic
    # bytes of the captured launch and of the benchmark's launch; they must
    # be the bench's own figures, and a capture of a smaller M is scaled by
    # exactly their ratio (the weight re-reads grow with M)
    import dataclasses
    import json
    import os
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for key, e in rec.items():
        name, _, j = key.partition(":")
        layer = WORKLOADS[name].layers[int(j)]
        assert e["kernel"].startswith("qgemm_kernel<" + layer.fmt + ",")
        assert os.path.exists(os.path.join(bench.ROOT, e["capture"]))
        b, cap = bench.profiled_traffic(name, int(j), layer.M)
        fresh = e["source_sha"] == bench.gemm_source_sha()
        assert (b is not None) == fresh
        if "M" in e:
            small = dataclasses.replace(layer, M=e["M"])
            assert e["algorithmic_bytes_captured"] == bench.gemm_bytes(small)
            assert e["algorithmic_bytes_full"] == bench.gemm_bytes(layer)
            if fresh:
                ratio = e["algorithmic_bytes_full"] / e["algorithmic_bytes_captured"]
                assert b == int(float(e["dram_bytes_per_launch"]) * ratio)
                assert cap == e["capture"]
        else:
            assert e["algorithmic_bytes"] == bench.gemm_bytes(layer)
            if fresh:
                assert b == e["dram_bytes_per_launch"]
