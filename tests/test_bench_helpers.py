"""bench.py's helper logic on CPU: the tensor peak per dtype, the code-only source hash
that keys the committed profiles, the profile lookup, and the HBM/tensor bound choice."""
import bench
import synth


def test_tensor_peak_per_dtype():
    pk = {"bf16_tflops": 1000.0, "hbm_gbs": 6000.0, "source": "measured"}
    assert bench.tensor_peak(pk, synth.WORKLOADS["seq4096_b8_h32_d128"])[0] == 1000.0
    assert bench.tensor_peak(pk, synth.WORKLOADS["seq4096_b8_h32_d128_f16"])[0] == 1000.0
    peak, src = bench.tensor_peak(pk, synth.WORKLOADS["seq4096_b8_h32_d128_fp8"])
    f8 = bench.fp8_peak()
    if f8 is not None:   # the measured E4M3 GEMM figure committed under profiles/
        assert peak == f8 and "measured E4M3" in src and 1.5 * 1638.2 < f8 < 2.5 * 1638.2
    else:                # else the nominal dense fp8 / bf16 ratio
        assert peak == 2000.0 and "x 2" in src


def test_code_only_ignores_comments_not_code():
    a = "int f(int x) { return x + 1; }  // add one\n/* block\n comment */\n"
    b = "// header\nint f(int x) {\n    return x + 1;\n}\n"
    c = "int f(int x) { return x + 2; }\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_profiled_traffic_requires_matching_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc123")
    f = prof / f"{bench.KERNEL_NAME}_w.md"
    f.write_text("kernel_source_hash: abc123\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic("w") == 12345.0
    f.write_text("kernel_source_hash: 0000\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic("w") is None            # stale: the kernel changed since
    assert bench.profiled_traffic("missing") is None


def test_decode_is_byte_bound_and_headline_tensor_bound():
    pk = bench.FALLBACK_PEAKS
    for name, bytes_bound in [("decode_b4_hq32_hkv8_nq16_nk32k_d128", True), ("seq4096_b8_h32_d128", False)]:
        w = synth.WORKLOADS[name]
        t_bytes = w.io_bytes / (pk["hbm_gbs"] * 1e9)
        t_flops = w.flops / (bench.tensor_peak(pk, w)[0] * 1e12)
        assert (t_bytes > t_flops) == bytes_bound, name
