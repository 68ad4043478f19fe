"""Host logic of bench.py on CPU: the kernel launches it claims per forward,
the bound it picks for the gate/up kernel's roofline, and the e4m3 peak it
measures against."""
import bench
import workloads as W

PEAKS = {"hbm_gbs": 6535.7, "bf16_tflops": 1630.1, "bf16_tflops_sustained": 1381.3}


def test_kernels_per_step_matches_the_profiled_launch_lists():
    # the ncu launch lists under profiles/ count 24 launches in two c2_prefill
    # steps and 26 in two c4_fp8 steps
    assert bench.kernels_per_step(W.CONFIGS["c2_prefill"], 148) == 12
    assert bench.kernels_per_step(W.CONFIGS["c4_fp8"], 148) == 13


def test_kernels_per_step_variants():
    s2 = W.CONFIGS["c2_prefill"]
    # small T: the router's K range is split (score pass + top-k instead of the merge)
    assert bench.kernels_per_step(W.CONFIGS["c1_decode"], 148) == bench.KERNELS_PER_STEP + 2
    # FP4 experts at full width: h quantised in the gate/up epilogue (as FP8)
    c1_fp4 = W.CONFIGS["c1_fp4"]
    c1_fp8 = W.LayerShape("d", T=c1_fp4.T, d_model=4096, d_lat=2048, n_experts=512, top_k=10, d_ff=2048,
                          n_routers=4, fp8=True)
    assert bench.kernels_per_step(c1_fp4, 148) == bench.kernels_per_step(c1_fp8, 148)
    # FP4 experts with a d_lat that does not split into 256-wide slices: a
    # quantiser pass over h follows the gate/up GEMM
    c0_fp4, c0_fp8 = W.CONFIGS["c0_fp4"], W.CONFIGS["c0_fp8"]
    assert bench.kernels_per_step(c0_fp4, 148) == bench.kernels_per_step(c0_fp8, 148) + 1
    # the bf16 layer: no quantiser
    assert bench.kernels_per_step(W.CONFIGS["c2_prefill"].with_T(16384), 148) == bench.kernels_per_step(s2, 148) - 1


def _probe(tflops=2600.0):
    bench._E4M3_PROBE.clear()
    if tflops is None:
        bench._E4M3_PROBE["dev"] = {"unavailable": "no e4m3 GEMM in this build"}
    else:
        bench._E4M3_PROBE["dev"] = {"tflops": tflops, "gemm": "probe"}


def test_gate_up_roofline_takes_the_larger_floor():
    _probe()
    # c2: weight bytes dominate (HBM); c3: 4x the rows on the same weights (tensor)
    r2 = bench.glu_roofline(W.CONFIGS["c2_prefill"], 2.0, 512, PEAKS, "measured", "dev")
    assert r2["bound"] == "hbm" and r2["unit"] == "GB/s"
    assert abs(r2["achieved"] - bench.glu_kernel_bytes(W.CONFIGS["c2_prefill"], 512) / 2e-3 / 1e9) < 1e-6
    r3 = bench.glu_roofline(W.CONFIGS["c3_skew"], 7.0, 512, PEAKS, "measured", "dev")
    assert r3["bound"] == "tensor" and r3["peak"] == PEAKS["bf16_tflops_sustained"]
    # e4m3 at prefill size: FLOPs against the probe; e2m1 at decode size: bytes
    r4 = bench.glu_roofline(W.CONFIGS["c4_fp8"], 2.1, 512, PEAKS, "measured", "dev")
    assert r4["bound"] == "tensor" and r4["peak"] == 2600.0
    assert abs(r4["frac"] - bench.glu_kernel_flops(W.CONFIGS["c4_fp8"]) / 2.1e-3 / 1e12 / 2600.0) < 1e-12
    r1 = bench.glu_roofline(W.CONFIGS["c1_fp4"], 0.5, 470, PEAKS, "measured", "dev")
    assert r1["bound"] == "hbm"
    # weight bytes: e2m1 half a byte, e4m3 one, bf16 two
    fp4 = bench.glu_kernel_bytes(W.CONFIGS["c1_fp4"], 470)
    fp8 = bench.glu_kernel_bytes(W.CONFIGS["c4_fp8"], 470)
    bf16 = bench.glu_kernel_bytes(W.CONFIGS["c1_decode"], 470)
    assert 4 * fp4 == 2 * fp8 == bf16 == 471 * 2 * 2048 * 2048 * 2


def test_e4m3_peak_falls_back_to_twice_the_sustained_bf16_peak():
    _probe(None)
    peak, kind, probe = bench.e4m3_peak("dev", PEAKS, "measured")
    assert peak == 2 * PEAKS["bf16_tflops_sustained"] and "assumed" in kind and "unavailable" in probe
    _probe(2500.0)
    peak, kind, _ = bench.e4m3_peak("dev", PEAKS, "measured")
    assert peak == 2500.0 and kind.startswith("measured")
    bench._E4M3_PROBE.clear()


def test_profiled_traffic_only_on_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    # a committed summary carries the hash of csrc/ it was captured on; any
    # other hash reads as "no traffic figure"
    (tmp_path / "profiles").mkdir()
    p = tmp_path / "profiles" / "k__w.json"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_hash", lambda: "abc")
    p.write_text('{"csrc_hash": "abc", "dram_bytes_per_launch_full": 123.0}')
    assert bench.profiled_traffic("k", "w") == 123.0
    p.write_text('{"csrc_hash": "old", "dram_bytes_per_launch_full": 123.0}')
    assert bench.profiled_traffic("k", "w") is None
    assert bench.profiled_traffic("missing", "w") is None
