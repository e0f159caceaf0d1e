"""Host-side pieces of bench.py's secondary lines (no GPU): the attention
roofline object and the oracle CPU baseline of a Light-Ulysses rank share."""
import bench


PEAKS = {"hbm_gbs": 6548.8, "bf16": 1628.7, "bf16_sustained": 1380.3, "source": "measured",
         "int8": 3000.0, "fp8": 3400.0, "int8_sustained": 2600.0, "fp8_sustained": 2900.0,
         "source_8bit": "measured"}


def test_attn_roofline_int8_and_bf16():
    r = bench.attn_roofline(2.0e12, 2.0, PEAKS, "int8fp8", 128)      # 1000 TFLOP/s
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    # the 8-bit burst peak is the larger of the measured int8 and fp8 figures
    assert r["achieved"] == 1000.0 and r["peak"] == 3400.0
    assert r["frac"] == round(1000.0 / 3400.0, 3)
    assert r["frac_of_sustained"] == round(1000.0 / 2900.0, 3)
    assert "tcgen05_peak_at_clock" not in r
    b = bench.attn_roofline(2.0e12, 2.0, PEAKS, "bf16", 128)
    assert b["peak"] == 1628.7 and b["kernel"] == "sparse_attn_kernel<128,bf16>"
    assert r["kernel"] == "sparse_attn_paired_kernel<128,int8fp8>"
    assert b["frac_of_sustained"] == round(1000.0 / 1380.3, 3)


def test_attn_roofline_tcgen05_rate_at_the_sampled_clock():
    # 8192 MAC/clk/SM x 2 x 148 SMs x 1965 MHz = 4764.9 TFLOP/s for 8-bit, half for bf16
    r = bench.attn_roofline(2.0e12, 2.0, PEAKS, "int8fp8", 128, sm_mhz=1965.0)
    assert r["tcgen05_peak_at_clock"] == round(2 * 8192 * 148 * 1965e6 / 1e12, 1)
    assert r["frac_of_tcgen05_at_clock"] == round(1000.0 / (2 * 8192 * 148 * 1965e6 / 1e12), 3)
    b = bench.attn_roofline(2.0e12, 2.0, PEAKS, "bf16", 128, sm_mhz=1965.0)
    assert b["tcgen05_peak_at_clock"] == round(8192 * 148 * 1965e6 / 1e12, 1)


def test_peaks_without_8bit_file_fall_back_to_twice_bf16_burst(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PEAKS_8BIT", str(tmp_path / "absent.json"))
    p = bench._peaks()
    assert p["int8"] == p["fp8"] == 2.0 * p["bf16"]
    assert p["int8_sustained"] == 2.0 * p["bf16_sustained"]


def test_attn_traffic_is_keyed_by_kernel_source(monkeypatch):
    import hashlib
    import os
    for mode in ("int8fp8", "bf16"):
        h = hashlib.sha256()
        for f in bench.ATTN_KERNEL[mode][1]:
            h.update(open(os.path.join(bench._CSRC, f), "rb").read())
        h = h.hexdigest()
        assert bench.attn_source_hash(mode) == h
        monkeypatch.setattr(bench, "ATTN_DRAM_BYTES", {"0" * 64: (1, "stale")})
        assert bench.attn_traffic(mode)[0] is None
        monkeypatch.setattr(bench, "ATTN_DRAM_BYTES", {h: (123, "capture")})
        assert bench.attn_traffic(mode) == (123, "capture")
    # the two modes run different kernels, so their keys differ
    assert bench.attn_source_hash("int8fp8") != bench.attn_source_hash("bf16")


def test_ulysses_cpu_sample_combines_exchange_and_attention():
    attn = {"value": 1e-3, "cores": 4, "sample": "fake attention rate"}   # 1 GFLOP/s
    flops = 1e9                                                            # 1 s of oracle attention
    r = bench.ulysses_cpu_sample(2, 1, 4, 64, 512, flops, sample_tokens=64, attn=attn)
    assert r["kind"] == "oracle" and r["unit"] == "TFLOP/s" and r["cores"] == 4
    # the exchange adds time, so the rate is below the attention-only rate
    assert 0 < r["value"] < 1e-3
    assert "64 of the shard's 256 tokens" in r["sample"]


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler_with(lines):
    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.lines = list(lines)
    return s.stop()


def test_clock_sampler_median_and_reasons():
    base = "0, {mhz}, 1965, 700.5, 0x0, {hw}, Not Active, Not Active, {pc}"
    lines = [base.format(mhz=m, hw="Not Active", pc="Not Active") for m in (1965, 1950, 1965)]
    r = _sampler_with(lines)
    assert r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0 and r["reasons"] == [] and r["samples"] == 3
    lines.append(base.format(mhz=1500, hw="Active", pc="Active"))
    r = _sampler_with(lines)
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert r["samples"] == 4 and r["sm_mhz"] == 1965.0


def test_clock_sampler_ignores_malformed_lines():
    r = _sampler_with(["garbage", "0, [N/A], 1965, 1, 0, a, b, c, d", ""])
    assert r["sm_mhz"] is None and r["samples"] == 0
