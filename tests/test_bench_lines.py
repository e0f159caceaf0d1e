"""Host-side pieces of bench.py's secondary lines (no GPU): the attention
roofline object and the oracle CPU baseline of a Light-Ulysses rank share."""
import bench


PEAKS = {"hbm_gbs": 6548.8, "bf16": 1628.7, "bf16_sustained": 1380.3, "source": "measured"}


def test_attn_roofline_int8_and_bf16():
    r = bench.attn_roofline(2.0e12, 2.0, PEAKS, "int8fp8", 128)      # 1000 TFLOP/s
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == 1000.0 and r["peak"] == 2760.6
    assert r["frac"] == round(1000.0 / 2760.6, 3)
    b = bench.attn_roofline(2.0e12, 2.0, PEAKS, "bf16", 128)
    assert b["peak"] == 1380.3 and b["kernel"] == "sparse_attn_kernel<128,bf16>"


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
