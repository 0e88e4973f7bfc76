"""The benchmark's host logic on CPU: algorithmic byte counts, the recorded-traffic
lookup keyed by the kernel source, and the clock sampler (with a fake NVML helper)."""
import subprocess
import sys
import time

import bench
from expert_ffn_layer_moe_b200.inputs import CONFIGS, MoEConfig


def test_byte_counts_by_hand():
    cfg = MoEConfig("b", N=10, H=64, I=128, E=4, k=2)          # R = 20
    # bf16: W1+W3 tiles of 3 touched experts + x_perm read + h written
    assert bench.gemm13_bytes(cfg, 3) == 3 * 2 * 128 * 64 * 2 + 20 * 64 * 2 + 20 * 128 * 2
    assert bench.gemm2_bytes(cfg, 3) == 3 * 64 * 128 * 2 + 20 * 128 * 2 + 20 * 64 * 2
    # e4m3 weights add a 4-byte scale per weight row; e4m3 activations a scale per activation row
    assert bench.gemm13_bytes(cfg, 3, 1) == 3 * 2 * 128 * 64 + 3 * 2 * 128 * 4 + 20 * 64 * 2 + 20 * 128 * 2
    assert bench.gemm13_bytes(cfg, 3, 1, 1) == (3 * 2 * 128 * 64 + 3 * 2 * 128 * 4 + 20 * 64 + 20 * 4
                                               + 20 * 128 * 2)
    assert bench.gemm2_bytes(cfg, 3, 1, 1) == 3 * 64 * 128 + 3 * 64 * 4 + 20 * 128 + 20 * 4 + 20 * 64 * 2
    # the layer: touched experts' weights + shared weights + router + x in + out
    s = MoEConfig("s", N=10, H=64, I=128, E=4, k=2, Is=192)
    assert bench.layer_bytes(s, 4) == 4 * 3 * 64 * 128 * 2 + 3 * 64 * 192 * 2 + 64 * 4 * 4 + 2 * 10 * 64 * 2


def test_headline_bytes_match_the_worked_example():
    # Mixtral-8x22B decode: 8 experts x 3 matrices of 6144 x 16384 bf16 = 4.83 GB per step
    cfg = CONFIGS["mixtral_8x22b_decode"]
    assert abs(bench.layer_bytes(cfg, 8) - 4.8359e9) < 1e6
    assert bench.gemm13_bytes(cfg, 8) == 3235282944


def test_traffic_lookup_follows_the_kernel_source(tmp_path):
    src = tmp_path / "k.cu"
    src.write_text("int f() { return 1; }\n")
    d0 = bench.kernel_source_digest(str(src))
    src.write_text("// a comment\n\nint f() { return 1; } /* another */\n")
    assert bench.kernel_source_digest(str(src)) == d0            # comments and blank lines do not count
    src.write_text("int f() { return 2; }\n")
    assert bench.kernel_source_digest(str(src)) != d0
    # a recorded line counts only while its digest is the kernel source's current one
    rec = tmp_path / "traffic.txt"
    rec.write_text(f"# comment\ngemm13 wl 123.0 {bench.kernel_source_digest(str(src))}\n"
                   f"gemm13 old 456.0 {d0}\n")
    assert bench.kernel_traffic("gemm13", "wl", str(rec), str(src)) == 123.0
    assert bench.kernel_traffic("gemm13", "old", str(rec), str(src)) is None     # source changed since
    assert bench.kernel_traffic("gemm13", "no_such_workload", str(rec), str(src)) is None


FAKE_NVML = r"""
import sys, time
print("ready", flush=True)
time.sleep(float(sys.argv[1]))
while True:
    print(time.time(), 1800, 1965, 700000, 0x4 | 0x20, flush=True)
    time.sleep(0.002)
"""


def _sampler_with_fake(delay):
    c = bench.ClockSampler(0)
    c.proc = subprocess.Popen([sys.executable, "-c", FAKE_NVML, str(delay)], stdout=subprocess.PIPE, text=True)
    assert c.proc.stdout.readline().strip() == "ready"
    return c


def test_clock_sampler_keeps_a_sample_for_a_short_region():
    c = _sampler_with_fake(0.05)                  # the helper's first sample comes after the region
    with c:
        time.sleep(0.001)
    s = c.summary()
    assert s is not None and s["samples"] >= 1
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965 and s["power_w_max"] == 700.0
    assert s["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]


def test_clock_sampler_region_samples():
    c = _sampler_with_fake(0.0)
    time.sleep(0.02)
    with c:
        time.sleep(0.05)
    s = c.summary()
    assert s["samples"] >= 5


def test_weight_rotation_covers_twice_l2():
    l2 = 126 << 20
    assert bench.rotation_copies(4.83e9, l2) == 1                # streamed from HBM anyway
    for wb in (6e6, 77e6, 200e6):                                # tiny, Qwen3-30B N=1, just under 2 x L2
        c = bench.rotation_copies(wb, l2)
        assert c >= 2 and c * wb >= 2 * l2 and (c - 1) * wb < 2 * l2
    big = bench.l2_note(4.83e9, 8, l2, 1)
    small = bench.l2_note(6e6, 8, l2, bench.rotation_copies(6e6, l2))
    assert big.startswith("inputs larger than L2") and small.startswith("weight rotation")


def test_oracle_sample_size():
    cfg = CONFIGS["qwen3_235b_a22b_skew"]
    assert bench.sample_size(cfg, 1e6, 15.0, 8) == cfg.N          # the whole batch fits
    n = bench.sample_size(cfg, 100.0, 15.0, 8)
    assert n == 1496 and n % 8 == 0                               # whole rounds of the threads
    assert bench.sample_size(cfg, 0.1, 15.0, 8) == 1
