"""Host-side pieces of bench.py that need no GPU: the clock summary and the
algorithmic byte / flop counts the roofline divides by."""
import bench
from latent_kv_decode_b200 import workloads as wl


def test_clock_summary_maps_nvml_reason_bits():
    c = bench.ClockSampler(0)
    c.samples = [(1965.0, 1965.0, 0x0), (1900.0, 1965.0, 0x4), (1305.0, 1965.0, 0x8 | 0x40)]
    s = c.summary()
    assert s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]


def test_clock_summary_reads_nvidia_smi_lines():
    c = bench.ClockSampler(0)
    c.lines = ["0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Active"]
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["reasons"] == ["sw_power_cap"]


def test_algorithmic_bytes_of_the_dsv3_step():
    # cache (B*Lk*(Ckv+Dr)*2) + wkv_b (H*(Dn+Vd)*Ckv*2) + q (B*H*(Dn+Dr)*2) + out (B*H*Vd*2)
    w = wl.Workload(name="shape", B=64, H=128, Q=1, Dn=128, Dr=64, Vd=128, Ckv=512, Lk=4096,
                    dtype="bf16", softmax_scale=1.0, q_nope=None, q_pe=None, kv_cache=None,
                    pe_cache=None, wkv_b=None)
    a = bench.algorithmic(w)
    assert a["step_bytes"] == 64 * 4096 * 576 * 2 + 128 * 256 * 512 * 2 + 64 * 128 * 192 * 2 + 64 * 128 * 128 * 2
    assert a["step_bytes"] == 340_787_200
    # QK 576-wide + PV 512-wide per (row, token); absorb + up-projection per row
    assert a["step_flops"] == 2 * 64 * 128 * 4096 * (576 + 512) + 2 * 64 * 128 * 512 * (128 + 128)


def test_code_hash_ignores_comments_but_not_code():
    src = 'int a = 1; // note\n/* block */ const char* s = "x // kept";\n'
    assert bench._code_only(src) == bench._code_only(src.replace("note", "other note"))
    assert bench._code_only(src) != bench._code_only(src.replace("a = 1", "a = 2"))
    assert '"x // kept"' in bench._code_only(src)


def test_committed_profiles_match_the_current_kernel_code():
    # each decode summary names its kernel's sources and the hash of their code
    # when it was captured; the bench reports its traffic only while they match.
    # A kernel edited after its capture shows up here as an expected failure
    # until the summary is taken again.
    import os
    import re
    import pytest
    stale = []
    for workload, lo, hi in [("dsv3_b64_lk4096", 3.0e8, 3.4e8), ("v41_fp4_sink_h64", 7.5e7, 9.0e7)]:
        txt = open(os.path.join(bench.ROOT, "profiles", f"decode_{workload}.md")).read()
        assert re.search(r"kernel sources:\s*\S+", txt) and re.search(r"dram bytes per launch:\s*[0-9.eE+]+", txt)
        t = bench.profiled_traffic(workload)
        if t is None:
            stale.append(workload)
        else:
            assert lo <= t <= hi
    if stale:
        pytest.xfail(f"profile summaries older than the kernel code: {stale}")


def test_spec_fraction_uses_the_datasheet_peak_of_the_unit():
    assert abs(bench.spec_fraction(4000.0, "GB/s") - 0.5) < 1e-12
    assert abs(bench.spec_fraction(1125.0, "TFLOP/s") - 0.5) < 1e-12


def test_algorithmic_bytes_of_the_grouped_w_o():
    # V4.1 shape: two 64 MiB bf16 factors, x (32, 64, 1, 512), z (32, 8192) out and back, y (32, 4096)
    byts, flops = bench.group_wo_algorithmic(32, 64, 1, 512, 8, 1024, 4096)
    assert byts == 2 * 64 * 2**20 + 32 * 64 * 512 * 2 + 2 * 32 * 8192 * 2 + 32 * 4096 * 2
    assert byts == 137_625_600
    assert flops == 2 * 32 * (8 * 1024 * 4096 + 4096 * 8192)


def test_profiled_traffic_is_read_only_while_the_sources_match(tmp_path, monkeypatch):
    # a summary carries the hash of the kernel code it was captured with; the
    # bench reports its DRAM bytes only while the sources still hash to it
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "group_wo_wl.md").write_text(
        "kernel sources: a.cu b.cuh\nkernel source hash: `0123456789abcdef` (code)\n"
        "dram bytes per call: 1.5e8 (both passes)\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files: "0123456789abcdef")
    assert bench.profiled_traffic("wl", kernel="group_wo", per="call") == 1.5e8
    assert bench.profiled_traffic("wl", kernel="group_wo", per="launch") is None
    assert bench.profiled_traffic("other", kernel="group_wo", per="call") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files: "fedcba9876543210")
    assert bench.profiled_traffic("wl", kernel="group_wo", per="call") is None
