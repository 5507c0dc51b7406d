"""Host logic of bench.py that needs no GPU: the roofline's DRAM traffic is taken from a
committed ncu summary only while the summarised kernel's own sources are unchanged."""
import os

import bench


def _write(dirpath, kernel, workload, sha, nbytes):
    os.makedirs(os.path.join(dirpath, "profiles"), exist_ok=True)
    with open(os.path.join(dirpath, "profiles", f"{kernel}_{workload}.md"), "w") as f:
        f.write(f"# summary\n\nsource_sha: {sha}   (hash)\ndram_bytes_per_launch: {nbytes}\n")


def test_source_hash_is_per_kernel():
    shas = {k: bench.kernel_source_sha(k) for k in bench.KERNEL_SOURCES}
    assert len(set(shas.values())) == len(shas)         # each kernel hashes its own file
    assert all(len(v) == 16 for v in shas.values())
    assert bench.kernel_source_sha("act_quant") == bench.kernel_source_sha("act_quant")


def test_profiled_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda k: {"program_kernel": "aaaa",
                                                              "ternary_gemm": "bbbb"}[k])
    _write(tmp_path, "program_kernel", "wl", "aaaa", 1234)
    _write(tmp_path, "ternary_gemm", "wl", "cccc", 99)          # stale: sources changed since
    assert bench.profiled_traffic("program_kernel", "wl") == 1234.0
    assert bench.profiled_traffic("ternary_gemm", "wl") is None
    assert bench.profiled_traffic("program_kernel", "other") is None   # no summary
    assert bench.profiled_traffic("spin_kernel", "wl") is None         # not a profiled kernel


def test_committed_summaries_name_a_hash_and_traffic():
    root = os.path.dirname(os.path.abspath(bench.__file__))
    for name in ("program_kernel_hgrn370m_block_t64.md", "program_kernel_hgrn1p3b_decode_t8.md",
                 "ternary_gemm_hgrn1p3b_prefill_t32768.md", "mlgru_hgrn1p3b_mlgru_t32768.md",
                 "backward_hgrn1p3b_layer_backward_t8192.md"):
        text = open(os.path.join(root, "profiles", name), encoding="utf-8").read()
        assert "source_sha:" in text and "dram_bytes_per_launch:" in text, name


def test_mlgru_roofline_takes_the_binding_bound():
    # 32768 x 2048 fp16 call: 537 MB (82 us at 6546 GB/s) and 8 x 67.1 M special-function
    # operations (115 us at 16 x 148 x 1965 MHz): the special-function unit binds
    T, H = 32768, 2048
    r = bench.mlgru_roofline(T, H, False, 0.259, 6545.9, {"sm_mhz": 1965.0})
    assert r["bound"] == "alu" and r["other_bound"]["bound"] == "hbm"
    assert r["ops_per_call"] == 8 * T * H
    assert abs(r["peak"] - 16 * 148 * 1.965e9 / 1e12) < 1e-3
    assert abs(r["frac"] - 8 * T * H / 0.259e-3 / (16 * 148 * 1.965e9)) < 1e-4
    assert abs(r["other_bound"]["frac"] - bench.mlgru_bytes(T, H) / 0.259e-3 / 6545.9e9) < 1e-4
    # one token: the output pass alone, five operations per element; 16 KB at the copy rate
    # (2.5 ns) outlasts 10240 operations at the unit's rate (2.2 ns), so HBM is the bound
    r1 = bench.mlgru_roofline(1, H, False, 0.0066, 6545.9, {})
    assert r1["bound"] == "hbm" and r1["other_bound"]["ops_per_call"] == 5 * H
    assert r1["other_bound"]["frac_of_clock_scaled_peak"] is None
