"""Host logic of bench.py's roofline object: which roof binds a kernel at its
arithmetic intensity, and the achieved figure against that roof."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth_inputs as si  # noqa: E402

PEAKS = {"bf16_tflops": 1650.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}


def test_long_segments_are_tensor_bound():
    wl = si.varlen_gqa()
    F = wl.fwd_flops()
    fwd_ms, bwd_ms = F / 1e15 * 1e3, 2.5 * F / 0.9e15 * 1e3  # 1000 and 900 TF/s
    # a short timed region: the burst peak is the roof
    k, r = bench.kernel_rooflines(wl, fwd_ms, bwd_ms, PEAKS, "measured", 0.05)
    assert k["attn_fwd"]["bound"] == "tensor" and k["attn_bwd_main"]["bound"] == "tensor"
    assert r["kernel"] == "attn_bwd_main" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - 900.0) < 1e-6 and abs(r["frac"] - 900.0 / 1650.0) < 1e-9
    assert r["peak"] == 1650.0 and "burst" in r["peak_kind"]
    assert abs(r["frac_of_sustained"] - 900.0 / 1400.0) < 1e-9


def test_long_timed_region_uses_sustained_peak():
    wl = si.d256_gqa8(131072, False)
    F = wl.fwd_flops()
    k, r = bench.kernel_rooflines(wl, F / 1.3e15 * 1e3, 2.5 * F / 0.7e15 * 1e3, PEAKS,
                                  "measured", 16.0)
    assert r["kernel"] == "attn_bwd_main" and r["peak"] == 1400.0
    assert "sustained" in r["peak_kind"]
    assert abs(r["frac"] - 700.0 / 1400.0) < 1e-9 and abs(r["frac_of_burst"] - 700 / 1650) < 1e-9


def test_short_segments_forward_is_hbm_bound():
    wl = si.short_segments(128, 16384)
    # bytes: Q, O 32 heads and K, V 8 heads of 16384 rows x 256 bytes, LSE 4 bytes per row-head
    assert wl.fwd_bytes(True) == 256 * (2 * 16384 * 32 + 2 * 16384 * 8) + 4 * 32 * 16384
    assert wl.bwd_main_bytes() == 256 * (2 * 16384 * 32 + 4 * 16384 * 8) + 8 * 32 * 16384
    fwd_ms = wl.fwd_bytes(True) / 5e12 * 1e3  # 5 TB/s
    k, r = bench.kernel_rooflines(wl, fwd_ms, 0.5 * fwd_ms, PEAKS, "measured", 0.05)
    assert k["attn_fwd"]["bound"] == "hbm"
    assert r["kernel"] == "attn_fwd" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - 5000.0) < 1e-6 and abs(r["frac"] - 5000.0 / 6500.0) < 1e-9


def test_source_hash_ignores_comments_only():
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "x//y /* z */";\n'
    assert bench.strip_c_comments(src) == 'int a = 1; const char* s = "x//y /* z */";'
    assert bench.strip_c_comments(src) == bench.strip_c_comments(
        src.replace("// note", "// another note"))
    assert bench.strip_c_comments(src) != bench.strip_c_comments(src.replace("a = 1", "a = 2"))


def test_kernel_source_sets_cover_their_headers():
    # every kernel's recorded traffic is tied to the files it is compiled from:
    # the ABI file, the PTX wrappers and its own kernel headers, and those exist
    csrc = os.path.join(ROOT, "exact_attention_129_b200", "csrc")
    for kernel, names in bench.KERNEL_SOURCES.items():
        assert {"api.cu", "ptx.cuh"} <= set(names), kernel
        for n in names:
            assert os.path.exists(os.path.join(csrc, n)), (kernel, n)
    assert any("fwd" in n for n in bench.KERNEL_SOURCES["attn_fwd"])
    assert not any("fwd" in n for n in bench.KERNEL_SOURCES["attn_bwd_main"])
    # a kernel's hash is over its own files only, and the whole-library hash differs
    assert bench.library_source_hash("attn_fwd") != bench.library_source_hash("attn_bwd_main")
    assert bench.library_source_hash() not in (bench.library_source_hash("attn_fwd"),
                                               bench.library_source_hash("attn_bwd_main"))
