"""Host-side pieces of bench.py that need no GPU: the CPU baselines of the
backward and cell modes (bounded oracle samples), and the source hash that
ties a committed profile to the forward kernels."""
import os
import shutil

import bench
from dynamic_convolution_b200 import synth


def test_cpu_baseline_backward_small():
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_inputs(cfg)
    r = bench.cpu_baseline_backward(cfg, inp, synth.make_upstream_grad(cfg)[1], nb=2)
    assert r["value"] > 0 and r["kind"] == "oracle" and r["unit"] == "images/s"


def test_cpu_baseline_cells_small():
    cfg = synth.CONFIGS["tiny_fp32"]
    ci = synth.make_cell_inputs(cfg, 4, 6)
    r = bench.cpu_baseline_cells(cfg, ci, 4, 6, nb=2)
    assert r["value"] > 0 and r["cores"] == 1


def test_source_hash_covers_the_forward_unit_only(tmp_path):
    """On a copy of the sources: the hash changes with the code of a forward
    header and not with a backward or cell source (those compile in other
    translation units), nor with a comment or blank lines anywhere."""
    src = os.path.join(bench.ROOT, "dynamic_convolution_b200", "csrc")
    dst = tmp_path / "csrc"
    shutil.copytree(src, dst)
    base = bench.kernel_source_hash(str(dst))
    assert base == bench.kernel_source_hash()
    for fn, changes in (("conv_tc.cuh", True), ("internal.h", True), ("backward.cu", False),
                        ("backward_kernels.cuh", False), ("cells_kernels.cuh", False)):
        path = dst / fn
        orig = path.read_bytes()
        path.write_bytes(orig + b"\nstatic const int hash_probe_value = 1;\n")
        assert (bench.kernel_source_hash(str(dst)) != base) == changes, fn
        path.write_bytes(orig + b"\n// a comment\n/* and a block\n comment */\n\n")
        assert bench.kernel_source_hash(str(dst)) == base, fn
        path.write_bytes(orig)


def test_roofline_bound_per_configuration():
    """Tensor-bound only where the conv FLOP per algorithmic byte exceeds the
    ridge of the two peaks (dense bf16 layers); the fraction is achieved / peak."""
    peaks = {"hbm_gbs": 6553.6, "bf16_tflops": 1672.7}
    want = {"tiny_fp32": "hbm", "resnet18_3x3": "tensor", "effnet_expand_1x1": "hbm",
            "effnet_dw_5x5": "hbm", "deep_3x3_tau30": "tensor", "large_n64": "hbm"}
    for name, bound in want.items():
        cfg = synth.CONFIGS[name]
        got, algo = bench.bound_of(cfg, peaks)
        assert got == bound, name
        r = bench.roofline_entry(cfg, 0.05, "k", peaks, "measured", None)
        if bound == "tensor":
            assert abs(r["achieved"] - cfg.conv_flops / 5e-5 / 1e12) < 1e-6 * r["achieved"]
        else:
            assert abs(r["achieved"] - algo / 5e-5 / 1e9) < 1e-6 * r["achieved"]
        assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    # the algorithmic bytes of the deep 3x3 layer: x + y + experts, bf16
    cfg = synth.CONFIGS["deep_3x3_tau30"]
    assert bench.bound_of(cfg, peaks)[1] == 2 * (2 * 256 * 14 * 14 * 256 + 16 * 256 * 9 * 256)
