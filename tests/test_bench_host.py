"""Host-side logic of bench.py that needs no GPU: the code-only source hash that
keys the stored ncu traffic, and the lookup of that traffic."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_and_whitespace_but_keeps_code():
    a = "int f(int x) {  // twice\n    return 2 * x; /* the\n double */\n}\n"
    b = "int f(int x) { return 2 * x; }"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(b.replace("2", "3"))
    # comment markers inside literals are code
    s = 'const char *u = "http://x"; char c = \'/\';'
    assert "http://x" in bench._code_only(s)


def _copy_sources(dst):
    for sub in ("sub_quadratic_attention_b200/csrc", "include"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(dst, sub))


def test_source_hash_ignores_a_comment_edit_and_sees_a_code_edit(tmp_path, monkeypatch):
    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.source_hash()
    f = tmp_path / "sub_quadratic_attention_b200" / "csrc" / "api.cu"
    text = f.read_text()
    f.write_text("// an added comment line\n" + text)
    assert bench.source_hash() == h0
    f.write_text(text.replace("return SPECTRE_OK;", "return SPECTRE_OK; ", 1) + "\nstatic int extra;\n")
    assert bench.source_hash() != h0


def test_traffic_is_used_only_under_its_source_hash(tmp_path, monkeypatch):
    _copy_sources(tmp_path)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash()
    lines = ["# workload source_hash kernel dram_bytes_per_step",
             f"wl {h} rows_fwd 100", f"wl {h} slices 200", f"wl {h} rows_inv_ln 50",
             "wl 000000000000 rows_fwd 999", f"part {h} rows_fwd 1"]
    (tmp_path / "profiles" / "traffic.txt").write_text("\n".join(lines) + "\n")
    total, per = bench.ncu_traffic("wl")
    assert total == 350 and per == {"rows_fwd": 100.0, "slices": 200.0, "rows_inv_ln": 50.0}
    assert bench.ncu_traffic("other")[0] is None
    assert bench.ncu_traffic("part")[0] is None    # only a complete step counts


def test_dominant_kernel_roofline_arithmetic():
    """bf16 long's figures: 335.81 MB of algorithmic bytes over B L C =
    33,554,432 elements (10.008 B each); the slice pass is dominant with two
    launches in 0.2 ms per step, so a launch moves half the elements'
    bytes in 0.1 ms."""
    names = ["rows_fwd", "slices", "rows_inv_ln"]
    r = bench.dominant_roofline(335_810_560, 33_554_432, [0.1378, 0.2000, 0.0846], [2, 2, 1],
                                {"slices": 527_414_272.0}, names, 6554.6)
    assert r["kernel"] == "slices" and r["units_per_launch"] == 16_777_216
    assert abs(r["bytes_per_unit"] - 10.0079) < 1e-3
    assert abs(r["launch_ms"] - 0.1) < 1e-9
    assert abs(r["achieved"] - 335.81056 / 0.2) < 0.01          # GB/s
    assert abs(r["frac"] - (335.81056 / 0.2) / 6554.6) < 1e-4
    assert r["traffic"] == 527_414_272.0 / 2
    r2 = bench.dominant_roofline(100.0, 10, [1.0, 0.5, 3.0], [2, 2, 1], {}, names, 1000.0)
    assert r2["kernel"] == "rows_inv_ln" and r2["traffic"] is None


def test_block_view_keeps_memory_and_scales_F():
    import torch

    from sub_quadratic_attention_b200.workloads import custom, make_inputs

    w = custom(2, 256, 2, 4, 65, dtype="bf16")
    inp = make_inputs(w)
    pw, b = bench.block_view(w, inp, 64)
    assert (pw.B, pw.L, pw.C, pw.F) == (8, 64, 8, 16)        # F keeps the fraction 65/256 of L
    for k in ("q", "k", "v", "x"):
        assert b[k].shape == (8, 64, 8) and b[k].data_ptr() == inp[k].data_ptr()
    assert torch.equal(b["G"], inp["G"][:, :33]) and b["G"].is_contiguous()
    assert pw.algorithmic_bytes() == 5 * 2 * 256 * 8 * 2 + 2 * 16 * 4 + 2 * 8 * 4
    cfg = bench.config_dict(w, 1, pw)
    assert cfg["block_len"] == 64 and cfg["L"] == 256 and cfg["F"] == 16
    import pytest

    with pytest.raises(SystemExit):
        bench.block_view(w, inp, 100)


def test_alu_ceiling_and_method_flops():
    from sub_quadratic_attention_b200.workloads import DCT_WORKLOADS, WORKLOADS

    f = bench.method_flops(WORKLOADS["bf16_long"])
    assert abs(f / 1e9 - 5.76) < 0.02                 # about 5.8 GFLOP per step
    r = bench.alu_roofline(f, 0.5, 1965)
    assert abs(r["peak"] - 148 * 128 * 2 * 1.965e9 / 1e12) < 0.01
    assert abs(r["achieved"] - f / 0.5e-3 / 1e12) < 1e-3 and r["bound"] == "alu"
    assert bench.alu_roofline(f, 0.5, None)["peak"] == r["peak"]
    w = DCT_WORKLOADS["dct_d1024"]
    assert bench.dct_method_flops(w) == w.T * (5 * 1024 * 10 + 40 * 1024)
