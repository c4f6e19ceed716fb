"""Host logic of bench.py that needs no GPU: the kernel-code fingerprint that decides
whether the committed ncu DRAM counters still describe the kernel."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

SRC = """// header comment
#include "x.h"
/* block
   comment */
__global__ void k(int* a) {  // trailing comment
  a[0] = 1;
}
"""


def _fp(tmp_path, text):
    p = tmp_path / "k.cu"
    p.write_text(text)
    old = bench.KERNEL_SRC
    try:
        bench.KERNEL_SRC = str(p)
        return bench.kernel_sha()
    finally:
        bench.KERNEL_SRC = old


def test_fingerprint_ignores_comments_and_whitespace(tmp_path):
    base = _fp(tmp_path, SRC)
    edited = SRC.replace("// header comment", "// a different header\n// over two lines")
    edited = edited.replace("/* block\n   comment */", "/* reworded */")
    edited = edited.replace("  a[0] = 1;", "      a[0]  =  1 ;")
    assert _fp(tmp_path, edited) == base


def test_fingerprint_follows_code(tmp_path):
    base = _fp(tmp_path, SRC)
    assert _fp(tmp_path, SRC.replace("a[0] = 1;", "a[0] = 2;")) != base
    assert _fp(tmp_path, SRC.replace("int* a", "long* a")) != base


def test_current_kernel_fingerprint_is_well_formed():
    fp = bench.kernel_sha()
    assert len(fp) == 16 and int(fp, 16) >= 0


def test_gpus_flag_must_match_the_launched_ranks(monkeypatch, capsys):
    """`--gpus N` is only honoured through torchrun's WORLD_SIZE; a mismatch is refused
    instead of silently running one replica."""
    import pytest
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    bench.check_world(bench.parse_args(["--gpus", "1"]))  # one rank, as launched
    with pytest.raises(SystemExit) as e:
        bench.check_world(bench.parse_args(["--gpus", "8"]))
    assert e.value.code == 2 and "--gpus 8" in capsys.readouterr().err
    monkeypatch.setenv("WORLD_SIZE", "4")
    bench.check_world(bench.parse_args(["--gpus", "4"]))


def test_key_tile_periods_of_the_tower_layers():
    """The per-clock guard's denominator: on 148 SMs the full layer (1 x 16384 tokens, 16
    heads) makes 1024 units of 128 key tiles, 7 on the busiest CTA; the window layer (16 x
    1024) makes 1024 units of 8 key tiles, also 7 per CTA."""
    import bench
    import workloads
    full = workloads.cu_from_lengths([16384])
    window = workloads.cu_from_lengths([1024] * 16)
    assert bench.key_tile_periods(full, 16, 148) == 7 * 128
    assert bench.key_tile_periods(window, 16, 148) == 7 * 8
    # fewer units than SMs: one unit per CTA
    assert bench.key_tile_periods(workloads.cu_from_lengths([1024]), 16, 148) == 8


def test_measured_peaks_names_its_source(tmp_path, monkeypatch):
    """The roofline's peak comes from MEASURED_PEAKS.json when present, else the stated
    fallback, and the label says which."""
    import json
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peak, hbm, src = bench.measured_peaks()
    assert (peak, hbm) == (1590.0, 6650.0) and src.startswith("fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1608.2, "hbm_gbs": 6539.0}))
    peak, hbm, src = bench.measured_peaks()
    assert (peak, hbm) == (1608.2, 6539.0) and "MEASURED_PEAKS.json" in src and not src.startswith("fallback")
