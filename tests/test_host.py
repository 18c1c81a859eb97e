"""Host-side checks that need no GPU: the geometry shared by the kernels, the library's exported
symbols, and argument validation that must reject bad calls before any CUDA call."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_geometry_invariants(tmp_path):
    exe = tmp_path / "geometry_check"
    subprocess.check_call(["g++", "-O1", "-std=c++17", os.path.join(ROOT, "tests", "geometry_check.cpp"), "-o", str(exe)])
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout


@pytest.fixture(scope="module")
def lib():
    from block_causal_linear_relu_b200 import build
    build.build()
    import block_causal_linear_relu_b200 as sv
    return sv.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "svlinattn.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\*]+\s+\*?(sv_\w+)\s*\(", text, re.M)))


def test_header_and_binding_agree():
    import block_causal_linear_relu_b200 as sv
    assert _declared() == sorted(sv.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    nm = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (sv_\w+)", nm))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)
    assert lib.sv_version() == 100
    assert lib.sv_last_error() is not None


def test_validation_rejects_before_any_launch(lib):
    # null pointers and bad sizes are refused on the host with no CUDA call (no GPU here)
    vp = ctypes.c_void_p
    f = lib.sv_linattn_fwd
    fake = vp(256 * 1024)
    assert f(None, fake, fake, fake, 1, 1, 128, 128, 0, 1e-6, fake, 1 << 30, None) == 1
    assert b"q is NULL" in lib.sv_last_error()
    assert f(fake, fake, fake, fake, 1, 1, 0, 128, 0, 1e-6, fake, 1 << 30, None) == 1      # N = 0
    assert f(fake, fake, fake, fake, 1, 1, 128, 100, 0, 1e-6, fake, 1 << 30, None) == 2    # bf16 D=100
    assert f(fake, fake, fake, fake, 1, 1, 128, 36, 0, 1e-6, fake, 1 << 30, None) == 2     # bf16 D=36
    assert f(fake, fake, fake, fake, 1, 1, 128, 136, 0, 1e-6, fake, 1 << 30, None) == 2    # bf16 D>128
    assert f(fake, fake, fake, fake, 1, 1, 128, 129, 1, 1e-6, fake, 1 << 30, None) == 2    # f32 D>128
    assert f(fake, fake, fake, fake, 1, 1, 128, 128, 7, 1e-6, fake, 1 << 30, None) == 2    # dtype
    assert f(fake, vp(256 * 1024 + 2), fake, fake, 1, 1, 128, 128, 0, 1e-6, fake, 1 << 30, None) == 1  # misaligned
    assert b"16-byte aligned" in lib.sv_last_error()
    bc = lib.sv_block_causal_attn
    assert bc(fake, fake, fake, fake, 1, 1, 128, 128, 0, 0, 1e-6, None, None, None, None, fake, 1 << 30, None) == 1
    assert b"block_len" in lib.sv_last_error()
    assert bc(fake, fake, fake, fake, 1, 1, 128, 128, 64, 0, float("nan"), None, None, None, None, fake, 1 << 30, None) == 1
    assert bc(fake, fake, fake, fake, 1, 1, 128, 128, 64, 0, 1e-6, vp(256 * 1024 + 1), None, None, None, fake, 1 << 30, None) == 1
    cs = lib.sv_cache_step
    assert cs(fake, fake, fake, fake, 1, 1, 128, 128, 0, 1e-6, None, fake, 1, fake, 1 << 30, None) == 1
    assert b"S is NULL" in lib.sv_last_error()
    su = lib.sv_block_state_update
    assert su(fake, fake, 1, 1, 128, 128, 0, fake, None, fake, 1 << 30, None) == 1
    assert lib.sv_workspace_init(None, 0, None) == 1


def test_rope_arguments_are_checked_before_any_launch(lib):
    vp = ctypes.c_void_p
    from block_causal_linear_relu_b200._native import SvRope3d

    assert lib.sv_rope3d_table_bytes(60, 23, 40, 128) == (60 + 23 + 40) * 64 * 8
    assert lib.sv_rope3d_table_bytes(60, 23, 40, 127) == 0 and b"even" in lib.sv_last_error()
    assert lib.sv_rope3d_table_bytes(0, 23, 40, 128) == 0
    fake = vp(256 * 1024)
    tab = lib.sv_rope3d_table
    n = (60 + 23 + 40) * 64 * 8
    assert tab(fake, n, 60, 23, 40, 128, 22, 21, 20, 10000.0, None) == 1  # pairs sum to 63, not 64
    assert b"pairs" in lib.sv_last_error()
    assert tab(fake, n - 8, 60, 23, 40, 128, 22, 21, 21, 10000.0, None) == 1  # table too small
    assert tab(fake, n, 60, 23, 40, 128, 22, 21, 21, 1.0, None) == 1  # base must exceed 1
    assert tab(vp(256 * 1024 + 8), n, 60, 23, 40, 128, 22, 21, 21, 10000.0, None) == 1  # misaligned
    f = lib.sv_block_causal_attn_rope

    def call(desc, N=2760 * 3, D=128):
        return f(fake, fake, fake, fake, 1, 20, N, D, 2760, 0, 1e-6, None, None, None, None,
                 None if desc is None else ctypes.byref(desc), fake, 1 << 30, None)

    good = dict(table=256 * 1024, frames=9, height=23, width=40, D=128, pairs_t=22, pairs_h=21, pairs_w=21, frame0=0)
    assert call(None) == 1 and b"NULL" in lib.sv_last_error()
    assert call(SvRope3d(**{**good, "frame0": 1})) == 1  # tokens reach frame 9 of a 9-frame table
    assert b"frame0" in lib.sv_last_error()
    assert call(SvRope3d(**{**good, "D": 112})) == 1  # table built for another D
    assert call(SvRope3d(**{**good, "pairs_w": 20})) == 1
    assert call(SvRope3d(**{**good, "table": 256 * 1024 + 8})) == 1
    assert call(SvRope3d(**{**good, "height": 0})) == 1
    assert call(SvRope3d(**good), D=100) == 2  # bf16 D must be a multiple of 8 (checked first)


def test_binding_rope_helpers(lib):
    # the binding's table size and default pair split (host only); the split agrees with the oracle's
    import block_causal_linear_relu_b200 as sv
    from oracle import rope as R

    assert sv.sv_rope3d_table_bytes(60, 23, 40, 128) == (60 + 23 + 40) * 64 * 8
    with pytest.raises(sv.SvError, match="even"):
        sv.sv_rope3d_table_bytes(60, 23, 40, 127)
    for D in (8, 24, 64, 112, 128):
        assert sv.rope_pairs(D) == R.default_pairs(D)
        assert 2 * sum(sv.rope_pairs(D)) == D


def test_oracle_rates_of_the_other_configurations():
    # the bench's CPU-baseline leg for the other configurations: every sample runs and gives a rate
    import bench

    r = bench.oracle_rates_other(0.0)
    assert set(r) == {"480p_bidir", "720p_stream", "720p_prefill_rope", "720p_temporal_conv", "sv2_projections"}
    for v in r.values():
        assert v["value"] > 0 and v["unit"] and "1 run(s)" in v["sample"]


def test_binding_rejects_bad_tensors_before_the_library():
    # the binding's single pass of checks: host tensors, wrong rank, mismatched shape or dtype and
    # non-contiguous tensors raise before any library or CUDA call
    import torch

    import block_causal_linear_relu_b200 as sv
    from block_causal_linear_relu_b200 import _native as nat

    q = torch.zeros(1, 2, 64, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device"):
        nat._qkv(q, q, q)
    with pytest.raises(ValueError, match="CUDA device"):
        sv.sv_linattn_fwd(q, q, q, o=q)


def test_cpu_baseline_cycles_over_heads_until_its_budget():
    # the CPU oracle baseline keeps cycling over the workload's heads until its time budget is
    # spent (more heads than the workload holds), and max_heads caps it
    import bench
    from block_causal_linear_relu_b200.inputs import draw_qkv

    saved = (bench.H, bench.N, bench.L)
    try:
        bench.H, bench.N, bench.L = 2, 96, 32
        q, k, v = draw_qkv((1, 2, 96, 16), 0, "bf16")
        rate, heads, ntok, secs = bench.oracle_rate(q, k, v, 0.2)
        assert heads > bench.H and ntok == 96 and secs >= 0.2 and rate > 0
        _, heads1, _, _ = bench.oracle_rate(q, k, v, 0.0, max_heads=1)
        assert heads1 == 1
    finally:
        bench.H, bench.N, bench.L = saved
