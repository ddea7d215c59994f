"""Host-side pieces of bench.py that decide what its JSON line reports: the algorithmic work
per step, the quantizer's bytes, which kernel a stage names, and when a committed ncu summary
still describes the current kernel sources (its DRAM traffic is reported only then)."""
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _case(M, N, K, g=256, A=None, **extra):
    return types.SimpleNamespace(M=M, N=N, K=K, g=g, A=A, extra=extra)


def test_code_only_ignores_comments_and_whitespace():
    a = "int f(int x) { // one\n  return x + 1; /* two\n three */ }\n"
    b = "int f(int x)\n{\n\treturn x + 1;   }  // another comment\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(a.replace("x + 1", "x + 2"))


def test_kernel_source_hash_covers_each_family():
    hashes = {k: bench.kernel_source_hash(k) for k in bench.KERNEL_SOURCES}
    assert all(len(h) == 16 for h in hashes.values())
    # families built from different files hash differently
    assert len(set(hashes.values())) == len(hashes)


def test_profiled_traffic_only_for_current_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    os.makedirs(tmp_path / "profiles")
    # a fixed hash stands for the current sources' hash
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: "0123456789abcdef")
    p = tmp_path / "profiles" / "gemm_up_wl.md"
    p.write_text("# x\n\n- kernel: `k`\n- kernel_source_hash: `0123456789abcdef`\n"
                 "- dram_bytes_per_launch: `113711104`\n")
    assert bench.profiled_traffic("gemm_up", "gemm_s8", "wl") == 113711104.0
    p.write_text(p.read_text().replace("0123456789abcdef", "fedcba9876543210"))
    assert bench.profiled_traffic("gemm_up", "gemm_s8", "wl") is None     # stale
    assert bench.profiled_traffic("gemm_down", "gemm_s8", "wl") is None   # absent


def test_workload_ops():
    # MLP pair: two GEMMs of 2 M N K (up [M,K]x[N,K]^T, down [M,N]x[K,N]^T)
    ops, extra = bench.workload_ops(_case(4608, 10240, 3840), "dit_mlp_4608x3840x10240")
    assert ops == 2 * 2 * 4608 * 10240 * 3840 and extra == 0
    # LoRA: int8 ops, and the bf16 adapter flops reported beside them
    A = types.SimpleNamespace(shape=(3072, 64))
    ops, extra = bench.workload_ops(_case(8192, 12288, 3072, A=A), "peft_lora_8192x12288x3072_r64")
    assert ops == 2 * 8192 * 12288 * 3072
    assert extra == 2 * 8192 * 3072 * 64 + 2 * 8192 * 64 * 12288
    # input gradient: dy [M, N] x qW [N, K]
    ops, _ = bench.workload_ops(_case(4096, 3072, 3072), "grad_dit_attn_4096x3072x3072")
    assert ops == 2 * 4096 * 3072 * 3072
    # attention: int8 QK and bf16 PV, 2 L^2 D per head each
    ops, _ = bench.workload_ops(_case(4608, 24, 128, attn=True, B=1), "attn_flux_b1_l4608_h24_d128")
    assert ops == 2 * 2 * 24 * 4608 * 4608 * 128


def test_rotquant_bytes_and_kernel_names():
    # 2K read + K codes + 4 bytes of scale per row
    assert bench.rotquant_bytes(4608, 3840) == 4608 * (3 * 3840 + 4) == 53102592
    c = _case(4608, 10240, 3840)
    assert bench.rotquant_kernel_name(c, 3840, False, False) == "rotquant_run_kernel<256,false,V8>"
    assert bench.rotquant_kernel_name(c, 32768, False, True) == "rotquant_run_kernel<256,true,V8>"
    assert bench.rotquant_kernel_name(c, 65536, False, False) == "rotquant_kernel<256,false,false>"
    assert bench.rotquant_kernel_name(c, 12288, True, False) == "rotquant_persistent_kernel<1,true,false>"
    assert bench.rotquant_kernel_name(c, 20480, True, False) == "rotquant_kernel<1,true,false>"


@pytest.mark.parametrize("mhz,expect", [(1965, 1.0), (1830, 1830 / 1965), (None, None)])
def test_clock_scaled_fraction_matches_the_clock(mhz, expect):
    peak = bench.clock_scaled_peak(4500.0, {"sm_mhz": mhz, "sm_max_mhz": 1965})
    if expect is None:
        assert peak is None
    else:
        assert peak == pytest.approx(4500.0 * expect)
