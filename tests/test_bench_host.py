"""Host-side logic of bench.py and of the Python binding that needs no GPU:
workload definitions and byte models, the committed ncu traffic table, and
argument checks that fail before any library call."""
import json
import os

import pytest
import torch

import bench
import workloads
import weight_only_quantization_rtn_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_group_sizes_and_byte_models():
    assert bench.group_of(0, 4096) == 4096 and bench.group_of(128, 4096) == 128
    # 7B-shaped layer at M=1, g=128 asym: codes + scales + zeros + X + Y
    assert bench.algorithmic_bytes(1, 11008, 4096, 128, False) == 23983616
    assert bench.input_bytes(1, 11008, 4096, 128, False) + 2 * 11008 == 23983616
    # per-channel: one scale and one zero per row
    assert bench.algorithmic_bytes(1, 4096, 11008, 11008, False) == \
        4096 * 11008 // 2 + 4 * 4096 + 2 * 11008 + 2 * 4096
    # symmetric: no zeros
    assert bench.algorithmic_bytes(1, 28672, 8192, 128, True) == \
        28672 * 8192 // 2 + 2 * 28672 * 64 + 2 * 8192 + 2 * 28672


def test_workload_table():
    for name, (wl, M, g, sym, half, bits) in bench.WORKLOAD_DEFS.items():
        assert half in ("hbm", "tensor") and bits in (4, 8)
        # the bound follows the arithmetic intensity against the ridge of the
        # measured peaks (≈1646 TFLOP/s over ≈6.55 TB/s: about 250 flop per byte)
        L = wl.layers[0]
        intensity = 2 * M * L.N * L.K / bench.algorithmic_bytes(M, L.N, L.K, bench.group_of(g, L.K), sym, bits)
        assert (half == "hbm") == (intensity < 250), (name, intensity)
        for layer in wl.layers:
            assert layer.K % bench.group_of(g, layer.K) == 0
        assert bench.workload_name(wl, M, g).endswith("_per_channel") == (g == 0)
        assert bench.workload_name(wl, M, g, sym, bits).startswith("w8a16_") == (bits == 8)
    # 8-bit codes: one byte per weight
    assert bench.algorithmic_bytes(1, 28672, 8192, 128, False, 8) == \
        28672 * 8192 + 4 * 28672 * 64 + 2 * 8192 + 2 * 28672
    assert bench.WORKLOAD_DEFS["decode7b"][0] is workloads.DECODE_7B
    assert bench.WORKLOAD_DEFS["prefill"][1] == 2048


def test_traffic_table_points_at_committed_profiles():
    table = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    for key, entry in table.items():
        kernel, workload = key.split(":")
        assert kernel in bench.KERNEL_SOURCES and (workload in bench.WORKLOAD_DEFS or workload in bench.EXTRAS)
        src = entry["source"].split(" ")[0]
        assert os.path.exists(os.path.join(ROOT, src)), src
        assert entry["dram_bytes_per_launch"] > 0
        # a value is reported only while the kernel's sources are unchanged
        current = entry["kernel_source_digest"] == bench.kernel_source_digest(kernel)
        assert (bench.ncu_traffic(key) is not None) == current
    assert "gemv_decode_kernel:decode7b" in table and "gemm_tc_kernel:prefill" in table


def test_kernel_source_digest_tracks_listed_files():
    for kernel, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(ROOT, "weight_only_quantization_rtn_b200", "csrc", f))
        d = bench.kernel_source_digest(kernel)
        assert len(d) == 16 and d == bench.kernel_source_digest(kernel)


@pytest.mark.parametrize("fn,args", [
    (w4.quantize8, (torch.zeros(4, 128, dtype=torch.bfloat16), 128, False)),        # host tensor
    (w4.quantize8, (torch.zeros(4, 128, dtype=torch.float32), 128, False)),         # wrong dtype
    (w4.quantize, (torch.zeros(4, 128, dtype=torch.bfloat16), 128, False)),
    (w4.dequantize8, (torch.zeros(4, 128, dtype=torch.uint8), torch.zeros(4, 1, dtype=torch.bfloat16),
                      torch.zeros(4, 1, dtype=torch.bfloat16), 128, False)),
    (w4.gemm8, (torch.zeros(1, 128, dtype=torch.bfloat16), torch.zeros(4, 128, dtype=torch.uint8),
                torch.zeros(4, 1, dtype=torch.bfloat16), torch.zeros(4, 1, dtype=torch.bfloat16),
                128, False)),
])
def test_binding_rejects_host_or_mistyped_tensors(fn, args):
    """The binding checks dtype, rank, device and contiguity before calling the
    library, so these fail on any machine without launching anything."""
    with pytest.raises((TypeError, ValueError)):
        fn(*args)


def test_quantize_rejects_k_not_multiple_of_g():
    W = torch.zeros(4, 96, dtype=torch.bfloat16)
    with pytest.raises((TypeError, ValueError)):
        w4.quantize8(W, 64, False)
