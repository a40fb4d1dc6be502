"""The benchmark's algorithmic work (the roofline numerators) against figures worked out by hand
from the layer shapes, not from the benchmark's own formulas.

Shapes: "Scion-35B-A3B" model card, Model Overview (d = 2048, 256 experts, top-8 + one shared
expert, expert width 512) and Weight Representation (PQ2_0: 34 bytes per 128 weights);
"Scion-FlashNext-176B-A6B" model card, Model Overview (d = 3072, 512 experts, top-10 + one
shared, width 768) and Weight Representation (PTQ1_0: 28 bytes per 128 weights); rank-512
moe_out correction ("Scion: ternary MoE quantization with trained corrections", Method).

Per decode forward the kernels must move each active expert's three packed matrices once, the
dense weights once (router and delta [E][d], shared gate/up/down [Fs][d], correction A [r][d] and
B [d][r], all two bytes per weight), x in (bf16) and out (fp32).  Per prefill token the tensor
cores do 2 flops per multiply-add of k routed experts (3 d F each), the shared expert (3 d Fs),
router + delta (2 E d) and the correction (2 r d).
"""
import pytest

import bench
from workloads import synth


def test_packed_expert_bytes():
    # three matrices of F x d weights at 34/128 (PQ2_0) or 28/128 (PTQ1_0) bytes per weight
    a3b, fn = synth.CONFIGS["a3b_decode"], synth.CONFIGS["flashnext_decode"]
    assert bench.workload_bytes(a3b, 0, 1) - bench.workload_bytes(a3b, 0, 0) == 835_584  # 3*512*2048*34/128
    assert bench.workload_bytes(fn, 0, 1) - bench.workload_bytes(fn, 0, 0) == 1_548_288  # 3*768*3072*28/128


@pytest.mark.parametrize("name,fixed", [
    # (2*256*2048 + 3*512*2048) * 2 B + (512*2048 + 2048*512) * 2 B
    ("a3b_decode", 8_388_608 + 4_194_304),
    # (2*512*3072 + 3*768*3072) * 2 B + 2 * 512*3072 * 2 B
    ("flashnext_decode", 20_447_232 + 6_291_456),
])
def test_fixed_bytes(name, fixed):
    assert bench.workload_bytes(synth.CONFIGS[name], 0, 0) == fixed


@pytest.mark.parametrize("name,T,U,mb", [
    ("a3b_decode", 1, 8, 19.279872),          # 8 experts + 12.58 MB + 2048 * 6 B
    ("a3b_decode", 64, 220, 197.197824),      # 220 * 835584 + 12582912 + 64 * 2048 * 6
    ("flashnext_decode", 1, 10, 42.24),       # 10 experts + 26.74 MB + 3072 * 6 B
    ("flashnext_decode", 64, 367, 596.140032),  # 367 * 1548288 + 26738688 + 64 * 3072 * 6
])
def test_decode_bytes(name, T, U, mb):
    assert bench.workload_bytes(synth.CONFIGS[name], T, U) == pytest.approx(mb * 1e6, abs=1)


def test_packed_correction_bytes():
    # A and B as PQ2_0 blocks: 2 * 512 * 2048 weights at 34/128 bytes instead of 2 bytes
    cfg = synth.CONFIGS["a3b_decode"]
    diff = bench.workload_bytes(cfg, 0, 0) - bench.workload_bytes(cfg, 0, 0, cb=34 / 128)
    assert diff == pytest.approx(2 * 512 * 2048 * (2 - 34 / 128))


@pytest.mark.parametrize("name,gf", [
    # 2 * 4096 * (8*3*2048*512 + 3*2048*512 + 2*256*2048 + 2*512*2048)
    ("a3b_prefill", 257.69803776),
    # 2 * 16384 * (10*3*3072*768 + 3*3072*768 + 2*512*3072 + 2*512*3072)
    ("flashnext_prefill", 2757.369004032),
])
def test_prefill_flops(name, gf):
    cfg = synth.CONFIGS[name]
    assert bench.workload_flops(cfg, cfg.tokens[0]) == pytest.approx(gf * 1e9, abs=1)


def test_stage_flops_add_up():
    """The per-stage GEMM flops of a bf16-router layer cover the forward's flops exactly."""
    cfg = synth.CONFIGS["a3b_prefill"]
    T = cfg.tokens[0]
    st = bench.stage_flops(cfg, T)
    parts = st["xproj"] + st["gateup"] + st["down_routed"] + st["down_dense"]
    assert parts == bench.workload_flops(cfg, T)
