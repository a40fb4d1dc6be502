"""The oracle's correction branch on the attention output ("Scion: ternary MoE quantization with
trained corrections", The idea: rank-512 branches on the attention output and the MoE block
output; Findings: the attention-output branch is a plain low-rank adapter on the attention
output projection), pinned against numpy matrix products built from the generating values --
bf16 factors from their bit patterns (torch's bfloat16), ternary factors from their codes and
fp16 scales (numpy's float16), never from the packed bytes the oracle reads.  d_in != d_out, so a
transposed factor or a swapped axis fails."""
import numpy as np
import pytest

import oracle
from tests.helpers import bf16, f16
from workloads import synth


def _v(T, d_in, seed):
    rng = np.random.default_rng(seed)
    return synth.to_bf16_bits(rng.standard_normal((T, d_in), dtype=np.float32))


def test_bf16_factors_match_numpy():
    T, d_in, d_out, r = 5, 384, 256, 48
    rng = np.random.default_rng(3)
    a = synth.normal_bf16(rng, (r, d_in), 0.02)
    b = synth.normal_bf16(rng, (d_out, r), 0.02)
    v = _v(T, d_in, 4)
    base = rng.standard_normal((T, d_out))
    out, z = oracle.attn_corr(v, a, b, d_in, d_out, r, base=base)
    z_ref = bf16(v) @ bf16(a).T
    np.testing.assert_allclose(z, z_ref, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out, base + z_ref @ bf16(b).T, rtol=1e-12, atol=1e-14)


def test_packed_factors_match_numpy_from_codes():
    T, d_in, d_out, r = 3, 256, 384, 128
    rng = np.random.default_rng(5)
    ca, sa = synth.ternary_codes(rng, (r, d_in)), synth.group_scales(rng, (r, d_in // 128))
    cb, sb = synth.ternary_codes(rng, (d_out, r)), synth.group_scales(rng, (d_out, r // 128))
    a_ref = ca.astype(np.float64) * np.repeat(f16(sa), 128, axis=1)
    b_ref = cb.astype(np.float64) * np.repeat(f16(sb), 128, axis=1)
    v = _v(T, d_in, 6)
    out, z = oracle.attn_corr(v, oracle.pack(synth.PQ2_0, ca, sa), oracle.pack(synth.PQ2_0, cb, sb), d_in, d_out, r,
                              packed=1)
    np.testing.assert_allclose(z, bf16(v) @ a_ref.T, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out, bf16(v) @ a_ref.T @ b_ref.T, rtol=1e-12, atol=1e-15)


def test_zero_branch_returns_base_and_branch_is_linear():
    T, d_in, d_out, r = 4, 128, 256, 128
    rng = np.random.default_rng(7)
    zeros = oracle.pack(synth.PQ2_0, np.zeros((r, d_in), np.int8), synth.group_scales(rng, (r, 1)))
    cb, sb = synth.ternary_codes(rng, (d_out, r)), synth.group_scales(rng, (d_out, 1))
    bp = oracle.pack(synth.PQ2_0, cb, sb)
    v = _v(T, d_in, 8)
    base = rng.standard_normal((T, d_out))
    out, z = oracle.attn_corr(v, zeros, bp, d_in, d_out, r, packed=1, base=base)
    assert (z == 0).all()
    np.testing.assert_array_equal(out, base)
    # doubling v (exact in bf16) doubles the branch
    ca, sa = synth.ternary_codes(rng, (r, d_in)), synth.group_scales(rng, (r, 1))
    ap = oracle.pack(synth.PQ2_0, ca, sa)
    o1, _ = oracle.attn_corr(v, ap, bp, d_in, d_out, r, packed=1)
    o2, _ = oracle.attn_corr(synth.to_bf16_bits(2 * bf16(v).astype(np.float32)), ap, bp, d_in, d_out, r, packed=1)
    np.testing.assert_allclose(o2, 2 * o1, rtol=1e-13, atol=1e-15)


def test_rejects_bad_shapes():
    v = _v(2, 128, 1)
    a = np.zeros((16, 128), np.uint16)
    b = np.zeros((128, 16), np.uint16)
    with pytest.raises(RuntimeError):  # packed factors need d_in and r multiples of 128
        oracle.attn_corr(v, a, b, 128, 128, 16, packed=1)
