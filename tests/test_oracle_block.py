"""Pins for the oracle's block forward against library routines, brute force on tiny
inputs, special cases and invariants.  Each is chosen so that a plausible slip in
the oracle (a dropped router delta, a transposed down projection, a wrong group
or expert index, a sign error in SiLU, a missing shared or correction term, a
wrong top-k tie rule) fails at least one of them."""
import math

import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle
from tests.helpers import bf16, f16, oracle_layer_from
from workloads import synth


def small_cfg(fmt=synth.PQ2_0, router_f32=False, E=6, k=3, d=256, F=128, Fs=128, r=16):
    return synth.Config("small", 9, d, E, k, F, Fs, fmt, r, router_f32, [5], 1)


def numpy_block(cfg, L, x_bits, norm_topk=1, corr_on_output=False, sh_gate_vec=None):
    """The block written with numpy/scipy primitives, straight from the generated codes
    and scales (never from packed bytes)."""
    x = bf16(x_bits)
    conv = (lambda a: a.astype(np.float64)) if cfg.router_f32 else bf16
    logits = x @ conv(L["w_router"]).T + x @ conv(L["w_delta"]).T
    T, E, k = x.shape[0], cfg.n_experts, cfg.top_k

    def W(name):
        c = L[name + "_codes"].astype(np.float64)
        s = np.repeat(f16(L[name + "_scales"]), 128, axis=-1)
        return c * s

    Wg, Wu, Wdn = W("gate"), W("up"), W("down")
    out = np.zeros((T, cfg.d))
    ids_all = np.zeros((T, k), np.int64)
    for t in range(T):
        ids = np.argsort(-logits[t], kind="stable")[:k]
        ids_all[t] = ids
        if norm_topk:
            g = softmax(logits[t, ids])
        else:
            g = softmax(logits[t])[ids]
        for j, e in enumerate(ids):
            a = Wg[e] @ x[t]
            b = Wu[e] @ x[t]
            out[t] += g[j] * (Wdn[e] @ (a * expit(a) * b))
        if cfg.shared_ffn:
            a = bf16(L["sh_gate"]) @ x[t]
            b = bf16(L["sh_up"]) @ x[t]
            ys = bf16(L["sh_down"]) @ (a * expit(a) * b)
            if sh_gate_vec is not None:
                ys = ys * expit(bf16(sh_gate_vec) @ x[t])
            out[t] += ys
        if cfg.rank:
            inp = out[t].copy() if corr_on_output else x[t]
            out[t] += bf16(L["corr_b"]) @ (bf16(L["corr_a"]) @ inp)
    return out, ids_all


def _rel(a, b):
    return np.abs(a - b).max() / np.abs(b).max()


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("router_f32", [False, True])
def test_brute_force_block(fmt, router_f32):
    cfg = small_cfg(fmt, router_f32)
    L = synth.layer_host(cfg)
    x = synth.x_host(cfg, 5)
    out, ids, g = oracle.forward(oracle_layer_from(cfg, L), x)
    ref, ref_ids = numpy_block(cfg, L, x)
    np.testing.assert_array_equal(ids, ref_ids)
    assert _rel(out, ref) < 1e-12


@pytest.mark.parametrize("variant", ["norm_topk0", "corr_on_output", "sh_gate_vec"])
def test_brute_force_readings(variant):
    cfg = small_cfg(synth.PQ2_0)
    L = synth.layer_host(cfg)
    x = synth.x_host(cfg, 4)
    kw, nk = {}, {}
    if variant == "norm_topk0":
        kw["norm_topk"] = nk["norm_topk"] = 0
    elif variant == "corr_on_output":
        kw["corr_on_output"] = 1
        nk["corr_on_output"] = True
    else:
        v = synth.normal_bf16(synth.rng_for(3), (cfg.d,), 0.05)
        kw["sh_gate_vec"] = nk["sh_gate_vec"] = v
    out, _, _ = oracle.forward(oracle_layer_from(cfg, L, **kw), x)
    ref, _ = numpy_block(cfg, L, x, **nk)
    assert _rel(out, ref) < 1e-12


def test_dense_cross_form():
    """Sum over all experts with masked gates equals the sparse top-k form."""
    for fmt in (synth.PQ2_0, synth.PTQ1_0):
        cfg = small_cfg(fmt, E=7, k=3)
        L = synth.layer_host(cfg)
        x = synth.x_host(cfg, 4)
        lay = oracle_layer_from(cfg, L)
        out, _, _ = oracle.forward(lay, x)
        dense = oracle.forward_dense(lay, x)
        assert _rel(out, dense) < 1e-12


def test_topk_matches_stable_argsort():
    rng = np.random.default_rng(1)
    for _ in range(200):
        E = int(rng.integers(1, 40))
        k = int(rng.integers(1, E + 1))
        logits = rng.integers(-3, 4, size=E).astype(np.float64)  # many ties
        got = oracle.topk(logits, k)
        ref = np.argsort(-logits, kind="stable")[:k]
        np.testing.assert_array_equal(got, ref)


def test_gates_are_softmax():
    rng = np.random.default_rng(2)
    for _ in range(50):
        E = int(rng.integers(2, 64))
        k = int(rng.integers(1, E + 1))
        logits = rng.normal(size=E) * 3
        ids = np.argsort(-logits, kind="stable")[:k]
        np.testing.assert_allclose(oracle.gates(logits, ids, 1), softmax(logits[ids]), rtol=1e-14)
        np.testing.assert_allclose(oracle.gates(logits, ids, 0), softmax(logits)[ids], rtol=1e-14)
        assert abs(oracle.gates(logits, ids, 1).sum() - 1) < 1e-14


def test_group_matches_stable_sort():
    rng = np.random.default_rng(3)
    for E, T, k in [(8, 16, 2), (256, 64, 8), (512, 300, 10), (5, 1, 5)]:
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        counts, offsets, perm = oracle.group(ids, E)
        np.testing.assert_array_equal(counts, np.bincount(ids.ravel(), minlength=E))
        np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
        np.testing.assert_array_equal(perm, np.argsort(ids.ravel(), kind="stable"))


def test_single_expert_is_plain_swiglu_mlp():
    """E = k = 1, no shared expert, no correction: the block is a SwiGLU MLP (gate 1).
    Reference: pure-Python loops over the dequantized weights."""
    cfg = small_cfg(synth.PTQ1_0, E=1, k=1, d=128, F=128, Fs=0, r=0)
    L = synth.layer_host(cfg)
    x = synth.x_host(cfg, 2)
    out, ids, g = oracle.forward(oracle_layer_from(cfg, L), x)
    assert (ids == 0).all() and (g == 1.0).all()
    xv = bf16(x)
    sg, su, sd = f16(L["gate_scales"])[0], f16(L["up_scales"])[0], f16(L["down_scales"])[0]
    cg, cu, cd = L["gate_codes"][0], L["up_codes"][0], L["down_codes"][0]
    for t in range(2):
        h = []
        for f in range(128):
            a = sum(float(cg[f, i]) * sg[f, i // 128] * xv[t, i] for i in range(128))
            b = sum(float(cu[f, i]) * su[f, i // 128] * xv[t, i] for i in range(128))
            h.append(a / (1.0 + math.exp(-a)) * b)
        for i in range(128):
            y = sum(float(cd[i, f]) * sd[i, f // 128] * h[f] for f in range(128))
            assert abs(out[t, i] - y) <= 1e-12 * max(1.0, abs(y))


def test_zero_codes_leave_shared_plus_correction():
    cfg = small_cfg(synth.PQ2_0)
    L = synth.layer_host(cfg)
    for n in ("gate", "up", "down"):
        L[n + "_codes"][:] = 0
    x = synth.x_host(cfg, 3)
    out, _, _ = oracle.forward(oracle_layer_from(cfg, L), x)
    xv = bf16(x)
    a, b = xv @ bf16(L["sh_gate"]).T, xv @ bf16(L["sh_up"]).T
    ref = (a * expit(a) * b) @ bf16(L["sh_down"]).T + (xv @ bf16(L["corr_a"]).T) @ bf16(L["corr_b"]).T
    assert _rel(out, ref) < 1e-12


def test_k_equals_E_gates_are_full_softmax():
    cfg = small_cfg(synth.PQ2_0, E=4, k=4, Fs=0, r=0)
    L = synth.layer_host(cfg)
    x = synth.x_host(cfg, 3)
    lay = oracle_layer_from(cfg, L)
    logits, ids, g = oracle.route(lay, x)
    for t in range(3):
        np.testing.assert_allclose(g[t], softmax(logits[t])[ids[t]], rtol=1e-14)
        assert sorted(ids[t].tolist()) == [0, 1, 2, 3]


def test_router_logits_match_numpy():
    cfg = synth.CONFIGS["tiny"]
    L = synth.layer_host(cfg)
    x = synth.x_host(cfg, 16)
    logits, _, _ = oracle.route(oracle_layer_from(cfg, L), x)
    xv = bf16(x)
    ref = xv @ L["w_router"].astype(np.float64).T + xv @ L["w_delta"].astype(np.float64).T
    np.testing.assert_allclose(logits, ref, rtol=1e-12, atol=1e-14)


def test_expert_relabelling_invariance():
    """Permuting the expert labels (router rows and banks together) permutes ids only."""
    cfg = small_cfg(synth.PTQ1_0, E=6, k=2)
    L = synth.layer_host(cfg)
    x = synth.x_host(cfg, 4)
    out, ids, g = oracle.forward(oracle_layer_from(cfg, L), x)
    pi = np.array([3, 0, 5, 1, 4, 2])  # new label of old expert e is where(pi == e)
    L2 = dict(L)
    for key in ("w_router", "w_delta", "gate_codes", "gate_scales", "up_codes", "up_scales",
                "down_codes", "down_scales"):
        L2[key] = np.ascontiguousarray(L[key][pi])
    out2, ids2, g2 = oracle.forward(oracle_layer_from(cfg, L2), x)
    np.testing.assert_array_equal(pi[ids2], ids)
    np.testing.assert_allclose(g2, g, rtol=1e-14)
    assert _rel(out2, out) < 1e-13


def test_tokens_are_independent_and_empty_batch():
    cfg = small_cfg(synth.PQ2_0)
    L = synth.layer_host(cfg)
    lay = oracle_layer_from(cfg, L)
    x = synth.x_host(cfg, 5)
    out, _, _ = oracle.forward(lay, x)
    for t in range(5):
        o1, _, _ = oracle.forward(lay, x[t:t + 1])
        np.testing.assert_array_equal(o1[0], out[t])
    o0, i0, g0 = oracle.forward(lay, x[:0])
    assert o0.shape == (0, cfg.d) and i0.shape == (0, cfg.top_k)


def test_expert_hidden_matches_forward():
    """oracle.expert (one expert, one token) is the term the forward sums."""
    cfg = small_cfg(synth.PQ2_0, Fs=0, r=0, k=1)
    L = synth.layer_host(cfg)
    lay = oracle_layer_from(cfg, L)
    x = synth.x_host(cfg, 2)
    out, ids, g = oracle.forward(lay, x)
    for t in range(2):
        _, y = oracle.expert(lay, int(ids[t, 0]), x[t])
        np.testing.assert_allclose(out[t], y, rtol=1e-14, atol=1e-300)


def test_packed_correction_matches_numpy_from_codes():
    """Ternary correction factors in PQ2_0 blocks: the oracle's z = A x and c = B z from the
    packed bytes against numpy from the generating codes and scales (groups of 128 along each
    factor's reduction axis: d for A, r for B), and the block with the packed correction minus
    the block without any correction is c."""
    cfg = small_cfg(fmt=synth.PTQ1_0, r=256)
    L = synth.layer_host(cfg)
    rng = np.random.default_rng(31)
    ca = synth.ternary_codes(rng, (cfg.rank, cfg.d))
    sa = synth.group_scales(rng, (cfg.rank, cfg.d // 128))
    cb = synth.ternary_codes(rng, (cfg.d, cfg.rank))
    sb = synth.group_scales(rng, (cfg.d, cfg.rank // 128))
    ol = oracle_layer_from(cfg, L)
    ol.corr_a, ol.corr_b, ol.corr_packed = oracle.pack(synth.PQ2_0, ca, sa), oracle.pack(synth.PQ2_0, cb, sb), 1
    x = synth.x_host(cfg, 5)
    z, c = oracle.corr(ol, x)
    A = ca.astype(np.float64) * np.repeat(f16(sa), 128, axis=1)
    B = cb.astype(np.float64) * np.repeat(f16(sb), 128, axis=1)
    xv = bf16(x)
    np.testing.assert_allclose(z, xv @ A.T, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(c, z @ B.T, rtol=1e-10, atol=1e-14)
    out, _, _ = oracle.forward(ol, x)
    ol0 = oracle_layer_from(cfg, L)
    ol0.rank, ol0.corr_a, ol0.corr_b = 0, None, None
    out0, _, _ = oracle.forward(ol0, x)
    np.testing.assert_allclose(out - out0, c, rtol=1e-9, atol=1e-12)


def test_expert_parallel_parts_sum_to_the_block():
    """The parts an expert-parallel layout computes: routed terms of disjoint expert ranges that
    cover all experts, plus the dense part (shared expert + correction) once, add up to the block
    output; the dense part alone is the shared expert's output plus the correction's; an empty
    range contributes nothing."""
    cfg = synth.Config("ep", 41, 256, 12, 3, 128, 128, synth.PQ2_0, 16, False, [8], 1)
    L = synth.layer_host(cfg)
    ol = oracle_layer_from(cfg, L)
    x = synth.x_host(cfg, 9)
    full, _, _ = oracle.forward(ol, x)
    parts = [oracle.forward_part(ol, x, lo, n, oracle.ROUTED) for lo, n in ((0, 5), (5, 4), (9, 3))]
    dense = oracle.forward_part(ol, x, 0, 0, oracle.DENSE)
    np.testing.assert_allclose(sum(parts) + dense, full, rtol=1e-12, atol=1e-12)
    _, ys = oracle.shared(ol, x)
    _, c = oracle.corr(ol, x)
    np.testing.assert_allclose(dense, ys + c, rtol=1e-12, atol=1e-13)
    assert (oracle.forward_part(ol, x, 4, 0, oracle.ROUTED) == 0).all()
    np.testing.assert_allclose(oracle.forward_part(ol, x, 0, 12, oracle.ROUTED | oracle.DENSE), full, rtol=1e-12,
                               atol=1e-13)
