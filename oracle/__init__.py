"""CPU fp64 oracle for the ternary MoE block -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product library never calls it, and this
package imports nothing from the product library: the two share no code.

The arithmetic lives in ``scion_oracle.c`` (plain C, fp64, OpenMP over
independent tokens / experts).  This module compiles it with gcc on first use
(or via :func:`build`) and wraps it with numpy arrays.

Arrays use the storage dtypes of the pages' formats: bf16 and fp16 values are
passed as their uint16 bit patterns; packed banks are uint8 blocks of 34 B
(PQ2_0) or 28 B (PTQ1_0) per 128 weights, laid out row-major with the groups of
128 running along each row's reduction axis ("Scion-35B-A3B" model card, Weight
Representation; "Scion-FlashNext-176B-A6B" model card, Weight Representation).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "scion_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

PQ2_0 = 0
PTQ1_0 = 1
OK, EINVAL, ENOMEM, EFORMAT = 0, -1, -2, -4


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (plain -O2, no -march)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(C.Structure):
    _fields_ = [
        ("d", C.c_int), ("n_experts", C.c_int), ("top_k", C.c_int), ("ffn", C.c_int),
        ("shared_ffn", C.c_int), ("rank", C.c_int), ("fmt", C.c_int), ("router_f32", C.c_int),
        ("norm_topk", C.c_int), ("corr_on_output", C.c_int),
        ("w_router", C.c_void_p), ("w_delta", C.c_void_p),
        ("gate_exps", C.c_void_p), ("up_exps", C.c_void_p), ("down_exps", C.c_void_p),
        ("sh_gate", C.c_void_p), ("sh_up", C.c_void_p), ("sh_down", C.c_void_p),
        ("sh_gate_vec", C.c_void_p), ("corr_a", C.c_void_p), ("corr_b", C.c_void_p),
        ("corr_packed", C.c_int),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = C.CDLL(_LIB)
            vp, i64, ci = C.c_void_p, C.c_int64, C.c_int
            lib.oracle_f16_to_f64.restype = C.c_double
            lib.oracle_f16_to_f64.argtypes = [C.c_uint16]
            lib.oracle_bf16_to_f64.restype = C.c_double
            lib.oracle_bf16_to_f64.argtypes = [C.c_uint16]
            lib.oracle_block_bytes.restype = C.c_long
            lib.oracle_block_bytes.argtypes = [ci]
            for name in ("oracle_pq2_pack", "oracle_ptq1_pack"):
                getattr(lib, name).restype = ci
                getattr(lib, name).argtypes = [vp, vp, i64, vp]
            for name in ("oracle_pq2_unpack", "oracle_ptq1_unpack"):
                getattr(lib, name).restype = ci
                getattr(lib, name).argtypes = [vp, i64, vp, vp]
            lib.oracle_dequant_row.restype = ci
            lib.oracle_dequant_row.argtypes = [ci, vp, ci, vp]
            lib.oracle_router_logits_one.restype = None
            lib.oracle_router_logits_one.argtypes = [C.POINTER(_Layer), vp, vp]
            lib.oracle_topk.restype = None
            lib.oracle_topk.argtypes = [vp, ci, ci, vp]
            lib.oracle_gates.restype = None
            lib.oracle_gates.argtypes = [vp, ci, ci, vp, ci, vp]
            lib.oracle_group.restype = None
            lib.oracle_group.argtypes = [vp, ci, ci, ci, vp, vp, vp]
            lib.oracle_expert_one.restype = ci
            lib.oracle_expert_one.argtypes = [C.POINTER(_Layer), ci, vp, vp, vp]
            lib.oracle_route.restype = ci
            lib.oracle_route.argtypes = [C.POINTER(_Layer), vp, ci, vp, vp, vp]
            lib.oracle_moe_forward.restype = ci
            lib.oracle_moe_forward.argtypes = [C.POINTER(_Layer), vp, ci, vp, vp, vp]
            lib.oracle_moe_forward_part.restype = ci
            lib.oracle_moe_forward_part.argtypes = [C.POINTER(_Layer), vp, ci, ci, ci, ci, vp]
            lib.oracle_moe_forward_dense.restype = ci
            lib.oracle_moe_forward_dense.argtypes = [C.POINTER(_Layer), vp, ci, vp]
            lib.oracle_shared.restype = ci
            lib.oracle_shared.argtypes = [C.POINTER(_Layer), vp, ci, vp, vp]
            lib.oracle_corr.restype = ci
            lib.oracle_corr.argtypes = [C.POINTER(_Layer), vp, ci, vp, vp]
            lib.oracle_f64_to_f16_nonneg.restype = C.c_uint16
            lib.oracle_f64_to_f16_nonneg.argtypes = [C.c_double]
            lib.oracle_quantize.restype = ci
            lib.oracle_quantize.argtypes = [ci, vp, i64, ci, vp, vp]
            lib.oracle_attn_corr.restype = ci
            lib.oracle_attn_corr.argtypes = [ci, ci, ci, ci, vp, vp, vp, ci, vp, vp, vp]
            _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


# ----------------------------------------------------------------- scalars
def f16_to_f64(bits: int) -> float:
    return _load().oracle_f16_to_f64(int(bits))


def bf16_to_f64(bits: int) -> float:
    return _load().oracle_bf16_to_f64(int(bits))


def block_bytes(fmt: int) -> int:
    return int(_load().oracle_block_bytes(int(fmt)))


# -------------------------------------------------------------- containers
def pack(fmt: int, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """codes: int8 [..., K] in {-1,0,1} (K % 128 == 0); scales: uint16 [..., K/128].
    Returns uint8 [..., K/128 * block_bytes]."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    n_groups = codes.size // 128
    assert scales.size == n_groups
    bb = block_bytes(fmt)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] // 128 * bb,), dtype=np.uint8)
    fn = _load().oracle_pq2_pack if fmt == PQ2_0 else _load().oracle_ptq1_pack
    st = fn(_ptr(codes), _ptr(scales), n_groups, _ptr(out))
    if st != OK:
        raise ValueError("oracle pack failed: %d" % st)
    return out


def unpack(fmt: int, blocks: np.ndarray):
    """Inverse of :func:`pack`.  Returns (codes int8 [..., K], scales uint16 [..., K/128], status)."""
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    bb = block_bytes(fmt)
    n_groups = blocks.size // bb
    codes = np.empty(blocks.shape[:-1] + (blocks.shape[-1] // bb * 128,), dtype=np.int8)
    scales = np.empty(blocks.shape[:-1] + (blocks.shape[-1] // bb,), dtype=np.uint16)
    fn = _load().oracle_pq2_unpack if fmt == PQ2_0 else _load().oracle_ptq1_unpack
    st = fn(_ptr(blocks), n_groups, _ptr(codes), _ptr(scales))
    return codes, scales, int(st)


def dequant_rows(fmt: int, blocks: np.ndarray, K: int) -> np.ndarray:
    """Packed rows [R, K/128*bb] -> fp64 [R, K] = code * scale."""
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8).reshape(-1, blocks.shape[-1])
    out = np.empty((blocks.shape[0], K), dtype=np.float64)
    lib = _load()
    for r in range(blocks.shape[0]):
        row = np.ascontiguousarray(blocks[r])
        st = lib.oracle_dequant_row(fmt, _ptr(row), K, out[r].ctypes.data)
        if st != OK:
            raise ValueError("invalid code in row %d" % r)
    return out


# ------------------------------------------------------------------- layer
@dataclass
class OracleLayer:
    """Host copy of one MoE block in the interchange layout."""
    d: int
    n_experts: int
    top_k: int
    ffn: int
    fmt: int
    w_router: np.ndarray               # [E, d] float32 or uint16 (bf16 bits)
    w_delta: np.ndarray                # same dtype as w_router
    gate_exps: np.ndarray              # uint8 [E, ffn, d/128*bb]
    up_exps: np.ndarray                # uint8 [E, ffn, d/128*bb]
    down_exps: np.ndarray              # uint8 [E, d, ffn/128*bb]
    shared_ffn: int = 0
    sh_gate: Optional[np.ndarray] = None   # uint16 bf16 [Fs, d]
    sh_up: Optional[np.ndarray] = None     # uint16 bf16 [Fs, d]
    sh_down: Optional[np.ndarray] = None   # uint16 bf16 [d, Fs]
    sh_gate_vec: Optional[np.ndarray] = None  # uint16 bf16 [d]
    rank: int = 0
    corr_a: Optional[np.ndarray] = None    # uint16 bf16 [r, d], or uint8 PQ2_0 blocks [r, d/128*34]
    corr_b: Optional[np.ndarray] = None    # uint16 bf16 [d, r], or uint8 PQ2_0 blocks [d, r/128*34]
    norm_topk: int = 1
    corr_on_output: int = 0
    corr_packed: int = 0                   # 1: the correction factors are the PQ2_0 blocks

    def _c(self) -> _Layer:
        rf32 = 1 if self.w_router.dtype == np.float32 else 0
        for name in ("w_router", "w_delta", "gate_exps", "up_exps", "down_exps", "sh_gate", "sh_up",
                     "sh_down", "sh_gate_vec", "corr_a", "corr_b"):
            a = getattr(self, name)
            if a is not None and not a.flags["C_CONTIGUOUS"]:
                setattr(self, name, np.ascontiguousarray(a))
        L = _Layer()
        L.d, L.n_experts, L.top_k, L.ffn = self.d, self.n_experts, self.top_k, self.ffn
        L.shared_ffn, L.rank, L.fmt, L.router_f32 = self.shared_ffn, self.rank, self.fmt, rf32
        L.norm_topk, L.corr_on_output = self.norm_topk, self.corr_on_output
        L.w_router, L.w_delta = _ptr(self.w_router), _ptr(self.w_delta)
        L.gate_exps, L.up_exps, L.down_exps = _ptr(self.gate_exps), _ptr(self.up_exps), _ptr(self.down_exps)
        L.sh_gate, L.sh_up, L.sh_down = _ptr(self.sh_gate), _ptr(self.sh_up), _ptr(self.sh_down)
        L.sh_gate_vec, L.corr_a, L.corr_b = _ptr(self.sh_gate_vec), _ptr(self.corr_a), _ptr(self.corr_b)
        L.corr_packed = self.corr_packed
        return L


def _x(layer: OracleLayer, x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    assert x.ndim == 2 and x.shape[1] == layer.d
    return x


def route(layer: OracleLayer, x: np.ndarray):
    """Returns (logits fp64 [T,E], ids int32 [T,k], gates fp64 [T,k])."""
    x = _x(layer, x)
    T = x.shape[0]
    logits = np.empty((T, layer.n_experts), np.float64)
    ids = np.empty((T, layer.top_k), np.int32)
    gates = np.empty((T, layer.top_k), np.float64)
    L = layer._c()
    st = _load().oracle_route(C.byref(L), _ptr(x), T, _ptr(logits), _ptr(ids), _ptr(gates))
    if st != OK:
        raise RuntimeError("oracle_route: %d" % st)
    return logits, ids, gates


def topk(logits_row: np.ndarray, k: int) -> np.ndarray:
    row = np.ascontiguousarray(logits_row, dtype=np.float64)
    ids = np.empty(k, np.int32)
    _load().oracle_topk(_ptr(row), row.size, k, _ptr(ids))
    return ids


def gates(logits_row: np.ndarray, ids: np.ndarray, norm_topk: int = 1) -> np.ndarray:
    row = np.ascontiguousarray(logits_row, dtype=np.float64)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    g = np.empty(ids.size, np.float64)
    _load().oracle_gates(_ptr(row), row.size, ids.size, _ptr(ids), int(norm_topk), _ptr(g))
    return g


def group(ids: np.ndarray, n_experts: int):
    """Histogram / exclusive scan / stable scatter of ids [T,k].
    Returns (counts [E], offsets [E+1], perm [T*k] with entries t*k+j)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    counts = np.empty(n_experts, np.int32)
    offsets = np.empty(n_experts + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    _load().oracle_group(_ptr(ids), T, k, n_experts, _ptr(counts), _ptr(offsets), _ptr(perm))
    return counts, offsets, perm


def expert(layer: OracleLayer, e: int, x_row: np.ndarray):
    """One expert on one token: (h fp64 [ffn], y fp64 [d])."""
    x_row = np.ascontiguousarray(x_row, dtype=np.uint16).reshape(-1)
    h = np.empty(layer.ffn, np.float64)
    y = np.empty(layer.d, np.float64)
    L = layer._c()
    st = _load().oracle_expert_one(C.byref(L), int(e), _ptr(x_row), _ptr(h), _ptr(y))
    if st != OK:
        raise RuntimeError("oracle_expert_one: %d" % st)
    return h, y


def forward(layer: OracleLayer, x: np.ndarray):
    """The block forward.  Returns (out fp64 [T,d], ids int32 [T,k], gates fp64 [T,k])."""
    x = _x(layer, x)
    T = x.shape[0]
    out = np.zeros((T, layer.d), np.float64)
    ids = np.zeros((T, layer.top_k), np.int32)
    g = np.zeros((T, layer.top_k), np.float64)
    if T == 0:
        return out, ids, g
    L = layer._c()
    st = _load().oracle_moe_forward(C.byref(L), _ptr(x), T, _ptr(out), _ptr(ids), _ptr(g))
    if st != OK:
        raise RuntimeError("oracle_moe_forward: %d" % st)
    return out, ids, g


ROUTED, DENSE = 1, 2


def forward_part(layer: OracleLayer, x: np.ndarray, expert_lo: int = 0, n_local: Optional[int] = None,
                 parts: int = ROUTED | DENSE) -> np.ndarray:
    """The part of the block one expert-parallel rank computes: the routed terms of the experts in
    [expert_lo, expert_lo + n_local) (parts & ROUTED) and the shared expert + correction (parts &
    DENSE).  Disjoint ranges covering all experts plus one dense part sum to forward()."""
    x = _x(layer, x)
    n_local = layer.n_experts - expert_lo if n_local is None else n_local
    out = np.zeros((x.shape[0], layer.d), np.float64)
    if x.shape[0] == 0:
        return out
    L = layer._c()
    st = _load().oracle_moe_forward_part(C.byref(L), _ptr(x), x.shape[0], int(expert_lo), int(n_local), int(parts),
                                         _ptr(out))
    if st != OK:
        raise RuntimeError("oracle_moe_forward_part: %d" % st)
    return out


def forward_dense(layer: OracleLayer, x: np.ndarray) -> np.ndarray:
    """Cross-form over all E experts with masked gates (tiny sizes only)."""
    x = _x(layer, x)
    out = np.zeros((x.shape[0], layer.d), np.float64)
    L = layer._c()
    st = _load().oracle_moe_forward_dense(C.byref(L), _ptr(x), x.shape[0], _ptr(out))
    if st != OK:
        raise RuntimeError("oracle_moe_forward_dense: %d" % st)
    return out


def shared(layer: OracleLayer, x: np.ndarray):
    """Shared expert: (h fp64 [T,Fs], y fp64 [T,d])."""
    x = _x(layer, x)
    T = x.shape[0]
    h = np.empty((T, layer.shared_ffn), np.float64)
    y = np.empty((T, layer.d), np.float64)
    L = layer._c()
    st = _load().oracle_shared(C.byref(L), _ptr(x), T, _ptr(h), _ptr(y))
    if st != OK:
        raise RuntimeError("oracle_shared: %d" % st)
    return h, y


def corr(layer: OracleLayer, x: np.ndarray):
    """Correction on the block input: (z fp64 [T,r], c fp64 [T,d])."""
    x = _x(layer, x)
    T = x.shape[0]
    z = np.empty((T, layer.rank), np.float64)
    y = np.empty((T, layer.d), np.float64)
    L = layer._c()
    st = _load().oracle_corr(C.byref(L), _ptr(x), T, _ptr(z), _ptr(y))
    if st != OK:
        raise RuntimeError("oracle_corr: %d" % st)
    return z, y


def attn_corr(v: np.ndarray, a: np.ndarray, b: np.ndarray, d_in: int, d_out: int, rank: int, packed: int = 0,
              base: Optional[np.ndarray] = None):
    """The correction branch on the attention output ("Scion: ternary MoE quantization with trained
    corrections", The idea and Findings): z = A v, out = base + B z.  v: bf16 bits [T, d_in];
    a, b: bf16 bits [rank, d_in] / [d_out, rank] or (packed) PQ2_0 blocks; base fp64 [T, d_out] or
    None.  Returns (out fp64 [T, d_out], z fp64 [T, rank])."""
    v = np.ascontiguousarray(v, dtype=np.uint16)
    assert v.ndim == 2 and v.shape[1] == d_in
    T = v.shape[0]
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    out = np.empty((T, d_out), np.float64)
    z = np.empty((T, rank), np.float64)
    bs = None if base is None else np.ascontiguousarray(base, dtype=np.float64)
    st = _load().oracle_attn_corr(d_in, d_out, rank, int(packed), _ptr(a), _ptr(b), _ptr(v), T, _ptr(bs), _ptr(out),
                                  _ptr(z))
    if st != OK:
        raise RuntimeError("oracle_attn_corr: %d" % st)
    return out, z


ABSMEAN = 0
LLOYD = 1


def f64_to_f16(v: float) -> int:
    """Nearest binary16 bit pattern of a finite v >= 0 (ties to even)."""
    return int(_load().oracle_f64_to_f16_nonneg(float(v)))


def quantize(method: int, w: np.ndarray, iters: int = 30):
    """Ternary codes int8 [n, 128] and fp16 scales (uint16 bits) [n] of fp32 groups w [n, 128]
    ("Scion: ternary MoE quantization with trained corrections", Findings; "Scion-35B-A3B" model
    card, Highlights): ABSMEAN (s = mean |w|, codes by rounding w / s) or LLOYD (centroid /
    nearest-level rounds from the absmean start).  Decisions in fp64; see scion_oracle.c."""
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(-1, 128)
    n = w.shape[0]
    codes = np.empty((n, 128), np.int8)
    scales = np.empty(n, np.uint16)
    st = _load().oracle_quantize(int(method), _ptr(w), n, int(iters), _ptr(codes), _ptr(scales))
    if st != OK:
        raise ValueError("oracle_quantize failed: %d" % st)
    return codes, scales


def cores_used() -> int:
    """Threads the OpenMP loops will use (OMP_NUM_THREADS or all online CPUs)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.isdigit():
        return int(env)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
