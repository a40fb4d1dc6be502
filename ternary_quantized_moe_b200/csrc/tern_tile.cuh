// tern_tile.cuh -- register-level building blocks of the weight-streaming (decode) kernels:
// the per-format B-operand column orders, the in-register unpack of PQ2_0 / PTQ1_0 codes
// into mma.sync A fragments, and one 16-row x 128-column tile times up to 8 tokens.
//
// Containers ("Scion-35B-A3B" model card, Weight Representation: PQ2_0, 2-bit codes +
// fp16 scale per 128; "Scion-FlashNext-176B-A6B" model card, Weight Representation:
// PTQ1_0, base-3 trits + fp16 scale per 128); bit orders as in include/scion.h.
#pragma once

#include "scion_internal.cuh"

namespace scion {

constexpr uint32_t kMagic = 0x64006400u;  // fp16x2 (1024, 1024)

// ------------------------------------------------------------ fragment orders
// Within each 128-column group the B operand (x or h, fp16) is stored permuted so
// that lane (n, c) finds the 64 bytes it needs for the whole group contiguously:
// element index idx = 32c + ... (see frag_index_*).
//  PQ2_0  (m16n8k16, 8 steps s): idx = 32c + 4s + q  <->  column 32c + s + 8q.
//  PTQ1_0 (m16n8k8, 16 steps s): idx = 32c + 2s + h  <->
//         s < 15: column 5(6c + m + 3h) + j with m = s/5, j = s%5;  s = 15: 120 + 2c + h.
__device__ __forceinline__ int frag_col(int fmt, int idx) {
  int c = idx >> 5, w = idx & 31;
  if (fmt == SCION_PQ2_0) {
    int s = w >> 2, q = w & 3;
    return 32 * c + s + 8 * q;
  }
  int s = w >> 1, h = w & 1;
  if (s == 15) return 120 + 2 * c + h;
  int m = s / 5, j = s % 5;
  return 5 * (6 * c + m + 3 * h) + j;
}

__device__ __forceinline__ int frag_index(int fmt, int col) {
  if (fmt == SCION_PQ2_0) {
    int c = col >> 5, rem = col & 31;
    return 32 * c + 4 * (rem & 7) + (rem >> 3);
  }
  if (col >= 120) {
    int rho = col - 120;
    return 32 * (rho >> 1) + 30 + (rho & 1);
  }
  int Q = col / 5, j = col % 5, c = Q / 6, mm = Q % 6;
  int m = mm % 3, h = mm / 3;
  return 32 * c + 2 * (5 * m + j) + h;
}

// Stored order of a B group row (SCION_BROW halves): lane (n, c) consumes the 32 elements
// idx = 32c + w (w = 0..31) as four 16-byte chunks w / 8; chunk i of lane-column c is stored at
// halves 32i + 8c, so the four lane-columns of one 16-byte load read 64 contiguous bytes.
__device__ __forceinline__ int brow_pos_of(int c, int w) { return 32 * (w >> 3) + 8 * c + (w & 7); }
// column held by stored position p
__device__ __forceinline__ int brow_col(int fmt, int p) {
  const int w = 8 * (p >> 5) + (p & 7), c = (p >> 3) & 3;
  return frag_col(fmt, 32 * c + w);
}
// stored position of column col
__device__ __forceinline__ int brow_pos(int fmt, int col) {
  const int idx = frag_index(fmt, col);
  return brow_pos_of(idx >> 5, idx & 31);
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_stream32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];\n" : "=r"(v) : "l"(p));
  return v;
}


// ================================================================= ternary tiles
// PQ2_0 unpack without per-step shifts: for pair s < 5 the 2-bit field sits at bits
// 2s..2s+1 of each 16-bit half, so ((w & (3 << 2s)) | (1024,1024)) is the fp16 value
// 1024 + 4^s b and subtracting (1024 + 4^s) leaves 4^s (b - 1) exactly; pairs 5..7 do
// the same on w >> 10.  The factor 4^f(s) (f(s) = s < 5 ? s : s - 5) is divided out of
// the B operand when it is written (an exact power-of-two scaling of the fp16 values).
__device__ __forceinline__ int pq2_f(int s) { return s < 5 ? s : s - 5; }
__device__ __forceinline__ float pq2_bscale(int idx) { return exp2f(-2.0f * pq2_f((idx & 31) >> 2)); }
// the same factor for stored position p of a B group row
__device__ __forceinline__ float brow_bscale(int p) { return exp2f(-2.0f * pq2_f(((p >> 5) * 8 + (p & 7)) >> 2)); }

template <int S>
__device__ __forceinline__ uint32_t pq2_pair_nf(uint32_t w, uint32_t w10) {
  constexpr int f = S < 5 ? S : S - 5;
  constexpr uint32_t mask = 0x00030003u << (2 * f);
  constexpr uint32_t biash = 0x6400u + (1u << (2 * f));  // fp16 bits of 1024 + 4^f (exact, < 2048)
  const __half2 v = u32_as_h2(lop3_and_or(S < 5 ? w : w10, mask, kMagic));
  return h2_as_u32(__hsub2(v, u32_as_h2(biash | (biash << 16))));
}

// PQ2_0 unpack to fp16 subnormals (one AND per two weights).  Masking the field of pair s
// (bits 2f..2f+1 of each 16-bit half, f = s < 5 ? s : s - 5, pairs 5..7 taken from w >> 10)
// leaves the bit pattern b * 4^f with a zero exponent field: the fp16 subnormal
// b * 4^f * 2^-24, where b = code + 1 is the stored field (0..2).  With the B operand
// pre-scaled by 4^-f the MMA sums 2^-24 * b * x; starting the accumulator at
// -2^-24 * sum(x) (the group-row tail) leaves 2^-24 * sum(code * x).
template <int S>
__device__ __forceinline__ uint32_t pq2_pair_sub(uint32_t w, uint32_t w10) {
  constexpr int f = S < 5 ? S : S - 5;
  return (S < 5 ? w : w10) & (0x00030003u << (2 * f));
}

// Registers of one 16-row x 128-column sub-tile block for lane (r8, c).
template <int FMT>
struct TileRegs;
template <>
struct TileRegs<SCION_PQ2_0> {
  uint4 w;
  uint32_t sc;
  __device__ __forceinline__ void load(const uint8_t* blk, int lane) {
    w = ldg_stream(blk + 16 * lane);
    sc = ldg_stream32(blk + 512 + 4 * (lane >> 2));
  }
  // from a sub-tile block staged in shared memory (shared-window address)
  __device__ __forceinline__ void load_shared(uint32_t blk, int lane) {
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                 : "r"(blk + 16 * lane));
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(sc) : "r"(blk + 512 + 4 * (lane >> 2)));
  }
};
template <>
struct TileRegs<SCION_PTQ1_0> {
  uint32_t q0, q1, q2, rem, sc;
  __device__ __forceinline__ void load(const uint8_t* blk, int lane) {
    q0 = ldg_stream32(blk + 12 * lane);
    q1 = ldg_stream32(blk + 12 * lane + 4);
    q2 = ldg_stream32(blk + 12 * lane + 8);
    rem = ldg_stream32(blk + 384 + 4 * (lane >> 2));
    sc = ldg_stream32(blk + 416 + 4 * (lane >> 2));
  }
  __device__ __forceinline__ void load_shared(uint32_t blk, int lane) {
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(q0) : "r"(blk + 12 * lane));
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(q1) : "r"(blk + 12 * lane + 4));
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(q2) : "r"(blk + 12 * lane + 8));
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(rem) : "r"(blk + 384 + 4 * (lane >> 2)));
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(sc) : "r"(blk + 416 + 4 * (lane >> 2)));
  }
};

// PTQ1_0: 5 base-3 digits of two quintet bytes held as fp16 (1024+v) halves.
// floor(v/3) = round(v*fp16(1/3) + 682.5 - ...) lands on 1024 + floor(v/3) exactly for
// v < 243; digit - 1 = V - 3*V' + 2047.  Exact for every byte value (checked on all 243).
struct Ptq1Digits {
  __half2 V;
  __device__ __forceinline__ uint32_t next() {
    const __half2 third = __float2half2_rn(0.333251953125f);
    const __half2 c1 = __float2half2_rn(682.5f);
    const __half2 m3 = __float2half2_rn(-3.0f);
    const __half2 c2047 = __float2half2_rn(2047.0f);
    __half2 Vn = __hfma2(V, third, c1);
    __half2 code = __hadd2(__hfma2(Vn, m3, V), c2047);
    V = Vn;
    return h2_as_u32(code);
  }
};

__device__ __forceinline__ __half2 ptq1_v0(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t p;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(p) : "r"(a), "r"(b), "r"(sel));
  return u32_as_h2(lop3_and_or(p, 0x00ff00ffu, kMagic));
}

// PTQ1_0 tile for the ring kernels: the digit chains, then eight MMAs issued without `volatile`
// (independent tiles of a stage can interleave).
__device__ __forceinline__ void tile_mma_ptq1_nv(const TileRegs<SCION_PTQ1_0>& t, const uint32_t (&b)[16],
                                                 float (&acc)[4], int c) {
  const uint32_t sel_r[3] = {0x0300u, 0x0401u, 0x0502u};
  const uint32_t sel_h[3] = {0x0502u, 0x0603u, 0x0704u};
  uint32_t ar[16], ah[16];
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    Ptq1Digits dr{ptq1_v0(t.q0, t.q1, sel_r[m])}, dh{ptq1_v0(t.q1, t.q2, sel_h[m])};
#pragma unroll
    for (int j = 0; j < 5; ++j) ar[5 * m + j] = dr.next(), ah[5 * m + j] = dh.next();
  }
  ar[15] = ptq1_rem_pair(t.rem, 2 * c);
  ah[15] = ptq1_rem_pair(t.rem, 2 * c + 8);
  float g[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int s2 = 0; s2 < 8; ++s2) {
    const uint32_t fa[4] = {ar[2 * s2], ah[2 * s2], ar[2 * s2 + 1], ah[2 * s2 + 1]};
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(g[0]), "+f"(g[1]), "+f"(g[2]), "+f"(g[3])
        : "r"(fa[0]), "r"(fa[1]), "r"(fa[2]), "r"(fa[3]), "r"(b[2 * s2]), "r"(b[2 * s2 + 1]));
  }
  const float2 sf = __half22float2(u32_as_h2(t.sc));
  acc[0] = fmaf(sf.x, g[0], acc[0]);
  acc[1] = fmaf(sf.x, g[1], acc[1]);
  acc[2] = fmaf(sf.y, g[2], acc[2]);
  acc[3] = fmaf(sf.y, g[3], acc[3]);
}

// acc += scale_row * (codes . B) for one loaded tile and one token tile of 8.
// b: the lane's 64 bytes of the group (16 u32) in fragment order.
template <int FMT>
__device__ __forceinline__ void tile_mma(const TileRegs<FMT>& t, const uint32_t (&b)[16], float (&acc)[4], int c) {
  float g[4] = {0.f, 0.f, 0.f, 0.f};
  if constexpr (FMT == SCION_PQ2_0) {
    const uint32_t x10 = t.w.x >> 10, y10 = t.w.y >> 10, z10 = t.w.z >> 10, w10 = t.w.w >> 10;
#define SCION_PQ2_STEP(S)                                                                          \
  {                                                                                                \
    const uint32_t fa[4] = {pq2_pair_nf<S>(t.w.x, x10), pq2_pair_nf<S>(t.w.z, z10),                \
                            pq2_pair_nf<S>(t.w.y, y10), pq2_pair_nf<S>(t.w.w, w10)};               \
    mma_f16_16816(g, fa, b[2 * S], b[2 * S + 1]);                                                  \
  }
    SCION_PQ2_STEP(0) SCION_PQ2_STEP(1) SCION_PQ2_STEP(2) SCION_PQ2_STEP(3)
    SCION_PQ2_STEP(4) SCION_PQ2_STEP(5) SCION_PQ2_STEP(6) SCION_PQ2_STEP(7)
#undef SCION_PQ2_STEP
  } else {
    // row r quintets: q0.b0..b3, q1.b0, q1.b1;  row r+8: q1.b2, q1.b3, q2.b0..b3.
    // half2 slot j (j < 15) = digit j%5 of the quintet pair m = j/5: (Q[m], Q[m+3]); slot 15 =
    // this lane's two remainder trits.  Slots (2s, 2s+1) feed the k16 step s.
    const uint32_t sel_r[3] = {0x0300u, 0x0401u, 0x0502u};  // pairs (Q[m], Q[m+3]) from (q0, q1)
    const uint32_t sel_h[3] = {0x0502u, 0x0603u, 0x0704u};  // from (q1, q2)
    uint32_t ar[16], ah[16];
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      Ptq1Digits dr{ptq1_v0(t.q0, t.q1, sel_r[m])}, dh{ptq1_v0(t.q1, t.q2, sel_h[m])};
#pragma unroll
      for (int j = 0; j < 5; ++j) ar[5 * m + j] = dr.next(), ah[5 * m + j] = dh.next();
    }
    ar[15] = ptq1_rem_pair(t.rem, 2 * c);
    ah[15] = ptq1_rem_pair(t.rem, 2 * c + 8);
#pragma unroll
    for (int s2 = 0; s2 < 8; ++s2) {
      const uint32_t fa[4] = {ar[2 * s2], ah[2 * s2], ar[2 * s2 + 1], ah[2 * s2 + 1]};
      mma_f16_16816(g, fa, b[2 * s2], b[2 * s2 + 1]);
    }
  }
  const float s_lo = __half2float(__ushort_as_half(uint16_t(t.sc & 0xffff)));
  const float s_hi = __half2float(__ushort_as_half(uint16_t(t.sc >> 16)));
  acc[0] = fmaf(s_lo, g[0], acc[0]);
  acc[1] = fmaf(s_lo, g[1], acc[1]);
  acc[2] = fmaf(s_hi, g[2], acc[2]);
  acc[3] = fmaf(s_hi, g[3], acc[3]);
}

// PQ2_0, subnormal unpack: acc += scale_row * 2^-24 * (codes . B) for one tile and one token
// tile of 8.  xn0 / xn1 = -2^-24 * (group sum of B) of the lane's token columns 2c, 2c+1.
__device__ __forceinline__ void tile_mma_pq2_sub(const TileRegs<SCION_PQ2_0>& t, const uint32_t (&b)[16],
                                                 float (&acc)[4], float xn0, float xn1) {
  float g[4] = {xn0, xn1, xn0, xn1};
  const uint32_t x10 = t.w.x >> 10, y10 = t.w.y >> 10, z10 = t.w.z >> 10, w10 = t.w.w >> 10;
#define SCION_PQ2_SUB_STEP(S)                                                                      \
  {                                                                                                \
    const uint32_t fa[4] = {pq2_pair_sub<S>(t.w.x, x10), pq2_pair_sub<S>(t.w.z, z10),              \
                            pq2_pair_sub<S>(t.w.y, y10), pq2_pair_sub<S>(t.w.w, w10)};             \
    mma_f16_16816(g, fa, b[2 * S], b[2 * S + 1]);                                                  \
  }
  SCION_PQ2_SUB_STEP(0) SCION_PQ2_SUB_STEP(1) SCION_PQ2_SUB_STEP(2) SCION_PQ2_SUB_STEP(3)
  SCION_PQ2_SUB_STEP(4) SCION_PQ2_SUB_STEP(5) SCION_PQ2_SUB_STEP(6) SCION_PQ2_SUB_STEP(7)
#undef SCION_PQ2_SUB_STEP
  const float s_lo = __half2float(__ushort_as_half(uint16_t(t.sc & 0xffff)));
  const float s_hi = __half2float(__ushort_as_half(uint16_t(t.sc >> 16)));
  acc[0] = fmaf(s_lo, g[0], acc[0]);
  acc[1] = fmaf(s_lo, g[1], acc[1]);
  acc[2] = fmaf(s_hi, g[2], acc[2]);
  acc[3] = fmaf(s_hi, g[3], acc[3]);
}

// B fragment of one group for lane (n, c): its 64 bytes of row `row` (or zeros); group rows are
// SCION_BROW halves apart.
__device__ __forceinline__ void load_b(const __half* base, int64_t row_stride_h, int row, int g, int c,
                                       uint32_t (&b)[16]) {
  if (row >= 0) {
    const __half* rp = base + int64_t(row) * row_stride_h + int64_t(g) * SCION_BROW + 8 * c;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(rp + 32 * i);
      b[4 * i] = v.x, b[4 * i + 1] = v.y, b[4 * i + 2] = v.z, b[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) b[i] = 0u;
  }
}

}  // namespace scion
