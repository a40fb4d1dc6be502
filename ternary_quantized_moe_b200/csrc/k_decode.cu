// k_decode.cu -- weight-streaming kernels for one pass of up to SCION_TDEC tokens.
//
// The block ("Scion: ternary MoE quantization with trained corrections", The idea;
// "Scion-35B-A3B" and "Scion-FlashNext-176B-A6B" model cards, Model Overview and
// Weight Representation):
//   out[t] = sum_j g_tj W_d,e (silu(W_g,e x_t) * (W_u,e x_t)) + S(x_t) + B (A x_t)
// with W = code * scale, codes in {-1,0,+1}, one fp16 scale per 128 weights.
//
// Kernels (each weight byte is read from HBM once per pass):
//   xproj        dense bf16 rows that read x: router + router delta (-> logits),
//                shared gate/up (-> SwiGLU hidden) and correction A (-> z).  Split-K
//                over CTAs, the last CTA of a unit reduces and applies the epilogue.
//                An extra CTA column writes x in fragment order (fp16) and zeroes out.
//   gateup       ternary gate/up of every active expert, fused SwiGLU -> h (fp16).
//   down_routed  ternary down projection, gate-weighted scatter-add into out.
//   down_dense   [shared down | correction B] (fp16 copy) over [h_s | z], added to out.
//
// Tensor-core use: warp-level mma.sync with the weights as the 16-row A operand (codes
// unpacked in registers straight from 128-bit loads) and up to 8 tokens as N.  Codes
// enter the MMA as exact fp16 {-1,0,+1}; each 128-column group accumulates separately
// and is scaled by its fp16 group scale in fp32.
#include <math.h>

#include "scion_internal.cuh"

namespace scion {
namespace {

constexpr uint32_t kMagic = 0x64006400u;   // fp16x2 (1024, 1024)
constexpr uint32_t kPq2Bias = 0x64016401u; // fp16x2 (1025, 1025)

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

// ========================================================================= xproj
struct XProjArgs {
  const __nv_bfloat16* x;
  int T, d, E, Fs, r, Kd;  // Kd = padded row stride of hz
  int fmt;
  const __nv_bfloat16 *w_router, *w_delta, *sh_gate, *sh_up, *corr_a;
  const XUnit* units;
  int n_units, n_chunks;
  float* partial;
  unsigned* count;
  float* logits;
  __half* hz;
  __half* xfrag;  // [T][d/128][128] fp16 in fragment order
  float* out;     // zeroed here
};

// One CTA = (unit, 512-column chunk); 4 warps x 128 columns.  NT = token tiles of 8.
template <int NT>
__global__ void __launch_bounds__(128) xproj_kernel(XProjArgs a) {
  __shared__ float red[4][2][NT][32][4];
  __shared__ int last_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, c = lane & 3;
  const int chunk = blockIdx.y;
  const int kbase = chunk * SCION_XPROJ_KC;

  if (blockIdx.x == a.n_units) {
    // aux column: x in fragment order for this chunk's groups, and zero out.
    const int g0 = kbase >> 7, g1 = min(a.d, kbase + SCION_XPROJ_KC) >> 7;
    const int per_tok = (g1 - g0) * 128;
    for (int i = threadIdx.x; i < a.T * per_tok; i += blockDim.x) {
      int t = i / per_tok, rem = i % per_tok, g = g0 + rem / 128, idx = rem % 128;
      int col = g * 128 + frag_col(a.fmt, idx);
      a.xfrag[(int64_t(t) * (a.d >> 7) + g) * 128 + idx] = __float2half_rn(__bfloat162float(a.x[int64_t(t) * a.d + col]));
    }
    const int64_t n4 = int64_t(a.T) * a.d / 4;
    float4* o4 = reinterpret_cast<float4*>(a.out);
    for (int64_t i = int64_t(chunk) * blockDim.x + threadIdx.x; i < n4; i += int64_t(a.n_chunks) * blockDim.x)
      o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }

  const XUnit u = a.units[blockIdx.x];
  const __nv_bfloat16* mats[2];
  int nmat, nacc, nrows;
  if (u.kind == kUnitRouter) {
    mats[0] = a.w_router, mats[1] = a.w_delta, nmat = 2, nacc = 1, nrows = a.E;
  } else if (u.kind == kUnitSwiglu) {
    mats[0] = a.sh_gate, mats[1] = a.sh_up, nmat = 2, nacc = 2, nrows = a.Fs;
  } else {
    mats[0] = a.corr_a, mats[1] = a.corr_a, nmat = 1, nacc = 1, nrows = a.r;
  }

  float acc[2][NT][4];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][nt][i] = 0.f;

  const int kw = kbase + warp * 128;
  if (kw < a.d) {
    const int row_a = u.row0 + g8, row_b = u.row0 + g8 + 8;
    const bool ok_a = row_a < nrows, ok_b = row_b < nrows;
    const bool second_acc = (u.kind == kUnitSwiglu);
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      if (m >= nmat) break;
      const __nv_bfloat16* W = mats[m];
      uint4 wa[4], wb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = kw + 32 * q + 8 * c;
        wa[q] = ok_a ? ldg_stream(W + int64_t(row_a) * a.d + kk) : make_uint4(0, 0, 0, 0);
        wb[q] = ok_b ? ldg_stream(W + int64_t(row_b) * a.d + kk) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tok = nt * 8 + g8;
        uint4 xb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          xb[q] = tok < a.T ? *reinterpret_cast<const uint4*>(a.x + int64_t(tok) * a.d + kw + 32 * q + 8 * c)
                            : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t fa0[4] = {wa[q].x, wb[q].x, wa[q].y, wb[q].y};
          uint32_t fa1[4] = {wa[q].z, wb[q].z, wa[q].w, wb[q].w};
          if (m == 1 && second_acc) {
            mma_bf16_16816(acc[1][nt], fa0, xb[q].x, xb[q].y);
            mma_bf16_16816(acc[1][nt], fa1, xb[q].z, xb[q].w);
          } else {
            mma_bf16_16816(acc[0][nt], fa0, xb[q].x, xb[q].y);
            mma_bf16_16816(acc[0][nt], fa1, xb[q].z, xb[q].w);
          }
        }
      }
    }
  }
  // reduce the 4 warps
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][m][nt][lane][i] = acc[m][nt][i];
  __syncthreads();

  // thread -> (nt, lane) pairs; NT*32 pairs over 128 threads
  const int npairs = NT * 32;
  float* part = a.partial + (int64_t(blockIdx.x) * a.n_chunks) * (2 * 16 * SCION_TDEC);
  for (int p = threadIdx.x; p < npairs; p += blockDim.x) {
    int nt = p >> 5, ln = p & 31;
    for (int m = 0; m < nacc; ++m)
      for (int i = 0; i < 4; ++i) {
        float v = red[0][m][nt][ln][i] + red[1][m][nt][ln][i] + red[2][m][nt][ln][i] + red[3][m][nt][ln][i];
        int row = (ln >> 2) + 8 * (i >> 1), tok = nt * 8 + 2 * (ln & 3) + (i & 1);
        red[0][m][nt][ln][i] = v;
        if (a.n_chunks > 1) part[(int64_t(chunk) * 2 + m) * 16 * SCION_TDEC + row * SCION_TDEC + tok] = v;
      }
  }
  if (a.n_chunks > 1) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned prev = atomicAdd(&a.count[blockIdx.x], 1u);
      last_flag = (prev == unsigned(a.n_chunks - 1));
    }
    __syncthreads();
    if (!last_flag) return;
    __threadfence();
  } else {
    __syncthreads();
  }

  // epilogue: thread -> (row, tok)
  const int nrows_u = 16;
  for (int p = threadIdx.x; p < nrows_u * a.T; p += blockDim.x) {
    int row = p / a.T, tok = p % a.T;
    int grow = u.row0 + row;
    if (grow >= nrows) continue;
    float v[2] = {0.f, 0.f};
    if (a.n_chunks > 1) {
      for (int ch = 0; ch < a.n_chunks; ++ch)
        for (int m = 0; m < nacc; ++m)
          v[m] += __ldcg(&part[(int64_t(ch) * 2 + m) * 16 * SCION_TDEC + row * SCION_TDEC + tok]);
    } else {
      int nt = tok >> 3, ln = (row & 7) * 4 + ((tok & 7) >> 1), i = (row >> 3) * 2 + (tok & 1);
      for (int m = 0; m < nacc; ++m) v[m] = red[0][m][nt][ln][i];
    }
    if (u.kind == kUnitRouter) {
      a.logits[int64_t(tok) * a.E + grow] = v[0];
    } else if (u.kind == kUnitSwiglu) {
      a.hz[int64_t(tok) * a.Kd + grow] = __float2half_rn(silu_f(v[0]) * v[1]);
    } else {
      a.hz[int64_t(tok) * a.Kd + a.Fs + grow] = __float2half_rn(v[0]);
    }
  }
  if (a.n_chunks > 1 && threadIdx.x == 0) a.count[blockIdx.x] = 0;
}

// ================================================================= ternary tiles
// Unpack one PQ2_0 code word into the A register pair for step s:
// ((w >> 2s) & 0x00030003) | (1024,1024) -> (1024+b) halves; minus 1025 -> b - 1.
__device__ __forceinline__ uint32_t pq2_pair(uint32_t w, int s) {
  __half2 v = u32_as_h2(lop3_and_or(w >> (2 * s), 0x00030003u, kMagic));
  return h2_as_u32(__hsub2(v, u32_as_h2(kPq2Bias)));
}

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

__device__ __forceinline__ int trit_of(int v, int digit) {
  for (int i = 0; i < digit; ++i) v /= 3;
  return v % 3;
}

// Remainder step of PTQ1_0: trits 120+2c and 121+2c of a row, from (q24, tail).
__device__ __forceinline__ uint32_t ptq1_rem_pair(uint32_t q24, uint32_t tail, int c) {
  int rlo = 2 * c, rhi = 2 * c + 1;
  int tlo = rlo < 5 ? trit_of(int(q24), rlo) : trit_of(int(tail), rlo - 5);
  int thi = rhi < 5 ? trit_of(int(q24), rhi) : trit_of(int(tail), rhi - 5);
  return h2_as_u32(__halves2half2(__int2half_rn(tlo - 1), __int2half_rn(thi - 1)));
}

// Accumulate one 16-row x 128-column ternary tile against NT token tiles.
// acc[nt] += scale_row * (codes . B).  `blk` = sub-tile block; `bfr` = B fragments
// (16 u32 per token tile: the lane's 64 bytes of the group).
template <int FMT, int NT>
__device__ __forceinline__ void tile_mma(const uint8_t* blk, const uint4 (&bfr)[NT][4], float (&acc)[NT][4],
                                         int lane) {
  const int r8 = lane >> 2, c = lane & 3;
  float g[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) g[nt][i] = 0.f;
  uint32_t sc;
  if constexpr (FMT == SCION_PQ2_0) {
    const uint4 w = ldg_stream(blk + 16 * lane);
    sc = ldg_stream32(blk + 512 + 4 * r8);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      uint32_t fa[4] = {pq2_pair(w.x, s), pq2_pair(w.z, s), pq2_pair(w.y, s), pq2_pair(w.w, s)};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t* b = reinterpret_cast<const uint32_t*>(&bfr[nt][0]);
        mma_f16_16816(g[nt], fa, b[2 * s], b[2 * s + 1]);
      }
    }
  } else {
    const uint32_t q0 = ldg_stream32(blk + 12 * lane), q1 = ldg_stream32(blk + 12 * lane + 4),
                   q2 = ldg_stream32(blk + 12 * lane + 8);
    const uint32_t rem = ldg_stream32(blk + 384 + 4 * r8);
    sc = ldg_stream32(blk + 416 + 4 * r8);
    // row r quintets: q0.b0..b3, q1.b0, q1.b1;  row r+8: q1.b2, q1.b3, q2.b0..b3
    // pair m = (Q[m], Q[m+3]); selector nibble order: byte0 <- idx0, byte2 <- idx2
    const uint32_t sel_r[3] = {0x0300u, 0x0401u, 0x0502u};  // from (q0, q1)
    const uint32_t sel_h[3] = {0x0502u, 0x0603u, 0x0704u};  // from (q1, q2)
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      Ptq1Digits dr{ptq1_v0(q0, q1, sel_r[m])}, dh{ptq1_v0(q1, q2, sel_h[m])};
#pragma unroll
      for (int j = 0; j < 5; ++j) {
        const int s = 5 * m + j;
        uint32_t a0 = dr.next(), a1 = dh.next();
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint32_t* b = reinterpret_cast<const uint32_t*>(&bfr[nt][0]);
          mma_f16_1688(g[nt], a0, a1, b[s]);
        }
      }
    }
    uint32_t a0 = ptq1_rem_pair(rem & 0xff, (rem >> 8) & 0xff, c);
    uint32_t a1 = ptq1_rem_pair((rem >> 16) & 0xff, rem >> 24, c);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t* b = reinterpret_cast<const uint32_t*>(&bfr[nt][0]);
      mma_f16_1688(g[nt], a0, a1, b[15]);
    }
  }
  const float s_lo = __half2float(__ushort_as_half(uint16_t(sc & 0xffff)));
  const float s_hi = __half2float(__ushort_as_half(uint16_t(sc >> 16)));
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    acc[nt][0] = fmaf(s_lo, g[nt][0], acc[nt][0]);
    acc[nt][1] = fmaf(s_lo, g[nt][1], acc[nt][1]);
    acc[nt][2] = fmaf(s_hi, g[nt][2], acc[nt][2]);
    acc[nt][3] = fmaf(s_hi, g[nt][3], acc[nt][3]);
  }
}

// B fragments of one group for NT token tiles: lane (n, c) reads 64 contiguous bytes of
// token n's group (fragment order) or zeros past the last token.
template <int NT>
__device__ __forceinline__ void load_bfrag(const __half* base, int64_t tok_stride_h, const int (&tok)[NT], int G,
                                           int g, int lane, uint4 (&bfr)[NT][4]) {
  const int c = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    if (tok[nt] >= 0) {
      const uint4* p = reinterpret_cast<const uint4*>(base + int64_t(tok[nt]) * tok_stride_h + int64_t(g) * 128 + 32 * c);
#pragma unroll
      for (int i = 0; i < 4; ++i) bfr[nt][i] = p[i];
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) bfr[nt][i] = make_uint4(0, 0, 0, 0);
    }
  }
}

// ======================================================================= gate/up
struct GateUpArgs {
  const uint8_t* bank;  // gate/up bank
  const __half* xfrag;  // [T][Gd][128]
  const int32_t *active, *n_active, *counts, *offsets, *perm;
  int d, F, k, Gd, fmt;
  __half* hfrag;  // [T*k][GF][128] fragment order of the down format
};

constexpr int kGuWarps = 8;
constexpr int kGuNT = 2;

template <int FMT>
__global__ void __launch_bounds__(kGuWarps * 32) gateup_kernel(GateUpArgs a) {
  __shared__ float red[kGuWarps][2][kGuNT][32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = blockIdx.y;
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  const int p0 = a.offsets[e], ne = a.counts[e];
  const int ft = blockIdx.x, rt = ft >> 3, sub = ft & 7;
  const int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  const uint8_t* tile0 = a.bank + (int64_t(e) * (a.F >> 7) + rt) * a.Gd * 2 * 8 * tb + int64_t(sub) * tb;
  const int GF = a.F >> 7;

  for (int pc = 0; pc < ne; pc += 8 * kGuNT) {
    const int nn = min(8 * kGuNT, ne - pc);
    int tok[kGuNT];
#pragma unroll
    for (int nt = 0; nt < kGuNT; ++nt) {
      int i = nt * 8 + (lane >> 2);
      tok[nt] = i < nn ? a.perm[p0 + pc + i] / a.k : -1;
    }
    float accg[kGuNT][4], accu[kGuNT][4];
#pragma unroll
    for (int nt = 0; nt < kGuNT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) accg[nt][i] = accu[nt][i] = 0.f;
    for (int g = warp; g < a.Gd; g += kGuWarps) {
      uint4 bfr[kGuNT][4];
      load_bfrag<kGuNT>(a.xfrag, int64_t(a.Gd) * 128, tok, a.Gd, g, lane, bfr);
      const uint8_t* blk = tile0 + int64_t(g) * 2 * 8 * tb;
      if (nn > 8) {
        tile_mma<FMT, kGuNT>(blk, bfr, accg, lane);
        tile_mma<FMT, kGuNT>(blk + 8 * tb, bfr, accu, lane);
      } else {
        tile_mma<FMT, 1>(blk, reinterpret_cast<uint4(&)[1][4]>(bfr), reinterpret_cast<float(&)[1][4]>(accg), lane);
        tile_mma<FMT, 1>(blk + 8 * tb, reinterpret_cast<uint4(&)[1][4]>(bfr), reinterpret_cast<float(&)[1][4]>(accu),
                         lane);
      }
    }
#pragma unroll
    for (int nt = 0; nt < kGuNT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        red[warp][0][nt][lane][i] = accg[nt][i];
        red[warp][1][nt][lane][i] = accu[nt][i];
      }
    __syncthreads();
    // thread -> (nt, lane, i) : kGuNT*32*4 = 256 outputs
    {
      const int idx = threadIdx.x;
      const int nt = idx >> 7, ln = (idx >> 2) & 31, i = idx & 3;
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int w = 0; w < kGuWarps; ++w) {
        gs += red[w][0][nt][ln][i];
        us += red[w][1][nt][ln][i];
      }
      const int row = (ln >> 2) + 8 * (i >> 1), tcol = nt * 8 + 2 * (ln & 3) + (i & 1);
      if (tcol < nn) {
        const int f = ft * 16 + row;
        const int64_t p = p0 + pc + tcol;
        a.hfrag[(p * GF + (f >> 7)) * 128 + frag_index(a.fmt, f & 127)] = __float2half_rn(silu_f(gs) * us);
      }
    }
    __syncthreads();
  }
}

// ======================================================================== down
struct DownArgs {
  const uint8_t* bank;  // down bank
  const __half* hfrag;  // [T*k][GF][128]
  const int32_t *active, *n_active, *counts, *offsets, *perm;
  const float* gates;
  int d, F, k, GF;
  float* out;
};

constexpr int kDnWarps = 4;
constexpr int kDnNT = 2;

template <int FMT>
__global__ void __launch_bounds__(kDnWarps * 32) down_routed_kernel(DownArgs a) {
  __shared__ float red[kDnWarps][kDnNT][32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = blockIdx.y;
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  const int p0 = a.offsets[e], ne = a.counts[e];
  const int dt = blockIdx.x, rt = dt >> 3, sub = dt & 7;
  const int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  const uint8_t* tile0 = a.bank + (int64_t(e) * (a.d >> 7) + rt) * a.GF * 8 * tb + int64_t(sub) * tb;

  for (int pc = 0; pc < ne; pc += 8 * kDnNT) {
    const int nn = min(8 * kDnNT, ne - pc);
    int pos[kDnNT];
#pragma unroll
    for (int nt = 0; nt < kDnNT; ++nt) {
      int i = nt * 8 + (lane >> 2);
      pos[nt] = i < nn ? p0 + pc + i : -1;
    }
    float acc[kDnNT][4];
#pragma unroll
    for (int nt = 0; nt < kDnNT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    for (int g = warp; g < a.GF; g += kDnWarps) {
      uint4 bfr[kDnNT][4];
      load_bfrag<kDnNT>(a.hfrag, int64_t(a.GF) * 128, pos, a.GF, g, lane, bfr);
      const uint8_t* blk = tile0 + int64_t(g) * 8 * tb;
      if (nn > 8)
        tile_mma<FMT, kDnNT>(blk, bfr, acc, lane);
      else
        tile_mma<FMT, 1>(blk, reinterpret_cast<uint4(&)[1][4]>(bfr), reinterpret_cast<float(&)[1][4]>(acc), lane);
    }
#pragma unroll
    for (int nt = 0; nt < kDnNT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][nt][lane][i] = acc[nt][i];
    __syncthreads();
    for (int idx = threadIdx.x; idx < kDnNT * 32 * 4; idx += blockDim.x) {
      const int nt = idx >> 7, ln = (idx >> 2) & 31, i = idx & 3;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kDnWarps; ++w) v += red[w][nt][ln][i];
      const int row = (ln >> 2) + 8 * (i >> 1), tcol = nt * 8 + 2 * (ln & 3) + (i & 1);
      if (tcol < nn) {
        const int entry = a.perm[p0 + pc + tcol];
        const int t = entry / a.k;
        atomicAdd(&a.out[int64_t(t) * a.d + dt * 16 + row], a.gates[entry] * v);
      }
    }
    __syncthreads();
  }
}

// [sh_down | corr_b] (fp16 [d][Kd]) x hz ([T][Kd] fp16, natural order) -> out += .
// One CTA per 16 output rows; 8 warps split K in 32-column chunks.
struct DenseArgs {
  const __half* w;  // [d][Kd]
  const __half* hz; // [T][Kd]
  int d, Kd, T;
  float* out;
};

template <int NT>
__global__ void __launch_bounds__(256) down_dense_kernel(DenseArgs a) {
  __shared__ float red[8][NT][32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g8 = lane >> 2, c = lane & 3;
  const int row0 = blockIdx.x * 16;
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
  for (int kc = warp * 32; kc < a.Kd; kc += 8 * 32) {
    const uint4 wa = ldg_stream(a.w + int64_t(row0 + g8) * a.Kd + kc + 8 * c);
    const uint4 wb = ldg_stream(a.w + int64_t(row0 + g8 + 8) * a.Kd + kc + 8 * c);
    uint32_t fa0[4] = {wa.x, wb.x, wa.y, wb.y};
    uint32_t fa1[4] = {wa.z, wb.z, wa.w, wb.w};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int tok = nt * 8 + g8;
      uint4 xb = tok < a.T ? *reinterpret_cast<const uint4*>(a.hz + int64_t(tok) * a.Kd + kc + 8 * c)
                           : make_uint4(0, 0, 0, 0);
      mma_f16_16816(acc[nt], fa0, xb.x, xb.y);
      mma_f16_16816(acc[nt], fa1, xb.z, xb.w);
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][nt][lane][i] = acc[nt][i];
  __syncthreads();
  for (int idx = threadIdx.x; idx < NT * 128; idx += blockDim.x) {
    const int nt = idx >> 7, ln = (idx >> 2) & 31, i = idx & 3;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[w][nt][ln][i];
    const int row = (ln >> 2) + 8 * (i >> 1), tok = nt * 8 + 2 * (ln & 3) + (i & 1);
    if (tok < a.T) atomicAdd(&a.out[int64_t(tok) * a.d + row0 + row], v);
  }
}

__global__ void unfrag_kernel(int fmt, const __half* __restrict__ src, int64_t n, __half* __restrict__ dst) {
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int64_t grp = i >> 7;
  int col = int(i & 127);
  dst[grp * 128 + col] = src[grp * 128 + frag_index(fmt, col)];
}

}  // namespace

// ------------------------------------------------------------------- launchers
cudaError_t launch_xproj(const scion_layer* L, const __nv_bfloat16* x, int T, float* out, cudaStream_t s) {
  XProjArgs a;
  a.x = x;
  a.T = T, a.d = L->d, a.E = L->E, a.Fs = L->Fs, a.r = L->r, a.Kd = L->Kd, a.fmt = L->fmt;
  a.w_router = static_cast<const __nv_bfloat16*>(L->desc.w_router);
  a.w_delta = static_cast<const __nv_bfloat16*>(L->desc.w_router_delta);
  a.sh_gate = static_cast<const __nv_bfloat16*>(L->desc.sh_gate);
  a.sh_up = static_cast<const __nv_bfloat16*>(L->desc.sh_up);
  a.corr_a = static_cast<const __nv_bfloat16*>(L->desc.corr_a);
  a.units = L->xunits, a.n_units = L->n_xunits, a.n_chunks = L->n_xchunks;
  a.partial = L->xpartial, a.count = L->xcount, a.logits = L->logits, a.hz = L->hz, a.xfrag = L->xfrag, a.out = out;
  dim3 grid(L->n_xunits + 1, L->n_xchunks);
  const int nt = (T + 7) / 8;
  switch (nt) {
    case 1: xproj_kernel<1><<<grid, 128, 0, s>>>(a); break;
    case 2: xproj_kernel<2><<<grid, 128, 0, s>>>(a); break;
    case 3: case 4: xproj_kernel<4><<<grid, 128, 0, s>>>(a); break;
    default: xproj_kernel<8><<<grid, 128, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_gateup(const scion_layer* L, const __nv_bfloat16* /*x*/, int T, cudaStream_t s) {
  GateUpArgs a;
  a.bank = L->gu_bank, a.xfrag = L->xfrag;
  a.active = L->active, a.n_active = L->n_active, a.counts = L->counts, a.offsets = L->offsets, a.perm = L->perm;
  a.d = L->d, a.F = L->F, a.k = L->k, a.Gd = L->Gd, a.fmt = L->fmt;
  a.hfrag = L->h;
  const int slots = min(L->E, T * L->k);
  dim3 grid(L->F / 16, slots);
  if (L->fmt == SCION_PQ2_0)
    gateup_kernel<SCION_PQ2_0><<<grid, kGuWarps * 32, 0, s>>>(a);
  else
    gateup_kernel<SCION_PTQ1_0><<<grid, kGuWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_down_routed(const scion_layer* L, int T, float* out, cudaStream_t s) {
  DownArgs a;
  a.bank = L->dn_bank, a.hfrag = L->h;
  a.active = L->active, a.n_active = L->n_active, a.counts = L->counts, a.offsets = L->offsets, a.perm = L->perm;
  a.gates = L->gates;
  a.d = L->d, a.F = L->F, a.k = L->k, a.GF = L->GF, a.out = out;
  const int slots = min(L->E, T * L->k);
  dim3 grid(L->d / 16, slots);
  if (L->fmt == SCION_PQ2_0)
    down_routed_kernel<SCION_PQ2_0><<<grid, kDnWarps * 32, 0, s>>>(a);
  else
    down_routed_kernel<SCION_PTQ1_0><<<grid, kDnWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_down_dense(const scion_layer* L, int T, float* out, cudaStream_t s) {
  if (L->Kdense == 0) return cudaSuccess;
  DenseArgs b;
  b.w = L->dense_down, b.hz = L->hz, b.d = L->d, b.Kd = L->Kd, b.T = T, b.out = out;
  const int nt = (T + 7) / 8;
  dim3 g2(L->d / 16);
  switch (nt) {
    case 1: down_dense_kernel<1><<<g2, 256, 0, s>>>(b); break;
    case 2: down_dense_kernel<2><<<g2, 256, 0, s>>>(b); break;
    case 3: case 4: down_dense_kernel<4><<<g2, 256, 0, s>>>(b); break;
    default: down_dense_kernel<8><<<g2, 256, 0, s>>>(b); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_unfrag(int fmt, const __half* src, int rows, int G, __half* dst, cudaStream_t s) {
  int64_t n = int64_t(rows) * G * 128;
  if (n == 0) return cudaSuccess;
  unfrag_kernel<<<unsigned((n + 255) / 256), 256, 0, s>>>(fmt, src, n, dst);
  return cudaGetLastError();
}

cudaError_t configure_kernels() {
  cudaError_t e = configure_route_kernels();
  return e != cudaSuccess ? e : configure_prefill_kernels();
}

}  // namespace scion
