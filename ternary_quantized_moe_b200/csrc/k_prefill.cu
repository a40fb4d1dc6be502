// k_prefill.cu -- the large-batch (prefill) path on the 5th-generation tensor cores.
//
// Same block as the decode path ("Scion: ternary MoE quantization with trained
// corrections", The idea; "Scion-35B-A3B" / "Scion-FlashNext-176B-A6B" model cards,
// Model Overview and Weight Representation), organised as GEMMs with the weights as
// the 128-row A operand and tokens as N ("swap-AB", so an expert with n tokens costs
// N = round_up(n, 16) columns instead of a 128-row tile):
//
//   x16       x (bf16) -> fp16 in the container's column order (B operand of gate/up)
//   dense     tcgen05 GEMM with both operands loaded by TMA (128B swizzle):
//               x-projection  router + delta -> logits; shared gate/up -> SwiGLU; corr A -> z
//               dense down    [shared down | correction B] x [h_s | z] -> out (store)
//   route     top-k per token (warp per token), then one CTA groups the T*k entries by
//             expert (histogram, scan, stable scatter) and lists 128-token tiles
//   ternary   tcgen05 grouped GEMM over the routed tiles: packed code blocks arrive by
//             bulk copy, four warps expand them to fp16 (code * scale, exact) in the
//             swizzled layout, gathered token rows arrive by cp.async:
//               gate/up  -> SwiGLU -> h (fp16)
//               down     -> out += gate * y   (fp32 red.add)
//
// Column orders (the A expansion and the B rows must agree):
//   PQ2_0 : inside every 16 columns, position 2s+h holds column s + 8h (s < 8, h < 2)
//   PTQ1_0: inside every 128 columns, position 2q+h (q < 60) holds column 10(q/5) + 5h + q%5,
//           positions 120..127 hold columns 120..127.
#include <cudaTypedefs.h>
#include <float.h>
#include <math.h>

#include <string.h>

#include "tc_common.cuh"

namespace scion {

namespace {

using namespace tc;

constexpr int kBM = 128;  // weight rows per tile
constexpr int kBN = 128;  // tokens per tile
constexpr int kThreads = 256;

// ------------------------------------------------------------- column orders
__device__ __forceinline__ int perm_pos(int fmt, int col) {  // physical column -> position
  if (fmt == SCION_PQ2_0) {
    int c16 = col & 15;
    return (col & ~15) | (2 * (c16 & 7) + (c16 >> 3));
  }
  int g = col & ~127, k = col & 127;
  if (k >= 120) return col;
  int i = k / 10, r = k % 10;
  return g | (2 * (5 * i + r % 5) + r / 5);
}

__global__ void x16_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, int fmt, __half* __restrict__ xp) {
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  // n = T*d; columns are permuted within their own row (d % 128 == 0)
  int64_t base = i & ~int64_t(127);
  int col = int(i & 127);
  xp[base + perm_pos(fmt, col)] = __float2half_rn(__bfloat162float(x[i]));
}

// ---------------------------------------------------------------- dense GEMM
enum DenseEpi : int { kEpiLogits = 0, kEpiSwiglu = 1, kEpiPlain = 2, kEpiStore = 3 };

struct DenseUnit {
  int epi;     // DenseEpi
  int na;      // A matrices in this unit (1 or 2)
  int map1;    // accumulator of the second matrix (0 = same as the first)
  int mat0, mat1;  // indices into the A tensor-map table
  int row0;    // first weight row
  int nrows;   // valid rows of the matrices
  int col0;    // output column offset (hz column, logit column or out column)
};

struct DenseParams {
  CUtensorMap a[6];  // A matrices, box {64, 128}
  CUtensorMap b;     // B (tokens x K), box {64, 128}
  const DenseUnit* units;
  int K, T, ab_bf16;
  float* logits;  int ld_logits;
  __half* hz;     int ld_hz;
  float* out;     int ld_out;
  int* err;
};

constexpr int kDenseStages = 4;
constexpr int kBK = 64;

__global__ void __launch_bounds__(kThreads, 1) dense_gemm_kernel(const __grid_constant__ DenseParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kDenseStages], empty[kDenseStages], accf;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DenseUnit u = p.units[blockIdx.x];
  const int tok0 = blockIdx.y * kBN;
  const int na = u.na;
  const int nacc = (na == 2 && u.map1 == 1) ? 2 : 1;
  const uint32_t a_bytes = kBM * kBK * 2, b_bytes = kBN * kBK * 2;
  const uint32_t stage_bytes = 2 * a_bytes + b_bytes;
  const int nk = p.K / kBK;
  const uint32_t ncols = nacc == 2 ? 2 * kBN : kBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDenseStages; ++s) mbar_init(&full[s], 1), mbar_init(&empty[s], 1);
    mbar_init(&accf, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&tmem_slot, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kDenseStages;
      if (kb >= kDenseStages && !mbar_wait(&empty[s], ((kb / kDenseStages) - 1) & 1, &abort_flag, p.err)) break;
      uint8_t* st = smem + s * stage_bytes;
      mbar_arrive_expect_tx(&full[s], na * a_bytes + b_bytes);
      tma_load_2d(st, &p.a[u.mat0], kb * kBK, u.row0, &full[s]);
      if (na == 2) tma_load_2d(st + a_bytes, &p.a[u.mat1], kb * kBK, u.row0, &full[s]);
      tma_load_2d(st + 2 * a_bytes, &p.b, kb * kBK, tok0, &full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    const uint32_t idesc = umma_idesc(kBM, kBN, p.ab_bf16);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kDenseStages;
      if (!mbar_wait(&full[s], (kb / kDenseStages) & 1, &abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t st = smem_u32(smem + s * stage_bytes);
#pragma unroll
      for (int k16 = 0; k16 < kBK / 16; ++k16) {
        const uint64_t db = umma_desc_sw128(st + 2 * a_bytes + 32 * k16);
        const uint64_t da0 = umma_desc_sw128(st + 32 * k16);
        umma_f16(tmem, da0, db, idesc, (kb | k16) != 0);
        if (na == 2) {
          const uint64_t da1 = umma_desc_sw128(st + a_bytes + 32 * k16);
          const uint32_t acc = u.map1 ? tmem + kBN : tmem;
          umma_f16(acc, da1, db, idesc, u.map1 ? uint32_t((kb | k16) != 0) : 1u);
        }
      }
      umma_commit(&empty[s]);
    }
    umma_commit(&accf);
  } else if (warp >= 4) {
    // ---------------- epilogue: TMEM lanes 32q..32q+31 = weight rows
    const int q = warp - 4;
    if (mbar_wait(&accf, 0, &abort_flag, p.err) && !abort_flag) {
      tc_fence_after();
      const int row = q * 32 + lane;
      const int grow = u.row0 + row;
      const bool rok = grow < u.nrows;
      for (int c = 0; c < kBN / 16; ++c) {
        float v0[16], v1[16];
        const uint32_t ta = tmem + (uint32_t(q * 32) << 16) + c * 16;
        tmem_ld16(ta, v0);
        if (nacc == 2) tmem_ld16(ta + kBN, v1);
        if (!rok) continue;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = tok0 + c * 16 + i;
          if (t >= p.T) break;
          if (u.epi == kEpiLogits) {
            p.logits[int64_t(t) * p.ld_logits + u.col0 + grow] = v0[i];
          } else if (u.epi == kEpiSwiglu) {
            p.hz[int64_t(t) * p.ld_hz + u.col0 + grow] = __float2half_rn(silu_f(v0[i]) * v1[i]);
          } else if (u.epi == kEpiPlain) {
            p.hz[int64_t(t) * p.ld_hz + u.col0 + grow] = __float2half_rn(v0[i]);
          } else {
            p.out[int64_t(t) * p.ld_out + u.col0 + grow] = v0[i];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace
}  // namespace scion

namespace scion {
namespace {

// -------------------------------------------------------------- ternary GEMM
struct TernTile {
  int e;   // expert
  int c0;  // first token (within the expert's group) of this 128-token tile
};

struct TernParams {
  const uint8_t* bank;  // re-tiled gate/up bank (na = 2) or down bank (na = 1)
  int fmt, na, G, R;    // groups along K, rows per expert matrix
  const __half* bsrc;   // B rows: x16 [T][d] (gate/up) or h [T*k][F] (down)
  int ldb;
  const TernTile* tiles;
  const int32_t* n_tiles;
  const int32_t *counts, *offsets, *perm;
  const float* gates;
  int k;
  __half* h;  int F;     // gate/up output
  float* out; int d;     // down output
  int* err;
};

constexpr int kTernStages = 2;
constexpr uint32_t kAtom = 128 * 128;  // bytes of one 128-row x 64-column swizzled atom

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Expand row t (0..127) of one 128-row x 128-column group from its PQ2_0 sub-tile block
// into the swizzled fp16 A tile (2 atoms).  Values are code * scale, exact in fp16.
__device__ __forceinline__ void expand_pq2_row(const uint8_t* codes, int t, uint32_t a_tile) {
  const uint8_t* blk = codes + (t >> 4) * kPq2Tile;
  const int rho = t & 15, r8 = rho & 7, hi = rho >> 3;
  const __half2 sc = __half2half2(__ushort_as_half(*reinterpret_cast<const uint16_t*>(blk + 512 + 4 * r8 + 2 * hi)));
  const __half2 bias = u32_as_h2(0x64016401u);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint2 w2 = *reinterpret_cast<const uint2*>(blk + 16 * (4 * r8 + c) + 8 * hi);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t w = half ? w2.y : w2.x;
      const int m = 2 * c + half;  // container word: columns 16m .. 16m+15
      uint32_t v[8];
#pragma unroll
      for (int s = 0; s < 8; ++s)
        v[s] = h2_as_u32(__hmul2(__hsub2(u32_as_h2(lop3_and_or(w >> (2 * s), 0x00030003u, 0x64006400u)), bias), sc));
      const int j0 = 2 * m;  // 16-byte chunk index along the 128 columns
      st_shared_v4(a_tile + (j0 >> 3) * kAtom + sw128_offset(t, j0 & 7), v[0], v[1], v[2], v[3]);
      st_shared_v4(a_tile + ((j0 + 1) >> 3) * kAtom + sw128_offset(t, (j0 + 1) & 7), v[4], v[5], v[6], v[7]);
    }
  }
}

__device__ __forceinline__ int trit_at(int v, int digit) {
  for (int i = 0; i < digit; ++i) v /= 3;
  return v % 3;
}

// Same for PTQ1_0: quintet pairs (2i, 2i+1) give positions 10i + j | 10i + 5 + j through
// the exact fp16 base-3 digit recurrence; columns 120..127 come from byte 24 and the tail.
__device__ __forceinline__ void expand_ptq1_row(const uint8_t* codes, int t, uint32_t a_tile) {
  const uint8_t* blk = codes + (t >> 4) * kPtq1Tile;
  const int rho = t & 15, r8 = rho & 7, hi = rho >> 3;
  const __half2 sc = __half2half2(__ushort_as_half(*reinterpret_cast<const uint16_t*>(blk + 416 + 4 * r8 + 2 * hi)));
  const __half2 third = __float2half2_rn(0.333251953125f), c1 = __float2half2_rn(682.5f);
  const __half2 m3 = __float2half2_rn(-3.0f), c2047 = __float2half2_rn(2047.0f);
  uint32_t v[64];
#pragma unroll
  for (int i = 0; i < 12; ++i) {
    const int q = 2 * i;
    const uint32_t x = *reinterpret_cast<const uint16_t*>(blk + 12 * (4 * r8 + q / 6) + 6 * hi + q % 6);
    uint32_t pr;
    asm("prmt.b32 %0, %1, 0, 0x4140;" : "=r"(pr) : "r"(x));
    __half2 V = u32_as_h2(pr | 0x64006400u);
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      __half2 Vn = __hfma2(V, third, c1);
      __half2 code = __hadd2(__hfma2(Vn, m3, V), c2047);
      V = Vn;
      v[5 * i + j] = h2_as_u32(__hmul2(code, sc));
    }
  }
  const int q24 = blk[384 + 4 * r8 + 2 * hi], tail = blk[384 + 4 * r8 + 2 * hi + 1];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int k0 = 2 * m, k1 = 2 * m + 1;  // columns 120 + k
    const int t0 = k0 < 5 ? trit_at(q24, k0) : trit_at(tail, k0 - 5);
    const int t1 = k1 < 5 ? trit_at(q24, k1) : trit_at(tail, k1 - 5);
    v[60 + m] = h2_as_u32(__hmul2(__halves2half2(__int2half_rn(t0 - 1), __int2half_rn(t1 - 1)), sc));
  }
#pragma unroll
  for (int j = 0; j < 16; ++j)
    st_shared_v4(a_tile + (j >> 3) * kAtom + sw128_offset(t, j & 7), v[4 * j], v[4 * j + 1], v[4 * j + 2],
                 v[4 * j + 3]);
}

template <int FMT, int NA>
__global__ void __launch_bounds__(kThreads, 1) tern_gemm_kernel(const __grid_constant__ TernParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t codes_full[kTernStages], b_full[kTernStages], a_full[kTernStages], empty[kTernStages], accf;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  if (int(blockIdx.x) >= *p.n_tiles) return;
  const TernTile tile = p.tiles[blockIdx.x];
  const int rt = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p0 = p.offsets[tile.e];
  const int nn = min(kBN, p.counts[tile.e] - tile.c0);
  const int nmma = (nn + 15) & ~15;
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  constexpr uint32_t a_bytes = 2 * kAtom, b_bytes = 2 * kAtom, c_bytes = 8 * tb;
  constexpr uint32_t stage_bytes = (NA * a_bytes + b_bytes + NA * c_bytes + 1023) & ~1023u;  // atoms 1024-aligned
  constexpr uint32_t ncols = NA * kBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTernStages; ++s) {
      mbar_init(&codes_full[s], 1);
      mbar_init(&b_full[s], 32);
      mbar_init(&a_full[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&accf, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&tmem_slot, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // ---------------- producer: packed code blocks (bulk copy) + gathered B rows (cp.async)
    const __half* rows[kBN / 32];
#pragma unroll
    for (int i = 0; i < kBN / 32; ++i) {
      const int r = lane + 32 * i;
      rows[i] = nullptr;
      if (r < nn) {
        const int64_t src = NA == 2 ? int64_t(p.perm[p0 + tile.c0 + r] / p.k) : int64_t(p0 + tile.c0 + r);
        rows[i] = p.bsrc + src * p.ldb;
      }
    }
    const int64_t mat_stride = int64_t(8) * tb;
    const int64_t grp_stride = NA * mat_stride;
    const uint8_t* ebase = p.bank + (int64_t(tile.e) * (p.R >> 7) + rt) * p.G * grp_stride;
    for (int kb = 0; kb < p.G; ++kb) {
      const int s = kb % kTernStages;
      if (kb >= kTernStages && !mbar_wait(&empty[s], ((kb / kTernStages) - 1) & 1, &abort_flag, p.err)) break;
      uint8_t* st = smem + s * stage_bytes;
      if (lane == 0) {
        mbar_arrive_expect_tx(&codes_full[s], NA * c_bytes);
#pragma unroll
        for (int m = 0; m < NA; ++m)
          bulk_load(st + NA * a_bytes + b_bytes + m * c_bytes, ebase + kb * grp_stride + m * mat_stride, c_bytes,
                    &codes_full[s]);
      }
      const uint32_t bt = smem_u32(st + NA * a_bytes);
#pragma unroll
      for (int i = 0; i < kBN / 32; ++i) {
        const int r = lane + 32 * i;
        if (rows[i]) {
          const __half* src = rows[i] + kb * 128;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t dst = bt + (j >> 3) * kAtom + sw128_offset(r, j & 7);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src + 8 * j) : "memory");
          }
        }
      }
      cp_async_arrive_noinc(&b_full[s]);
    }
    cp_async_wait_all();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc = umma_idesc(kBM, nmma, 0);
      for (int kb = 0; kb < p.G; ++kb) {
        const int s = kb % kTernStages;
        const uint32_t par = (kb / kTernStages) & 1;
        if (!mbar_wait(&a_full[s], par, &abort_flag, p.err)) break;
        if (!mbar_wait(&b_full[s], par, &abort_flag, p.err)) break;
        tc_fence_after();
        fence_proxy_async();
        const uint32_t st = sbase + s * stage_bytes;
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16) {
          const uint32_t off = (k16 >> 2) * kAtom + 32 * (k16 & 3);
          const uint64_t db = umma_desc_sw128(st + NA * a_bytes + off);
#pragma unroll
          for (int m = 0; m < NA; ++m)
            umma_f16(tmem + m * kBN, umma_desc_sw128(st + m * a_bytes + off), db, idesc, (kb | k16) != 0);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(&accf);
    }
  } else if (warp >= 4) {
    // ---------------- expansion (one weight row per thread), then the epilogue
    const int t = threadIdx.x - 128;
    for (int kb = 0; kb < p.G; ++kb) {
      const int s = kb % kTernStages;
      if (!mbar_wait(&codes_full[s], (kb / kTernStages) & 1, &abort_flag, p.err)) break;
      const uint8_t* st = smem + s * stage_bytes;
#pragma unroll
      for (int m = 0; m < NA; ++m) {
        const uint8_t* codes = st + NA * a_bytes + b_bytes + m * c_bytes;
        const uint32_t at = sbase + s * stage_bytes + m * a_bytes;
        if constexpr (FMT == SCION_PQ2_0)
          expand_pq2_row(codes, t, at);
        else
          expand_ptq1_row(codes, t, at);
      }
      fence_proxy_async();
      mbar_arrive(&a_full[s]);
    }
    const int q = warp - 4;
    if (mbar_wait(&accf, 0, &abort_flag, p.err) && !abort_flag) {
      tc_fence_after();
      const int row = q * 32 + lane;
      const int grow = rt * kBM + row;
      for (int c = 0; c * 16 < nn; ++c) {
        float v0[16], v1[16];
        const uint32_t ta = tmem + (uint32_t(q * 32) << 16) + c * 16;
        tmem_ld16(ta, v0);
        if (NA == 2) tmem_ld16(ta + kBN, v1);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int n = c * 16 + i;
          if (n >= nn) break;
          const int pos = p0 + tile.c0 + n;
          if constexpr (NA == 2) {
            p.h[int64_t(pos) * p.F + perm_pos(FMT, grow)] = __float2half_rn(silu_f(v0[i]) * v1[i]);
          } else {
            const int entry = p.perm[pos];
            atomicAdd(&p.out[int64_t(entry / p.k) * p.d + grow], p.gates[entry] * v0[i]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// ------------------------------------------------------------------- routing
__device__ __forceinline__ void argmax_merge2(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) v = v2, i = i2;
}

// One warp per token: top-k (ties -> lower id), gates.  smem: vals[8][E].
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                   int norm_topk, int32_t* __restrict__ ids, float* __restrict__ gates) {
  extern __shared__ float vals_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  float* vals = vals_all + warp * E;
  const float* row = logits + int64_t(t) * E;
  float mx = -INFINITY;
  for (int e = lane; e < E; e += 32) {
    float v = row[e];
    if (!(v >= -FLT_MAX)) v = -FLT_MAX;
    vals[e] = v;
    mx = fmaxf(mx, v);
  }
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float zall = 0.f;
  if (!norm_topk) {
    for (int e = lane; e < E; e += 32) zall += expf(vals[e] - mx);
    for (int o = 16; o; o >>= 1) zall += __shfl_xor_sync(0xffffffffu, zall, o);
  }
  __syncwarp();
  float my_v = -INFINITY;
  int my_id = -1;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) argmax_merge2(bv, bi, vals[e], e);
    for (int o = 16; o; o >>= 1) {
      float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
      int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
      argmax_merge2(bv, bi, v2, i2);
    }
    if (lane == j) my_v = bv, my_id = bi;
    __syncwarp();
    if (lane == (bi & 31)) vals[bi] = -INFINITY;
    __syncwarp();
  }
  const float top = __shfl_sync(0xffffffffu, my_v, 0);
  float ex = 0.f;
  if (lane < k) ex = norm_topk ? expf(my_v - top) : expf(my_v - mx);
  float z = ex;
  for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (!norm_topk) z = zall;
  if (lane < k) {
    ids[int64_t(t) * k + lane] = my_id;
    gates[int64_t(t) * k + lane] = ex / z;
  }
}

constexpr int kGroupWarps = 16;

// One CTA: histogram per warp-range, scan, stable scatter, and the 128-token tile list.
// smem: hist[kGroupWarps][E] int32 | tot[E] | tscan[E]
__global__ void __launch_bounds__(kGroupWarps * 32) group_kernel(const int32_t* __restrict__ ids, int T, int E, int k,
                                                                 int32_t* __restrict__ counts,
                                                                 int32_t* __restrict__ offsets,
                                                                 int32_t* __restrict__ perm,
                                                                 TernTile* __restrict__ tiles,
                                                                 int32_t* __restrict__ n_tiles) {
  extern __shared__ int32_t gsm[];
  int32_t* hist = gsm;                  // [W][E]
  int32_t* tot = gsm + kGroupWarps * E; // [E]
  __shared__ int32_t wsum[kGroupWarps], wtile[kGroupWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nthr = blockDim.x;
  const int n = T * k;
  const int per = (n + kGroupWarps - 1) / kGroupWarps;
  const int i0 = min(n, warp * per), i1 = min(n, i0 + per);
  for (int i = threadIdx.x; i < kGroupWarps * E; i += nthr) hist[i] = 0;
  __syncthreads();
  for (int i = i0 + lane; i < i1; i += 32) atomicAdd(&hist[warp * E + ids[i]], 1);
  __syncthreads();
  // per expert: total, and per-warp exclusive prefix (in place)
  for (int e = threadIdx.x; e < E; e += nthr) {
    int run = 0;
    for (int w = 0; w < kGroupWarps; ++w) {
      int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    tot[e] = run;
    counts[e] = run;
  }
  __syncthreads();
  // exclusive scan of totals and of tile counts: each warp scans a contiguous slice
  const int eper = (E + kGroupWarps - 1) / kGroupWarps;
  const int e0 = min(E, warp * eper), e1 = min(E, e0 + eper);
  int ls = 0, lt = 0;
  for (int e = e0 + lane; e < e1; e += 32) ls += tot[e], lt += (tot[e] + kBN - 1) / kBN;
  for (int o = 16; o; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o), lt += __shfl_xor_sync(0xffffffffu, lt, o);
  if (lane == 0) wsum[warp] = ls, wtile[warp] = lt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0, b = 0;
    for (int w = 0; w < kGroupWarps; ++w) {
      int x = wsum[w], y = wtile[w];
      wsum[w] = a, wtile[w] = b;
      a += x, b += y;
    }
    offsets[E] = a;
    *n_tiles = b;
  }
  __syncthreads();
  if (lane == 0) {
    int run = wsum[warp], trun = wtile[warp];
    for (int e = e0; e < e1; ++e) {
      const int c = tot[e];
      offsets[e] = run;
      for (int c0 = 0; c0 < c; c0 += kBN) tiles[trun++] = TernTile{e, c0};
      tot[e] = run;  // becomes the expert's base offset
      run += c;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kGroupWarps * E; i += nthr) hist[i] += tot[i % E];
  __syncthreads();
  // stable scatter: warp w walks its range in order
  const unsigned ltm = (1u << lane) - 1u;
  int32_t* cur = hist + warp * E;
  for (int base = i0; base < i1; base += 32) {
    const int i = base + lane;
    const int e = i < i1 ? ids[i] : -1 - lane;
    const unsigned mask = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(mask & ltm);
    const int c = i < i1 ? cur[e] : 0;
    __syncwarp();
    if (i < i1) {
      perm[c + rank] = i;
      if (rank == 0) cur[e] = c + __popc(mask);
    }
    __syncwarp();
  }
}

}  // namespace
}  // namespace scion

// ====================================================================== host side
namespace scion {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

size_t tern_smem(int na, int fmt) {
  const size_t tb = fmt == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  const size_t stage = (size_t(na) * 2 * kAtom + 2 * kAtom + na * 8 * tb + 1023) & ~size_t(1023);
  return kTernStages * stage + 1024;
}
constexpr size_t kDenseSmem = kDenseStages * (2 * 128 * 64 * 2 + 128 * 64 * 2) + 1024;

}  // namespace

// K-major [rows][K] 2-byte matrix, box {64 columns, 128 rows}, 128-byte swizzle.
int make_tmap_2d(CUtensorMap* map, const void* ptr, int bf16, int64_t rows, int64_t K) {
  auto fn = encode_fn();
  if (!fn) return SCION_ECUDA;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (K * 2) % 16) return SCION_EINVAL;
  cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(K * 2)};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SCION_OK : SCION_ECUDA;
}

cudaError_t configure_prefill_kernels() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(dense_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kDenseSmem))))
    return e;
  if ((e = cudaFuncSetAttribute(tern_gemm_kernel<SCION_PQ2_0, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(tern_smem(2, SCION_PQ2_0)))))
    return e;
  if ((e = cudaFuncSetAttribute(tern_gemm_kernel<SCION_PQ2_0, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(tern_smem(1, SCION_PQ2_0)))))
    return e;
  if ((e = cudaFuncSetAttribute(tern_gemm_kernel<SCION_PTQ1_0, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(tern_smem(2, SCION_PTQ1_0)))))
    return e;
  if ((e = cudaFuncSetAttribute(tern_gemm_kernel<SCION_PTQ1_0, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(tern_smem(1, SCION_PTQ1_0)))))
    return e;
  if ((e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024))) return e;
  return cudaFuncSetAttribute(group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

__global__ void unperm_prefill_kernel(int fmt, const __half* __restrict__ src, int64_t n, __half* __restrict__ dst) {
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t base = i & ~int64_t(127);
  dst[i] = src[base + perm_pos(fmt, int(i & 127))];
}

cudaError_t launch_unperm_prefill(int fmt, const __half* src, int64_t n, __half* dst, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  unperm_prefill_kernel<<<unsigned((n + 255) / 256), 256, 0, s>>>(fmt, src, n, dst);
  return cudaGetLastError();
}

size_t prefill_unit_bytes() { return sizeof(DenseUnit); }
size_t prefill_tile_bytes() { return sizeof(TernTile); }

// Builds the dense unit tables (host) for the x-projection and the dense down GEMM.
void prefill_units(const scion_layer* L, void* xunits_host, int* n_x, void* dunits_host, int* n_d) {
  DenseUnit* xu = static_cast<DenseUnit*>(xunits_host);
  DenseUnit* du = static_cast<DenseUnit*>(dunits_host);
  int nx = 0, nd = 0;
  // A map table: 0 router, 1 delta, 2 sh_gate, 3 sh_up, 4 corr_a, 5 dense_down
  if (!L->desc.router_fp32)
    for (int r0 = 0; r0 < L->E; r0 += 128) xu[nx++] = DenseUnit{kEpiLogits, 2, 0, 0, 1, r0, L->E, 0};
  for (int r0 = 0; r0 < L->Fs; r0 += 128) xu[nx++] = DenseUnit{kEpiSwiglu, 2, 1, 2, 3, r0, L->Fs, 0};
  for (int r0 = 0; r0 < L->r; r0 += 128) xu[nx++] = DenseUnit{kEpiPlain, 1, 0, 4, 4, r0, L->r, L->Fs};
  if (L->Kdense)
    for (int r0 = 0; r0 < L->d; r0 += 128) du[nd++] = DenseUnit{kEpiStore, 1, 0, 5, 5, r0, L->d, 0};
  *n_x = nx;
  *n_d = nd;
}

int prefill_max_units(const scion_layer* L) { return (L->E + 127) / 128 + (L->Fs + 127) / 128 + (L->r + 127) / 128 + L->d / 128; }

cudaError_t launch_prefill_stage(int stage, const scion_layer* L, const __nv_bfloat16* x, int T, float* out,
                                 cudaStream_t s) {
  const PrefillState& P = *L->pre;
  switch (stage) {
    case SCION_STAGE_X16: {
      const int64_t n = int64_t(T) * L->d;
      x16_kernel<<<unsigned((n + 255) / 256), 256, 0, s>>>(x, n, L->fmt, P.x16);
      return cudaGetLastError();
    }
    case SCION_STAGE_XPROJ: {
      if (P.n_xunits == 0) return cudaSuccess;
      DenseParams dp;
      memcpy(dp.a, P.maps, sizeof(dp.a));
      if (make_tmap_2d(&dp.b, x, 1, T, L->d) != SCION_OK) return cudaErrorInvalidValue;
      dp.units = static_cast<const DenseUnit*>(P.xunits), dp.K = L->d, dp.T = T, dp.ab_bf16 = 1;
      dp.logits = P.logits, dp.ld_logits = L->E, dp.hz = P.hz, dp.ld_hz = L->Kd, dp.out = nullptr, dp.ld_out = 0;
      dp.err = L->err;
      dim3 grid(P.n_xunits, (T + kBN - 1) / kBN);
      dense_gemm_kernel<<<grid, kThreads, kDenseSmem, s>>>(dp);
      return cudaGetLastError();
    }
    case SCION_STAGE_ROUTE: {
      topk_kernel<<<(T + 7) / 8, 256, sizeof(float) * 8 * L->E, s>>>(P.logits, T, L->E, L->k, L->desc.norm_topk,
                                                                    P.ids, P.gates);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      const size_t gsm = sizeof(int32_t) * (size_t(kGroupWarps) * L->E + L->E);
      group_kernel<<<1, kGroupWarps * 32, gsm, s>>>(P.ids, T, L->E, L->k, P.counts, P.offsets, P.perm,
                                                   static_cast<TernTile*>(P.tiles), P.n_tiles);
      return cudaGetLastError();
    }
    case SCION_STAGE_GATEUP: {
      TernParams tp;
      tp.bank = L->gu_bank, tp.fmt = L->fmt, tp.na = 2, tp.G = L->Gd, tp.R = L->F;
      tp.bsrc = P.x16, tp.ldb = L->d;
      tp.tiles = static_cast<const TernTile*>(P.tiles), tp.n_tiles = P.n_tiles;
      tp.counts = P.counts, tp.offsets = P.offsets, tp.perm = P.perm, tp.gates = P.gates, tp.k = L->k;
      tp.h = P.h, tp.F = L->F, tp.out = nullptr, tp.d = L->d, tp.err = L->err;
      const int max_tiles = (T * L->k + kBN - 1) / kBN + L->E;
      dim3 grid(max_tiles, L->F / kBM);
      if (L->fmt == SCION_PQ2_0)
        tern_gemm_kernel<SCION_PQ2_0, 2><<<grid, kThreads, tern_smem(2, L->fmt), s>>>(tp);
      else
        tern_gemm_kernel<SCION_PTQ1_0, 2><<<grid, kThreads, tern_smem(2, L->fmt), s>>>(tp);
      return cudaGetLastError();
    }
    case SCION_STAGE_DOWN_DENSE: {
      if (P.n_dunits == 0) return cudaMemsetAsync(out, 0, sizeof(float) * size_t(T) * L->d, s);
      DenseParams dp;
      memcpy(dp.a, P.maps, sizeof(dp.a));
      dp.b = P.hz_map;
      dp.units = static_cast<const DenseUnit*>(P.dunits), dp.K = L->Kd, dp.T = T, dp.ab_bf16 = 0;
      dp.logits = nullptr, dp.ld_logits = 0, dp.hz = nullptr, dp.ld_hz = 0, dp.out = out, dp.ld_out = L->d;
      dp.err = L->err;
      dim3 grid(P.n_dunits, (T + kBN - 1) / kBN);
      dense_gemm_kernel<<<grid, kThreads, kDenseSmem, s>>>(dp);
      return cudaGetLastError();
    }
    case SCION_STAGE_DOWN_ROUTED: {
      TernParams tp;
      tp.bank = L->dn_bank, tp.fmt = L->fmt, tp.na = 1, tp.G = L->GF, tp.R = L->d;
      tp.bsrc = P.h, tp.ldb = L->F;
      tp.tiles = static_cast<const TernTile*>(P.tiles), tp.n_tiles = P.n_tiles;
      tp.counts = P.counts, tp.offsets = P.offsets, tp.perm = P.perm, tp.gates = P.gates, tp.k = L->k;
      tp.h = nullptr, tp.F = L->F, tp.out = out, tp.d = L->d, tp.err = L->err;
      const int max_tiles = (T * L->k + kBN - 1) / kBN + L->E;
      dim3 grid(max_tiles, L->d / kBM);
      if (L->fmt == SCION_PQ2_0)
        tern_gemm_kernel<SCION_PQ2_0, 1><<<grid, kThreads, tern_smem(1, L->fmt), s>>>(tp);
      else
        tern_gemm_kernel<SCION_PTQ1_0, 1><<<grid, kThreads, tern_smem(1, L->fmt), s>>>(tp);
      return cudaGetLastError();
    }
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace scion
