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
//   route     top-k per token (warp per token) with a histogram of the selections, one CTA
//             scans it and lists the token tiles (128 or 160 tokens), and each entry takes
//             its position inside its expert's segment
//   ternary   tcgen05 grouped GEMM over the routed tiles: packed code blocks arrive by
//             bulk copy, eight warps expand them to fp16 (code * scale, exact) straight into
//             tensor memory (the A operand), token rows arrive by cp.async (gathered x16 rows)
//             or TMA (h, already in routed order):
//               gate/up  -> SwiGLU -> h (fp16)
//               down     -> y (fp16, one row per routed entry)
//   combine   out = base + the gate-weighted sum of each token's k rows of y
//
// Column orders (the A expansion and the B rows must agree):
//   PQ2_0 : inside every 16 columns, position 2s+h holds column s + 8h (s < 8, h < 2)
//   PTQ1_0: each 64-column half of a 128-column group is self-contained: quintets 12h..12h+11
//           in pairs, then remainder trits 4h..4h+3 (see perm_pos).
#include <cudaTypedefs.h>
#include <float.h>
#include <math.h>

#include <string.h>

#include <vector>

#include "tc_common.cuh"
#include "tc_order.cuh"
#include "topk_warp.cuh"

namespace scion {

namespace {

using namespace tc;

constexpr int kBM = 128;  // weight rows per tile
constexpr int kBN = 128;  // tokens per tile
constexpr int kThreads = 384;   // dense GEMM: TMA warp, MMA warp, 2 idle, 8 epilogue warps
constexpr int kDenseEpi = 256;  // epilogue threads (two warps per TMEM lane quarter)

// x (bf16) -> fp16 x 2^s_t in the container's column order (PQ2_0: times the factor of its
// position), s_t the token's range exponent (token_shift of its largest magnitude, written to
// xexp).  One warp per token: the whole row's coalesced 16-byte loads are issued first (pairs of
// 128-column groups, 16 bytes per lane), their maximum fixes s_t, then each pair goes through
// shared memory, where each lane gathers the columns of its 8 output positions and stores 16
// bytes.  d <= 4096 (16 pairs).
constexpr int kXPairs = 16;
__device__ __forceinline__ uint32_t max_mag8(uint4 v) {
  const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu), __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}
// init_out: also set out[t] = resid[t] (or zero) -- for layers without shared expert and
// correction, whose routed down projection only adds into out.
template <int FMT>
__global__ void __launch_bounds__(256) x16_kernel(const __nv_bfloat16* __restrict__ x, int T, int d,
                                                  __half* __restrict__ xp, int32_t* __restrict__ xexp,
                                                  int init_out, const float* resid, float* out) {
  __shared__ __align__(16) __nv_bfloat16 buf[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gl = lane >> 4, p0 = 8 * (lane & 15);  // group of the pair, first output position
  const int G = d >> 7, n_pairs = (G + 1) / 2;
  for (int t = blockIdx.x * 8 + warp; t < T; t += gridDim.x * 8) {
    const __nv_bfloat16* row = x + int64_t(t) * d;
    uint4 v[kXPairs];
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < kXPairs; ++i) {
      // past the last group (an odd group count leaves the last pair half empty) nothing moves
      const bool ok = i < n_pairs && 2 * i + gl < G;
      v[i] = ok ? __ldg(reinterpret_cast<const uint4*>(row + i * 256) + lane) : make_uint4(0u, 0u, 0u, 0u);
      mx = max(mx, max_mag8(v[i]));
    }
    const int sh = token_shift(__reduce_max_sync(0xffffffffu, mx));
    if (lane == 0) xexp[t] = sh;
    const float xs = pow2i(sh);
    __half* orow = xp + int64_t(t) * d;
#pragma unroll
    for (int i = 0; i < kXPairs; ++i) {
      if (i >= n_pairs) break;
      __syncwarp();
      *reinterpret_cast<uint4*>(&buf[warp][8 * lane]) = v[i];
      __syncwarp();
      __align__(16) __half o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int p = p0 + e;
        const float f = __bfloat162float(buf[warp][128 * gl + pos_col(FMT, p)]) * xs;
        o[e] = __float2half_rn(f);
      }
      if (2 * i + gl < G) reinterpret_cast<uint4*>(orow + i * 256)[lane] = *reinterpret_cast<const uint4*>(o);
    }
    if (init_out && resid != out) {
      float4* o4 = reinterpret_cast<float4*>(out + int64_t(t) * d);
      const float4* r4 = reinterpret_cast<const float4*>(resid + int64_t(t) * d);
      for (int j = lane; j < d / 4; j += 32) o4[j] = resid ? r4[j] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// Ternary correction factors (PQ2_0 blocks [rows][K/128], 2-bit codes + fp16 scale) -> fp16
// code * scale, exact.  order < 0: natural column order; otherwise the column order of the
// layer's x16 operand for expert format `order`, so that a GEMM against x16 computes A x.  dst == nullptr only counts.  Invalid codes (3)
// and values past the fp16 range are counted into *bad.
__global__ void dequant_corr_kernel(const uint8_t* __restrict__ blocks, int rows, int K, __half* __restrict__ dst,
                                    int ld, int order, unsigned long long* __restrict__ bad) {
  const int64_t n = int64_t(rows) * K;
  unsigned nbad = 0;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int row = int(i / K), col = int(i % K), j = col & 127;
    const uint8_t* blk = blocks + (int64_t(row) * (K >> 7) + (col >> 7)) * 34;
    const int field = (blk[j >> 2] >> (2 * (j & 3))) & 3;
    const float sc = __half2float(__ushort_as_half(uint16_t(blk[32] | (blk[33] << 8))));
    float v = field == 3 ? 0.f : float(field - 1) * sc;
    nbad += field == 3;
    const int pos = order >= 0 ? perm_pos(order, col) : col;
    const __half hv = __float2half_rn(v);
    nbad += __hisinf(hv) != 0;
    if (dst) dst[int64_t(row) * ld + pos] = hv;
  }
  if (nbad) atomicAdd(bad, (unsigned long long)nbad);
}

// ---------------------------------------------------------------- dense GEMM
enum DenseEpi : int { kEpiLogits = 0, kEpiSwiglu = 1, kEpiPlain = 2, kEpiStore = 3 };

struct DenseUnit {
  int epi;     // DenseEpi
  int na;      // A matrices in this unit (1 or 2); units with 2 run 128-token tiles, the others 256
  int map1;    // accumulator of the second matrix (0 = same as the first)
  int mat0, mat1;  // indices into the A tensor-map table
  int row0;    // first weight row
  int nrows;   // valid rows of the matrices
  int col0;    // output column offset (hz column, logit column or out column)
  int b16;     // 1: fp16 operands with B = DenseParams::b16 (x16; the ternary correction A's units)
};

struct DenseParams {
  CUtensorMap a[6];  // A matrices, box {64, 128}
  CUtensorMap b;     // B (tokens x K), box {64, 128}
  CUtensorMap b16;   // B of the units with b16 set: x16 (tokens x K fp16)
  const DenseUnit* units;
  int n_units2;      // units with two A matrices (listed first)
  int n_units;
  int K, T, ab_bf16;
  float* logits;  int ld_logits;
  __half* hz;     int ld_hz;
  float* out;     int ld_out;
  const float* resid;  // kEpiStore: added to the stored value (same layout as out; may equal out)
  const int32_t* xexp;  // range exponent s_t of each token: hz rows are stored times 2^hz_shift(s_t)
  int has_corr;         // the layer has a correction (hz_shift's choice)
  int has_shared;       // the layer has a shared expert (hz_shift's choice)
  int z_only;           // the correction branch alone: z rows are stored times 2^s_t
  int* err;
};

constexpr int kDenseStages = 4;
constexpr int kBK = 64;
constexpr uint32_t kDenseStage = 3 * 128 * kBK * 2;  // 48 KB: two A boxes + one B box, or one A + two B

// Tile t of the persistent schedule: 256-token block b = t / per_block; inside a block the
// two-matrix units come first with two 128-token tiles each, then the one-matrix units with
// one 256-token tile each.  Every role derives the same sequence from the same arithmetic.
struct DenseTile {
  int unit, tok0, ntok;  // ntok = 128 or 256 (tokens past T are not stored)
};
__device__ __forceinline__ DenseTile dense_tile(const DenseParams& p, int t) {
  const int per_block = 2 * p.n_units2 + (p.n_units - p.n_units2);
  const int b = t / per_block, r = t % per_block;
  DenseTile d;
  if (r < 2 * p.n_units2) {
    d.unit = r >> 1, d.tok0 = 256 * b + 128 * (r & 1), d.ntok = 128;
  } else {
    d.unit = p.n_units2 + (r - 2 * p.n_units2), d.tok0 = 256 * b, d.ntok = 256;
  }
  return d;
}

// Persistent tcgen05 GEMM over (weight-row unit, token block) tiles: one TMA producer thread,
// one MMA thread, four epilogue warps; the stage ring runs on across tiles and the fp32
// accumulator is double-buffered in tensor memory (2 x 256 columns), so the epilogue of a tile
// overlaps the main loop of the next.
__global__ void __launch_bounds__(kThreads, 1) dense_gemm_kernel(const __grid_constant__ DenseParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1024-aligned, still __shared__
  __shared__ uint64_t full[kDenseStages], empty[kDenseStages], acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_block = 2 * p.n_units2 + (p.n_units - p.n_units2);
  const int n_tiles = per_block * ((p.T + 255) / 256);
  const int nk = p.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDenseStages; ++s) mbar_init(&full[s], 1), mbar_init(&empty[s], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&acc_full[i], 1), mbar_init(&acc_empty[i], kDenseEpi);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    int ks = 0;  // running k-block counter (ring position)
    for (int t = blockIdx.x; t < n_tiles && !abort_flag; t += gridDim.x) {
      const DenseTile dt = dense_tile(p, t);
      if (dt.tok0 >= p.T) continue;
      const DenseUnit u = p.units[dt.unit];
      const uint32_t bytes = u.na * 128 * kBK * 2 + dt.ntok * kBK * 2;
      for (int kb = 0; kb < nk; ++kb, ++ks) {
        const int s = ks % kDenseStages;
        if (ks >= kDenseStages && !mbar_wait(&empty[s], ((ks / kDenseStages) - 1) & 1, &abort_flag, p.err)) break;
        uint8_t* st = smem + s * kDenseStage;
        mbar_arrive_expect_tx(&full[s], bytes);
        tma_load_2d(st, &p.a[u.mat0], kb * kBK, u.row0, &full[s]);
        uint8_t* bdst = st + 128 * kBK * 2;
        if (u.na == 2) {
          tma_load_2d(bdst, &p.a[u.mat1], kb * kBK, u.row0, &full[s]);
          bdst += 128 * kBK * 2;
        }
        const CUtensorMap* bm = u.b16 ? &p.b16 : &p.b;
        tma_load_2d(bdst, bm, kb * kBK, dt.tok0, &full[s]);
        if (dt.ntok == 256) tma_load_2d(bdst + 128 * kBK * 2, bm, kb * kBK, dt.tok0 + 128, &full[s]);
      }
    }
    // copies of the last ring positions may still be in flight if a consumer gave up
    for (int i = max(0, ks - kDenseStages); i < ks; ++i) mbar_drain(&full[i % kDenseStages], (i / kDenseStages) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int ks = 0, li = 0;
    for (int t = blockIdx.x; t < n_tiles && !abort_flag; t += gridDim.x) {
      const DenseTile dt = dense_tile(p, t);
      if (dt.tok0 >= p.T) continue;
      const DenseUnit u = p.units[dt.unit];
      const int ab = li & 1;
      if (li >= 2 && !mbar_wait(&acc_empty[ab], ((li >> 1) - 1) & 1, &abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t acc = tmem + 256 * ab;
      const uint32_t idesc = umma_idesc(kBM, dt.ntok, u.b16 ? 0 : p.ab_bf16);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb, ++ks) {
        const int s = ks % kDenseStages;
        if (!mbar_wait(&full[s], (ks / kDenseStages) & 1, &abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * kDenseStage);
        const uint32_t bst = st + u.na * 128 * kBK * 2;
#pragma unroll
        for (int k16 = 0; k16 < kBK / 16; ++k16) {
          const uint64_t db = umma_desc_sw128(bst + 32 * k16);
          umma_f16(acc, umma_desc_sw128(st + 32 * k16), db, idesc, (kb | k16) != 0);
          if (u.na == 2) {
            const uint64_t da1 = umma_desc_sw128(st + 128 * kBK * 2 + 32 * k16);
            umma_f16(u.map1 ? acc + 128 : acc, da1, db, idesc, u.map1 ? uint32_t((kb | k16) != 0) : 1u);
          }
        }
        umma_commit(&empty[s]);
      }
      if (!ok) break;
      umma_commit(&acc_full[ab]);
      ++li;
    }
    // every MMA issued above has finished before TMEM is released
    umma_commit(&mma_done);
    mbar_drain(&mma_done, 0);
  } else if (warp >= 4) {
    // ---------------- epilogue: TMEM lanes 32q..32q+31 = weight rows; the two warps of a lane
    // quarter take alternate 16-token chunks.  Each thread writes its row's element of every
    // token (consecutive rows across the lanes: one contiguous segment per warp and token).
    const int q = warp & 3, half = (warp - 4) >> 2;
    const int row = q * 32 + lane;
    int li = 0;
    // no abort-flag test in the loop condition: the epilogue threads leave only together, by the vote
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
      const DenseTile dt = dense_tile(p, t);
      if (dt.tok0 >= p.T) continue;
      const DenseUnit u = p.units[dt.unit];
      const int ab = li & 1;
      if (!named_bar_and(1, kDenseEpi, mbar_wait(&acc_full[ab], (li >> 1) & 1, &abort_flag, p.err))) break;
      tc_fence_after();
      const int grow = u.row0 + row;
      const bool rok = grow < u.nrows;
      const uint32_t acc = tmem + 256 * ab + (uint32_t(q * 32) << 16);
      const int nt = min(dt.ntok, p.T - dt.tok0);
      const int64_t col = u.col0 + grow;
      for (int c = half; c * 16 < nt; c += 2) {
        float v0[16], v1[16];
        if (u.epi == kEpiSwiglu)
          tmem_ld16x2(acc + c * 16, acc + 128 + c * 16, v0, v1);
        else
          tmem_ld16(acc + c * 16, v0);
        const int n16 = min(16, nt - c * 16);
        const int64_t t0 = dt.tok0 + c * 16;
        // per-token factors of the hz rows (see hz_shift): stored times 2^p, read back times 2^-p;
        // the units against x16 (ternary correction A) accumulate x 2^s_t.  One load per lane,
        // shared by shuffles (the whole warp takes part, before rows past the unit drop out).
        float tf[16];
        if (u.epi != kEpiLogits) {
          const int my_sh = lane < n16 ? p.xexp[t0 + lane] : 0;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int sh = __shfl_sync(0xffffffffu, my_sh, i);
            const int e = p.z_only ? sh : hz_shift(sh, p.has_shared, p.has_corr);
            tf[i] = pow2i(u.epi == kEpiStore ? -e : (u.b16 ? e - sh : e));
          }
        }
        if (!rok) continue;
        if (u.epi == kEpiLogits) {
          float* dst = p.logits + t0 * p.ld_logits + col;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i < n16) dst[int64_t(i) * p.ld_logits] = v0[i];
        } else if (u.epi == kEpiStore) {
          float* dst = p.out + t0 * p.ld_out + col;
          if (p.resid) {
            const float* rs = p.resid + t0 * p.ld_out + col;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (i < n16) dst[int64_t(i) * p.ld_out] = v0[i] * tf[i] + rs[int64_t(i) * p.ld_out];
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (i < n16) dst[int64_t(i) * p.ld_out] = v0[i] * tf[i];
          }
        } else {
          __half* dst = p.hz + t0 * p.ld_hz + col;
          const bool sw = u.epi == kEpiSwiglu;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i < n16) dst[int64_t(i) * p.ld_hz] = __float2half_rn((sw ? silu_f(v0[i]) * v1[i] : v0[i]) * tf[i]);
        }
      }
      // accumulator drained: hand it back to the MMA thread
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
      ++li;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace
}  // namespace scion

namespace scion {
namespace {

// -------------------------------------------------------------- ternary GEMM
struct __align__(16) TernTile {
  int e;     // expert
  int c0;    // first token (within the expert's group) of this tile
  int n;     // tokens in the tile (1..TN, TN = 128 or 160)
  int pos0;  // routed-order position of its first token (offsets[e] + c0)
};

__device__ __forceinline__ TernTile load_tile(const TernTile* tiles, int i) {
  const int4 v = __ldg(reinterpret_cast<const int4*>(tiles) + i);
  return TernTile{v.x, v.y, v.z, v.w};
}

// out[0..3] += (a, b, c, d): one 16-byte fp32 reduction (16-byte aligned address).
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

struct TernParams {
  CUtensorMap bmap;     // down projection: B = h [T*k][F], box {64, box_rows}
  int box_rows;         // rows of one TMA box of B (the tile width)
  const uint8_t* bank;  // re-tiled gate/up bank (na = 2) or down bank (na = 1)
  int fmt, na, G, R;    // groups along K, rows per expert matrix
  const __half* bsrc;   // B rows: x16 [T][d] (gate/up) or h [T*k][F] (down)
  int ldb;
  const TernTile* tiles;
  const int32_t* n_tiles;
  const int32_t *counts, *offsets, *perm;
  const float* gperm;   // [T*k] gate of the entry at each routed position, times 2^(-2 s_t)
  int k;
  const int32_t* pexp;  // [T*k] range exponent s_t of the token of each routed position (gate/up B rows are x 2^s_t)
  __half* h;  int F;     // gate/up output, h 2^(2 s_t), one row per routed position
  // down output: y != nullptr -> one fp16 row per routed (token, slot), [T*k][d], gates applied
  // by the combine; otherwise out[t] += gate 2^(-2 s_t) y with fp32 reductions
  __half* y;  int d;
  float* out;
  int* err;
};

constexpr int kBN3 = 160;      // tokens per tile of batches whose experts average kMid160 or more
constexpr int kMid160 = 112;   // mean tokens per expert from which both ternary GEMMs take kBN3 tiles

// Expand half h (64 columns) of row t (0..127) of one 128-row group from its sub-tile block
// into 32 registers of fp16 pairs, in position order (v[i] = positions 2i, 2i+1 of the half).
// Values are code * scale, exact in fp16.
__device__ __forceinline__ void expand_pq2_half(uint32_t codes, int t, int h, uint32_t (&out)[32]) {
  const uint32_t blk = codes + (t >> 4) * kPq2Tile;
  const int rho = t & 15, r8 = rho & 7, hi = rho >> 3;
  const __half2 sc = __half2half2(__ushort_as_half(uint16_t(lds_u16(blk + 512 + 4 * r8 + 2 * hi))));
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = 2 * h + cc;  // container code bytes 8c .. 8c+7 = words 2c, 2c+1
    const uint2 w2 = lds_v2(blk + 16 * (4 * r8 + c) + 8 * hi);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t w = half ? w2.y : w2.x, w10 = w >> 10;
      // pair s = columns (s, s + 8): the field at bits 2f..2f+1 of each 16-bit half (f = s, or
      // s - 5 in w >> 10) ORed into the fp16 pattern of 2^(10-2f) (exponent field 25 - 2f, whose
      // mantissa unit is 4^-f) reads 2^(10-2f) + b; minus 2^(10-2f) + 1, times the scale, is
      // code * scale exactly, so the B operands carry no factor
      uint32_t v[8];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int f = s < 5 ? s : s - 5;
        const uint32_t magic = uint32_t(25 - 2 * f) << 10, bias = magic | (1u << (2 * f));
        v[s] = h2_as_u32(__hmul2(__hsub2(u32_as_h2(lop3_and_or(s < 5 ? w : w10, 0x00030003u << (2 * f),
                                                               magic | (magic << 16))),
                                         u32_as_h2(bias | (bias << 16))),
                                 sc));
      }
      const int j0 = 2 * (2 * cc + half);  // 8-position chunk index inside the half
#pragma unroll
      for (int i = 0; i < 8; ++i) out[4 * j0 + i] = v[i];
    }
  }
}

__device__ __forceinline__ void expand_ptq1_half(uint32_t codes, int t, int h, uint32_t (&v)[32]) {
  const uint32_t blk = codes + (t >> 4) * kPtq1Tile;
  const int rho = t & 15, r8 = rho & 7, hi = rho >> 3;
  const __half2 sc = __half2half2(__ushort_as_half(uint16_t(lds_u16(blk + 416 + 4 * r8 + 2 * hi))));
  const __half2 third = __float2half2_rn(0.333251953125f), c1 = __float2half2_rn(682.5f);
  const __half2 m3 = __float2half2_rn(-3.0f), c2047 = __float2half2_rn(2047.0f);
#pragma unroll
  for (int i = 0; i < 6; ++i) {
    const int q = 12 * h + 2 * i;
    const uint32_t x = lds_u16(blk + 12 * (4 * r8 + q / 6) + 6 * hi + q % 6);
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
  {
    // remainder trits (columns 120..127) as 2-bit fields: bytes (even trits, odd trits) of this row;
    // half h takes trits 4h .. 4h + 3
    const uint32_t x = (lds_u32(blk + 384 + 4 * r8) >> (8 * hi)) & 0x00ff00ffu;
    const uint32_t r0 = ptq1_rem_pair(x, 4 * h), r1 = ptq1_rem_pair(x, 4 * h + 2);
    v[30] = h2_as_u32(__hmul2(u32_as_h2(r0), sc));
    v[31] = h2_as_u32(__hmul2(u32_as_h2(r1), sc));
  }
}

// Pipeline granularity: one 128-column code group along K ("group" = two 64-column halves).
// TN = tokens per tile: 128, or 160 when the experts average at least kMid160 tokens (a tile then
// holds nearly all of an expert's tokens, so its codes are seldom expanded a second time for a
// tile of a few tokens).
template <int FMT, int NA, int TN = kBN>
struct TernRing {
  static constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  // shared memory: B groups (two 64-column K blocks of TN swizzled 128-byte rows) and packed
  // code groups
  static_assert(TN == kBN || TN == kBN3, "tile width");
  static constexpr int kB = 4;
  static constexpr int kC = 4;
  static constexpr uint32_t b_kblock = uint32_t(TN) * 128;  // bytes of one 64-column K block of B
  static constexpr uint32_t b_bytes = 2 * b_kblock;
  static constexpr uint32_t c_bytes = NA * 8 * tb;
  static constexpr uint32_t b_off = 0, c_off = kB * b_bytes;
  // down projection: per epilogue warp a 16-token x 32-row fp32 tile, read back as 4-row vectors
  // for the 16-byte reductions into out
  static constexpr uint32_t e_off = c_off + kC * c_bytes;
  static constexpr uint32_t bytes = e_off + (NA == 1 ? 8 * 16 * 32 * 4 : 0);
  // tensor memory: accumulators, then the ring of expanded A groups
  // gate/up: one NA x TN accumulator; down: two TN-column accumulators (ping-pong)
  static constexpr int n_acc = NA == 1 ? 2 : 1;
  static constexpr uint32_t acc_cols = NA * TN;
  // ring entries of expanded A: one group of all NA matrices, or (160-token gate/up tiles,
  // whose accumulators leave 192 columns) one matrix of a group, EPG entries per group
  static constexpr int EPG = TN == kBN3 ? NA : 1;
  static constexpr int MPE = NA / EPG;           // matrices per entry
  static constexpr int kA = TN == kBN3 ? 3 : (NA == 2 ? 2 : 4);
  static constexpr uint32_t a_cols = MPE * 64;   // one entry: MPE matrices x 64 columns (128 fp16 per lane)
  static constexpr uint32_t a_col0 = n_acc * acc_cols;
  static constexpr uint32_t tmem_cols = 512;
  static_assert(a_col0 + kA * a_cols <= tmem_cols, "TMEM budget");
};

constexpr int kTernThreads = 640;  // 20 warps: codes, MMA, 2 x B rows, 8 expansion, 8 epilogue
constexpr int kEpiThreads = 256;

// Persistent grouped GEMM: CTA b walks the work items b, b + gridDim.x, ... where item =
// (token tile of up to TN tokens, 128-row weight tile).  The expansion warps decode the packed codes of each
// 128-column group straight into tensor memory (one weight row per TMEM lane), and the MMA
// reads A from there and the tokens (B) from shared memory.  All roles walk the same item
// sequence; rings carry over from one item to the next.  The MMA issuer waits on a single
// barrier per group: the expansion side folds the B-ready condition into its own arrival.
template <int FMT, int NA, int TN = kBN>
__global__ void __launch_bounds__(kTernThreads, 1) tern_gemm_kernel(const __grid_constant__ TernParams p) {
  using R = TernRing<FMT, NA, TN>;
  constexpr bool kBTma = NA == 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1024-aligned, still __shared__
  __shared__ uint64_t c_full[R::kC], c_empty[R::kC], a_full[R::kA], a_empty[R::kA], b_full[R::kB], b_empty[R::kB];
  __shared__ uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int RT = p.R >> 7;                     // 128-row weight tiles per expert matrix
  const int n_items = *p.n_tiles * RT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < R::kC; ++i) mbar_init(&c_full[i], 1), mbar_init(&c_empty[i], 256);
    for (int i = 0; i < R::kA; ++i) mbar_init(&a_full[i], 256), mbar_init(&a_empty[i], 1);
    for (int i = 0; i < R::kB; ++i) mbar_init(&b_full[i], kBTma ? 1 : 64), mbar_init(&b_empty[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&acc_full[i], 1), mbar_init(&acc_empty[i], kEpiThreads);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&tmem_slot, R::tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // ---------------- packed code blocks, one 128-row group per bulk copy and matrix
    if (lane == 0) {
      const int64_t mat_stride = int64_t(8) * R::tb, grp_stride = NA * mat_stride;
      int gs = 0;  // running group counter
      for (int item = blockIdx.x; item < n_items && !abort_flag; item += gridDim.x) {
        const TernTile tile = load_tile(p.tiles, item / RT);
        const int rt = item % RT;
        const uint8_t* ebase = p.bank + (int64_t(tile.e) * RT + rt) * p.G * grp_stride;
        for (int g = 0; g < p.G; ++g, ++gs) {
          const int s = gs % R::kC;
          if (gs >= R::kC && !mbar_wait(&c_empty[s], ((gs / R::kC) - 1) & 1, &abort_flag, p.err)) break;
          uint8_t* dst = smem + R::c_off + s * R::c_bytes;
          mbar_arrive_expect_tx(&c_full[s], R::c_bytes);
#pragma unroll
          for (int m = 0; m < NA; ++m)
            bulk_load(dst + m * mat_stride, ebase + g * grp_stride + m * mat_stride, mat_stride, &c_full[s]);
        }
      }
      // the last kC groups issued may still be in flight if a consumer gave up: let them land
      for (int i = max(0, gs - R::kC); i < gs; ++i) mbar_drain(&c_full[i % R::kC], (i / R::kC) & 1);
    }
  } else if (kBTma && warp == 2) {
    // ---------------- B rows are contiguous (h in routed order): two TMA boxes per group
    if (lane == 0) {
      int gs = 0;
      for (int item = blockIdx.x; item < n_items && !abort_flag; item += gridDim.x) {
        const TernTile tile = load_tile(p.tiles, item / RT);
        // boxes of box_rows rows (128-byte rows, swizzle atoms of 8 rows: consecutive boxes
        // stack into one TN-row operand); rows past the tile's tokens are loaded but never stored
        const int nbox = p.box_rows >= TN ? 1 : (tile.n + p.box_rows - 1) / p.box_rows;
        const uint32_t box_bytes = uint32_t(min(p.box_rows, TN)) * 128;
        for (int g = 0; g < p.G; ++g, ++gs) {
          const int s = gs % R::kB;
          if (gs >= R::kB && !mbar_wait(&b_empty[s], ((gs / R::kB) - 1) & 1, &abort_flag, p.err)) break;
          uint8_t* dst = smem + R::b_off + s * R::b_bytes;
          mbar_arrive_expect_tx(&b_full[s], 2 * nbox * box_bytes);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb)  // 64-column K blocks of the group
            for (int bx = 0; bx < nbox; ++bx)
              tma_load_2d(dst + kb * R::b_kblock + bx * box_bytes, &p.bmap, g * 128 + 64 * kb,
                          tile.pos0 + bx * p.box_rows, &b_full[s]);
        }
      }
      for (int i = max(0, gs - R::kB); i < gs; ++i) mbar_drain(&b_full[i % R::kB], (i / R::kB) & 1);
    }
  } else if (!kBTma && (warp == 2 || warp == 3)) {
    // ---------------- gathered B rows (tokens of the tile), 128 columns (two atoms) per group;
    // warp 2 takes rows 0..63, warp 3 rows 64..127.  Lanes 2m and 2m+1 copy the two 16-byte
    // halves of one 32-byte sector of the same row, so every request is a whole L2 sector:
    // lane (m, hf) handles rows rbase + m + 16i (i < 4), 16-byte chunks 2j + hf (j < 8).
    constexpr int kRows = TN / 32;   // rows per lane pair
    const int rbase = (warp - 2) * (TN / 2) + (lane >> 1), hf = lane & 1;
    constexpr int kLag = R::kB / 2;  // groups in flight per thread before the oldest is published
    int gs = 0;                      // running group counter
    for (int item = blockIdx.x; item < n_items && !abort_flag; item += gridDim.x) {
      const TernTile tile = load_tile(p.tiles, item / RT);
      const __half* rows[kRows];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int r = rbase + 16 * i;
        rows[i] = r < tile.n ? p.bsrc + int64_t(p.perm[tile.pos0 + r] / p.k) * p.ldb + 8 * hf : nullptr;
      }
      for (int g = 0; g < p.G; ++g, ++gs) {
        const int s = gs % R::kB;
        if (gs >= R::kB && !mbar_wait(&b_empty[s], ((gs / R::kB) - 1) & 1, &abort_flag, p.err)) break;
        const uint32_t bt = sbase + R::b_off + s * R::b_bytes;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          if (!rows[i]) continue;
          const int r = rbase + 16 * i;
          const __half* src = rows[i] + g * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int ch = 2 * j + hf;  // 16-byte chunk of the row's 256 bytes
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(bt + (ch >> 3) * R::b_kblock + sw128_offset(r, ch & 7)),
                         "l"(src + 16 * j)
                         : "memory");
          }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        // group gs - kLag has landed: make it visible to the tensor cores (async proxy), then publish it
        if (gs >= kLag) {
          asm volatile("cp.async.wait_group %0;" ::"n"(kLag) : "memory");
          fence_proxy_async();
          mbar_arrive(&b_full[(gs - kLag) % R::kB]);
        }
      }
    }
    cp_async_wait_all();
    fence_proxy_async();
    for (int i = max(0, gs - kLag); i < gs; ++i) mbar_arrive(&b_full[i % R::kB]);
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: A from tensor memory, B from shared memory
      int gs = 0, es = 0, li = 0;  // running group, A-entry and item counters
      TernTile next = blockIdx.x < n_items ? load_tile(p.tiles, blockIdx.x / RT) : TernTile{};
      for (int item = blockIdx.x; item < n_items && !abort_flag; item += gridDim.x, ++li) {
        const TernTile tile = next;  // loaded one item ahead: no global-load latency between items
        if (item + int(gridDim.x) < n_items) next = load_tile(p.tiles, (item + gridDim.x) / RT);
        const uint32_t idesc = umma_idesc(kBM, (tile.n + 15) & ~15, 0);
        const int ab = li % R::n_acc;
        if (li >= R::n_acc && !mbar_wait(&acc_empty[ab], ((li / R::n_acc) - 1) & 1, &abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + ab * R::acc_cols;
        bool ok = true;
        for (int g = 0; g < p.G && ok; ++g, ++gs) {
          const int sb = gs % R::kB;
          const uint32_t bt = sbase + R::b_off + sb * R::b_bytes;
#pragma unroll
          for (int eg = 0; eg < R::EPG; ++eg, ++es) {
            const int sa = es % R::kA;
            // A expanded and (folded into the group's first arrival) B landed
            if (!(ok = mbar_wait(&a_full[sa], (es / R::kA) & 1, &abort_flag, p.err))) break;
            tc_fence_after();
            const uint32_t at = tmem + R::a_col0 + sa * R::a_cols;
#pragma unroll
            for (int k16 = 0; k16 < 8; ++k16) {
              const uint64_t db = umma_desc_sw128(bt + (k16 >> 2) * R::b_kblock + 32 * (k16 & 3));
#pragma unroll
              for (int m = 0; m < R::MPE; ++m)
                umma_ts(acc + (eg * R::MPE + m) * TN, at + m * 64 + 8 * k16, db, idesc, (g | k16) != 0);
            }
            umma_commit(&a_empty[sa]);
          }
          if (ok) umma_commit(&b_empty[sb]);
        }
        umma_commit(&acc_full[ab]);
      }
      // every MMA issued above has finished before TMEM is released
      umma_commit(&mma_done);
      mbar_drain(&mma_done, 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------- expansion: two warpgroups; group `part` decodes the 64-column half
    // h == part of every code group, thread t of a warpgroup decoding weight row t into TMEM lane t
    const int part = (warp - 4) >> 2;
    const int t = (threadIdx.x - 128) & 127;
    const bool b_watch = part == 0 && t == 0;  // this thread also waits for the group's B rows
    const uint32_t lane_base = tmem + (uint32_t((warp & 3) * 32) << 16) + R::a_col0 + part * 32;
    int gs = 0, es = 0;  // running code-group and A-entry counters
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok && !abort_flag; item += gridDim.x) {
      for (int g = 0; g < p.G && ok; ++g, ++gs) {
        const int sc = gs % R::kC;
        if (!(ok = mbar_wait(&c_full[sc], (gs / R::kC) & 1, &abort_flag, p.err))) break;
        const uint32_t codes = sbase + R::c_off + sc * R::c_bytes;
#pragma unroll
        for (int eg = 0; eg < R::EPG; ++eg, ++es) {
          const int sa = es % R::kA;
          if (es >= R::kA && !(ok = mbar_wait(&a_empty[sa], ((es / R::kA) - 1) & 1, &abort_flag, p.err))) break;
          tc_fence_after();
#pragma unroll
          for (int m = 0; m < R::MPE; ++m) {
            const int mat = eg * R::MPE + m;
            uint32_t v[32];
            if constexpr (FMT == SCION_PQ2_0)
              expand_pq2_half(codes + mat * 8 * R::tb, t, part, v);
            else
              expand_ptq1_half(codes + mat * 8 * R::tb, t, part, v);
            tmem_st32(lane_base + sa * R::a_cols + m * 64, v);
          }
          tmem_wait_st();
          tc_fence_before();
          if (eg == R::EPG - 1) mbar_arrive(&c_empty[sc]);
          if (eg == 0 && b_watch && !(ok = mbar_wait(&b_full[gs % R::kB], (gs / R::kB) & 1, &abort_flag, p.err)))
            break;
          mbar_arrive(&a_full[sa]);
        }
      }
    }
  } else if (warp >= 12) {
    // ---------------- epilogue: TMEM lane quarter q = weight rows 32q .. 32q+31, 16 tokens per
    // chunk; the two warps of a quarter take alternate chunks.  Stores go straight to global
    // memory.
    const int q = warp & 3, half = (warp - 12) >> 2;
    const int row = q * 32 + lane;
    const int pcol = perm_pos(FMT, row);  // gate/up: position of this row inside its 128-column group of h
    int li = 0;
    // no abort-flag test in the loop condition: the epilogue threads leave only together, by the vote
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++li) {
      const TernTile tile = load_tile(p.tiles, item / RT);
      const int rt = item % RT;
      const int64_t pos0 = tile.pos0;
      const int nn = tile.n;
      const int ab = li % R::n_acc;
      if (!named_bar_and(1, kEpiThreads, mbar_wait(&acc_full[ab], (li / R::n_acc) & 1, &abort_flag, p.err))) break;
      tc_fence_after();
      const uint32_t acc = tmem + ab * R::acc_cols + (uint32_t(q * 32) << 16);
      for (int c = half; c * 16 < nn; c += 2) {
        float v0[16], v1[16];
        if constexpr (NA == 2)
          tmem_ld16x2(acc + c * 16, acc + TN + c * 16, v0, v1);
        else
          tmem_ld16(acc + c * 16, v0);
        const int n0 = c * 16;
        if constexpr (NA == 2) {
          __half* dst = p.h + (pos0 + n0) * p.F + int64_t(rt) * kBM + pcol;
          // range exponents of the chunk's 16 tokens: one load per lane, shared by shuffles; the
          // common case (every token in the unscaled band) skips the scaling
          const int my_sh = (lane < 16 && n0 + lane < nn) ? p.pexp[pos0 + n0 + lane] : 0;
          if (__all_sync(0xffffffffu, my_sh == 0)) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n0 + i < nn) dst[int64_t(i) * p.F] = __float2half_rn(silu_f(v0[i]) * v1[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int sh = __shfl_sync(0xffffffffu, my_sh, i);  // the sums are of x 2^sh
              if (n0 + i < nn)
                dst[int64_t(i) * p.F] = __float2half_rn(silu_f(v0[i] * pow2i(-sh)) * (v1[i] * pow2i(sh)));
            }
          }
        } else if (p.y) {
          __half* dst = p.y + (pos0 + n0) * p.d + int64_t(rt) * kBM + row;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (n0 + i < nn) dst[int64_t(i) * p.d] = __float2half_rn(v0[i]);
        } else {
          // gate-weighted scatter-add: the warp's 32 rows x 16 tokens go through shared memory and
          // come back as (token, 4 consecutive rows) vectors, one 16-byte fp32 reduction each
          float* ts = reinterpret_cast<float*>(smem + R::e_off) + (warp - 12) * 512;
#pragma unroll
          for (int i = 0; i < 16; ++i) ts[i * 32 + lane] = v0[i];
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = (lane >> 3) + 4 * j, g4 = lane & 7;  // token i of the chunk, rows 4 g4 .. 4 g4 + 3
            if (n0 + i < nn) {
              const float4 w = *reinterpret_cast<const float4*>(ts + i * 32 + 4 * g4);
              const int pos = int(pos0) + n0 + i;
              const int t = p.perm[pos] / p.k;
              const float gg = p.gperm[pos];
              red_add_v4(p.out + int64_t(t) * p.d + int64_t(rt) * kBM + q * 32 + 4 * g4, gg * w.x, gg * w.y,
                         gg * w.z, gg * w.w);
            }
          }
          __syncwarp();
        }
      }
      // accumulator drained: hand it back to the MMA warp
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, R::tmem_cols);
  }
}

// ------------------------------------------------------------------- routing
// One warp per token, `tpw` tokens per warp (more for long batches, so that each CTA's
// histogram covers more selections), logits in registers.  The expert histogram is counted in
// shared memory and added to the global one once per CTA and expert (a hot expert of a skewed
// router would otherwise take one global atomic per selection).
template <int VPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                   int norm_topk, int tpw, int32_t* __restrict__ ids,
                                                   float* __restrict__ gates, int32_t* __restrict__ counts, int elo,
                                                   int El) {
  extern __shared__ int32_t hist[];  // [El]: the handle's local experts
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < El; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  for (int i = 0; i < tpw; ++i) {
    const int t = (blockIdx.x * tpw + i) * 8 + warp;
    if (t >= T) break;
    warp_topk<VPL>(logits + int64_t(t) * E, E, k, norm_topk, lane, ids + int64_t(t) * k, gates + int64_t(t) * k);
    __syncwarp();
    if (lane < k) {
      const unsigned le = unsigned(ids[int64_t(t) * k + lane] - elo);
      if (le < unsigned(El)) atomicAdd(&hist[le], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < El; e += blockDim.x)
    if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

// Grouping by expert.  The order of the tokens inside an expert's segment is free (each token
// column of the grouped GEMMs is computed independently, and the combine sums a token's k rows
// in slot order), so the scatter takes positions with one atomic per entry.
//
// One CTA: exclusive scan of the histogram, the per-expert cursors, and the token tiles of the
// two ternary GEMMs (w tokens: 128 or 160).
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) group_scan_kernel(const int32_t* __restrict__ counts, int E,
                                                                  int32_t* __restrict__ offsets,
                                                                  int32_t* __restrict__ cursor,
                                                                  TernTile* __restrict__ tiles,
                                                                  int32_t* __restrict__ n_tiles, int w) {
  __shared__ int32_t wsum[kScanThreads / 32], wtile[kScanThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (E + kScanThreads - 1) / kScanThreads;  // experts per thread, contiguous
  const int e0 = min(E, threadIdx.x * per), e1 = min(E, e0 + per);
  int cs = 0, ts = 0;
  for (int e = e0; e < e1; ++e) {
    const int c = counts[e];
    cs += c, ts += (c + w - 1) / w;
  }
  // block-wide exclusive scan of (cs, ts)
  int ic = cs, it = ts;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int c2 = __shfl_up_sync(0xffffffffu, ic, o), t2 = __shfl_up_sync(0xffffffffu, it, o);
    if (lane >= o) ic += c2, it += t2;
  }
  if (lane == 31) wsum[warp] = ic, wtile[warp] = it;
  __syncthreads();
  if (warp == 0) {
    int a = wsum[lane], b = wtile[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a2 = __shfl_up_sync(0xffffffffu, a, o), x2 = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) a += a2, b += x2;
    }
    wsum[lane] = a, wtile[lane] = b;
    if (lane == 31) offsets[E] = a, *n_tiles = b;
  }
  __syncthreads();
  int run = (warp ? wsum[warp - 1] : 0) + ic - cs;
  int trun = (warp ? wtile[warp - 1] : 0) + it - ts;
  for (int e = e0; e < e1; ++e) {
    const int c = counts[e];
    offsets[e] = run;
    cursor[e] = run;
    for (int c0 = 0; c0 < c; c0 += w) tiles[trun++] = TernTile{e, c0, min(w, c - c0), run + c0};
    run += c;
  }
}

// Positions inside the experts' segments: `ept` (<= kScatterMaxPerThread) entries per thread.
// Each CTA ranks its entries per expert in shared memory, then reserves one block of positions
// per expert it touches with a single global atomic.
constexpr int kScatterMaxPerThread = 8;
__global__ void __launch_bounds__(256) group_scatter_kernel(const int32_t* __restrict__ ids, int n, int E, int ept,
                                                            int32_t* __restrict__ cursor, int32_t* __restrict__ perm,
                                                            int32_t* __restrict__ inv, int k,
                                                            const float* __restrict__ gates,
                                                            const int32_t* __restrict__ xexp,
                                                            float* __restrict__ gperm, int32_t* __restrict__ pexp,
                                                            int elo) {
  extern __shared__ int32_t sh[];  // cnt[E], base[E]
  int32_t *cnt = sh, *base = sh + E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  int id[kScatterMaxPerThread], local[kScatterMaxPerThread];
  const int i0 = blockIdx.x * 256 * ept + threadIdx.x;
#pragma unroll
  for (int j = 0; j < kScatterMaxPerThread; ++j) {
    const int i = i0 + 256 * j;
    // local expert of the entry; entries of another rank's experts get no position (inv = -1)
    id[j] = j < ept && i < n ? ids[i] - elo : -1;
    if (id[j] >= E) id[j] = -1;
    if (j < ept && i < n && id[j] < 0) inv[i] = -1;
    local[j] = id[j] >= 0 ? atomicAdd(&cnt[id[j]], 1) : 0;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (cnt[e]) base[e] = atomicAdd(&cursor[e], cnt[e]);
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kScatterMaxPerThread; ++j) {
    if (id[j] < 0) continue;
    const int i = i0 + 256 * j, pos = base[id[j]] + local[j];
    const int sh = xexp[i / k];
    perm[pos] = i;
    inv[i] = pos;
    pexp[pos] = sh;
    gperm[pos] = gates[i] * pow2i(-2 * sh);
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

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

int dense_grid(const DenseParams& dp) {
  const int n_tiles = (2 * dp.n_units2 + (dp.n_units - dp.n_units2)) * ((dp.T + 255) / 256);
  return max(1, min(n_tiles, num_sms()));
}

template <int FMT, int NA, int TN>
size_t tern_smem_t() {
  return TernRing<FMT, NA, TN>::bytes + 1024;
}
template <int FMT>
size_t tern_smem_f(int na, int tn) {
  if (na == 2) return tn == kBN3 ? tern_smem_t<FMT, 2, kBN3>() : tern_smem_t<FMT, 2, kBN>();
  return tn == kBN3 ? tern_smem_t<FMT, 1, kBN3>() : tern_smem_t<FMT, 1, kBN>();
}
size_t tern_smem(int na, int fmt, int tn = kBN) {
  return fmt == SCION_PQ2_0 ? tern_smem_f<SCION_PQ2_0>(na, tn) : tern_smem_f<SCION_PTQ1_0>(na, tn);
}
// Tile width of both ternary GEMMs: 160 tokens when the experts average at least kMid160 tokens
// (fewer tiles of a few tokens past 128, each of which expands all of its expert's codes again),
// 128 otherwise.
int tile_width(int64_t Tk, int E) { return Tk >= int64_t(kMid160) * E ? kBN3 : kBN; }
constexpr size_t kDenseSmem = kDenseStages * kDenseStage + 1024;

}  // namespace

// K-major [rows][K] 2-byte matrix, box {64 columns, box_rows rows}, 128-byte swizzle.
int make_tmap_2d(CUtensorMap* map, const void* ptr, int bf16, int64_t rows, int64_t K, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return SCION_ECUDA;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (K * 2) % 16) return SCION_EINVAL;
  cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(K * 2)};
  cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
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
  if ((e = cudaFuncSetAttribute(tern_gemm_kernel<SCION_PQ2_0, 2, kBN3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(tern_smem(2, SCION_PQ2_0, kBN3)))))
    return e;
  if ((e = cudaFuncSetAttribute(tern_gemm_kernel<SCION_PQ2_0, 1, kBN3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(tern_smem(1, SCION_PQ2_0, kBN3)))))
    return e;
  if ((e = cudaFuncSetAttribute(tern_gemm_kernel<SCION_PTQ1_0, 1, kBN3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(tern_smem(1, SCION_PTQ1_0, kBN3)))))
    return e;
  if ((e = cudaFuncSetAttribute(tern_gemm_kernel<SCION_PTQ1_0, 2, kBN3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(tern_smem(2, SCION_PTQ1_0, kBN3)))))
    return e;
  return cudaSuccess;
}

// out[t] = base[t] + sum over slots j < k (in slot order) of gates[t][j] y[inv[t k + j]];
// base = out (the dense down projection stored its part there, residual included), the
// residual (a layer without shared expert and correction), or zero.  One CTA per token.
__global__ void __launch_bounds__(256) combine_kernel(const __half* __restrict__ y, const int32_t* __restrict__ inv,
                                                     const float* __restrict__ gates, int k, int d,
                                                     const int32_t* __restrict__ xexp, const float* base, float* out) {
  const int t = blockIdx.x;
  const int32_t* iv = inv + int64_t(t) * k;
  const float* gt = gates + int64_t(t) * k;
  const float ys = pow2i(-2 * xexp[t]);  // the rows of y are of the hidden h 2^(2 s_t)
  // each thread: 8 columns (one 16-byte load per routed row); the k rows' loads are issued in
  // batches of 8 before any of them is used, so each thread keeps 8 loads in flight
  for (int c8 = threadIdx.x; c8 < d / 8; c8 += blockDim.x) {
    float acc[8];
    if (base) {
      const float4 b0 = reinterpret_cast<const float4*>(base + int64_t(t) * d)[2 * c8];
      const float4 b1 = reinterpret_cast<const float4*>(base + int64_t(t) * d)[2 * c8 + 1];
      acc[0] = b0.x, acc[1] = b0.y, acc[2] = b0.z, acc[3] = b0.w;
      acc[4] = b1.x, acc[5] = b1.y, acc[6] = b1.z, acc[7] = b1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    }
    for (int j0 = 0; j0 < k; j0 += 8) {
      uint4 raw[8];
      float g[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j0 + j < k && iv[j0 + j] >= 0) {  // (an entry of another rank's expert has no row)
          raw[j] = reinterpret_cast<const uint4*>(y + int64_t(iv[j0 + j]) * d)[c8];
          g[j] = gt[j0 + j] * ys;
        } else {
          raw[j] = make_uint4(0u, 0u, 0u, 0u);
          g[j] = 0.f;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 v = __half22float2(u32_as_h2(w[q]));
          acc[2 * q] = fmaf(g[j], v.x, acc[2 * q]);
          acc[2 * q + 1] = fmaf(g[j], v.y, acc[2 * q + 1]);
        }
      }
    }
    float4* o = reinterpret_cast<float4*>(out + int64_t(t) * d);
    o[2 * c8] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[2 * c8 + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// h in the tcgen05 column order -> natural order.  pos_scaled: the values carry the PQ2_0
// position factor 4^-f (the tensor-core decode's h), divided out here.
__global__ void unperm_prefill_kernel(int fmt, int pos_scaled, const __half* __restrict__ src, int64_t n,
                                      __half* __restrict__ dst) {
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t base = i & ~int64_t(127);
  const int p = perm_pos(fmt, int(i & 127));
  const float v = __half2float(src[base + p]);
  dst[i] = __float2half_rn(pos_scaled && fmt == SCION_PQ2_0 ? v / pq2_pos_scale(p) : v);
}

cudaError_t launch_unperm_prefill(int fmt, int pos_scaled, const __half* src, int64_t n, __half* dst, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  unperm_prefill_kernel<<<unsigned((n + 255) / 256), 256, 0, s>>>(fmt, pos_scaled, src, n, dst);
  return cudaGetLastError();
}

size_t prefill_unit_bytes() { return sizeof(DenseUnit); }
size_t prefill_tile_bytes() { return sizeof(TernTile); }

// Builds the dense unit tables (host) for the x-projection and the dense down GEMM.
cudaError_t launch_dequant_corr(const uint8_t* blocks, int rows, int K, __half* dst, int ld, int order,
                                int64_t* bad, cudaStream_t s) {
  const int64_t n = int64_t(rows) * K;
  if (n == 0) return cudaSuccess;
  const unsigned grid = unsigned(std::min<int64_t>((n + 255) / 256, int64_t(num_sms()) * 16));
  dequant_corr_kernel<<<grid, 256, 0, s>>>(blocks, rows, K, dst, ld, order, reinterpret_cast<unsigned long long*>(bad));
  return cudaGetLastError();
}

void prefill_units(const scion_layer* L, void* xunits_host, int* n_x, void* dunits_host, int* n_d) {
  DenseUnit* xu = static_cast<DenseUnit*>(xunits_host);
  DenseUnit* du = static_cast<DenseUnit*>(dunits_host);
  int nx = 0, nd = 0;
  // A map table: 0 router, 1 delta, 2 sh_gate, 3 sh_up, 4 corr_a, 5 dense_down
  // the dense kernel expects the two-matrix units first
  if (!L->desc.router_fp32)
    for (int r0 = 0; r0 < L->E; r0 += 128) xu[nx++] = DenseUnit{kEpiLogits, 2, 0, 0, 1, r0, L->E, 0};
  for (int r0 = 0; r0 < L->Fs; r0 += 128) xu[nx++] = DenseUnit{kEpiSwiglu, 2, 1, 2, 3, r0, L->Fs, 0};
  // ternary correction factors: A's exact fp16 copy (x16 column order) against x16
  const int b16 = L->desc.corr_packed ? 1 : 0;
  for (int r0 = 0; r0 < L->r; r0 += 128) xu[nx++] = DenseUnit{kEpiPlain, 1, 0, 4, 4, r0, L->r, L->Fs, b16};
  if (L->Kdense)
    for (int r0 = 0; r0 < L->d; r0 += 128) du[nd++] = DenseUnit{kEpiStore, 1, 0, 5, 5, r0, L->d, 0};
  *n_x = nx;
  *n_d = nd;
}

bool prefill_dense_down(const scion_layer* L) { return (L->parts & SCION_PART_DENSE) && L->pre->n_dunits > 0; }

int prefill_max_units(const scion_layer* L) { return (L->E + 127) / 128 + (L->Fs + 127) / 128 + (L->r + 127) / 128 + L->d / 128; }

cudaError_t launch_prefill_stage(int stage, const scion_layer* L, const __nv_bfloat16* x, int T, float* out,
                                 const float* resid, cudaStream_t s) {
  const PrefillState& P = *L->pre;
  switch (stage) {
    case SCION_STAGE_X16: {
      const unsigned grid = unsigned(std::min((T + 7) / 8, num_sms() * 8));
      // without a dense down projection (which stores out first) the fused routed down
      // projection only adds into out: set it here
      const int init = !prefill_dense_down(L) && !L->deterministic && (L->parts & SCION_PART_ROUTED);
      if (L->fmt == SCION_PQ2_0)
        x16_kernel<SCION_PQ2_0><<<grid, 256, 0, s>>>(x, T, L->d, P.x16, P.xexp, init, resid, out);
      else
        x16_kernel<SCION_PTQ1_0><<<grid, 256, 0, s>>>(x, T, L->d, P.x16, P.xexp, init, resid, out);
      return cudaGetLastError();
    }
    case SCION_STAGE_XPROJ: {
      // units of the selected parts: router units, then shared gate/up and correction units
      const bool routed = L->parts & SCION_PART_ROUTED, dense = L->parts & SCION_PART_DENSE;
      const int u0 = routed ? 0 : P.n_xrouter, u1 = dense ? P.n_xunits : P.n_xrouter;
      if (u1 <= u0) return cudaSuccess;
      DenseParams dp;
      memcpy(dp.a, P.maps, sizeof(dp.a));
      if (make_tmap_2d(&dp.b, x, 1, T, L->d) != SCION_OK) return cudaErrorInvalidValue;
      dp.units = static_cast<const DenseUnit*>(P.xunits) + u0, dp.K = L->d, dp.T = T, dp.ab_bf16 = 1;
      dp.n_units = u1 - u0;
      // two-matrix units (router + delta, shared gate/up) come first
      dp.n_units2 = (routed ? P.n_xrouter : 0) + (dense ? (L->Fs + 127) / 128 : 0);
      dp.logits = P.logits, dp.ld_logits = L->E, dp.hz = P.hz, dp.ld_hz = L->Kd, dp.out = nullptr, dp.ld_out = 0;
      dp.resid = nullptr;
      dp.xexp = P.xexp, dp.has_corr = L->r > 0, dp.has_shared = L->Fs > 0, dp.z_only = 0;
      dp.err = L->err;
      if (L->desc.corr_packed) dp.b16 = P.x16_map;
      dense_gemm_kernel<<<dense_grid(dp), kThreads, kDenseSmem, s>>>(dp);
      return cudaGetLastError();
    }
    case SCION_STAGE_ROUTE: {
      const int vpl = (L->E + 31) / 32;
      // at least two CTAs per SM for the top-k and one for the scatter, then fewer global atomics
      const int tpw = max(1, min(2, T / (8 * 2 * num_sms())));
      const int n = T * L->k, ept = max(1, min(kScatterMaxPerThread, n / (256 * num_sms())));
      cudaError_t e = cudaMemsetAsync(P.counts, 0, sizeof(int32_t) * L->El, s);
      if (e != cudaSuccess) return e;
#define SCION_TOPK(V) \
  topk_kernel<V><<<(T + 8 * tpw - 1) / (8 * tpw), 256, sizeof(int32_t) * L->El, s>>>( \
      P.logits, T, L->E, L->k, L->desc.norm_topk, tpw, P.ids, P.gates, P.counts, L->elo, L->El)
      if (vpl <= 1) SCION_TOPK(1);
      else if (vpl <= 2) SCION_TOPK(2);
      else if (vpl <= 4) SCION_TOPK(4);
      else if (vpl <= 8) SCION_TOPK(8);
      else if (vpl <= 16) SCION_TOPK(16);
      else if (vpl <= 32) SCION_TOPK(32);
      else SCION_TOPK(64);
#undef SCION_TOPK
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      group_scan_kernel<<<1, kScanThreads, 0, s>>>(P.counts, L->El, P.offsets, P.cursor,
                                                  static_cast<TernTile*>(P.tiles), P.n_tiles,
                                                  tile_width(int64_t(T) * L->k, L->E));
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      group_scatter_kernel<<<(n + 256 * ept - 1) / (256 * ept), 256, 2 * sizeof(int32_t) * L->El, s>>>(
          P.ids, n, L->El, ept, P.cursor, P.perm, P.inv, L->k, P.gates, P.xexp, P.gperm, P.pexp, L->elo);
      return cudaGetLastError();
    }
    case SCION_STAGE_GATEUP: {
      TernParams tp;
      tp.bank = L->gu_bank, tp.fmt = L->fmt, tp.na = 2, tp.G = L->Gd, tp.R = L->F;
      tp.bsrc = P.x16, tp.ldb = L->d;
      const bool mid = tile_width(int64_t(T) * L->k, L->E) == kBN3;
      tp.tiles = static_cast<const TernTile*>(P.tiles), tp.n_tiles = P.n_tiles;
      tp.counts = P.counts, tp.offsets = P.offsets, tp.perm = P.perm, tp.gperm = P.gperm, tp.k = L->k;
      tp.pexp = P.pexp, tp.box_rows = kBN, tp.out = nullptr;
      tp.h = P.h, tp.F = L->F, tp.y = nullptr, tp.d = L->d, tp.err = L->err;
      const dim3 grid(num_sms());
      if (L->fmt == SCION_PQ2_0 && mid)
        tern_gemm_kernel<SCION_PQ2_0, 2, kBN3><<<grid, kTernThreads, tern_smem(2, L->fmt, kBN3), s>>>(tp);
      else if (L->fmt == SCION_PQ2_0)
        tern_gemm_kernel<SCION_PQ2_0, 2><<<grid, kTernThreads, tern_smem(2, L->fmt), s>>>(tp);
      else if (mid)
        tern_gemm_kernel<SCION_PTQ1_0, 2, kBN3><<<grid, kTernThreads, tern_smem(2, L->fmt, kBN3), s>>>(tp);
      else
        tern_gemm_kernel<SCION_PTQ1_0, 2><<<grid, kTernThreads, tern_smem(2, L->fmt), s>>>(tp);
      return cudaGetLastError();
    }
    case SCION_STAGE_COMBINE: {
      combine_kernel<<<T, 256, 0, s>>>(P.y, P.inv, P.gates, L->k, L->d, P.xexp, prefill_dense_down(L) ? out : resid,
                                       out);
      return cudaGetLastError();
    }
    case SCION_STAGE_DOWN_DENSE: {
      if (P.n_dunits == 0) return cudaSuccess;
      DenseParams dp;
      memcpy(dp.a, P.maps, sizeof(dp.a));
      dp.b = P.hz_map;
      dp.units = static_cast<const DenseUnit*>(P.dunits), dp.K = L->Kd, dp.T = T, dp.ab_bf16 = 0;
      dp.n_units = P.n_dunits, dp.n_units2 = 0;
      dp.logits = nullptr, dp.ld_logits = 0, dp.hz = nullptr, dp.ld_hz = 0, dp.out = out, dp.ld_out = L->d;
      dp.resid = resid;
      dp.xexp = P.xexp, dp.has_corr = L->r > 0, dp.has_shared = L->Fs > 0, dp.z_only = 0;
      dp.err = L->err;
      dense_gemm_kernel<<<dense_grid(dp), kThreads, kDenseSmem, s>>>(dp);
      return cudaGetLastError();
    }
    case SCION_STAGE_DOWN_ROUTED: {
      TernParams tp;
      tp.bank = L->dn_bank, tp.fmt = L->fmt, tp.na = 1, tp.G = L->GF, tp.R = L->d;
      tp.bsrc = P.h, tp.ldb = L->F;
      const int wd = tile_width(int64_t(T) * L->k, L->E);
      tp.tiles = static_cast<const TernTile*>(P.tiles), tp.n_tiles = P.n_tiles;
      tp.counts = P.counts, tp.offsets = P.offsets, tp.perm = P.perm, tp.gperm = P.gperm, tp.k = L->k;
      tp.pexp = P.pexp, tp.box_rows = wd;
      // fused gate-weighted scatter-add into out, or (deterministic) one row per entry for the combine
      tp.out = out, tp.y = L->deterministic ? P.y : nullptr;
      tp.h = nullptr, tp.F = L->F, tp.d = L->d, tp.err = L->err;
      if (make_tmap_2d(&tp.bmap, P.h, 0, int64_t(T) * L->k, L->F, wd) != SCION_OK)
        return cudaErrorInvalidValue;
      const dim3 grid(num_sms());
#define SCION_DOWN(F, W) tern_gemm_kernel<F, 1, W><<<grid, kTernThreads, tern_smem(1, F, W), s>>>(tp)
      if (L->fmt == SCION_PQ2_0)
        wd == kBN3 ? SCION_DOWN(SCION_PQ2_0, kBN3) : SCION_DOWN(SCION_PQ2_0, kBN);
      else
        wd == kBN3 ? SCION_DOWN(SCION_PTQ1_0, kBN3) : SCION_DOWN(SCION_PTQ1_0, kBN);
#undef SCION_DOWN
      return cudaGetLastError();
    }
    default:
      return cudaErrorInvalidValue;
  }
}

// ---------------------------------------- correction branch on the attention output
// Tensor-core path: v -> fp16 (PTQ1_0 column order, no per-position factors) with the range
// exponents, z = A v into hz (A bf16 against v bf16, or packed A's exact fp16 copy in the same
// column order against v16), then out = base + B z with B's fp16 copy.
int corr_prefill_setup(CorrState* C, cudaStream_t s) {
  std::vector<DenseUnit> uz, uo;
  for (int r0 = 0; r0 < C->r; r0 += 128) uz.push_back(DenseUnit{kEpiPlain, 1, 0, 4, 4, r0, C->r, 0, C->packed});
  for (int r0 = 0; r0 < C->d_out; r0 += 128) uo.push_back(DenseUnit{kEpiStore, 1, 0, 5, 5, r0, C->d_out, 0, 0});
  C->n_units_z = int(uz.size()), C->n_units_o = int(uo.size());
  int st;
  if (cudaMalloc(&C->units_z, sizeof(DenseUnit) * uz.size()) != cudaSuccess) return SCION_ENOMEM;
  if (cudaMalloc(&C->units_o, sizeof(DenseUnit) * uo.size()) != cudaSuccess) return SCION_ENOMEM;
  C->device_bytes += sizeof(DenseUnit) * (uz.size() + uo.size());
  if (cudaMemcpyAsync(C->units_z, uz.data(), sizeof(DenseUnit) * uz.size(), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(C->units_o, uo.data(), sizeof(DenseUnit) * uo.size(), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)  // the host vectors go out of scope
    return SCION_ECUDA;
  if (C->packed) {
    if ((st = make_tmap_2d(&C->map_a, C->a16, 0, C->r, C->d_in))) return st;
  } else if ((st = make_tmap_2d(&C->map_a, C->a, 1, C->r, C->d_in))) {
    return st;
  }
  if ((st = make_tmap_2d(&C->map_b16, C->b16, 0, C->d_out, C->Kd))) return st;
  if ((st = make_tmap_2d(&C->map_v16, C->v16, 0, C->max_tokens, C->d_in))) return st;
  return make_tmap_2d(&C->map_hz, C->hz, 0, C->max_tokens, C->Kd);
}

cudaError_t launch_corr_prefill(const CorrState* C, const __nv_bfloat16* v, int T, const float* base, float* out,
                                cudaStream_t s) {
  const unsigned grid = unsigned(std::min((T + 7) / 8, num_sms() * 8));
  x16_kernel<SCION_PTQ1_0><<<grid, 256, 0, s>>>(v, T, C->d_in, C->v16, C->xexp, 0, nullptr, nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  DenseParams dp;
  memset(&dp, 0, sizeof(dp));
  dp.a[4] = C->map_a, dp.a[5] = C->map_b16;
  if (!C->packed && make_tmap_2d(&dp.b, v, 1, T, C->d_in) != SCION_OK) return cudaErrorInvalidValue;
  dp.b16 = C->map_v16;
  dp.units = static_cast<const DenseUnit*>(C->units_z), dp.n_units = C->n_units_z, dp.n_units2 = 0;
  dp.K = C->d_in, dp.T = T, dp.ab_bf16 = 1;
  dp.hz = C->hz, dp.ld_hz = C->Kd, dp.xexp = C->xexp, dp.z_only = 1, dp.err = C->err;
  dense_gemm_kernel<<<dense_grid(dp), kThreads, kDenseSmem, s>>>(dp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  DenseParams dq;
  memset(&dq, 0, sizeof(dq));
  dq.a[5] = C->map_b16, dq.b = C->map_hz;
  dq.units = static_cast<const DenseUnit*>(C->units_o), dq.n_units = C->n_units_o, dq.n_units2 = 0;
  dq.K = C->Kd, dq.T = T, dq.ab_bf16 = 0;
  dq.out = out, dq.ld_out = C->d_out, dq.resid = base, dq.xexp = C->xexp, dq.z_only = 1, dq.err = C->err;
  dense_gemm_kernel<<<dense_grid(dq), kThreads, kDenseSmem, s>>>(dq);
  return cudaGetLastError();
}

}  // namespace scion
