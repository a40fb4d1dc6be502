// k_tdec.cu -- the expert GEMMs of decode batches on the 5th-generation tensor cores.
//
// Same arithmetic as the other expert kernels ("Scion-35B-A3B" and "Scion-FlashNext-176B-A6B"
// model cards, Weight Representation: codes in {-1, 0, +1} with one fp16 scale per 128 weights;
// "Scion: ternary MoE quantization with trained corrections", Serving notes: k experts per
// token), shaped for decode batches, where an active expert sees a few tokens and the kernel is
// bound by streaming its codes:
//
//  * work item = (tile of up to 16 tokens of one expert, 128 weight rows); the routing lists the
//    tiles.  A persistent CTA walks items; codes arrive by bulk copy, one 128 x 128 group of each
//    matrix per stage.
//  * eight expansion warps turn each group into the MMA's A operand straight in tensor memory,
//    one weight row per TMEM lane, at one instruction per two weights: PQ2_0 fields are masked
//    into fp16 subnormals b 4^f 2^-24 (b = code + 1, the B operand carries 4^-f), PTQ1_0 digits
//    come out of the base-3 digit chain as exact fp16 codes.  No scale is applied here.
//  * one thread issues tcgen05.mma (M = 128 rows, N = 16 tokens, K = 128) per group into its own
//    accumulator slot; the epilogue warps fold each group into registers as
//    acc += scale(row, group) * (2^24 D - X) (PQ2_0, X = the group sum of the B row) or
//    acc += scale * D (PTQ1_0), then finish the item: SwiGLU into the hidden rows (gate/up, with
//    their group sums for the down projection) or the gate-weighted 16-byte fp32 reductions into
//    out (down).
#include "tc_common.cuh"
#include "tc_order.cuh"

namespace scion {
namespace {

using namespace tc;

constexpr int kTN = kDecTile;     // tokens per tile = the MMA N
constexpr int kTdThreads = 512;   // warp 0 codes, 1 MMA, 2-3 B rows, 4-11 expansion, 12-15 epilogue
constexpr int kTdEpi = 128;
constexpr float kTwo24 = 16777216.0f;

struct TdecParams {
  CUtensorMap bmap;      // down: B = hidden rows [T*k][F] (tcgen05 order), box {64 columns, 16 rows}
  const uint8_t* bank;   // re-tiled gate/up bank (NA = 2) or down bank (NA = 1)
  int G, R;              // 128-groups along K, rows per expert matrix
  const __half* bsrc;    // gate/up: x [T][d] in the tcgen05 order (fp16, x 2^s_t, PQ2_0: times 4^-f)
  int ldb;
  const int4* tiles;     // {expert, first token of the expert, tokens, first routed position}
  const int32_t* n_tiles;
  const int32_t* perm;
  int k;
  const float* gperm;    // gate of each routed position, times 2^(-2 s_t)
  const int32_t* pexp;   // range exponent of the token of each routed position
  const float* bsum;     // PQ2_0: group sums of the B rows times 4^f -- gate/up [T][G] by token, down [T*k][G] by position
  __half* h;             // gate/up: hidden rows [T*k][F] (tcgen05 order, PQ2_0 times 4^-f), h 2^(2 s_t)
  float* hsum;           // gate/up: their group sums [T*k][F/128] (PQ2_0)
  int F;
  float* out;            // down: out[t] += gate y
  int d;
  int* err;
};

template <int FMT, int NA>
struct TdRing {
  static constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  static constexpr uint32_t mat_bytes = 8 * tb;     // one 128-row x 128-column group of one matrix
  static constexpr uint32_t c_bytes = NA * mat_bytes;
  static constexpr int kC = 8;                      // code stages
  static constexpr uint32_t b_kblock = kTN * 128;   // one 64-column K block of 16 token rows (128B swizzle)
  static constexpr uint32_t b_bytes = 2 * b_kblock;
  static constexpr int kB = 8;                      // B stages
  static constexpr int kD = 4;                      // accumulator slots, one group each
  static constexpr uint32_t d_cols = NA * kTN;
  static constexpr uint32_t a_cols = NA * 64;       // one group of all matrices (128 fp16 per lane each)
  static constexpr uint32_t a_col0 = kD * d_cols;
  static constexpr int kA = int((512 - a_col0) / a_cols);
  static constexpr uint32_t b_off = 0, c_off = kB * b_bytes, e_off = c_off + kC * c_bytes;
  static constexpr uint32_t bytes = e_off + 4 * kTN * 32 * 4;  // epilogue staging of the down reductions
  static_assert(kA >= 2, "TMEM budget");
};

__device__ __forceinline__ int4 load_td_tile(const int4* tiles, int i) { return __ldg(tiles + i); }

// PQ2_0: half h (64 columns) of row t of one 128-row group (sub-tile blocks in shared memory)
// as fp16 subnormal pairs b 4^f 2^-24, in the tcgen05 position order (v[i] = positions 2i, 2i+1).
__device__ __forceinline__ void expand_pq2_sub(uint32_t codes, int t, int h, uint32_t (&out)[32]) {
  const uint32_t blk = codes + (t >> 4) * kPq2Tile;
  const int rho = t & 15, r8 = rho & 7, hi = rho >> 3;
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = 2 * h + cc;  // container code bytes 8c .. 8c+7
    const uint2 w2 = lds_v2(blk + 16 * (4 * r8 + c) + 8 * hi);
#pragma unroll
    for (int hw = 0; hw < 2; ++hw) {
      const uint32_t w = hw ? w2.y : w2.x, w10 = w >> 10;
      const int j0 = 2 * (2 * cc + hw);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int f = s < 5 ? s : s - 5;
        out[4 * j0 + s] = (s < 5 ? w : w10) & (0x00030003u << (2 * f));
      }
    }
  }
}

// PTQ1_0: half h of row t as exact fp16 codes (digit - 1) in the tcgen05 position order.
__device__ __forceinline__ void expand_ptq1_codes(uint32_t codes, int t, int h, uint32_t (&v)[32]) {
  const uint32_t blk = codes + (t >> 4) * kPtq1Tile;
  const int rho = t & 15, r8 = rho & 7, hi = rho >> 3;
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
      const __half2 Vn = __hfma2(V, third, c1);
      v[5 * i + j] = h2_as_u32(__hadd2(__hfma2(Vn, m3, V), c2047));
      V = Vn;
    }
  }
  // remainder trits (columns 120..127) as 2-bit fields: bytes (even trits, odd trits) of this row
  const uint32_t x = (lds_u32(blk + 384 + 4 * r8) >> (8 * hi)) & 0x00ff00ffu;
  v[30] = ptq1_rem_pair(x, 4 * h);
  v[31] = ptq1_rem_pair(x, 4 * h + 2);
}

// fp16 group scale of row t of a 128-row group of one matrix, from the re-tiled bank in global memory.
template <int FMT>
__device__ __forceinline__ float row_scale(const uint8_t* grp, int t) {
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  constexpr int soff = FMT == SCION_PQ2_0 ? 512 : 416;
  const int rho = t & 15;
  return __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short*>(
      grp + (t >> 4) * tb + soff + 4 * (rho & 7) + 2 * (rho >> 3)))));
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

template <int FMT, int NA>
__global__ void __launch_bounds__(kTdThreads, 1) tdec_kernel(const __grid_constant__ TdecParams p) {
  using R = TdRing<FMT, NA>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1024-aligned
  __shared__ uint64_t c_full[R::kC], c_empty[R::kC], a_full[R::kA], a_empty[R::kA], b_full[R::kB], b_empty[R::kB];
  __shared__ uint64_t d_full[R::kD], d_empty[R::kD], mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int RT = p.R >> 7;
  const int64_t grp_stride = int64_t(R::c_bytes);

  if (threadIdx.x == 0) {
    for (int i = 0; i < R::kC; ++i) mbar_init(&c_full[i], 1), mbar_init(&c_empty[i], 256);
    for (int i = 0; i < R::kA; ++i) mbar_init(&a_full[i], 256), mbar_init(&a_empty[i], 1);
    for (int i = 0; i < R::kB; ++i) mbar_init(&b_full[i], NA == 1 ? 1 : 64), mbar_init(&b_empty[i], 1);
    for (int i = 0; i < R::kD; ++i) mbar_init(&d_full[i], 1), mbar_init(&d_empty[i], kTdEpi);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the prologue above overlaps the previous kernel's tail; everything below reads its outputs
  pdl_trigger();
  pdl_wait();
  const int n_items = *p.n_tiles * RT;
  const uint32_t tmem = tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // ---------------- packed code groups, one bulk copy per matrix
    if (lane == 0) {
      int gs = 0;
      for (int item = blockIdx.x; item < n_items && !abort_flag; item += gridDim.x) {
        const int4 tile = load_td_tile(p.tiles, item / RT);
        const uint8_t* ebase = p.bank + (int64_t(tile.x) * RT + item % RT) * p.G * grp_stride;
        for (int g = 0; g < p.G; ++g, ++gs) {
          const int s = gs % R::kC;
          if (gs >= R::kC && !mbar_wait(&c_empty[s], ((gs / R::kC) - 1) & 1, &abort_flag, p.err)) break;
          uint8_t* dst = smem + R::c_off + s * R::c_bytes;
          mbar_arrive_expect_tx(&c_full[s], R::c_bytes);
#pragma unroll
          for (int m = 0; m < NA; ++m)
            bulk_load(dst + m * R::mat_bytes, ebase + g * grp_stride + m * R::mat_bytes, R::mat_bytes, &c_full[s]);
        }
      }
      for (int i = max(0, gs - R::kC); i < gs; ++i) mbar_drain(&c_full[i % R::kC], (i / R::kC) & 1);
    }
  } else if (NA == 1 && warp == 2) {
    // ---------------- down: the tile's hidden rows (routed positions), two 16-row TMA boxes per group
    if (lane == 0) {
      int gs = 0;
      for (int item = blockIdx.x; item < n_items && !abort_flag; item += gridDim.x) {
        const int pos0 = load_td_tile(p.tiles, item / RT).w;
        for (int g = 0; g < p.G; ++g, ++gs) {
          const int s = gs % R::kB;
          if (gs >= R::kB && !mbar_wait(&b_empty[s], ((gs / R::kB) - 1) & 1, &abort_flag, p.err)) break;
          uint8_t* dst = smem + R::b_off + s * R::b_bytes;
          mbar_arrive_expect_tx(&b_full[s], R::b_bytes);
          tma_load_2d(dst, &p.bmap, g * 128, pos0, &b_full[s]);
          tma_load_2d(dst + R::b_kblock, &p.bmap, g * 128 + 64, pos0, &b_full[s]);
        }
      }
      for (int i = max(0, gs - R::kB); i < gs; ++i) mbar_drain(&b_full[i % R::kB], (i / R::kB) & 1);
    }
  } else if (NA == 2 && (warp == 2 || warp == 3)) {
    // ---------------- gate/up: the tile's x rows gathered with cp.async, 16 rows x 256 bytes per
    // group; thread j copies 16-byte chunks 4 (j & 3) .. + 3 of row j >> 2
    const int j = threadIdx.x - 64, r = j >> 2, q4 = j & 3;
    constexpr int kLag = R::kB / 2;
    int gs = 0;
    for (int item = blockIdx.x; item < n_items && !abort_flag; item += gridDim.x) {
      const int4 tile = load_td_tile(p.tiles, item / RT);
      const __half* row = r < tile.z ? p.bsrc + int64_t(p.perm[tile.w + r] / p.k) * p.ldb : nullptr;
      for (int g = 0; g < p.G; ++g, ++gs) {
        const int s = gs % R::kB;
        if (gs >= R::kB && !mbar_wait(&b_empty[s], ((gs / R::kB) - 1) & 1, &abort_flag, p.err)) break;
        if (row) {
          const uint32_t bt = sbase + R::b_off + s * R::b_bytes;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int ch = 4 * q4 + cc;  // 16-byte chunk of the group row (8 columns)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(bt + (ch >> 3) * R::b_kblock +
                                                                             sw128_offset(r, ch & 7)),
                         "l"(row + g * 128 + 8 * ch)
                         : "memory");
          }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
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
    // ---------------- MMA issuer: A from tensor memory, B from shared memory, one slot per group
    if (lane == 0) {
      const uint32_t idesc = umma_idesc(128, kTN, 0);
      int gs = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok && !abort_flag; item += gridDim.x) {
        for (int g = 0; g < p.G && ok; ++g, ++gs) {
          const int sa = gs % R::kA, sb = gs % R::kB, sd = gs % R::kD;
          // A expanded and (folded into its arrival) B landed; the accumulator slot drained
          if (!(ok = mbar_wait(&a_full[sa], (gs / R::kA) & 1, &abort_flag, p.err))) break;
          if (gs >= R::kD && !(ok = mbar_wait(&d_empty[sd], ((gs / R::kD) - 1) & 1, &abort_flag, p.err))) break;
          tc_fence_after();
          const uint32_t bt = sbase + R::b_off + sb * R::b_bytes;
          const uint32_t at = tmem + R::a_col0 + sa * R::a_cols, dt = tmem + sd * R::d_cols;
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16) {
            const uint64_t db = umma_desc_sw128(bt + (k16 >> 2) * R::b_kblock + 32 * (k16 & 3));
#pragma unroll
            for (int m = 0; m < NA; ++m) umma_ts(dt + m * kTN, at + m * 64 + 8 * k16, db, idesc, k16 != 0);
          }
          umma_commit(&a_empty[sa]);
          umma_commit(&b_empty[sb]);
          umma_commit(&d_full[sd]);
        }
      }
      umma_commit(&mma_done);
      mbar_drain(&mma_done, 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------- expansion: NA = 2: warpgroup wg expands matrix wg (both halves of each row);
    // NA = 1: warpgroup wg expands half wg of the single matrix.  Thread t = weight row t = TMEM lane t.
    const int wg = (warp - 4) >> 2;
    const int t = (threadIdx.x - 128) & 127;
    const bool b_watch = wg == 0 && t == 0;  // this thread also waits for the group's B rows
    const uint32_t lane_base = tmem + (uint32_t((warp & 3) * 32) << 16) + R::a_col0;
    int gs = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok && !abort_flag; item += gridDim.x) {
      for (int g = 0; g < p.G && ok; ++g, ++gs) {
        const int sc = gs % R::kC, sa = gs % R::kA;
        if (!(ok = mbar_wait(&c_full[sc], (gs / R::kC) & 1, &abort_flag, p.err))) break;
        if (gs >= R::kA && !(ok = mbar_wait(&a_empty[sa], ((gs / R::kA) - 1) & 1, &abort_flag, p.err))) break;
        tc_fence_after();
        const uint32_t codes = sbase + R::c_off + sc * R::c_bytes;
        uint32_t v[32];
        if constexpr (NA == 2) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if constexpr (FMT == SCION_PQ2_0)
              expand_pq2_sub(codes + wg * R::mat_bytes, t, hh, v);
            else
              expand_ptq1_codes(codes + wg * R::mat_bytes, t, hh, v);
            tmem_st32(lane_base + sa * R::a_cols + wg * 64 + hh * 32, v);
          }
        } else {
          if constexpr (FMT == SCION_PQ2_0)
            expand_pq2_sub(codes, t, wg, v);
          else
            expand_ptq1_codes(codes, t, wg, v);
          tmem_st32(lane_base + sa * R::a_cols + wg * 32, v);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&c_empty[sc]);
        if (b_watch && !(ok = mbar_wait(&b_full[gs % R::kB], (gs / R::kB) & 1, &abort_flag, p.err))) break;
        mbar_arrive(&a_full[sa]);
      }
    }
  } else if (warp >= 12) {
    // ---------------- epilogue: thread = weight row (TMEM lane quarter q); per group it folds the
    // accumulator slot into registers with the row's group scale, then finishes the item
    const int q = warp & 3, row = q * 32 + lane;
    const int pcol = perm_pos(FMT, row);  // gate/up: position of this row inside its 128-column group of h
    const float hscale = FMT == SCION_PQ2_0 ? pq2_pos_scale(pcol) : 1.0f;
    int gs = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int4 tile = load_td_tile(p.tiles, item / RT);
      const int e = tile.x, nn = tile.z, pos0 = tile.w, rt = item % RT;
      const uint8_t* ebase = p.bank + (int64_t(e) * RT + rt) * p.G * grp_stride;
      // lane i < nn holds token i's position data
      const int my_pos = pos0 + min(lane, nn - 1);
      const int my_brow = NA == 2 ? p.perm[my_pos] / p.k : my_pos;  // row of the group sums
      float acc[NA][kTN];
#pragma unroll
      for (int m = 0; m < NA; ++m)
#pragma unroll
        for (int i = 0; i < kTN; ++i) acc[m][i] = 0.f;
      // the row's group scales and the tokens' group sums, kPre groups ahead (their loads from L2
      // are in flight while the earlier groups are folded)
      constexpr int kPre = 4;
      float scq[kPre][NA], xgq[kPre];
#pragma unroll
      for (int j = 0; j < kPre; ++j) {
#pragma unroll
        for (int m = 0; m < NA; ++m)
          scq[j][m] = j < p.G ? row_scale<FMT>(ebase + j * grp_stride + m * R::mat_bytes, row) : 0.f;
        xgq[j] = (FMT == SCION_PQ2_0 && j < p.G) ? p.bsum[int64_t(my_brow) * p.G + j] : 0.f;
      }
      for (int g = 0; g < p.G; ++g, ++gs) {
        const int sd = gs % R::kD;
        float sc[NA], xg;
        // rotate the prefetch ring (static indices: the ring shifts by one each group)
#pragma unroll
        for (int m = 0; m < NA; ++m) sc[m] = scq[0][m];
        xg = xgq[0];
#pragma unroll
        for (int j = 0; j + 1 < kPre; ++j) {
#pragma unroll
          for (int m = 0; m < NA; ++m) scq[j][m] = scq[j + 1][m];
          xgq[j] = xgq[j + 1];
        }
        {
          const int gn = g + kPre;
#pragma unroll
          for (int m = 0; m < NA; ++m)
            scq[kPre - 1][m] = gn < p.G ? row_scale<FMT>(ebase + gn * grp_stride + m * R::mat_bytes, row) : 0.f;
          xgq[kPre - 1] = (FMT == SCION_PQ2_0 && gn < p.G) ? p.bsum[int64_t(my_brow) * p.G + gn] : 0.f;
        }
        // no abort-flag test: the epilogue threads leave only together, by the vote
        if (!(ok = named_bar_and(1, kTdEpi, mbar_wait(&d_full[sd], (gs / R::kD) & 1, &abort_flag, p.err)))) break;
        tc_fence_after();
        float dv[NA][16];
        const uint32_t dt = tmem + (uint32_t(q * 32) << 16) + sd * R::d_cols;
        if constexpr (NA == 2)
          tmem_ld16x2(dt, dt + kTN, dv[0], dv[1]);
        else
          tmem_ld16(dt, dv[0]);
        tc_fence_before();
        mbar_arrive(&d_empty[sd]);
#pragma unroll
        for (int i = 0; i < kTN; ++i) {
          if (i >= nn) break;  // the tile's tokens only (nn is the same for the whole warp)
          if constexpr (FMT == SCION_PQ2_0) {
            const float x = __shfl_sync(0xffffffffu, xg, i);  // group sum of token i's B row
#pragma unroll
            for (int m = 0; m < NA; ++m) acc[m][i] = fmaf(sc[m], fmaf(dv[m][i], kTwo24, -x), acc[m][i]);
          } else {
#pragma unroll
            for (int m = 0; m < NA; ++m) acc[m][i] = fmaf(sc[m], dv[m][i], acc[m][i]);
          }
        }
      }
      if (!ok) break;
      const int my_sh = p.pexp[my_pos];
      if constexpr (NA == 2) {
        // SwiGLU of the scaled sums (h 2^(2 s_t)), stored in the tcgen05 order of the down projection
        __half* dst = p.h + int64_t(pos0) * p.F + int64_t(rt) * 128 + pcol;
#pragma unroll
        for (int i = 0; i < kTN; ++i) {
          const int sh = __shfl_sync(0xffffffffu, my_sh, i);
          const __half hv = __float2half_rn(silu_f(acc[0][i] * pow2i(-sh)) * (acc[1][i] * pow2i(sh)) * hscale);
          if (i < nn) dst[int64_t(i) * p.F] = hv;
          if (FMT == SCION_PQ2_0) {
            // the hidden row's group sum (B values times 4^f) over this item's 128 rows = one group
            float hs = i < nn ? __half2float(hv) / hscale : 0.f;
#pragma unroll
            for (int o = 16; o; o >>= 1) hs += __shfl_xor_sync(0xffffffffu, hs, o);
            if (lane == 0 && i < nn) atomicAdd(p.hsum + int64_t(pos0 + i) * (p.F >> 7) + rt, hs);
          }
        }
      } else {
        // gate-weighted scatter-add through shared memory as (token, 4 rows) 16-byte reductions
        const float my_g = p.gperm[my_pos];
        const int my_t = p.perm[my_pos] / p.k;
        float* ts = reinterpret_cast<float*>(smem + R::e_off) + q * (kTN * 32);
#pragma unroll
        for (int i = 0; i < kTN; ++i) ts[i * 32 + lane] = acc[0][i];
        __syncwarp();
#pragma unroll
        for (int j = 0; j < kTN / 4; ++j) {
          const int i = (lane >> 3) + 4 * j, g4 = lane & 7;
          const float gi = __shfl_sync(0xffffffffu, my_g, i);
          const int ti = __shfl_sync(0xffffffffu, my_t, i);
          if (i < nn) {
            const float4 w = *reinterpret_cast<const float4*>(ts + i * 32 + 4 * g4);
            red_add_v4(p.out + int64_t(ti) * p.d + int64_t(rt) * 128 + q * 32 + 4 * g4, gi * w.x, gi * w.y, gi * w.z,
                       gi * w.w);
          }
        }
        __syncwarp();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int num_sms_td() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <int FMT, int NA>
constexpr size_t td_smem() {
  return TdRing<FMT, NA>::bytes + 1024;
}

}  // namespace

cudaError_t configure_tdec_kernels() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(tdec_kernel<SCION_PQ2_0, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(td_smem<SCION_PQ2_0, 2>()))))
    return e;
  if ((e = cudaFuncSetAttribute(tdec_kernel<SCION_PQ2_0, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(td_smem<SCION_PQ2_0, 1>()))))
    return e;
  if ((e = cudaFuncSetAttribute(tdec_kernel<SCION_PTQ1_0, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(td_smem<SCION_PTQ1_0, 2>()))))
    return e;
  return cudaFuncSetAttribute(tdec_kernel<SCION_PTQ1_0, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(td_smem<SCION_PTQ1_0, 1>()));
}

cudaError_t launch_tdec(int na, const scion_layer* L, int T, float* out, cudaStream_t s) {
  TdecParams p;
  memset(&p, 0, sizeof(p));
  p.tiles = static_cast<const int4*>(L->dtiles), p.n_tiles = L->n_dtiles;
  p.perm = L->perm, p.k = L->k, p.gperm = L->gperm, p.pexp = L->pexp, p.F = L->F, p.d = L->d, p.err = L->err;
  if (na == 2) {
    p.bank = L->gu_bank, p.G = L->Gd, p.R = L->F, p.bsrc = L->x16d, p.ldb = L->d, p.bsum = L->xsum;
    p.h = L->hp, p.hsum = L->hsum;
  } else {
    p.bank = L->dn_bank, p.G = L->GF, p.R = L->d, p.bmap = L->hp_map, p.bsum = L->hsum, p.out = out;
  }
  const int Tk = T * L->k;
  const int max_tiles = Tk / kDecTile + std::min(L->El, Tk);
  const int items = max_tiles * (p.R / 128);
  const dim3 grid(std::max(1, std::min(items, num_sms_td())));
#define SCION_TD(F, NA) return launch_pdl(tdec_kernel<F, NA>, grid, dim3(kTdThreads), td_smem<F, NA>(), s, p)
  if (L->fmt == SCION_PQ2_0) {
    if (na == 2) SCION_TD(SCION_PQ2_0, 2);
    SCION_TD(SCION_PQ2_0, 1);
  }
  if (na == 2) SCION_TD(SCION_PTQ1_0, 2);
  SCION_TD(SCION_PTQ1_0, 1);
#undef SCION_TD
}

}  // namespace scion
