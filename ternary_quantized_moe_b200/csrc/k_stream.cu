// k_stream.cu -- expert kernels for batches of up to 64 tokens, fed by a TMA bulk-copy ring.
//
// Same arithmetic as the register-fed decode kernels (k_decode.cu): the expert SwiGLU
// gate/up and the gate-weighted down projection over ternary codes ("Scion-35B-A3B" and
// "Scion-FlashNext-176B-A6B" model cards, Weight Representation; "Scion: ternary MoE
// quantization with trained corrections", Serving notes: k experts per token).
//
// Work item = one active expert x 128 weight rows; a persistent CTA walks many.  In the
// re-tiled bank the 128 x 128 codes of one group (gate and up interleaved for the gate/up
// bank) are one contiguous block and consecutive groups follow each other, so a producer
// warp streams GPS groups per stage with one cp.async.bulk into an mbarrier ring, together
// with the fragment-ordered B rows (x or h, plus their group-sum tails) of the item's tokens.
// Eight consumer warps each own a 16-row sub-tile over the whole K range: codes come from
// shared memory, are unpacked in registers into mma.sync fragments (PQ2_0 as fp16
// subnormals, PTQ1_0 through the base-3 digit chain), and no cross-warp reduction is needed.
#include "tc_common.cuh"
#include "tern_tile.cuh"

namespace scion {
namespace {

using namespace tc;

constexpr int kRing = 4;    // stages in flight (two CTAs per SM; three CTAs of a three-stage ring
                            // measured slower)
constexpr int kCons = 8;    // consumer warps (one 16-row sub-tile each)
constexpr int kTok = 8;     // tokens per pass (one mma n-tile)
constexpr int kRowB = SCION_BROW * 2;  // bytes of one token's 128-column group row (fp16 + sum tail)
constexpr int kHdr = 256;   // stage header
constexpr float kTwoP24 = 16777216.0f;  // 2^24

// Written by the producer into every stage; the consumers are driven by it alone.
struct StageHdr {
  int nn;     // tokens of the pass (1..kTok); -1: no more work for this CTA
  int flags;  // bit 0: first stage of the pass, bit 1: last stage of the pass
  int rb;     // 128-row block of the item
  int ng;     // 128-column groups in this stage (1..GPS)
  int pos[kTok];     // gate/up: routed positions of the pass's tokens (last stage only)
  int orow[kTok];    // down: output token row (entry / k)
  float gate[kTok];  // down: gate of the entry times 2^(-2 s_t) (the hidden is h 2^(2 s_t))
};
static_assert(sizeof(StageHdr) <= kHdr, "stage header");

struct StreamArgs {
  const uint8_t* bank;
  const __half* bsrc;  // gate/up: xfrag [T][Gd][SCION_BROW]; down: h [T*k][GF][SCION_BROW]
  int bld;             // 128-column groups per B row (Gd or GF)
  const int4* slot_info;
  const int32_t *n_active, *perm;
  const float* gperm;  // gate of each routed position, times 2^(-2 s_t)
  const int32_t* pexp; // range exponent s_t of the token of each routed position
  const int32_t* any_scaled;  // nonzero when some token of the batch has s_t != 0 (written by the routing)
  int G, R, k, F, d, fmt;
  __half* hfrag;  // gate/up output
  float* out;     // down output
  int* err;
};

struct TokInfo {
  int pos, brow, orow;
  float gate;
};

// Groups per stage: two for the gate/up bank (each group holds both matrices), four for down.
template <int NMAT>
constexpr int gps() {
  return NMAT == 2 ? 2 : 4;
}
template <int FMT, int NMAT>
constexpr uint32_t code_bytes() {
  return NMAT * 8 * (FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile);
}
// B rows in a stage: token n at n * tok_stride + 16 * (n / 2).  The stride is 64 (mod 128)
// bytes, so tokens n and n + 1 fall on opposite halves of the shared-memory banks (a 16-byte
// load of lanes (n, 0..3) and (n + 1, 0..3) is conflict-free), and the 16-byte skew spreads the
// group-sum tails of tokens 0, 2, 4, 6 over different banks.
template <int NMAT>
constexpr uint32_t tok_stride() {
  return (gps<NMAT>() * kRowB + 63) / 128 * 128 + 64;
}
__device__ __forceinline__ uint32_t tok_off(uint32_t stride, int n) { return n * stride + 16 * (n >> 1); }
template <int FMT, int NMAT>
constexpr uint32_t stage_bytes() {
  return kHdr + gps<NMAT>() * code_bytes<FMT, NMAT>() + kTok * tok_stride<NMAT>() + 64;
}

// mma.sync m16n8k16 (fp16 in, fp32 accumulate) without `volatile`, so that independent
// accumulation chains of several tiles can be interleaved by the compiler.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Predicated shared-memory loads: lanes whose token lies past the pass's count issue no bank
// access and keep the old register contents (their accumulator columns are dropped later).
// lds_brow_if: the lane's 64 bytes of one B group row (four 16-byte chunks 64 bytes apart)
// under one predicate.
__device__ __forceinline__ void lds_brow_if(uint32_t (&r)[16], uint32_t addr, bool p) {
  asm volatile(
      "{\n .reg .pred q;\n setp.ne.u32 q, %17, 0;\n"
      " @q ld.shared.v4.u32 {%0,%1,%2,%3}, [%16];\n"
      " @q ld.shared.v4.u32 {%4,%5,%6,%7}, [%16+64];\n"
      " @q ld.shared.v4.u32 {%8,%9,%10,%11}, [%16+128];\n"
      " @q ld.shared.v4.u32 {%12,%13,%14,%15}, [%16+192];\n}\n"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
      : "r"(addr), "r"(uint32_t(p)));
}
__device__ __forceinline__ float ldsf_if(uint32_t addr, bool p) {
  float v = 0.f;
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %2, 0;\n @q ld.shared.f32 %0, [%1];\n}\n"
               : "+f"(v)
               : "r"(addr), "r"(uint32_t(p)));
  return v;
}

// Per-lane shared-memory offsets within a stage (loop invariant).
struct LaneOffs {
  uint32_t code;   // this warp's tile of matrix 0, lane's 16 bytes
  uint32_t scale;  // this warp's tile of matrix 0, the scales of rows r, r + 8
  uint32_t brow;   // B row of token n, lane-column c
  uint32_t tail0, tail1;  // group-sum tails of tokens 2c, 2c + 1
};

// First MMA of a chain: d = a b + c with c in other registers (no copies into the accumulator).
__device__ __forceinline__ void mma_f16_c(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, float c0,
                                          float c1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%10,%11};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c0), "f"(c1));
}

// One stage's groups [j0, j0 + J) for this warp: J x NMAT independent PQ2_0 tiles (subnormal
// unpack, accumulators started at the group-sum tails) or PTQ1_0 tiles (digit chain).
template <int FMT, int NMAT, int J>
__device__ __forceinline__ void stage_groups(uint32_t stg, const LaneOffs& o, int j0, int nn, int lane,
                                             float (&acc)[NMAT][4]) {
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  constexpr uint32_t cb = code_bytes<FMT, NMAT>();
  const int c = lane & 3, n = lane >> 2;
  uint32_t b[J][16];
#pragma unroll
  for (int j = 0; j < J; ++j) lds_brow_if(b[j], stg + o.brow + (j0 + j) * kRowB, n < nn);
  if constexpr (FMT == SCION_PQ2_0) {
    uint4 w[J][NMAT];
    uint32_t sc[J][NMAT];
    float g[J][NMAT][4], xn[J][2];
#pragma unroll
    for (int j = 0; j < J; ++j) {
      // -2^-24 * group sums of the lane's token columns 2c, 2c+1: the chains' start values
      xn[j][0] = ldsf_if(stg + o.tail0 + (j0 + j) * kRowB, 2 * c < nn);
      xn[j][1] = ldsf_if(stg + o.tail1 + (j0 + j) * kRowB, 2 * c + 1 < nn);
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        const uint32_t blk = stg + (j0 + j) * cb + m * 8 * tb;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(w[j][m].x), "=r"(w[j][m].y), "=r"(w[j][m].z), "=r"(w[j][m].w)
                     : "r"(blk + o.code));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(sc[j][m]) : "r"(blk + o.scale));
      }
    }
    uint32_t w10[J][NMAT][4];
#pragma unroll
    for (int j = 0; j < J; ++j)
#pragma unroll
      for (int m = 0; m < NMAT; ++m)
        w10[j][m][0] = w[j][m].x >> 10, w10[j][m][1] = w[j][m].y >> 10, w10[j][m][2] = w[j][m].z >> 10,
        w10[j][m][3] = w[j][m].w >> 10;
#define SCION_SUB_FA(S)                                                                                  \
  const uint32_t fa[4] = {pq2_pair_sub<S>(w[j][m].x, w10[j][m][0]), pq2_pair_sub<S>(w[j][m].z, w10[j][m][2]), \
                          pq2_pair_sub<S>(w[j][m].y, w10[j][m][1]), pq2_pair_sub<S>(w[j][m].w, w10[j][m][3])};
#pragma unroll
    for (int j = 0; j < J; ++j)
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        SCION_SUB_FA(0)
        mma_f16_c(g[j][m], fa, b[j][0], b[j][1], xn[j][0], xn[j][1]);
      }
#define SCION_SUB_STEP(S)                                                                              \
  _Pragma("unroll") for (int j = 0; j < J; ++j) _Pragma("unroll") for (int m = 0; m < NMAT; ++m) {     \
    SCION_SUB_FA(S)                                                                                    \
    mma_f16(g[j][m], fa, b[j][2 * S], b[j][2 * S + 1]);                                                \
  }
    SCION_SUB_STEP(1) SCION_SUB_STEP(2) SCION_SUB_STEP(3)
    SCION_SUB_STEP(4) SCION_SUB_STEP(5) SCION_SUB_STEP(6) SCION_SUB_STEP(7)
#undef SCION_SUB_STEP
#undef SCION_SUB_FA
#pragma unroll
    for (int j = 0; j < J; ++j)
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        const float2 sf = __half22float2(u32_as_h2(sc[j][m]));  // scales of rows r, r + 8
        acc[m][0] = fmaf(sf.x, g[j][m][0], acc[m][0]);
        acc[m][1] = fmaf(sf.x, g[j][m][1], acc[m][1]);
        acc[m][2] = fmaf(sf.y, g[j][m][2], acc[m][2]);
        acc[m][3] = fmaf(sf.y, g[j][m][3], acc[m][3]);
      }
  } else {
    // all code words of the stage's tiles first, then the digit chains and MMAs
    TileRegs<SCION_PTQ1_0> t[J][NMAT];
#pragma unroll
    for (int j = 0; j < J; ++j)
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        t[j][m].load_shared(stg + (j0 + j) * cb + m * 8 * tb + o.code - 16 * lane, lane);
      }
#pragma unroll
    for (int j = 0; j < J; ++j)
#pragma unroll
      for (int m = 0; m < NMAT; ++m) tile_mma_ptq1_nv(t[j][m], b[j], acc[m], c);
  }
}

// Persistent: CTA b walks a contiguous range of the items, item = (active slot, 128-row
// block).  One producer warp streams, per stage, GPS groups of the item's codes and the
// fragment-ordered B rows of up to kTok tokens into a ring of stages, each with a header that
// tells the consumers what it holds.
template <int FMT, int NMAT>
__global__ void __launch_bounds__((kCons + 1) * 32, 2) stream_kernel(const __grid_constant__ StreamArgs a) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kRing], empty[kRing];
  __shared__ int abort_flag;
  constexpr int GPS = gps<NMAT>();
  constexpr uint32_t cb = code_bytes<FMT, NMAT>();
  constexpr uint32_t sb = stage_bytes<FMT, NMAT>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int RB = a.R >> 7;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) mbar_init(&full[s], 1), mbar_init(&empty[s], kCons);
    abort_flag = 0;
    fence_barrier_init();
  }
  pdl_trigger();
  pdl_wait();
  __syncthreads();

  if (warp == kCons) {
    // ---------------- producer (all 32 lanes: lane i carries token i of the pass)
    const int n_items = *a.n_active * RB;
    auto slot_rec = [&](int item) { return item < n_items ? a.slot_info[item / RB] : make_int4(0, 0, 0, 0); };
    auto tok_info = [&](int4 si, int pc) {
      TokInfo t{0, 0, 0, 0.f};
      if (lane < min(kTok, si.z - pc)) {
        t.pos = si.y + pc + lane;
        t.orow = a.perm[t.pos] / a.k;
        if (NMAT == 1) t.gate = a.gperm[t.pos];
        t.brow = NMAT == 2 ? t.orow : t.pos;
      }
      return t;
    };
    // this CTA's items are a contiguous range, so consecutive items mostly share their slot and
    // its token records (loaded again only when the slot changes); the next slot's record is
    // fetched one slot ahead
    const int i0 = int(int64_t(n_items) * blockIdx.x / gridDim.x);
    const int i1 = int(int64_t(n_items) * (blockIdx.x + 1) / gridDim.x);
    int cur_slot = i0 / RB;
    int4 si_cur = slot_rec(i0), si_nxt = slot_rec((cur_slot + 1) * RB);
    TokInfo tk_cur = tok_info(si_cur, 0);
    int st = 0;  // running stage counter
    bool ok = true;
    for (int item = i0; item < i1 && ok; ++item) {
      if (item / RB != cur_slot) {
        cur_slot = item / RB;
        si_cur = si_nxt;
        si_nxt = slot_rec((cur_slot + 1) * RB);
        tk_cur = tok_info(si_cur, 0);
      }
      const int rb = item % RB;
      const uint8_t* src0 = a.bank + (int64_t(si_cur.x) * RB + rb) * a.G * cb;
      for (int pc = 0; pc < si_cur.z && ok; pc += kTok) {
        const TokInfo tk = pc == 0 ? tk_cur : tok_info(si_cur, pc);
        const int nn = min(kTok, si_cur.z - pc);
        for (int g0 = 0; g0 < a.G; g0 += GPS, ++st) {
          const int ng = min(GPS, a.G - g0);
          const int s = st % kRing;
          if (lane == 0 && st >= kRing) ok = mbar_wait(&empty[s], ((st / kRing) - 1) & 1, &abort_flag, a.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          uint8_t* stg = ring + s * sb;
          StageHdr* hd = reinterpret_cast<StageHdr*>(stg);
          const bool last = g0 + GPS >= a.G;
          if (last) {
            // the epilogue's per-token records, written by lane 0 so its arrive publishes them
#pragma unroll
            // (the producer's per-stage work bounds the ring: only what the epilogue reads)
            for (int i = 0; i < kTok; ++i) {
              if constexpr (NMAT == 2) {
                const int pos = __shfl_sync(0xffffffffu, tk.pos, i);
                if (lane == 0) hd->pos[i] = pos;
              } else {
                const int orow = __shfl_sync(0xffffffffu, tk.orow, i);
                const float gate = __shfl_sync(0xffffffffu, tk.gate, i);
                if (lane == 0) hd->orow[i] = orow, hd->gate[i] = gate;
              }
            }
          }
          if (lane == 0) {
            hd->nn = nn;
            hd->flags = (g0 == 0 ? 1 : 0) | (last ? 2 : 0);
            hd->rb = rb;
            hd->ng = ng;
            mbar_arrive_expect_tx(&full[s], ng * cb + nn * ng * kRowB);
          }
          __syncwarp();
          if (lane == 0) bulk_load(stg + kHdr, src0 + int64_t(g0) * cb, ng * cb, &full[s]);
          if (lane < nn)
            bulk_load(stg + kHdr + GPS * cb + tok_off(tok_stride<NMAT>(), lane),
                      a.bsrc + (int64_t(tk.brow) * a.bld + g0) * SCION_BROW, ng * kRowB, &full[s]);
        }
      }
    }
    if (lane == 0) {
      if (ok) {
        // end-of-work sentinel (the consumers wait for every earlier stage before reaching it)
        const int s = st % kRing;
        if (st < kRing || mbar_wait(&empty[s], ((st / kRing) - 1) & 1, &abort_flag, a.err)) {
          reinterpret_cast<StageHdr*>(ring + s * sb)->nn = -1;
          mbar_arrive(&full[s]);
        }
      } else {
        // a wait gave up: copies of the last kRing stages may still be in flight; let them land
        // before the CTA can exit (no sentinel was issued, so these are the barriers' latest phases)
        for (int i = max(0, st - kRing); i < st; ++i) mbar_drain(&full[i % kRing], (i / kRing) & 1);
      }
    }
    return;
  }

  // ---------------- consumers: warp w owns rows 16w .. 16w+15 of every item
  const bool scaled = NMAT == 2 && *a.any_scaled != 0;
  const int c = lane & 3;
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  LaneOffs lo;
  lo.code = kHdr + warp * tb + 16 * lane;
  lo.scale = kHdr + warp * tb + 512 + 4 * (lane >> 2);
  lo.brow = kHdr + GPS * cb + tok_off(tok_stride<NMAT>(), lane >> 2) + 16 * c;
  lo.tail0 = kHdr + GPS * cb + tok_off(tok_stride<NMAT>(), 2 * c) + 256;
  lo.tail1 = kHdr + GPS * cb + tok_off(tok_stride<NMAT>(), 2 * c + 1) + 256;
  const uint32_t ring_u32 = smem_u32(ring);
  // epilogue constants of this lane's rows r = 16 warp + lane / 4 and r + 8 (the same in every
  // 128-row block): stored position of the row in the hidden's group row and its 4^-f factor
  int hpos[2];
  float hsc[2], hinv[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    hpos[h] = brow_pos(FMT, warp * 16 + (lane >> 2) + 8 * h);
    hsc[h] = FMT == SCION_PQ2_0 ? brow_bscale(hpos[h]) : 1.0f;
    hinv[h] = 1.0f / hsc[h];
  }
  float acc[NMAT][4];
  for (int st = 0;; ++st) {
    const int s = st % kRing;
    if (!mbar_wait(&full[s], (st / kRing) & 1, &abort_flag, a.err)) break;
    const uint8_t* stgp = ring + s * sb;
    const uint32_t stg = ring_u32 + s * sb;
    const StageHdr* hd = reinterpret_cast<const StageHdr*>(stgp);
    const int nn = hd->nn;
    if (nn < 0) break;
    const int flags = hd->flags, ng = hd->ng;
    if (flags & 1) {
#pragma unroll
      for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;
    }
    // one group at a time (taking two per call measured slower: more registers, less overlap)
#pragma unroll
    for (int j = 0; j < GPS; ++j)
      if (j < ng) stage_groups<FMT, NMAT, 1>(stg, lo, j, nn, lane, acc);
    if (flags & 2) {
      // epilogue: this warp's 16 rows x the pass's tokens
      const int rb = hd->rb;
      constexpr float unit = FMT == SCION_PQ2_0 ? kTwoP24 : 1.0f;  // undo the subnormal 2^-24
      float hs[2] = {0.f, 0.f};  // PQ2_0: this lane's share of the hidden group sums (tokens 2c, 2c+1)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = warp * 16 + (lane >> 2) + 8 * (i >> 1);
        const int tcol = 2 * c + (i & 1);
        if constexpr (NMAT == 2) {
          float h;
          if (!scaled) {
            h = silu_f(acc[0][i] * unit) * (acc[1][i] * unit) * hsc[i >> 1];
          } else {  // some token of the batch is range-scaled: the sums are of x 2^sh
            const int sh = tcol < nn ? a.pexp[hd->pos[tcol]] : 0;
            h = silu_f(acc[0][i] * unit * pow2i(-sh)) * (acc[1][i] * unit * pow2i(sh)) * hsc[i >> 1];
          }
          const __half h16 = __float2half_rn(h);
          if (tcol < nn) a.hfrag[(int64_t(hd->pos[tcol]) * (a.F >> 7) + rb) * SCION_BROW + hpos[i >> 1]] = h16;
          if (FMT == SCION_PQ2_0) hs[i & 1] += __half2float(h16) * hinv[i >> 1];
        } else {
          if (tcol < nn)
            atomicAdd(&a.out[int64_t(hd->orow[tcol]) * a.d + rb * 128 + row], hd->gate[tcol] * (acc[0][i] * unit));
        }
      }
      if constexpr (NMAT == 2 && FMT == SCION_PQ2_0) {
        // sum over the warp's 16 rows, then add -2^-24 x that into the hidden rows' group-sum tails
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          hs[0] += __shfl_xor_sync(0xffffffffu, hs[0], o);
          hs[1] += __shfl_xor_sync(0xffffffffu, hs[1], o);
        }
        if (lane < 4) {
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (2 * c + j < nn)
              atomicAdd(reinterpret_cast<float*>(a.hfrag + (int64_t(hd->pos[2 * c + j]) * (a.F >> 7) + rb) *
                                                               SCION_BROW + 128),
                        -hs[j] * (1.0f / kTwoP24));
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

template <int FMT, int NMAT>
constexpr size_t stream_smem() {
  return size_t(kRing) * stage_bytes<FMT, NMAT>();
}

template <int FMT, int NMAT>
int stream_ctas_per_sm() {
  static int n = 0;
  if (!n) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, stream_kernel<FMT, NMAT>, (kCons + 1) * 32,
                                                      stream_smem<FMT, NMAT>()) != cudaSuccess || n < 1)
      n = 1;
  }
  return n;
}

int num_sms_stream() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <int FMT, int NMAT>
cudaError_t launch_stream(const StreamArgs& a, int max_items, cudaStream_t s) {
  const int grid = max(1, min(max_items, stream_ctas_per_sm<FMT, NMAT>() * num_sms_stream()));
  return launch_pdl(stream_kernel<FMT, NMAT>, dim3(grid), dim3((kCons + 1) * 32), stream_smem<FMT, NMAT>(), s, a);
}

template <int FMT, int NMAT>
cudaError_t set_smem() {
  return cudaFuncSetAttribute(stream_kernel<FMT, NMAT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(stream_smem<FMT, NMAT>()));
}

}  // namespace

cudaError_t configure_stream_kernels() {
  cudaError_t e;
  if ((e = set_smem<SCION_PQ2_0, 2>())) return e;
  if ((e = set_smem<SCION_PQ2_0, 1>())) return e;
  if ((e = set_smem<SCION_PTQ1_0, 2>())) return e;
  return set_smem<SCION_PTQ1_0, 1>();
}

cudaError_t launch_stream_gateup(const scion_layer* L, int T, cudaStream_t s) {
  StreamArgs a;
  a.bank = L->gu_bank, a.bsrc = L->xfrag, a.bld = L->Gd;
  a.slot_info = reinterpret_cast<const int4*>(L->slot_info), a.n_active = L->n_active, a.perm = L->perm;
  a.gperm = L->gperm, a.pexp = L->pexp, a.any_scaled = L->any_scaled, a.G = L->Gd, a.R = L->F, a.k = L->k, a.F = L->F, a.d = L->d, a.fmt = L->fmt;
  a.hfrag = L->h, a.out = nullptr, a.err = L->err;
  const int max_items = min(L->El, T * L->k) * (L->F / 128);
  if (L->fmt == SCION_PQ2_0) return launch_stream<SCION_PQ2_0, 2>(a, max_items, s);
  return launch_stream<SCION_PTQ1_0, 2>(a, max_items, s);
}

cudaError_t launch_stream_down(const scion_layer* L, int T, float* out, cudaStream_t s) {
  StreamArgs a;
  a.bank = L->dn_bank, a.bsrc = L->h, a.bld = L->GF;
  a.slot_info = reinterpret_cast<const int4*>(L->slot_info), a.n_active = L->n_active, a.perm = L->perm;
  a.gperm = L->gperm, a.pexp = L->pexp, a.any_scaled = L->any_scaled, a.G = L->GF, a.R = L->d, a.k = L->k, a.F = L->F, a.d = L->d, a.fmt = L->fmt;
  a.hfrag = nullptr, a.out = out, a.err = L->err;
  const int max_items = min(L->El, T * L->k) * (L->d / 128);
  if (L->fmt == SCION_PQ2_0) return launch_stream<SCION_PQ2_0, 1>(a, max_items, s);
  return launch_stream<SCION_PTQ1_0, 1>(a, max_items, s);
}

}  // namespace scion
