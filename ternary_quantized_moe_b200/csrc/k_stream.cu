// k_stream.cu -- expert kernels for batches of up to 64 tokens, fed by a TMA bulk-copy ring.
//
// Same arithmetic as the register-fed decode kernels (k_decode.cu): the expert SwiGLU
// gate/up and the gate-weighted down projection over ternary codes ("Scion-35B-A3B" and
// "Scion-FlashNext-176B-A6B" model cards, Weight Representation; "Scion: ternary MoE
// quantization with trained corrections", Serving notes: k experts per token).
//
// Work item = one active expert x 128 weight rows; a persistent CTA walks many.  In the
// re-tiled bank the 128 x 128 codes of one group (gate and up interleaved for the gate/up
// bank) are one contiguous block, so a producer warp streams group after group with
// cp.async.bulk into an mbarrier ring, together with the 256-byte fragment-ordered rows of the
// slot's tokens.  Eight consumer warps each own a 16-row sub-tile over the whole K range:
// codes come from shared memory, are unpacked in registers into mma.sync fragments, and no
// cross-warp reduction is needed.
#include "tc_common.cuh"
#include "tern_tile.cuh"

namespace scion {
namespace {

using namespace tc;

constexpr int kRing = 8;    // stages in flight
constexpr int kCons = 8;    // consumer warps (one 16-row sub-tile each)
constexpr int kTok = 8;     // tokens per pass (one mma n-tile)
constexpr int kRowB = 256;  // bytes of one token's 128-column group (fp16)
constexpr int kHdr = 256;   // stage header

// Written by the producer into every stage; the consumers are driven by it alone.
struct StageHdr {
  int nn;     // tokens of the pass (1..kTok); -1: no more work for this CTA
  int flags;  // bit 0: first group of the pass, bit 1: last group of the pass
  int rb;     // 128-row block of the item
  int pad;
  int pos[kTok];     // routed positions of the pass's tokens (last group only)
  int orow[kTok];    // output token row (entry / k)
  float gate[kTok];  // gate of the entry
};
static_assert(sizeof(StageHdr) <= kHdr, "stage header");

struct StreamArgs {
  const uint8_t* bank;
  const __half* bsrc;  // gate/up: xfrag [T][Gd][128]; down: hfrag [T*k][GF][128]
  int bld;             // 128-column groups per B row (Gd or GF)
  const int4* slot_info;
  const int32_t *n_active, *perm;
  const float* gperm;  // gate of each routed position
  int G, R, k, F, d, fmt;
  __half* hfrag;  // gate/up output
  float* out;     // down output
  int* err;
};

struct TokInfo {
  int pos, brow, orow;
  float gate;
};

// Persistent: CTA b walks the items b, b + gridDim.x, ... with item = (active slot, 128-row
// block).  One producer warp streams, per 128-column group, the item's codes and the
// fragment-ordered B rows of up to kTok tokens into a ring of stages, each with a header that
// tells the consumers what it holds; routing records are fetched one (tokens) and two (slot)
// items ahead, so no pointer chase sits between two items.
template <int FMT, int NMAT>
__global__ void __launch_bounds__((kCons + 1) * 32, 2) stream_kernel(const __grid_constant__ StreamArgs a) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kRing], empty[kRing];
  __shared__ int abort_flag;
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  constexpr uint32_t code_bytes = NMAT * 8 * tb;
  constexpr uint32_t stage_bytes = kHdr + code_bytes + kTok * kRowB;
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
        t.gate = a.gperm[t.pos];
        t.brow = NMAT == 2 ? t.orow : t.pos;
      }
      return t;
    };
    int4 si_cur = slot_rec(blockIdx.x), si_nxt = slot_rec(blockIdx.x + gridDim.x);
    TokInfo tk_cur = tok_info(si_cur, 0);
    int st = 0;  // running stage counter
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int4 si_n2 = slot_rec(item + 2 * gridDim.x);
      const TokInfo tk_nxt = tok_info(si_nxt, 0);
      const int rb = item % RB;
      const uint8_t* src0 = a.bank + (int64_t(si_cur.x) * RB + rb) * a.G * code_bytes;
      for (int pc = 0; pc < si_cur.z && ok; pc += kTok) {
        const TokInfo tk = pc == 0 ? tk_cur : tok_info(si_cur, pc);
        const int nn = min(kTok, si_cur.z - pc);
        for (int g = 0; g < a.G; ++g, ++st) {
          const int s = st % kRing;
          if (lane == 0 && st >= kRing) ok = mbar_wait(&empty[s], ((st / kRing) - 1) & 1, &abort_flag, a.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          uint8_t* stg = ring + s * stage_bytes;
          StageHdr* hd = reinterpret_cast<StageHdr*>(stg);
          if (g == a.G - 1) {
            // the epilogue's per-token records, written by lane 0 so its arrive publishes them
#pragma unroll
            for (int i = 0; i < kTok; ++i) {
              const int pos = __shfl_sync(0xffffffffu, tk.pos, i), orow = __shfl_sync(0xffffffffu, tk.orow, i);
              const float gate = __shfl_sync(0xffffffffu, tk.gate, i);
              if (lane == 0) hd->pos[i] = pos, hd->orow[i] = orow, hd->gate[i] = gate;
            }
          }
          if (lane == 0) {
            hd->nn = nn;
            hd->flags = (g == 0 ? 1 : 0) | (g == a.G - 1 ? 2 : 0);
            hd->rb = rb;
            mbar_arrive_expect_tx(&full[s], code_bytes + nn * kRowB);
          }
          __syncwarp();
          if (lane == 0) bulk_load(stg + kHdr, src0 + int64_t(g) * code_bytes, code_bytes, &full[s]);
          if (lane < nn)
            bulk_load(stg + kHdr + code_bytes + lane * kRowB, a.bsrc + (int64_t(tk.brow) * a.bld + g) * 128, kRowB,
                      &full[s]);
        }
      }
      si_cur = si_nxt, si_nxt = si_n2, tk_cur = tk_nxt;
    }
    if (lane == 0) {
      if (ok) {
        // end-of-work sentinel (the consumers wait for every earlier stage before reaching it)
        const int s = st % kRing;
        if (st < kRing || mbar_wait(&empty[s], ((st / kRing) - 1) & 1, &abort_flag, a.err)) {
          reinterpret_cast<StageHdr*>(ring + s * stage_bytes)->nn = -1;
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
  const int c = lane & 3, n = lane >> 2;
  const uint32_t ring_u32 = smem_u32(ring);
  float acc[NMAT][4];
  for (int st = 0;; ++st) {
    const int s = st % kRing;
    if (!mbar_wait(&full[s], (st / kRing) & 1, &abort_flag, a.err)) break;
    const StageHdr* hd = reinterpret_cast<const StageHdr*>(ring + s * stage_bytes);
    const int nn = hd->nn;
    if (nn < 0) break;
    const int flags = hd->flags;
    if (flags & 1) {
#pragma unroll
      for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;
    }
    const uint32_t stg = ring_u32 + s * stage_bytes;
    TileRegs<FMT> tr[NMAT];
#pragma unroll
    for (int m = 0; m < NMAT; ++m) tr[m].load_shared(stg + kHdr + m * 8 * tb + warp * tb, lane);
    {
      uint32_t b[16];
      if (n < nn) {
        const uint32_t bp = stg + kHdr + code_bytes + n * kRowB + 64 * c;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                       : "=r"(b[4 * i]), "=r"(b[4 * i + 1]), "=r"(b[4 * i + 2]), "=r"(b[4 * i + 3])
                       : "r"(bp + 16 * i));
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) b[i] = 0u;
      }
#pragma unroll
      for (int m = 0; m < NMAT; ++m) tile_mma<FMT>(tr[m], b, acc[m], c);
    }
    if (flags & 2) {
      // epilogue: this warp's 16 rows x the pass's tokens
      const int rb = hd->rb;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = warp * 16 + (lane >> 2) + 8 * (i >> 1);
        const int tcol = 2 * c + (i & 1);
        if (tcol >= nn) continue;
        if constexpr (NMAT == 2) {
          const int f = rb * 128 + row;
          const int idx = frag_index(FMT, f & 127);
          float h = silu_f(acc[0][i]) * acc[1][i];
          if (FMT == SCION_PQ2_0) h *= pq2_bscale(idx);
          a.hfrag[(int64_t(hd->pos[tcol]) * (a.F >> 7) + (f >> 7)) * 128 + idx] = __float2half_rn(h);
        } else {
          atomicAdd(&a.out[int64_t(hd->orow[tcol]) * a.d + rb * 128 + row], hd->gate[tcol] * acc[0][i]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

template <int FMT, int NMAT>
constexpr size_t stream_smem() {
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  return size_t(kRing) * (kHdr + NMAT * 8 * tb + kTok * kRowB);
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

}  // namespace

cudaError_t configure_stream_kernels() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(stream_kernel<SCION_PQ2_0, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(stream_smem<SCION_PQ2_0, 2>()))))
    return e;
  if ((e = cudaFuncSetAttribute(stream_kernel<SCION_PQ2_0, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(stream_smem<SCION_PQ2_0, 1>()))))
    return e;
  if ((e = cudaFuncSetAttribute(stream_kernel<SCION_PTQ1_0, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(stream_smem<SCION_PTQ1_0, 2>()))))
    return e;
  return cudaFuncSetAttribute(stream_kernel<SCION_PTQ1_0, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(stream_smem<SCION_PTQ1_0, 1>()));
}

cudaError_t launch_stream_gateup(const scion_layer* L, int T, cudaStream_t s) {
  StreamArgs a;
  a.bank = L->gu_bank, a.bsrc = L->xfrag, a.bld = L->Gd;
  a.slot_info = reinterpret_cast<const int4*>(L->slot_info), a.n_active = L->n_active, a.perm = L->perm;
  a.gperm = L->gperm, a.G = L->Gd, a.R = L->F, a.k = L->k, a.F = L->F, a.d = L->d, a.fmt = L->fmt;
  a.hfrag = L->h, a.out = nullptr, a.err = L->err;
  const int max_items = min(L->E, T * L->k) * (L->F / 128);
  if (L->fmt == SCION_PQ2_0) return launch_stream<SCION_PQ2_0, 2>(a, max_items, s);
  return launch_stream<SCION_PTQ1_0, 2>(a, max_items, s);
}

cudaError_t launch_stream_down(const scion_layer* L, int T, float* out, cudaStream_t s) {
  StreamArgs a;
  a.bank = L->dn_bank, a.bsrc = L->h, a.bld = L->GF;
  a.slot_info = reinterpret_cast<const int4*>(L->slot_info), a.n_active = L->n_active, a.perm = L->perm;
  a.gperm = L->gperm, a.G = L->GF, a.R = L->d, a.k = L->k, a.F = L->F, a.d = L->d, a.fmt = L->fmt;
  a.hfrag = nullptr, a.out = out, a.err = L->err;
  const int max_items = min(L->E, T * L->k) * (L->d / 128);
  if (L->fmt == SCION_PQ2_0) return launch_stream<SCION_PQ2_0, 1>(a, max_items, s);
  return launch_stream<SCION_PTQ1_0, 1>(a, max_items, s);
}

}  // namespace scion
