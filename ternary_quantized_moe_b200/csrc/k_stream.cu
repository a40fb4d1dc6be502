// k_stream.cu -- expert kernels for batches of up to 64 tokens, fed by a TMA bulk-copy ring.
//
// Same arithmetic as the register-fed decode kernels (k_decode.cu): the expert SwiGLU
// gate/up and the gate-weighted down projection over ternary codes ("Scion-35B-A3B" and
// "Scion-FlashNext-176B-A6B" model cards, Weight Representation; "Scion: ternary MoE
// quantization with trained corrections", Serving notes: k experts per token).
//
// One CTA = one active expert x 128 weight rows.  In the re-tiled bank the 128 x 128 codes
// of one group (gate and up interleaved for the gate/up bank) are one contiguous block, so a
// producer warp streams group after group with cp.async.bulk into an mbarrier ring, together
// with the 256-byte fragment-ordered rows of the slot's tokens.  Eight consumer warps each own
// a 16-row sub-tile over the whole K range: codes come from shared memory, are unpacked in
// registers into mma.sync fragments, and no cross-warp reduction is needed.
#include "tc_common.cuh"
#include "tern_tile.cuh"

namespace scion {
namespace {

using namespace tc;

constexpr int kRing = 8;           // stages in flight
constexpr int kCons = 8;           // consumer warps (one 16-row sub-tile each)
constexpr int kTok = 16;           // tokens per pass (two mma n-tiles)
constexpr int kRowB = 256;         // bytes of one token's 128-column group (fp16)

struct StreamArgs {
  const uint8_t* bank;
  const __half* bsrc;  // gate/up: xfrag [T][Gd][128]; down: hfrag [T*k][GF][128]
  int bld;             // 128-column groups per B row (Gd or GF)
  const int4* slot_info;
  const int32_t *n_active, *perm;
  const float* gates;
  int G, R, k, F, d, fmt;
  __half* hfrag;  // gate/up output
  float* out;     // down output
  int* err;
};

template <int FMT, int NMAT>
__global__ void __launch_bounds__((kCons + 1) * 32) stream_kernel(const __grid_constant__ StreamArgs a) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kRing], empty[kRing];
  __shared__ int abort_flag;
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  constexpr uint32_t code_bytes = NMAT * 8 * tb;
  constexpr uint32_t stage_bytes = code_bytes + kTok * kRowB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = blockIdx.y, rt = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) mbar_init(&full[s], 1), mbar_init(&empty[s], kCons);
    abort_flag = 0;
    fence_barrier_init();
  }
  pdl_trigger();
  pdl_wait();
  const int nact = *a.n_active;
  const int4 si = a.slot_info[slot];
  __syncthreads();
  if (slot >= nact) return;
  const int e = si.x, p0 = si.y, ne = si.z;
  const int npass = (ne + kTok - 1) / kTok;
  const int total = npass * a.G;
  const uint8_t* src0 = a.bank + (int64_t(e) * (a.R >> 7) + rt) * a.G * code_bytes;

  if (warp == kCons) {
    // ---------------- producer: codes of group g + the B rows of this pass's tokens
    if (lane == 0) {
      for (int it = 0; it < total; ++it) {
        const int s = it % kRing, pass = it / a.G, g = it % a.G;
        if (it >= kRing && !mbar_wait(&empty[s], ((it / kRing) - 1) & 1, &abort_flag, a.err)) break;
        const int nn = min(kTok, ne - pass * kTok);
        uint8_t* st = ring + s * stage_bytes;
        mbar_arrive_expect_tx(&full[s], code_bytes + nn * kRowB);
        bulk_load(st, src0 + int64_t(g) * code_bytes, code_bytes, &full[s]);
        for (int i = 0; i < nn; ++i) {
          const int pos = p0 + pass * kTok + i;
          const int64_t row = NMAT == 2 ? int64_t(a.perm[pos] / a.k) : int64_t(pos);
          bulk_load(st + code_bytes + i * kRowB, a.bsrc + (row * a.bld + g) * 128, kRowB, &full[s]);
        }
      }
    }
    return;
  }
  // ---------------- consumers
  const int c = lane & 3, n = lane >> 2;
  const uint32_t ring_u32 = smem_u32(ring);
  for (int pass = 0; pass < npass; ++pass) {
    const int nn = min(kTok, ne - pass * kTok);
    float acc[NMAT][2][4];
#pragma unroll
    for (int m = 0; m < NMAT; ++m)
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][t][i] = 0.f;
    for (int g = 0; g < a.G; ++g) {
      const int it = pass * a.G + g, s = it % kRing;
      if (!mbar_wait(&full[s], (it / kRing) & 1, &abort_flag, a.err)) break;
      const uint32_t st = ring_u32 + s * stage_bytes;
      TileRegs<FMT> tr[NMAT];
#pragma unroll
      for (int m = 0; m < NMAT; ++m) tr[m].load_shared(st + m * 8 * tb + warp * tb, lane);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t * 8 >= nn) break;
        uint32_t b[16];
        if (t * 8 + n < nn) {
          const uint32_t bp = st + code_bytes + (t * 8 + n) * kRowB + 64 * c;
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
        for (int m = 0; m < NMAT; ++m) tile_mma<FMT>(tr[m], b, acc[m][t], c);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (abort_flag) break;
    // epilogue: this warp's 16 rows x the pass's tokens
#pragma unroll
    for (int t = 0; t < 2; ++t) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = warp * 16 + (lane >> 2) + 8 * (i >> 1);
        const int tcol = t * 8 + 2 * c + (i & 1);
        if (tcol >= nn) continue;
        const int pos = p0 + pass * kTok + tcol;
        if constexpr (NMAT == 2) {
          const int f = rt * 128 + row;
          const int idx = frag_index(FMT, f & 127);
          float h = silu_f(acc[0][t][i]) * acc[1][t][i];
          if (FMT == SCION_PQ2_0) h *= pq2_bscale(idx);
          a.hfrag[(int64_t(pos) * (a.F >> 7) + (f >> 7)) * 128 + idx] = __float2half_rn(h);
        } else {
          const int entry = a.perm[pos];
          atomicAdd(&a.out[int64_t(entry / a.k) * a.d + rt * 128 + row], a.gates[entry] * acc[0][t][i]);
        }
      }
    }
  }
}

template <int FMT, int NMAT>
size_t stream_smem() {
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  return size_t(kRing) * (NMAT * 8 * tb + kTok * kRowB);
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
  a.gates = L->gates, a.G = L->Gd, a.R = L->F, a.k = L->k, a.F = L->F, a.d = L->d, a.fmt = L->fmt;
  a.hfrag = L->h, a.out = nullptr, a.err = L->err;
  const dim3 grid(L->F / 128, min(L->E, T * L->k));
  if (L->fmt == SCION_PQ2_0)
    return launch_pdl(stream_kernel<SCION_PQ2_0, 2>, grid, dim3((kCons + 1) * 32), stream_smem<SCION_PQ2_0, 2>(), s, a);
  return launch_pdl(stream_kernel<SCION_PTQ1_0, 2>, grid, dim3((kCons + 1) * 32), stream_smem<SCION_PTQ1_0, 2>(), s, a);
}

cudaError_t launch_stream_down(const scion_layer* L, int T, float* out, cudaStream_t s) {
  StreamArgs a;
  a.bank = L->dn_bank, a.bsrc = L->h, a.bld = L->GF;
  a.slot_info = reinterpret_cast<const int4*>(L->slot_info), a.n_active = L->n_active, a.perm = L->perm;
  a.gates = L->gates, a.G = L->GF, a.R = L->d, a.k = L->k, a.F = L->F, a.d = L->d, a.fmt = L->fmt;
  a.hfrag = nullptr, a.out = out, a.err = L->err;
  const dim3 grid(L->d / 128, min(L->E, T * L->k));
  if (L->fmt == SCION_PQ2_0)
    return launch_pdl(stream_kernel<SCION_PQ2_0, 1>, grid, dim3((kCons + 1) * 32), stream_smem<SCION_PQ2_0, 1>(), s, a);
  return launch_pdl(stream_kernel<SCION_PTQ1_0, 1>, grid, dim3((kCons + 1) * 32), stream_smem<SCION_PTQ1_0, 1>(), s, a);
}

}  // namespace scion
