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
#include <string.h>

#include "scion_internal.cuh"
#include "tc_order.cuh"
#include "tern_tile.cuh"

namespace scion {
namespace {


// ========================================================================= xproj
struct XProjArgs {
  const __nv_bfloat16* x;
  int T, d, E, Fs, r, Kd;  // Kd = padded row stride of hz
  int fmt;
  const __nv_bfloat16 *w_router, *w_delta, *sh_gate, *sh_up, *corr_a;
  const XUnit* units;  // this launch's units (a slice of the layer's table)
  int n_units, n_chunks;
  int n_aux;           // CTA columns after the units that run xproj_aux (0 or kXAux)
  float* logits;
  __half* hz;
  __half* xfrag;  // [T][d/128][SCION_BROW] fp16 x 2^s_t in fragment order + group sums
  int32_t* xexp;  // [T] range exponent s_t of each token (token_shift), written by the aux CTAs
  __half* x16;    // non-null: the aux CTAs write x 2^s_t here, [T][d] in the tcgen05 column order,
  float* xsum;    //   with its per-group sums of B * 4^f (PQ2_0) in xsum [T][d/128],
  float* hsum;    //   and zero the hidden's group sums hsum [T*k][F/128]
  __half* h;      // [T*k][F/128][SCION_BROW] expert hidden: group-sum tails zeroed here
  int k, GF;
  const uint8_t* corr_blocks;  // ternary correction A (PQ2_0 blocks [r][d/128]) or nullptr (bf16 corr_a)
  float* out;     // set here to the residual (or zero)
  const float* resid;  // nullptr: out starts at zero; may equal out (then out is left as it is)
  int z_only;          // the correction branch alone: z rows scaled by 2^s_t (not hz_shift), and the
                       // lead CTA of unit 0 writes each token's s_t to xexp
};

// One CTA = (unit, 512-column chunk); 8 warps x 64 columns.  NT = token tiles of 8.  The
// chunks of a unit are one thread-block cluster, reduced through distributed shared memory.
// kXAux extra CTA columns convert x to the fragment order and clear out and the hidden tails.
constexpr int kXRow = SCION_XPROJ_KC + 8;  // bf16 elements per staged token row (+16 B pad)
constexpr int kXAux = 8;
constexpr int kXThreads = 256;  // 8 warps x 64 columns

template <int NT>
constexpr size_t xproj_smem(int T) {
  return (size_t(T) * kXRow * 2 > size_t(8) * 2 * NT * 32 * 4 * 4) ? size_t(T) * kXRow * 2
                                                                    : size_t(8) * 2 * NT * 32 * 4 * 4;
}

// Largest magnitude of eight bf16 values, as the bit pattern of their absolute value.
__device__ __forceinline__ uint32_t max_mag8(uint4 v) {
  const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu), __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ void xproj_aux(const XProjArgs& a, int aux, int n_aux) {
  const int Gd = a.d >> 7, n_pairs = (Gd + 1) >> 1;
  const int lane = threadIdx.x & 31;
  const int gw = aux * (kXThreads / 32) + (threadIdx.x >> 5), nw = n_aux * (kXThreads / 32);
  // Warps share the tokens out (wpt warps per token, each a slice of its pairs of 128-column
  // groups).  Each warp streams its token's whole row once for the largest magnitude, which
  // fixes the range exponent s_t; each of its pairs is then read again (coalesced, from cache)
  // into shared memory, where lane (gl, part) gathers the 8 columns of its output positions in
  // group 2 pr + gl and writes x 2^s_t in the tcgen05 order (a.x16) or the fragment order with
  // the group sums of B * 4^f in the row tails.  (Nothing is held across the two passes: the
  // registers of this path would otherwise bound the x-projection CTAs' occupancy.)
  __shared__ __align__(16) __nv_bfloat16 pbuf[kXThreads / 32][256];
  __nv_bfloat16* buf = pbuf[threadIdx.x >> 5];
  const int wpt = max(1, nw / max(1, a.T));
  const int gl = lane >> 4, part = lane & 15;
  for (int job = gw; job < a.T * wpt; job += nw) {
    const int t = job / wpt, slice = job % wpt;
    const __nv_bfloat16* row = a.x + int64_t(t) * a.d;
    uint32_t mx = 0;
#pragma unroll 1
    for (int i = lane; i < a.d / 8; i += 32) mx = max(mx, max_mag8(*reinterpret_cast<const uint4*>(row + 8 * i)));
    const int sh = token_shift(__reduce_max_sync(0xffffffffu, mx));
    if (lane == 0 && slice == 0) a.xexp[t] = sh;
    const float xs = pow2i(sh);
    for (int pr = slice; pr < n_pairs; pr += wpt) {
      const int g = 2 * pr + gl;
      const bool ok = g < Gd;  // an odd group count leaves the last pair half empty
      const uint4 v = ok ? *reinterpret_cast<const uint4*>(row + 256 * pr + 8 * lane) : make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
      *reinterpret_cast<uint4*>(buf + 8 * lane) = v;
      __syncwarp();
      const __nv_bfloat16* src = buf + 128 * gl;
      __align__(16) __half o[8];
      float sum = 0.f;
      if (a.x16) {
        // tcgen05 order: positions 8 part .. 8 part + 7 of group g
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int q = 8 * part + e;
          const float f = __bfloat162float(src[pos_col(a.fmt, q)]) * xs;
          o[e] = __float2half_rn(a.fmt == SCION_PQ2_0 ? f * pq2_pos_scale(q) : f);
          if (a.fmt == SCION_PQ2_0) sum += __half2float(o[e]) / pq2_pos_scale(q);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int idx = part * 8 + e;
          const float f = __bfloat162float(src[brow_col(a.fmt, idx)]) * xs;
          if (a.fmt == SCION_PQ2_0) {
            const float up = 1.0f / brow_bscale(idx);
            o[e] = __float2half_rn(f / up);
            sum += __half2float(o[e]) * up;
          } else {
            o[e] = __float2half_rn(f);
          }
        }
      }
#pragma unroll
      for (int off = 8; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (!ok) continue;
      if (a.x16) {
        *reinterpret_cast<uint4*>(a.x16 + int64_t(t) * a.d + g * 128 + 8 * part) = *reinterpret_cast<const uint4*>(o);
        if (part == 0 && a.xsum && a.fmt == SCION_PQ2_0) a.xsum[int64_t(t) * Gd + g] = sum;
      } else {
        __half* dst = a.xfrag + (int64_t(t) * Gd + g) * SCION_BROW;
        *reinterpret_cast<uint4*>(dst + part * 8) = *reinterpret_cast<const uint4*>(o);
        if (part == 0)
          *reinterpret_cast<float4*>(dst + 128) = make_float4(-5.9604644775390625e-08f * sum, 0.f, 0.f, 0.f);
      }
    }
  }
  const int tid = aux * kXThreads + threadIdx.x, nth = n_aux * kXThreads;
  float4* o4 = reinterpret_cast<float4*>(a.out);
  if (!a.resid) {
    for (int64_t i = tid; i < int64_t(a.T) * a.d / 4; i += nth) o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else if (a.resid != a.out) {
    const float4* r4 = reinterpret_cast<const float4*>(a.resid);
    for (int64_t i = tid; i < int64_t(a.T) * a.d / 4; i += nth) o4[i] = r4[i];
  }
  // the expert hidden's group sums are accumulated by the gate/up epilogue
  for (int i = tid; i < a.T * a.k * a.GF; i += nth) {
    *reinterpret_cast<float4*>(a.h + int64_t(i) * SCION_BROW + 128) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (a.hsum) a.hsum[i] = 0.f;
  }
}

// Eight consecutive ternary codes (16 bits of a PQ2_0 block, low bits first: field 0/1/2 =
// -1/0/+1) as four bf16 pairs in column order.
__device__ __forceinline__ uint32_t tern_pair_bf16(uint32_t f) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(float(int(f & 3u) - 1), float(int((f >> 2) & 3u) - 1));
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ uint4 tern8_bf16(uint32_t c16) {
  return make_uint4(tern_pair_bf16(c16), tern_pair_bf16(c16 >> 4), tern_pair_bf16(c16 >> 8), tern_pair_bf16(c16 >> 12));
}

__device__ __forceinline__ uint32_t tern_pair_f16(uint32_t f) {
  const __half2 v = __floats2half2_rn(float(int(f & 3u) - 1), float(int((f >> 2) & 3u) - 1));
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ uint4 tern8_f16(uint32_t c16) {
  return make_uint4(tern_pair_f16(c16), tern_pair_f16(c16 >> 4), tern_pair_f16(c16 >> 8), tern_pair_f16(c16 >> 12));
}

template <int NT>
__global__ void __launch_bounds__(kXThreads) xproj_kernel(XProjArgs a) {
  extern __shared__ __align__(16) uint8_t xsm[];
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(xsm);  // [NT*8][kXRow], then the warp reduction
  __shared__ uint32_t tmax[SCION_TDEC];  // largest |x| bits of each token over this CTA's K chunk (T entries)
  __shared__ int tshift[SCION_TDEC];     // lead CTA: range exponent of each token
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, c = lane & 3;
  const int chunk = blockIdx.y;
  const int kbase = chunk * SCION_XPROJ_KC;

  pdl_trigger();
  if (blockIdx.x >= a.n_units) {
    pdl_wait();
    xproj_aux(a, (blockIdx.x - a.n_units) * a.n_chunks + chunk, a.n_aux * a.n_chunks);
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

  const int kw = kbase + warp * 64;
  const int row_a = u.row0 + g8, row_b = u.row0 + g8 + 8;
  const bool ok_a = row_a < nrows, ok_b = row_b < nrows;
  const bool active_warp = kw < a.d;
  // weights first (they do not depend on x): both matrices, this warp's 64 columns
  uint4 wa[2][2], wb[2][2];
  // ternary correction A: the warp's 64 columns lie in one group of 128 of each row's block, so
  // its partial sums take the group scales of rows row_a / row_b after the MMAs
  const bool tern = u.kind == kUnitPlain && a.corr_blocks != nullptr;
  float sc_a = 0.f, sc_b = 0.f;
  if (tern) {
    const int G = a.d >> 7, g = kw >> 7, hoff = kw & 127;
    const uint8_t* ba = a.corr_blocks + (int64_t(row_a) * G + g) * 34;
    const uint8_t* bb = a.corr_blocks + (int64_t(row_b) * G + g) * 34;
    const bool la = active_warp && ok_a, lb = active_warp && ok_b;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int j0 = hoff + 32 * q + 8 * c;  // first of the lane's 8 columns in the group
      wa[0][q] = la ? tern8_bf16(__ldg(reinterpret_cast<const unsigned short*>(ba + (j0 >> 2)))) : make_uint4(0, 0, 0, 0);
      wb[0][q] = lb ? tern8_bf16(__ldg(reinterpret_cast<const unsigned short*>(bb + (j0 >> 2)))) : make_uint4(0, 0, 0, 0);
      wa[1][q] = wb[1][q] = make_uint4(0, 0, 0, 0);
    }
    sc_a = la ? __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short*>(ba + 32)))) : 0.f;
    sc_b = lb ? __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short*>(bb + 32)))) : 0.f;
  } else {
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int kk = kw + 32 * q + 8 * c;
        const bool ld = active_warp && m < nmat;
        wa[m][q] = (ld && ok_a) ? ldg_stream(mats[m] + int64_t(row_a) * a.d + kk) : make_uint4(0, 0, 0, 0);
        wb[m][q] = (ld && ok_b) ? ldg_stream(mats[m] + int64_t(row_b) * a.d + kk) : make_uint4(0, 0, 0, 0);
      }
  }
  // the shared-expert and correction rows are stored scaled per token (hz_shift), which needs the
  // largest |x| of each token: each chunk's CTA finds it over its columns, the lead combines them
  const bool need_max = u.kind != kUnitRouter;
  pdl_wait();  // everything below reads x or writes the workspace
  // stage x[0..T)[kbase .. kbase+512) in shared memory (rows padded by 16 B: conflict-free reads)
  const int kchunks = min(SCION_XPROJ_KC, a.d - kbase) >> 3;  // 16-byte chunks per token row (<= 64)
  for (int i = threadIdx.x; i < a.T * 64; i += kXThreads) {
    const int t = i >> 6, j = i & 63;
    if (j >= kchunks) continue;
    const uint32_t dst = uint32_t(__cvta_generic_to_shared(xs + t * kXRow + 8 * j));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(a.x + int64_t(t) * a.d + kbase + 8 * j)
                 : "memory");
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  if (active_warp) {
    const bool second_acc = (u.kind == kUnitSwiglu);
    const int kwl = warp * 64;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      if (m >= nmat) break;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tok = nt * 8 + g8;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint4 xb = tok < a.T ? *reinterpret_cast<const uint4*>(xs + tok * kXRow + kwl + 32 * q + 8 * c)
                                     : make_uint4(0, 0, 0, 0);
          const uint32_t fa0[4] = {wa[m][q].x, wb[m][q].x, wa[m][q].y, wb[m][q].y};
          const uint32_t fa1[4] = {wa[m][q].z, wb[m][q].z, wa[m][q].w, wb[m][q].w};
          if (m == 1 && second_acc) {
            mma_bf16_16816(acc[1][nt], fa0, xb.x, xb.y);
            mma_bf16_16816(acc[1][nt], fa1, xb.z, xb.w);
          } else {
            mma_bf16_16816(acc[0][nt], fa0, xb.x, xb.y);
            mma_bf16_16816(acc[0][nt], fa1, xb.z, xb.w);
          }
        }
      }
    }
  }
  if (tern) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      acc[0][nt][0] *= sc_a, acc[0][nt][1] *= sc_a, acc[0][nt][2] *= sc_b, acc[0][nt][3] *= sc_b;
  }
  if (need_max)  // after the MMAs, while the x stage is still intact
    for (int t = warp; t < a.T; t += kXThreads / 32) {  // one warp per staged token row
      uint32_t m = 0;
      for (int j = lane; j < kchunks; j += 32) m = max(m, max_mag8(*reinterpret_cast<const uint4*>(xs + t * kXRow + 8 * j)));
      m = __reduce_max_sync(0xffffffffu, m);
      if (lane == 0) tmax[t] = m;
    }
  __syncthreads();  // the x stage is dead: its space holds the warp reduction
  float(*red)[2][NT][32][4] = reinterpret_cast<float(*)[2][NT][32][4]>(xsm);
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][m][nt][lane][i] = acc[m][nt][i];
  __syncthreads();

  // thread -> (nt, lane) pairs; sum the 8 warps into warp 0's slot
  for (int p = threadIdx.x; p < NT * 32; p += blockDim.x) {
    const int nt = p >> 5, ln = p & 31;
    for (int m = 0; m < nacc; ++m)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += red[w][m][nt][ln][i];
        red[0][m][nt][ln][i] = v;
      }
  }
  // the K chunks of a unit form one thread-block cluster: after a cluster barrier the chunk-0
  // CTA adds the other chunks' sums straight from their shared memory, then a second barrier
  // keeps them resident until it has read them
  cluster_sync();
  const bool lead = blockIdx.y == 0;
  // epilogue (chunk 0): thread -> (row, tok); all remote loads of the thread are issued together
  constexpr int kIt = 16 * SCION_TDEC / kXThreads;
  float v[kIt][2];
  if (lead && need_max) {
    // the tokens' largest |x| over all chunks (read beside the partial sums below; the cluster
    // barrier that follows orders these shared-memory writes before the epilogue reads them)
    for (int t = threadIdx.x; t < a.T; t += kXThreads) {
      uint32_t m = tmax[t];
      for (int ch = 1; ch < a.n_chunks; ++ch)
        m = max(m, ld_dsmem_u32(map_cluster_rank(smem_addr(&tmax[t]), ch)));
      const int sh = token_shift(m);
      tshift[t] = a.z_only ? sh : hz_shift(sh, a.Fs > 0, a.r > 0);
      if (a.z_only && blockIdx.x == 0) a.xexp[t] = sh;
    }
  }
  if (lead) {
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
      const int p = threadIdx.x + kXThreads * it;
      const int row = p / SCION_TDEC, tok = p % SCION_TDEC;
      v[it][0] = v[it][1] = 0.f;
      if (tok >= a.T) continue;
      const int nt = tok >> 3, ln = (row & 7) * 4 + ((tok & 7) >> 1), i = (row >> 3) * 2 + (tok & 1);
      for (int m = 0; m < nacc; ++m) {
        const uint32_t off = smem_addr(&red[0][m][nt][ln][i]);
        float sum = red[0][m][nt][ln][i];
        for (int ch = 1; ch < a.n_chunks; ++ch) sum += ld_dsmem_f32(map_cluster_rank(off, ch));
        v[it][m] = sum;
      }
    }
  }
  cluster_sync();
  if (!lead) return;
#pragma unroll
  for (int it = 0; it < kIt; ++it) {
    const int p = threadIdx.x + kXThreads * it;
    const int row = p / SCION_TDEC, tok = p % SCION_TDEC;
    if (tok >= a.T) continue;
    const int grow = u.row0 + row;
    if (grow >= nrows) continue;
    if (u.kind == kUnitRouter) {
      a.logits[int64_t(tok) * a.E + grow] = v[it][0];
    } else if (u.kind == kUnitSwiglu) {
      a.hz[int64_t(tok) * a.Kd + grow] = __float2half_rn(silu_f(v[it][0]) * v[it][1] * pow2i(tshift[tok]));
    } else {
      a.hz[int64_t(tok) * a.Kd + a.Fs + grow] = __float2half_rn(v[it][0] * pow2i(tshift[tok]));
    }
  }
}

// ======================================================================= gate/up
struct GateUpArgs {
  const uint8_t* bank;  // gate/up bank
  const __half* xfrag;  // [T][Gd][128]
  const int4* slot_info;
  const int32_t *n_active, *perm;
  const int32_t* pexp;  // [T*k] range exponent of the token of each routed position
  int d, F, k, Gd, fmt;
  __half* hfrag;  // [T*k][GF][128] fragment order of the down format, h 2^(2 s_t)
};

constexpr int kGuWarps = 8;

// CTA = (16 ffn rows, active-expert slot); the 8 warps split the d/128 groups, keep their
// groups' codes in registers, and run the slot's tokens 8 at a time.
template <int FMT, int GPW>
__device__ __forceinline__ void gateup_body(const GateUpArgs& a, int slot, int ft) {
  __shared__ float red[kGuWarps][2][32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, c = lane & 3;
  pdl_trigger();
  pdl_wait();
  const int nact = *a.n_active;
  const int4 si = a.slot_info[slot];
  if (slot >= nact) return;
  const int e = si.x, p0 = si.y, ne = si.z;
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  const uint8_t* tile0 = a.bank + ((int64_t(e) * (a.F >> 7) + (ft >> 3)) * a.Gd * 2 * 8 + (ft & 7)) * tb;
  TileRegs<FMT> rg[GPW], ru[GPW];
#pragma unroll
  for (int i = 0; i < GPW; ++i) {
    const int g = warp + kGuWarps * i;
    if (g < a.Gd) {
      const uint8_t* blk = tile0 + int64_t(g) * 2 * 8 * tb;
      rg[i].load(blk, lane);
      ru[i].load(blk + 8 * tb, lane);
    }
  }
  const int GF = a.F >> 7;
  for (int pc = 0; pc < ne; pc += 8) {
    const int nn = min(8, ne - pc);
    const int n = lane >> 2;
    const int tok = n < nn ? a.perm[p0 + pc + n] / a.k : -1;
    // the epilogue thread's token column is fixed: fetch its range exponent before the MMAs
    const int tcol_e = 2 * ((threadIdx.x >> 2) & 3) + (threadIdx.x & 1);
    const int sh_e = threadIdx.x < 128 && tcol_e < nn ? a.pexp[p0 + pc + tcol_e] : 0;
    float tg[4] = {0.f, 0.f, 0.f, 0.f}, tu[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < GPW; ++i) {
      const int g = warp + kGuWarps * i;
      if (g < a.Gd) {
        uint32_t b[16];
        load_b(a.xfrag, int64_t(a.Gd) * SCION_BROW, tok, g, c, b);
        tile_mma<FMT>(rg[i], b, tg, c);
        tile_mma<FMT>(ru[i], b, tu, c);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][0][lane][i] = tg[i], red[warp][1][lane][i] = tu[i];
    __syncthreads();
    if (threadIdx.x < 128) {
      const int ln = threadIdx.x >> 2, i = threadIdx.x & 3;
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int w = 0; w < kGuWarps; ++w) gs += red[w][0][ln][i], us += red[w][1][ln][i];
      const int row = (ln >> 2) + 8 * (i >> 1), tcol = 2 * (ln & 3) + (i & 1);
      if (tcol < nn) {
        const int f = ft * 16 + row;
        const int64_t pos = p0 + pc + tcol;
        const int idx = brow_pos(a.fmt, f & 127);
        float h = silu_f(gs * pow2i(-sh_e)) * (us * pow2i(sh_e));  // the sums are of x 2^sh_e
        if (a.fmt == SCION_PQ2_0) h *= brow_bscale(idx);
        a.hfrag[(pos * GF + (f >> 7)) * SCION_BROW + idx] = __float2half_rn(h);
      }
    }
    __syncthreads();
  }
}

template <int FMT, int GPW>
__global__ void __launch_bounds__(kGuWarps * 32) gateup_kernel(GateUpArgs a) {
  gateup_body<FMT, GPW>(a, blockIdx.y, blockIdx.x);
}

// ======================================================================== down
struct DownArgs {
  const uint8_t* bank;  // down bank
  const __half* hfrag;  // [T*k][GF][128]
  const int4* slot_info;
  const int32_t *n_active, *perm;
  const float* gperm;  // [T*k] gate of each routed position, times 2^(-2 s_t) (the hidden is h 2^(2 s_t))
  int d, F, k, GF;
  float* out;
};

constexpr int kDnWarps = 4;

template <int FMT, int GPW>
__global__ void __launch_bounds__(kDnWarps * 32) down_routed_kernel(DownArgs a) {
  __shared__ float red[kDnWarps][32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, c = lane & 3;
  const int slot = blockIdx.y;
  pdl_trigger();
  pdl_wait();
  const int nact = *a.n_active;
  const int4 si = a.slot_info[slot];
  if (slot >= nact) return;
  const int e = si.x, p0 = si.y, ne = si.z;
  const int dt = blockIdx.x;
  constexpr int tb = FMT == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile;
  const uint8_t* tile0 = a.bank + ((int64_t(e) * (a.d >> 7) + (dt >> 3)) * a.GF * 8 + (dt & 7)) * tb;
  TileRegs<FMT> rw[GPW];
#pragma unroll
  for (int i = 0; i < GPW; ++i) {
    const int g = warp + kDnWarps * i;
    if (g < a.GF) rw[i].load(tile0 + int64_t(g) * 8 * tb, lane);
  }
  for (int pc = 0; pc < ne; pc += 8) {
    const int nn = min(8, ne - pc);
    const int n = lane >> 2;
    const int pos = n < nn ? p0 + pc + n : -1;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < GPW; ++i) {
      const int g = warp + kDnWarps * i;
      if (g < a.GF) {
        uint32_t b[16];
        load_b(a.hfrag, int64_t(a.GF) * SCION_BROW, pos, g, c, b);
        tile_mma<FMT>(rw[i], b, acc, c);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][lane][i] = acc[i];
    __syncthreads();
    {
      const int ln = threadIdx.x >> 2, i = threadIdx.x & 3;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kDnWarps; ++w) v += red[w][ln][i];
      const int row = (ln >> 2) + 8 * (i >> 1), tcol = 2 * (ln & 3) + (i & 1);
      if (tcol < nn) {
        const int entry = a.perm[p0 + pc + tcol];
        atomicAdd(&a.out[int64_t(entry / a.k) * a.d + dt * 16 + row], a.gperm[p0 + pc + tcol] * v);
      }
    }
    __syncthreads();
  }
}

// [sh_down | corr_b] (fp16 [d][Kd]) x hz ([T][Kd] fp16, natural order) -> out += .
// CTA = (32 output rows, 256-column K chunk): the chunk of hz is staged in shared memory, the
// 8 warps take (16 rows, 64 columns) each with their weights loaded before the dependency
// wait, and the 4 K slices of each row pair are summed in shared memory before one fp32
// red.add per output.
struct DenseArgs {
  const __half* w;  // [d][Kd]
  const __half* hz; // [T][Kd]
  int d, Kd, T;
  float* out;
  // ternary correction B (PQ2_0 blocks [d][r/128]) read in place for columns Fs .. Fs + r
  // (nullptr: every column from w)
  const uint8_t* corr_b;
  int Fs, r;
  const int32_t* xexp;  // [T] range exponent of each token: hz rows hold 2^hz_shift(s_t, Fs > 0, r > 0) times their values
  int z_only;           // hz holds z 2^s_t alone (the correction branch on the attention output)
};

constexpr int kDnKc = 256;            // K columns per CTA
constexpr int kDnRowH = kDnKc + 32;   // staged hz row (halves): 576 B, rows 16 banks apart

template <int NT>
__device__ __forceinline__ void dense_body(const DenseArgs& a, int bx, int by) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __half* hs = reinterpret_cast<__half*>(dsm);                                 // [NT*8][kDnRowH]
  float* red = reinterpret_cast<float*>(dsm + NT * 8 * kDnRowH * sizeof(__half));  // [8][NT][32][4]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g8 = lane >> 2, c = lane & 3;
  const int row0 = bx * 32 + 16 * (warp & 1);
  const int kc0 = by * kDnKc;
  const int kw = kc0 + 64 * (warp >> 1);
  pdl_trigger();
  // weights first (they do not depend on earlier kernels): 64 columns of rows g8 and g8 + 8
  uint4 wa[2], wb[2];
  const bool kin = kw < a.Kd;
  // ternary correction columns: one group of 128 per warp slice, scaled after the MMAs
  const bool tern = a.corr_b != nullptr && kw >= a.Fs && kw < a.Fs + a.r;
  float sc_a = 0.f, sc_b = 0.f;
  if (tern) {
    const int Gr = a.r >> 7, kk = kw - a.Fs, g = kk >> 7, hoff = kk & 127;
    const uint8_t* ba = a.corr_b + (int64_t(row0 + g8) * Gr + g) * 34;
    const uint8_t* bb = a.corr_b + (int64_t(row0 + g8 + 8) * Gr + g) * 34;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int j0 = hoff + 32 * q + 8 * c;
      wa[q] = tern8_f16(__ldg(reinterpret_cast<const unsigned short*>(ba + (j0 >> 2))));
      wb[q] = tern8_f16(__ldg(reinterpret_cast<const unsigned short*>(bb + (j0 >> 2))));
    }
    sc_a = __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short*>(ba + 32))));
    sc_b = __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short*>(bb + 32))));
  } else {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      wa[q] = kin ? ldg_stream(a.w + int64_t(row0 + g8) * a.Kd + kw + 32 * q + 8 * c) : make_uint4(0, 0, 0, 0);
      wb[q] = kin ? ldg_stream(a.w + int64_t(row0 + g8 + 8) * a.Kd + kw + 32 * q + 8 * c) : make_uint4(0, 0, 0, 0);
    }
  }
  pdl_wait();
  const int kcols = min(kDnKc, a.Kd - kc0);  // multiple of 64
  for (int i = threadIdx.x; i < a.T * (kcols >> 3); i += blockDim.x) {
    const int t = i / (kcols >> 3), j = i % (kcols >> 3);
    const uint32_t dst = uint32_t(__cvta_generic_to_shared(hs + t * kDnRowH + 8 * j));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(a.hz + int64_t(t) * a.Kd + kc0 + 8 * j)
                 : "memory");
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
  if (kin) {
    const int kwl = kw - kc0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t fa0[4] = {wa[q].x, wb[q].x, wa[q].y, wb[q].y};
      const uint32_t fa1[4] = {wa[q].z, wb[q].z, wa[q].w, wb[q].w};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tok = nt * 8 + g8;
        const uint4 xb = tok < a.T ? *reinterpret_cast<const uint4*>(hs + tok * kDnRowH + kwl + 32 * q + 8 * c)
                                   : make_uint4(0, 0, 0, 0);
        mma_f16_16816(acc[nt], fa0, xb.x, xb.y);
        mma_f16_16816(acc[nt], fa1, xb.z, xb.w);
      }
    }
  }
  if (tern) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] *= sc_a, acc[nt][1] *= sc_a, acc[nt][2] *= sc_b, acc[nt][3] *= sc_b;
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[((warp * NT + nt) * 32 + lane) * 4 + i] = acc[nt][i];
  __syncthreads();
  // thread -> (row half h, nt, lane, i): sum the 4 K slices (warps h, h+2, h+4, h+6)
  for (int idx = threadIdx.x; idx < 2 * NT * 128; idx += blockDim.x) {
    const int h = idx / (NT * 128), rem = idx % (NT * 128);
    const int nt = rem >> 7, ln = (rem >> 2) & 31, i = rem & 3;
    float v = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) v += red[(((h + 2 * ks) * NT + nt) * 32 + ln) * 4 + i];
    const int row = bx * 32 + 16 * h + (ln >> 2) + 8 * (i >> 1), tok = nt * 8 + 2 * (ln & 3) + (i & 1);
    if (tok < a.T)
      atomicAdd(&a.out[int64_t(tok) * a.d + row],
                v * pow2i(a.z_only ? -a.xexp[tok] : -hz_shift(a.xexp[tok], a.Fs > 0, a.r > 0)));
  }
}

template <int NT>
__global__ void __launch_bounds__(256) down_dense_kernel(DenseArgs a) {
  dense_body<NT>(a, blockIdx.x, blockIdx.y);
}

// Batches below the ring kernels' threshold: the expert gate/up and the dense down projection
// (which needs only the x-projection) in one launch, so the dense part leaves the critical
// path.  Rows [0, gu_rows) of the grid are gate/up CTAs, the rows after them dense-down tiles
// (dense_x tiles of 32 output rows per K chunk).
template <int FMT, int GPW, int NT>
__global__ void __launch_bounds__(256) gateup_dense_kernel(GateUpArgs a, DenseArgs b, int gu_rows, int dense_x) {
  if (int(blockIdx.y) < gu_rows) {
    gateup_body<FMT, GPW>(a, blockIdx.y, blockIdx.x);
    return;
  }
  const int lin = (int(blockIdx.y) - gu_rows) * int(gridDim.x) + int(blockIdx.x);
  if (lin < dense_x * ((b.Kd + kDnKc - 1) / kDnKc)) dense_body<NT>(b, lin % dense_x, lin / dense_x);
}

template <int NT>
constexpr size_t down_dense_smem() {
  return size_t(NT) * 8 * kDnRowH * sizeof(__half) + size_t(8) * NT * 32 * 4 * sizeof(float);
}

__global__ void unfrag_kernel(int fmt, const __half* __restrict__ src, int64_t n, __half* __restrict__ dst) {
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int64_t grp = i >> 7;
  int col = int(i & 127);
  const int idx = brow_pos(fmt, col);
  float v = __half2float(src[grp * SCION_BROW + idx]);
  if (fmt == SCION_PQ2_0) v /= brow_bscale(idx);  // undo the exact power-of-two B pre-scaling
  dst[grp * 128 + col] = __float2half_rn(v);
}

}  // namespace

// ------------------------------------------------------------------- launchers
cudaError_t launch_xproj(const scion_layer* L, const __nv_bfloat16* x, int T, float* out, const float* resid,
                         int unit0, int n_units, bool aux, bool x16, cudaStream_t s) {
  XProjArgs a;
  a.resid = resid;
  a.x = x;
  a.T = T, a.d = L->d, a.E = L->E, a.Fs = L->Fs, a.r = L->r, a.Kd = L->Kd, a.fmt = L->fmt;
  a.w_router = static_cast<const __nv_bfloat16*>(L->desc.w_router);
  a.w_delta = static_cast<const __nv_bfloat16*>(L->desc.w_router_delta);
  a.sh_gate = static_cast<const __nv_bfloat16*>(L->desc.sh_gate);
  a.sh_up = static_cast<const __nv_bfloat16*>(L->desc.sh_up);
  a.corr_a = static_cast<const __nv_bfloat16*>(L->desc.corr_a);
  a.units = L->xunits + unit0, a.n_units = n_units, a.n_chunks = L->n_xchunks, a.n_aux = aux ? kXAux : 0;
  a.logits = L->logits, a.hz = L->hz, a.xfrag = L->xfrag, a.xexp = L->xexp, a.out = out;
  a.x16 = x16 ? L->x16d : nullptr;
  a.xsum = x16 ? L->xsum : nullptr;
  a.hsum = x16 ? L->hsum : nullptr;
  a.z_only = 0;
  a.corr_blocks = L->desc.corr_packed ? static_cast<const uint8_t*>(L->desc.corr_a) : nullptr;
  a.h = L->h, a.k = L->k, a.GF = L->GF;
  if (n_units + a.n_aux == 0) return cudaSuccess;
  dim3 grid(n_units + a.n_aux, L->n_xchunks);
  const dim3 cluster(1, L->n_xchunks, 1);
  const int nt = (T + 7) / 8;
  switch (nt) {
    case 1: return launch_pdl_cluster(xproj_kernel<1>, grid, dim3(kXThreads), cluster, xproj_smem<1>(T), s, a);
    case 2: return launch_pdl_cluster(xproj_kernel<2>, grid, dim3(kXThreads), cluster, xproj_smem<2>(T), s, a);
    case 3: case 4:
      return launch_pdl_cluster(xproj_kernel<4>, grid, dim3(kXThreads), cluster, xproj_smem<4>(T), s, a);
    default: return launch_pdl_cluster(xproj_kernel<8>, grid, dim3(kXThreads), cluster, xproj_smem<8>(T), s, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_gateup(const scion_layer* L, const __nv_bfloat16* /*x*/, int T, cudaStream_t s) {
  GateUpArgs a;
  a.bank = L->gu_bank, a.xfrag = L->xfrag;
  a.slot_info = reinterpret_cast<const int4*>(L->slot_info), a.n_active = L->n_active, a.perm = L->perm;
  a.d = L->d, a.F = L->F, a.k = L->k, a.Gd = L->Gd, a.fmt = L->fmt;
  a.hfrag = L->h, a.pexp = L->pexp;
  const int slots = min(L->El, T * L->k);
  const dim3 grid(L->F / 16, slots);
  const int gpw = (L->Gd + kGuWarps - 1) / kGuWarps;
#define SCION_GU(F_, G_) return launch_pdl(gateup_kernel<F_, G_>, grid, dim3(kGuWarps * 32), 0, s, a)
  if (L->fmt == SCION_PQ2_0) {
    if (gpw <= 1) SCION_GU(SCION_PQ2_0, 1); else if (gpw == 2) SCION_GU(SCION_PQ2_0, 2);
    else if (gpw == 3) SCION_GU(SCION_PQ2_0, 3); else if (gpw == 4) SCION_GU(SCION_PQ2_0, 4);
    else return cudaErrorInvalidValue;
  } else {
    if (gpw <= 1) SCION_GU(SCION_PTQ1_0, 1); else if (gpw == 2) SCION_GU(SCION_PTQ1_0, 2);
    else if (gpw == 3) SCION_GU(SCION_PTQ1_0, 3); else if (gpw == 4) SCION_GU(SCION_PTQ1_0, 4);
    else return cudaErrorInvalidValue;
  }
#undef SCION_GU
  return cudaGetLastError();
}

bool gateup_merges_dense(const scion_layer* L, int T) { return L->Kdense > 0 && (T + 7) / 8 <= 2; }

// The gate/up of the split-K path with the dense down projection in the same launch
// (gateup_merges_dense).
cudaError_t launch_gateup_dense(const scion_layer* L, int T, float* out, cudaStream_t s) {
  GateUpArgs a;
  a.bank = L->gu_bank, a.xfrag = L->xfrag;
  a.slot_info = reinterpret_cast<const int4*>(L->slot_info), a.n_active = L->n_active, a.perm = L->perm;
  a.d = L->d, a.F = L->F, a.k = L->k, a.Gd = L->Gd, a.fmt = L->fmt;
  a.hfrag = L->h, a.pexp = L->pexp;
  DenseArgs b;
  b.w = L->dense_down, b.hz = L->hz, b.d = L->d, b.Kd = L->Kd, b.T = T, b.out = out;
  b.corr_b = L->desc.corr_packed ? static_cast<const uint8_t*>(L->desc.corr_b) : nullptr, b.Fs = L->Fs, b.r = L->r;
  b.xexp = L->xexp, b.z_only = 0;
  const int slots = min(L->El, T * L->k);
  const int gx = L->F / 16, dense_x = L->d / 32;
  const int dense_tiles = dense_x * ((L->Kd + kDnKc - 1) / kDnKc);
  const dim3 grid(gx, slots + (dense_tiles + gx - 1) / gx);
  const int gpw = (L->Gd + kGuWarps - 1) / kGuWarps;
  const bool two = (T + 7) / 8 == 2;
#define SCION_GUD(F_, G_)                                                                                        \
  return two ? launch_pdl(gateup_dense_kernel<F_, G_, 2>, grid, dim3(kGuWarps * 32), down_dense_smem<2>(), s, a, b, \
                          slots, dense_x)                                                                        \
             : launch_pdl(gateup_dense_kernel<F_, G_, 1>, grid, dim3(kGuWarps * 32), down_dense_smem<1>(), s, a, b, \
                          slots, dense_x)
  if (L->fmt == SCION_PQ2_0) {
    if (gpw <= 1) SCION_GUD(SCION_PQ2_0, 1); else if (gpw == 2) SCION_GUD(SCION_PQ2_0, 2);
    else if (gpw == 3) SCION_GUD(SCION_PQ2_0, 3); else if (gpw == 4) SCION_GUD(SCION_PQ2_0, 4);
    else return cudaErrorInvalidValue;
  } else {
    if (gpw <= 1) SCION_GUD(SCION_PTQ1_0, 1); else if (gpw == 2) SCION_GUD(SCION_PTQ1_0, 2);
    else if (gpw == 3) SCION_GUD(SCION_PTQ1_0, 3); else if (gpw == 4) SCION_GUD(SCION_PTQ1_0, 4);
    else return cudaErrorInvalidValue;
  }
#undef SCION_GUD
  return cudaGetLastError();
}

cudaError_t launch_down_routed(const scion_layer* L, int T, float* out, cudaStream_t s) {
  DownArgs a;
  a.bank = L->dn_bank, a.hfrag = L->h;
  a.slot_info = reinterpret_cast<const int4*>(L->slot_info), a.n_active = L->n_active, a.perm = L->perm;
  a.gperm = L->gperm;
  a.d = L->d, a.F = L->F, a.k = L->k, a.GF = L->GF, a.out = out;
  const int slots = min(L->El, T * L->k);
  const dim3 grid(L->d / 16, slots);
  const int gpw = (L->GF + kDnWarps - 1) / kDnWarps;
#define SCION_DN(F_, G_) return launch_pdl(down_routed_kernel<F_, G_>, grid, dim3(kDnWarps * 32), 0, s, a)
  if (L->fmt == SCION_PQ2_0) {
    if (gpw <= 1) SCION_DN(SCION_PQ2_0, 1); else if (gpw == 2) SCION_DN(SCION_PQ2_0, 2);
    else if (gpw <= 4) SCION_DN(SCION_PQ2_0, 4);
    else return cudaErrorInvalidValue;
  } else {
    if (gpw <= 1) SCION_DN(SCION_PTQ1_0, 1); else if (gpw == 2) SCION_DN(SCION_PTQ1_0, 2);
    else if (gpw <= 4) SCION_DN(SCION_PTQ1_0, 4);
    else return cudaErrorInvalidValue;
  }
#undef SCION_DN
  return cudaGetLastError();
}

cudaError_t launch_down_dense(const scion_layer* L, int T, float* out, cudaStream_t s) {
  if (L->Kdense == 0) return cudaSuccess;
  DenseArgs b;
  b.w = L->dense_down, b.hz = L->hz, b.d = L->d, b.Kd = L->Kd, b.T = T, b.out = out;
  b.corr_b = L->desc.corr_packed ? static_cast<const uint8_t*>(L->desc.corr_b) : nullptr, b.Fs = L->Fs, b.r = L->r;
  b.xexp = L->xexp, b.z_only = 0;
  const int nt = (T + 7) / 8;
  const dim3 g2(L->d / 32, (L->Kd + kDnKc - 1) / kDnKc);
  switch (nt) {
    case 1: return launch_pdl(down_dense_kernel<1>, g2, dim3(256), down_dense_smem<1>(), s, b);
    case 2: return launch_pdl(down_dense_kernel<2>, g2, dim3(256), down_dense_smem<2>(), s, b);
    case 3: case 4: return launch_pdl(down_dense_kernel<4>, g2, dim3(256), down_dense_smem<4>(), s, b);
    default: return launch_pdl(down_dense_kernel<8>, g2, dim3(256), down_dense_smem<8>(), s, b);
  }
  return cudaGetLastError();
}

cudaError_t launch_corr_z(const CorrState* C, const __nv_bfloat16* v, int T, cudaStream_t s) {
  XProjArgs a;
  memset(&a, 0, sizeof(a));
  a.x = v, a.T = T, a.d = C->d_in, a.E = 0, a.Fs = 0, a.r = C->r, a.Kd = C->Kd, a.fmt = SCION_PQ2_0;
  a.corr_a = static_cast<const __nv_bfloat16*>(C->a);
  a.corr_blocks = C->packed ? static_cast<const uint8_t*>(C->a) : nullptr;
  a.units = C->xunits, a.n_units = C->n_xunits, a.n_chunks = C->n_xchunks, a.n_aux = 0;
  a.hz = C->hz, a.xexp = C->xexp, a.z_only = 1;
  const dim3 grid(C->n_xunits, C->n_xchunks), cluster(1, C->n_xchunks, 1);
  switch ((T + 7) / 8) {
    case 1: return launch_pdl_cluster(xproj_kernel<1>, grid, dim3(kXThreads), cluster, xproj_smem<1>(T), s, a);
    case 2: return launch_pdl_cluster(xproj_kernel<2>, grid, dim3(kXThreads), cluster, xproj_smem<2>(T), s, a);
    case 3: case 4:
      return launch_pdl_cluster(xproj_kernel<4>, grid, dim3(kXThreads), cluster, xproj_smem<4>(T), s, a);
    default: return launch_pdl_cluster(xproj_kernel<8>, grid, dim3(kXThreads), cluster, xproj_smem<8>(T), s, a);
  }
}

cudaError_t launch_corr_out(const CorrState* C, int T, float* out, cudaStream_t s) {
  DenseArgs b;
  memset(&b, 0, sizeof(b));
  b.w = C->b16, b.hz = C->hz, b.d = C->d_out, b.Kd = C->Kd, b.T = T, b.out = out;
  b.corr_b = C->packed ? static_cast<const uint8_t*>(C->b) : nullptr, b.Fs = 0, b.r = C->r;
  b.xexp = C->xexp, b.z_only = 1;
  const dim3 g2(C->d_out / 32, (C->Kd + kDnKc - 1) / kDnKc);
  switch ((T + 7) / 8) {
    case 1: return launch_pdl(down_dense_kernel<1>, g2, dim3(256), down_dense_smem<1>(), s, b);
    case 2: return launch_pdl(down_dense_kernel<2>, g2, dim3(256), down_dense_smem<2>(), s, b);
    case 3: case 4: return launch_pdl(down_dense_kernel<4>, g2, dim3(256), down_dense_smem<4>(), s, b);
    default: return launch_pdl(down_dense_kernel<8>, g2, dim3(256), down_dense_smem<8>(), s, b);
  }
}

cudaError_t launch_unfrag(int fmt, const __half* src, int rows, int G, __half* dst, cudaStream_t s) {
  int64_t n = int64_t(rows) * G * 128;
  if (n == 0) return cudaSuccess;
  unfrag_kernel<<<unsigned((n + 255) / 256), 256, 0, s>>>(fmt, src, n, dst);
  return cudaGetLastError();
}

cudaError_t configure_kernels() {
  const int xs_max = int(xproj_smem<8>(SCION_TDEC));
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(xproj_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, xs_max))) return e;
  if ((e = cudaFuncSetAttribute(xproj_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, xs_max))) return e;
  if ((e = cudaFuncSetAttribute(xproj_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, xs_max))) return e;
  if ((e = cudaFuncSetAttribute(xproj_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, xs_max))) return e;
  if ((e = cudaFuncSetAttribute(down_dense_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(down_dense_smem<1>()))))
    return e;
  if ((e = cudaFuncSetAttribute(down_dense_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(down_dense_smem<2>()))))
    return e;
  if ((e = cudaFuncSetAttribute(down_dense_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(down_dense_smem<4>()))))
    return e;
  if ((e = cudaFuncSetAttribute(down_dense_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(down_dense_smem<8>()))))
    return e;
  if ((e = configure_route_kernels())) return e;
  if ((e = configure_stream_kernels())) return e;
  if ((e = configure_tdec_kernels())) return e;
  return configure_prefill_kernels();
}

}  // namespace scion
