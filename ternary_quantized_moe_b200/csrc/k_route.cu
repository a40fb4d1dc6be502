// k_route.cu -- router logits (fp32 routers), top-k gating and token-to-expert grouping.
//
// Router: logit[t][e] = x_t . W_r[e] + x_t . D[e] ("Scion: ternary MoE quantization with
// trained corrections", The idea: router deltas; "Scion-35B-A3B" model card, Weight
// Representation: routers stay F32).  Top-k: the k largest logits ("Scion-35B-A3B"
// Model Overview: top-8 of 256; FlashNext Model Overview: top-10 of 512), ties to the
// lower expert id; gates = softmax over the selected logits (or the selected entries
// of a softmax over all E).  Grouping: histogram of the T*k ids, exclusive scan, and a
// stable scatter in (token, slot) order -- the per-expert token lists that the expert
// GEMMs consume ("Scion: ..." Serving notes: the expert matmul computes k experts per
// token).
#include <float.h>
#include <math.h>

#include "scion_internal.cuh"
#include "topk_warp.cuh"

namespace scion {
namespace {

constexpr int kRouteThreads = 256;

// One warp per (token, expert): FFMA in fp32 over d (no TF32).
__global__ void router_f32_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wr,
                                  const float* __restrict__ wd, int d, int E, float* __restrict__ logits) {
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int e = blockIdx.x * 8 + warp, t = blockIdx.y;
  if (e >= E) return;
  const __nv_bfloat16* xt = x + int64_t(t) * d;
  const float* a = wr + int64_t(e) * d;
  const float* b = wd + int64_t(e) * d;
  float sa = 0.f, sb = 0.f;
  for (int i = lane; i < d; i += 32) {
    float xv = __bfloat162float(xt[i]);
    sa = fmaf(xv, a[i], sa);
    sb = fmaf(xv, b[i], sb);
  }
  for (int o = 16; o; o >>= 1) {
    sa += __shfl_xor_sync(0xffffffffu, sa, o);
    sb += __shfl_xor_sync(0xffffffffu, sb, o);
  }
  if (lane == 0) logits[int64_t(t) * E + e] = sa + sb;
}

// Local index of expert e in the handle's range [lo, lo + nl), or -1 (an entry of another rank).
__device__ __forceinline__ int local_expert(int e, int lo, int nl) {
  const unsigned u = unsigned(e - lo);
  return u < unsigned(nl) ? int(u) : -1;
}

__device__ __forceinline__ void argmax_merge(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) {
    v = v2;
    i = i2;
  }
}

// Single CTA for one pass of T <= SCION_TDEC tokens.
// smem: vals[8][E] f32 | counts[E] | cursor[E] | ids[T*k]
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                              int norm_topk, int32_t* __restrict__ ids_out,
                                                              float* __restrict__ gates_out,
                                                              int32_t* __restrict__ counts_out,
                                                              int32_t* __restrict__ offsets_out,
                                                              int32_t* __restrict__ perm_out,
                                                              float* __restrict__ gperm_out,
                                                              int32_t* __restrict__ active_out,
                                                              int32_t* __restrict__ n_active_out,
                                                              const int32_t* __restrict__ xexp,
                                                              int32_t* __restrict__ pexp_out,
                                                              int32_t* __restrict__ any_scaled, int elo, int El) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = kRouteThreads / 32;
  float* vals = smem + warp * E;
  int32_t* counts = reinterpret_cast<int32_t*>(smem + nwarps * E);  // [El]
  int32_t* cursor = counts + El;
  int32_t* ids_s = cursor + El;  // local expert of each entry, -1 for another rank's

  for (int e = threadIdx.x; e < El; e += kRouteThreads) counts[e] = 0;

  // ---- top-k and gates, one warp per token
  for (int t = warp; t < T; t += nwarps) {
    const float* row = logits + int64_t(t) * E;
    float mx = -INFINITY;
    for (int e = lane; e < E; e += 32) {
      // NaN / -inf rank below every finite logit but above "taken" (-inf), so each of the
      // k rounds always selects an index in [0, E) that was not selected before.
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
      for (int e = lane; e < E; e += 32) argmax_merge(bv, bi, vals[e], e);
      for (int o = 16; o; o >>= 1) {
        float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
        int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
        argmax_merge(bv, bi, v2, i2);
      }
      if (lane == j) {
        my_v = bv;
        my_id = bi;
      }
      __syncwarp();
      if (lane == (bi & 31)) vals[bi] = -INFINITY;
      __syncwarp();
    }
    float top = __shfl_sync(0xffffffffu, my_v, 0);
    float ex = 0.f;
    if (lane < k) ex = norm_topk ? expf(my_v - top) : expf(my_v - mx);
    float z = ex;
    for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (!norm_topk) z = zall;
    if (lane < k) {
      ids_out[t * k + lane] = my_id;
      gates_out[t * k + lane] = ex / z;
      const int le = local_expert(my_id, elo, El);
      ids_s[t * k + lane] = le;
      if (le >= 0) atomicAdd(&counts[le], 1);
    }
    __syncwarp();
  }
  __syncthreads();

  // ---- exclusive scan of counts and the active-expert list (warp 0)
  if (warp == 0) {
    const int per = (El + 31) / 32;
    const int e0 = lane * per, e1 = min(El, e0 + per);
    int s = 0, a = 0;
    for (int e = e0; e < e1; ++e) {
      s += counts[e];
      a += counts[e] > 0;
    }
    int si = s, ai = a;
    for (int o = 1; o < 32; o <<= 1) {
      int s2 = __shfl_up_sync(0xffffffffu, si, o), a2 = __shfl_up_sync(0xffffffffu, ai, o);
      if (lane >= o) {
        si += s2;
        ai += a2;
      }
    }
    int run = si - s, arun = ai - a;
    for (int e = e0; e < e1; ++e) {
      int c = counts[e];
      offsets_out[e] = run;
      cursor[e] = run;
      counts_out[e] = c;
      if (c > 0) active_out[arun++] = e;
      run += c;
    }
    if (lane == 31) {
      offsets_out[El] = si;
      *n_active_out = ai;
    }
    int sc_any = 0;
    for (int t = lane; t < T; t += 32) sc_any |= xexp[t] != 0;
    sc_any = __any_sync(0xffffffffu, sc_any);
    if (lane == 0) *any_scaled = sc_any;
    __syncwarp();
    // ---- stable scatter in (token, slot) order, 32 entries at a time
    const int n = T * k;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < n; base += 32) {
      int i = base + lane;
      const bool mine = i < n && ids_s[i] >= 0;
      int e = mine ? ids_s[i] : -1 - lane;  // unique dummies never match real ids
      unsigned mask = __match_any_sync(0xffffffffu, e);
      int rank = __popc(mask & lt);
      int cur = mine ? cursor[e] : 0;
      __syncwarp();
      if (mine) {
        const int sh = xexp[i / k];
        perm_out[cur + rank] = i;
        gperm_out[cur + rank] = gates_out[i] * pow2i(-2 * sh);
        pexp_out[cur + rank] = sh;
        if (rank == 0) cursor[e] = cur + __popc(mask);
      }
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------- decode route
// One pass of T <= SCION_TDEC tokens (E <= 512).  Top-k and gates by one warp per token, then
// the grouping of the T*k entries inside one CTA's shared memory: histogram, exclusive scan,
// active-expert list with the per-slot records, and the stable scatter in (token, slot) order.
// Up to 32 tokens one CTA does everything; above that the top-k is spread over ceil(T/4) CTAs
// and the last one to finish stages the entries and groups them.

// The grouping of n = T k staged entries (T <= 64) by all threads of one CTA.  An expert appears
// at most once among a token's k entries (the top-k ids are distinct), so the rank of entry
// (t, j) among its expert's entries in the stable (token, slot) order is the number of earlier
// tokens that chose the expert: popc(tmask[e] & (2^t - 1)) with tmask[e] the expert's token bits.
// ids_s holds local expert indices (-1: an entry of another rank, not grouped); E = local experts.

// all threads: histogram and token bits of the staged entries (counts, tmask zeroed before)
__device__ __forceinline__ void group_count(const int32_t* ids_s, int n, int k, int tid, int nthr, int32_t* counts,
                                            unsigned long long* tmask) {
  for (int i = tid; i < n; i += nthr) {
    const int e = ids_s[i];
    if (e >= 0) {
      atomicAdd(&counts[e], 1);
      atomicOr(&tmask[e], 1ull << (i / k));
    }
  }
}

// warp 0: exclusive scan of the counts (cursor[e] = first position of expert e), the per-expert
// records, the active-expert list with its per-slot records, the tile list of the tensor-core
// decode kernels, and whether any token of the batch is range-scaled.
__device__ __forceinline__ void group_scan(const int32_t* xexp_s, int n, int k, int E, int lane, const int32_t* counts,
                                           int32_t* cursor, int32_t* __restrict__ counts_out,
                                           int32_t* __restrict__ offsets_out, int32_t* __restrict__ active_out,
                                           int32_t* __restrict__ n_active_out, int4* __restrict__ slot_info,
                                           int4* __restrict__ dtiles, int32_t* __restrict__ n_dtiles,
                                           int32_t* __restrict__ any_scaled) {
  const int per = (E + 31) / 32;
  const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
  int sc = 0, ac = 0, tc = 0;
  for (int e = e0; e < e1; ++e) sc += counts[e], ac += counts[e] > 0, tc += (counts[e] + kDecTile - 1) / kDecTile;
  int si = sc, ai = ac, ti = tc;
  for (int o = 1; o < 32; o <<= 1) {
    const int s2 = __shfl_up_sync(0xffffffffu, si, o), a2 = __shfl_up_sync(0xffffffffu, ai, o);
    const int t2 = __shfl_up_sync(0xffffffffu, ti, o);
    if (lane >= o) si += s2, ai += a2, ti += t2;
  }
  int run = si - sc, arun = ai - ac, trun = ti - tc;
  for (int e = e0; e < e1; ++e) {
    const int c = counts[e];
    offsets_out[e] = run;
    cursor[e] = run;
    counts_out[e] = c;
    if (c > 0) {
      active_out[arun] = e;
      slot_info[arun] = make_int4(e, run, c, 0);
      ++arun;
    }
    // tiles of the tensor-core decode kernels: {expert, first token, tokens, first position}
    if (dtiles)
      for (int c0 = 0; c0 < c; c0 += kDecTile) dtiles[trun++] = make_int4(e, c0, min(kDecTile, c - c0), run + c0);
    run += c;
  }
  if (lane == 31) {
    offsets_out[E] = si, *n_active_out = ai;
    if (dtiles) *n_dtiles = ti;
  }
  // whether any token of the batch is range-scaled (the expert epilogues skip the factors if not)
  int sc_any = 0;
  for (int t = lane; t < n / k; t += 32) sc_any |= xexp_s[t] != 0;
  sc_any = __any_sync(0xffffffffu, sc_any);
  if (lane == 0) *any_scaled = sc_any;
}

// all threads: each entry to its stable position.  Each routed position gets its token's range
// exponent (pexp_out) and its gate times 2^(-2 s_t) (gperm_out), the factor that takes the scaled
// expert hidden back to the block's units.
__device__ __forceinline__ void group_scatter(const int32_t* ids_s, const float* gates_s, const int32_t* xexp_s, int n,
                                              int k, int tid, int nthr, const int32_t* cursor,
                                              const unsigned long long* tmask, int32_t* __restrict__ perm_out,
                                              float* __restrict__ gperm_out, int32_t* __restrict__ pexp_out) {
  for (int i = tid; i < n; i += nthr) {
    const int e = ids_s[i];
    if (e < 0) continue;
    const int t = i / k;
    const int pos = cursor[e] + __popcll(tmask[e] & ((1ull << t) - 1ull));
    const int sh = xexp_s[t];
    perm_out[pos] = i;
    gperm_out[pos] = gates_s[i] * pow2i(-2 * sh);
    pexp_out[pos] = sh;
  }
}

// Single CTA (T <= 32): 1024 threads, one warp per token; 512 when each lane holds 16 logits,
// to keep the sorted lane lists in registers.
template <int VPL>
constexpr int rc_threads() {
  return VPL >= 16 ? 512 : 1024;
}

template <int VPL>
__global__ void __launch_bounds__(rc_threads<VPL>()) route_cta_kernel(
    const float* __restrict__ logits, int T, int E, int k, int norm_topk, int32_t* __restrict__ ids,
    float* __restrict__ gates, int32_t* __restrict__ counts_out, int32_t* __restrict__ offsets_out,
    int32_t* __restrict__ perm_out, float* __restrict__ gperm_out, int32_t* __restrict__ active_out,
    int32_t* __restrict__ n_active_out, int4* __restrict__ slot_info, const int32_t* __restrict__ xexp,
    int32_t* __restrict__ pexp_out, int4* __restrict__ dtiles, int32_t* __restrict__ n_dtiles,
    int32_t* __restrict__ any_scaled, int elo, int El) {
  extern __shared__ unsigned long long rs8[];  // tmask [El] | ids [T*k] | gates [T*k] | counts [El] | cursor [El] | xexp [T]
  const int n = T * k;
  unsigned long long* tmask = rs8;
  float* rs = reinterpret_cast<float*>(rs8 + El);
  int32_t* ids_s = reinterpret_cast<int32_t*>(rs);
  float* gates_s = rs + n;
  int32_t* counts = reinterpret_cast<int32_t*>(rs + 2 * n);
  int32_t* cursor = counts + El;
  int32_t* xexp_s = cursor + El;
  constexpr int kThr = rc_threads<VPL>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  for (int e = threadIdx.x; e < El; e += kThr) counts[e] = 0, tmask[e] = 0ull;
  pdl_wait();
  for (int t = threadIdx.x; t < T; t += kThr) xexp_s[t] = xexp[t];
  for (int t = warp; t < T; t += kThr / 32)
    warp_topk<VPL>(logits + int64_t(t) * E, E, k, norm_topk, lane, ids_s + t * k, gates_s + t * k);
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kThr) {
    ids[i] = ids_s[i];
    gates[i] = gates_s[i];
    ids_s[i] = local_expert(ids_s[i], elo, El);
  }
  __syncthreads();
  group_count(ids_s, n, k, threadIdx.x, kThr, counts, tmask);
  __syncthreads();
  if (warp == 0)
    group_scan(xexp_s, n, k, El, lane, counts, cursor, counts_out, offsets_out, active_out, n_active_out, slot_info,
               dtiles, n_dtiles, any_scaled);
  __syncthreads();
  group_scatter(ids_s, gates_s, xexp_s, n, k, threadIdx.x, kThr, cursor, tmask, perm_out, gperm_out, pexp_out);
}

// ceil(T/4) CTAs of 4 warps (T > 32); the last CTA to finish groups.
constexpr int kRmThreads = 128;

template <int VPL>
__global__ void __launch_bounds__(kRmThreads) route_multi_kernel(
    const float* __restrict__ logits, int T, int E, int k, int norm_topk, int32_t* __restrict__ ids,
    float* __restrict__ gates, int32_t* __restrict__ counts_out, int32_t* __restrict__ offsets_out,
    int32_t* __restrict__ perm_out, float* __restrict__ gperm_out, int32_t* __restrict__ active_out,
    int32_t* __restrict__ n_active_out, int4* __restrict__ slot_info, unsigned* __restrict__ done,
    const int32_t* __restrict__ xexp, int32_t* __restrict__ pexp_out, int4* __restrict__ dtiles,
    int32_t* __restrict__ n_dtiles, int32_t* __restrict__ any_scaled, int elo, int El) {
  extern __shared__ unsigned long long rs8[];  // tmask [El] | ids [T*k] | gates [T*k] | counts [El] | cursor [El] | xexp [T]
  __shared__ int last;
  const int n = T * k;
  unsigned long long* tmask = rs8;
  float* rs = reinterpret_cast<float*>(rs8 + El);
  int32_t* ids_s = reinterpret_cast<int32_t*>(rs);
  float* gates_s = rs + n;
  int32_t* counts = reinterpret_cast<int32_t*>(rs + 2 * n);
  int32_t* cursor = counts + El;
  int32_t* xexp_s = cursor + El;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kRmThreads / 32) + warp;
  pdl_trigger();
  pdl_wait();
  if (t < T) warp_topk<VPL>(logits + int64_t(t) * E, E, k, norm_topk, lane, ids + t * k, gates + t * k);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = (atomicAdd(done, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int e = threadIdx.x; e < El; e += kRmThreads) counts[e] = 0, tmask[e] = 0ull;
  for (int i = threadIdx.x; i < n; i += kRmThreads)
    ids_s[i] = local_expert(__ldcg(&ids[i]), elo, El), gates_s[i] = __ldcg(&gates[i]);
  for (int i = threadIdx.x; i < T; i += kRmThreads) xexp_s[i] = xexp[i];
  __syncthreads();
  group_count(ids_s, n, k, threadIdx.x, kRmThreads, counts, tmask);
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) *done = 0;
    group_scan(xexp_s, n, k, El, lane, counts, cursor, counts_out, offsets_out, active_out, n_active_out, slot_info,
               dtiles, n_dtiles, any_scaled);
  }
  __syncthreads();
  group_scatter(ids_s, gates_s, xexp_s, n, k, threadIdx.x, kRmThreads, cursor, tmask, perm_out, gperm_out, pexp_out);
}

size_t route_cta_smem(int T, int El, int k) {
  return sizeof(unsigned long long) * size_t(El) + sizeof(float) * (2 * size_t(T) * k + 2 * size_t(El) + size_t(T));
}

}  // namespace

cudaError_t launch_router_f32(const scion_layer* L, const __nv_bfloat16* x, int T, float* logits, cudaStream_t s) {
  dim3 grid((L->E + 7) / 8, T);
  router_f32_kernel<<<grid, 256, 0, s>>>(x, static_cast<const float*>(L->desc.w_router),
                                         static_cast<const float*>(L->desc.w_router_delta), L->d, L->E, logits);
  return cudaGetLastError();
}

cudaError_t launch_route(const scion_layer* L, int T, cudaStream_t s) {
  if (L->E <= 512) {
    const size_t smem = route_cta_smem(T, L->El, L->k);
    // tile list only for the tensor-core decode kernels (stream_min_tokens and up, option set)
    int4* dtl = (L->tc_decode && T >= L->stream_min_tokens) ? reinterpret_cast<int4*>(L->dtiles) : nullptr;
    const int vpl = (L->E + 31) / 32;
#define SCION_ROUTE_CTA(V)                                                                                     \
  return T <= 32 ? launch_pdl(route_cta_kernel<V>, dim3(1), dim3(rc_threads<V>()), smem, s, L->logits, T, L->E, \
                              L->k, L->desc.norm_topk, L->ids, L->gates, L->counts, L->offsets, L->perm,       \
                              L->gperm, L->active, L->n_active, reinterpret_cast<int4*>(L->slot_info), L->xexp, \
                              L->pexp, dtl, L->n_dtiles, L->any_scaled, L->elo, L->El)                         \
                 : launch_pdl(route_multi_kernel<V>, dim3((T + 3) / 4), dim3(kRmThreads), smem, s, L->logits, T, \
                              L->E, L->k, L->desc.norm_topk, L->ids, L->gates, L->counts, L->offsets, L->perm, \
                              L->gperm, L->active, L->n_active, reinterpret_cast<int4*>(L->slot_info),         \
                              L->route_done, L->xexp, L->pexp, dtl, L->n_dtiles,                               \
                              L->any_scaled, L->elo, L->El)
    if (vpl <= 1) SCION_ROUTE_CTA(1);
    else if (vpl <= 2) SCION_ROUTE_CTA(2);
    else if (vpl <= 4) SCION_ROUTE_CTA(4);
    else if (vpl <= 8) SCION_ROUTE_CTA(8);
    else SCION_ROUTE_CTA(16);
#undef SCION_ROUTE_CTA
    return cudaGetLastError();
  }
  size_t smem = sizeof(float) * (size_t(kRouteThreads / 32) * L->E) + sizeof(int32_t) * (2 * size_t(L->El)) +
                sizeof(int32_t) * size_t(T) * L->k;
  route_kernel<<<1, kRouteThreads, smem, s>>>(L->logits, T, L->E, L->k, L->desc.norm_topk, L->ids, L->gates,
                                               L->counts, L->offsets, L->perm, L->gperm, L->active, L->n_active,
                                               L->xexp, L->pexp, L->any_scaled, L->elo, L->El);
  if (cudaError_t e = cudaGetLastError()) return e;
  return launch_slot_info(L, s);
}

__global__ void slot_info_kernel(const int32_t* __restrict__ active, const int32_t* __restrict__ n_active,
                                 const int32_t* __restrict__ offsets, const int32_t* __restrict__ counts,
                                 int4* __restrict__ slot_info, int E) {
  const int n = *n_active;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int e = active[i];
    slot_info[i] = make_int4(e, offsets[e], counts[e], 0);
  }
}

cudaError_t launch_slot_info(const scion_layer* L, cudaStream_t s) {
  slot_info_kernel<<<(L->El + 255) / 256, 256, 0, s>>>(L->active, L->n_active, L->offsets, L->counts,
                                                        reinterpret_cast<int4*>(L->slot_info), L->El);
  return cudaGetLastError();
}

cudaError_t configure_route_kernels() {
  cudaError_t e;
  const int cta_max = int(route_cta_smem(SCION_TDEC, 512, 32));
  if ((e = cudaFuncSetAttribute(route_cta_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  if ((e = cudaFuncSetAttribute(route_cta_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  if ((e = cudaFuncSetAttribute(route_cta_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  if ((e = cudaFuncSetAttribute(route_cta_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  if ((e = cudaFuncSetAttribute(route_cta_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  if ((e = cudaFuncSetAttribute(route_multi_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  if ((e = cudaFuncSetAttribute(route_multi_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  if ((e = cudaFuncSetAttribute(route_multi_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  if ((e = cudaFuncSetAttribute(route_multi_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  if ((e = cudaFuncSetAttribute(route_multi_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, cta_max))) return e;
  return cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

}  // namespace scion
