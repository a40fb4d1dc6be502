// scion_abi.cu -- the extern "C" entry points of libscion (declared in include/scion.h).
//
// Everything here is argument checking, memory management and launch sequencing; the
// arithmetic of the block runs in the kernels of k_route.cu and k_decode.cu.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <new>
#include <vector>

#include "scion_internal.cuh"

namespace {

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SCION_OK;
  if (e == cudaErrorMemoryAllocation) return SCION_ENOMEM;
  return SCION_ECUDA;
}

#define SCION_TRY(expr)                 \
  do {                                  \
    cudaError_t e_ = (expr);            \
    if (e_ != cudaSuccess) {            \
      st = cuda_status(e_);             \
      goto fail;                        \
    }                                   \
  } while (0)

template <typename T>
cudaError_t dev_alloc(scion_layer* L, T** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return cudaSuccess;
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), bytes);
  if (e == cudaSuccess) L->device_bytes += bytes;
  return e;
}

void free_layer(scion_layer* L) {
  if (!L) return;
  void* ptrs[] = {L->gu_bank, L->dn_bank,  L->dense_down, L->xunits,  L->logits,    L->ids,       L->gates,
                  L->counts,  L->offsets,  L->perm,       L->active,  L->n_active,  L->h,         L->hz,
                  L->xfrag,   L->x_stage, L->out_stage, L->bad,       L->err,
                  L->slot_info, L->gperm, L->route_done, L->xexp, L->pexp, L->x16d, L->hp,
                  L->dtiles, L->n_dtiles, L->xsum, L->hsum, L->any_scaled};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  if (L->side) cudaStreamDestroy(L->side);
  if (L->ev_start) cudaEventDestroy(L->ev_start);
  if (L->ev_x) cudaEventDestroy(L->ev_x);
  if (L->ev_dense) cudaEventDestroy(L->ev_dense);
  if (L->pre) {
    scion::PrefillState* P = L->pre;
    void* pp[] = {P->xunits, P->dunits, P->logits, P->ids, P->gates, P->counts, P->offsets, P->perm, P->inv,
                  P->y, P->tiles, P->n_tiles, P->x16, P->h, P->hz, P->cursor, P->corr_a16, P->xexp, P->pexp, P->gperm};
    for (void* p : pp)
      if (p) cudaFree(p);
    delete P;
  }
  delete L;
}

// Buffers, unit tables and tensor maps of the tensor-core path (batches > SCION_TDEC).
int create_prefill(scion_layer* L, cudaStream_t s) {
  if (L->E > 2048) return SCION_EINVAL;  // grouping keeps one histogram row per warp in shared memory
  scion::PrefillState* P = new (std::nothrow) scion::PrefillState;
  if (!P) return SCION_ENOMEM;
  memset(P, 0, sizeof(*P));
  L->pre = P;
  const size_t T = L->max_tokens, Tk = T * L->k;
  const size_t max_tiles = (Tk + 127) / 128 + L->El;
  cudaError_t e;
#define PTRY(x)                              \
  if ((e = (x)) != cudaSuccess) return cuda_status(e)
  PTRY(dev_alloc(L, &P->logits, sizeof(float) * T * L->E));
  PTRY(dev_alloc(L, &P->ids, sizeof(int32_t) * Tk));
  PTRY(dev_alloc(L, &P->gates, sizeof(float) * Tk));
  PTRY(dev_alloc(L, &P->counts, sizeof(int32_t) * L->El));
  PTRY(dev_alloc(L, &P->offsets, sizeof(int32_t) * (L->El + 1)));
  PTRY(dev_alloc(L, &P->perm, sizeof(int32_t) * Tk));
  PTRY(dev_alloc(L, &P->inv, sizeof(int32_t) * Tk));
  PTRY(dev_alloc(L, &P->cursor, sizeof(int32_t) * L->El));
  PTRY(dev_alloc(L, &P->y, sizeof(__half) * Tk * L->d));
  PTRY(dev_alloc(L, reinterpret_cast<uint8_t**>(&P->tiles), scion::prefill_tile_bytes() * max_tiles));
  PTRY(dev_alloc(L, &P->n_tiles, sizeof(int32_t)));
  PTRY(dev_alloc(L, &P->x16, sizeof(__half) * T * L->d));
  PTRY(dev_alloc(L, &P->xexp, sizeof(int32_t) * T));
  PTRY(dev_alloc(L, &P->pexp, sizeof(int32_t) * Tk));
  PTRY(dev_alloc(L, &P->gperm, sizeof(float) * Tk));
  PTRY(dev_alloc(L, &P->h, sizeof(__half) * Tk * L->F));
  PTRY(dev_alloc(L, &P->hz, sizeof(__half) * T * (L->Kd ? L->Kd : 64)));
  PTRY(cudaMemsetAsync(P->hz, 0, sizeof(__half) * T * (L->Kd ? L->Kd : 64), s));
  const int max_units = scion::prefill_max_units(L);
  std::vector<uint8_t> xu(scion::prefill_unit_bytes() * max_units), du(scion::prefill_unit_bytes() * max_units);
  scion::prefill_units(L, xu.data(), &P->n_xunits, du.data(), &P->n_dunits);
  P->n_xrouter = L->desc.router_fp32 ? 0 : (L->E + 127) / 128;
  PTRY(dev_alloc(L, reinterpret_cast<uint8_t**>(&P->xunits), scion::prefill_unit_bytes() * max_units));
  PTRY(dev_alloc(L, reinterpret_cast<uint8_t**>(&P->dunits), scion::prefill_unit_bytes() * max_units));
  PTRY(cudaMemcpyAsync(P->xunits, xu.data(), xu.size(), cudaMemcpyHostToDevice, s));
  PTRY(cudaMemcpyAsync(P->dunits, du.data(), du.size(), cudaMemcpyHostToDevice, s));
  if (L->r && L->desc.corr_packed) {
    PTRY(dev_alloc(L, &P->corr_a16, sizeof(__half) * size_t(L->r) * L->d));
    PTRY(scion::launch_dequant_corr(static_cast<const uint8_t*>(L->desc.corr_a), L->r, L->d, P->corr_a16, L->d, L->fmt,
                                    L->bad, s));
  }
#undef PTRY
  int st;
  const scion_layer_desc& D = L->desc;
  if (!D.router_fp32) {
    if ((st = scion::make_tmap_2d(&P->maps[0], D.w_router, 1, L->E, L->d))) return st;
    if ((st = scion::make_tmap_2d(&P->maps[1], D.w_router_delta, 1, L->E, L->d))) return st;
  }
  if (L->Fs) {
    if ((st = scion::make_tmap_2d(&P->maps[2], D.sh_gate, 1, L->Fs, L->d))) return st;
    if ((st = scion::make_tmap_2d(&P->maps[3], D.sh_up, 1, L->Fs, L->d))) return st;
  }
  if (L->r && !D.corr_packed && (st = scion::make_tmap_2d(&P->maps[4], D.corr_a, 1, L->r, L->d))) return st;
  if (L->r && D.corr_packed) {
    if ((st = scion::make_tmap_2d(&P->maps[4], P->corr_a16, 0, L->r, L->d))) return st;
    if ((st = scion::make_tmap_2d(&P->x16_map, P->x16, 0, L->max_tokens, L->d))) return st;
  }
  if (L->Kd) {
    if ((st = scion::make_tmap_2d(&P->maps[5], L->dense_down, 0, L->d, L->Kd))) return st;
    if ((st = scion::make_tmap_2d(&P->hz_map, P->hz, 0, L->max_tokens, L->Kd))) return st;
  }
  return SCION_OK;
}

int check_desc(const scion_layer_desc* D, int max_tokens) {
  if (!D || max_tokens < 1) return SCION_EINVAL;
  if (D->d <= 0 || D->d % 128 || D->ffn <= 0 || D->ffn % 128) return SCION_EINVAL;
  // the decode x-projection reduces its 512-column chunks inside one thread-block cluster (<= 8)
  if (D->d > 8 * SCION_XPROJ_KC) return SCION_EINVAL;
  if (D->n_experts < 1 || D->n_experts > 4096 || D->top_k < 1 || D->top_k > D->n_experts || D->top_k > 32)
    return SCION_EINVAL;
  if (D->shared_ffn < 0 || D->shared_ffn % 128 || D->rank < 0 || D->rank % 16) return SCION_EINVAL;
  if (D->fmt != SCION_PQ2_0 && D->fmt != SCION_PTQ1_0) return SCION_EINVAL;
  if ((D->router_fp32 != 0 && D->router_fp32 != 1) || (D->norm_topk != 0 && D->norm_topk != 1)) return SCION_EINVAL;
  if (!D->w_router || !D->w_router_delta || !D->gate_exps || !D->up_exps || !D->down_exps) return SCION_EINVAL;
  if (D->shared_ffn > 0 && (!D->sh_gate || !D->sh_up || !D->sh_down)) return SCION_EINVAL;
  if (D->rank > 0 && (!D->corr_a || !D->corr_b)) return SCION_EINVAL;
  if (D->corr_packed != 0 && D->corr_packed != 1) return SCION_EINVAL;
  if (D->corr_packed && D->rank % 128) return SCION_EINVAL;  // groups of 128 along corr_b's rows
  if (D->corr_packed && D->rank && ((reinterpret_cast<uintptr_t>(D->corr_a) | reinterpret_cast<uintptr_t>(D->corr_b)) & 1))
    return SCION_EINVAL;  // blocks are read with 2-byte loads
  if (D->sh_gate_vec) return SCION_EINVAL;  // shared-expert sigmoid gate: not supported by the kernels yet
  // expert range of an expert-parallel rank (0 local experts: all of them)
  if (D->n_local_experts < 0 || D->expert_lo < 0 || (D->n_local_experts == 0 && D->expert_lo != 0) ||
      D->expert_lo + D->n_local_experts > D->n_experts)
    return SCION_EINVAL;
  return SCION_OK;
}

// ---- kernel timing for benchmarks (see scion_profile_begin in include/scion.h)
struct Profiler {
  bool on = false;
  std::vector<cudaEvent_t> ev;  // 2 per launch
  std::vector<int> stage;
  int used = 0;
};
Profiler g_prof;
std::atomic<long long> g_launches{0};

struct StageScope {
  cudaStream_t s;
  bool rec = false;
  StageScope(int stage, cudaStream_t st) : s(st) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (g_prof.on && g_prof.used < int(g_prof.stage.size())) {
      rec = true;
      g_prof.stage[g_prof.used] = stage;
      cudaEventRecord(g_prof.ev[2 * g_prof.used], s);
    }
  }
  ~StageScope() {
    if (rec) cudaEventRecord(g_prof.ev[2 * g_prof.used++ + 1], s);
  }
};

#define SCION_STAGE(stage, call)                     \
  do {                                               \
    cudaError_t e_;                                  \
    {                                                \
      StageScope scope_(stage, s);                   \
      e_ = (call);                                   \
    }                                                \
    if (e_ != cudaSuccess) return cuda_status(e_);   \
  } while (0)

// Whole batch on the tensor-core path (T > SCION_TDEC).
int forward_prefill(const scion_layer* L, const __nv_bfloat16* x, int T, float* out, const float* resid,
                    cudaStream_t s) {
  const bool routed = L->parts & SCION_PART_ROUTED;
  if (routed && L->desc.router_fp32)
    SCION_STAGE(SCION_STAGE_ROUTER_F32, scion::launch_router_f32(L, x, T, L->pre->logits, s));
  SCION_STAGE(SCION_STAGE_X16, scion::launch_prefill_stage(SCION_STAGE_X16, L, x, T, out, resid, s));
  SCION_STAGE(SCION_STAGE_XPROJ, scion::launch_prefill_stage(SCION_STAGE_XPROJ, L, x, T, out, resid, s));
  if (routed) {
    SCION_STAGE(SCION_STAGE_ROUTE, scion::launch_prefill_stage(SCION_STAGE_ROUTE, L, x, T, out, resid, s));
    SCION_STAGE(SCION_STAGE_GATEUP, scion::launch_prefill_stage(SCION_STAGE_GATEUP, L, x, T, out, resid, s));
  }
  if (scion::prefill_dense_down(L))
    SCION_STAGE(SCION_STAGE_DOWN_DENSE, scion::launch_prefill_stage(SCION_STAGE_DOWN_DENSE, L, x, T, out, resid, s));
  if (routed) {
    SCION_STAGE(SCION_STAGE_DOWN_ROUTED, scion::launch_prefill_stage(SCION_STAGE_DOWN_ROUTED, L, x, T, out, resid, s));
    if (L->deterministic)
      SCION_STAGE(SCION_STAGE_COMBINE, scion::launch_prefill_stage(SCION_STAGE_COMBINE, L, x, T, out, resid, s));
  }
  return SCION_OK;
}

// Same, but records the first failure in `status` and skips the launch once one has failed
// (used where work already forked onto the side stream must still be joined).
#define SCION_STAGE_INTO(status, stage, call)          \
  do {                                                 \
    if ((status) == SCION_OK) {                        \
      cudaError_t e_;                                  \
      {                                                \
        StageScope scope_(stage, s);                   \
        e_ = (call);                                   \
      }                                                \
      if (e_ != cudaSuccess) (status) = cuda_status(e_); \
    }                                                  \
  } while (0)

// One decode pass of T <= SCION_TDEC tokens.
int forward_pass(const scion_layer* L, const __nv_bfloat16* x, int T, float* out, const float* resid, cudaStream_t s) {
  // which parts of the block this forward computes (SCION_OPT_PARTS)
  const bool routed = L->parts & SCION_PART_ROUTED, dense = (L->parts & SCION_PART_DENSE) && L->Kdense;
  if (routed && L->desc.router_fp32)
    SCION_STAGE(SCION_STAGE_ROUTER_F32, scion::launch_router_f32(L, x, T, L->logits, s));
  const bool ring = T >= L->stream_min_tokens;
  // tcgen05 expert GEMMs instead of the bulk-copy ring kernels (their tiles come from the grouping
  // kernels of up to 512 experts)
  const bool tcd = ring && L->tc_decode && L->E <= 512;
  // Batches on the ring kernels split the dense work off the expert path: the caller's stream
  // runs the router part of the x-projection (with x's fragment rows and the clearing of out),
  // the layer's side stream the shared-expert / correction part of the x-projection (from the
  // start, beside the router part: it needs only x) and then, once out is cleared, the dense
  // down projection, beside routing and the expert kernels; the caller's stream joins it at the end.
  const bool side = routed && dense && ring;
  // x-projection units: router units first, then shared gate/up and correction A
  const int unit0 = routed ? 0 : L->n_xrouter;
  const int nx_main = routed ? ((dense && !side) ? L->n_xunits : L->n_xrouter) : (dense ? L->n_xunits - L->n_xrouter : 0);
  if (!side) {
    SCION_STAGE(SCION_STAGE_XPROJ, scion::launch_xproj(L, x, T, out, resid, unit0, nx_main, true, tcd && routed, s));
  }
  int st = SCION_OK;
  if (side) {
    // fork: the side stream starts after everything issued on the caller's stream so far (x ready)
    cudaError_t e = cudaEventRecord(L->ev_start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(L->side, L->ev_start, 0);
    if (e != cudaSuccess) return cuda_status(e);  // nothing was launched on the side stream
    // the router part first (the critical path), then the side stream's part
    SCION_STAGE_INTO(st, SCION_STAGE_XPROJ,
                     scion::launch_xproj(L, x, T, out, resid, unit0, nx_main, true, tcd && routed, s));
    int st_side = SCION_OK;
    {
      cudaStream_t s = L->side;  // SCION_STAGE_INTO launches and records on `s`
      SCION_STAGE_INTO(st_side, SCION_STAGE_XPROJ,
                       scion::launch_xproj(L, x, T, out, nullptr, L->n_xrouter, L->n_xunits - L->n_xrouter, false,
                                           false, s));
    }
    // the dense down projection adds into out after the caller's stream has cleared it (and
    // written the tokens' range exponents)
    if (st == SCION_OK && (e = cudaEventRecord(L->ev_x, s)) == cudaSuccess) e = cudaStreamWaitEvent(L->side, L->ev_x, 0);
    if (e != cudaSuccess && st == SCION_OK) st = cuda_status(e);
    if (st == SCION_OK) {
      cudaStream_t s = L->side;
      SCION_STAGE_INTO(st_side, SCION_STAGE_DOWN_DENSE, scion::launch_down_dense(L, T, out, s));
    }
    // the join is recorded whatever happened above, so that no later work on the caller's stream
    // (a retry, the next call) can overlap side-stream work that still writes out or hz
    if ((e = cudaEventRecord(L->ev_dense, L->side)) != cudaSuccess) {
      cudaStreamSynchronize(L->side);
      st_side = cuda_status(e);
    }
    if (st == SCION_OK) st = st_side;
  }
  // small batches: the dense down projection rides in the gate/up launch (it needs only the
  // x-projection), off the critical path of the routed kernels
  const bool merged = routed && dense && !ring && scion::gateup_merges_dense(L, T);
  if (routed) {
    SCION_STAGE_INTO(st, SCION_STAGE_ROUTE, scion::launch_route(L, T, s));
    SCION_STAGE_INTO(st, SCION_STAGE_GATEUP, tcd      ? scion::launch_tdec(2, L, T, out, s)
                                             : ring   ? scion::launch_stream_gateup(L, T, s)
                                             : merged ? scion::launch_gateup_dense(L, T, out, s)
                                                      : scion::launch_gateup(L, x, T, s));
    SCION_STAGE_INTO(st, SCION_STAGE_DOWN_ROUTED, tcd    ? scion::launch_tdec(1, L, T, out, s)
                                                  : ring ? scion::launch_stream_down(L, T, out, s)
                                                         : scion::launch_down_routed(L, T, out, s));
  }
  if (side) {
    const cudaError_t e = cudaStreamWaitEvent(s, L->ev_dense, 0);
    return st != SCION_OK ? st : cuda_status(e);
  }
  if (dense && !merged) SCION_STAGE_INTO(st, SCION_STAGE_DOWN_DENSE, scion::launch_down_dense(L, T, out, s));
  return st;
}

}  // namespace

extern "C" const char* scion_status_str(int status) {
  switch (status) {
    case SCION_OK: return "ok";
    case SCION_EINVAL: return "invalid argument";
    case SCION_ENOMEM: return "out of memory";
    case SCION_ECUDA: return "CUDA error";
    case SCION_EFORMAT: return "invalid code in a packed block";
    case SCION_ETIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

extern "C" int scion_pack_device(int fmt, const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out,
                                 int64_t* bad_count, void* stream) {
  if ((fmt != SCION_PQ2_0 && fmt != SCION_PTQ1_0) || n_groups < 0) return SCION_EINVAL;
  if (n_groups > 0 && (!codes || !scales || !out)) return SCION_EINVAL;
  return cuda_status(scion::launch_pack(fmt, codes, scales, n_groups, out, bad_count, as_stream(stream)));
}

extern "C" int scion_unpack_device(int fmt, const uint8_t* in, int64_t n_groups, int8_t* codes, uint16_t* scales,
                                   int64_t* bad_count, void* stream) {
  if ((fmt != SCION_PQ2_0 && fmt != SCION_PTQ1_0) || n_groups < 0) return SCION_EINVAL;
  if (n_groups > 0 && (!in || !codes || !scales)) return SCION_EINVAL;
  return cuda_status(scion::launch_unpack(fmt, in, n_groups, codes, scales, bad_count, as_stream(stream)));
}

extern "C" int scion_layer_create(const scion_layer_desc* desc, int max_tokens, void* stream, scion_layer** out) {
  if (!out) return SCION_EINVAL;
  *out = nullptr;
  int st = check_desc(desc, max_tokens);
  if (st != SCION_OK) return st;
  scion_layer* L = new (std::nothrow) scion_layer;
  if (!L) return SCION_ENOMEM;
  memset(L, 0, sizeof(*L));
  L->desc = *desc;
  L->d = desc->d, L->E = desc->n_experts, L->k = desc->top_k, L->F = desc->ffn;
  L->elo = desc->expert_lo, L->El = desc->n_local_experts ? desc->n_local_experts : desc->n_experts;
  L->parts = SCION_PART_ROUTED | SCION_PART_DENSE;
  L->Fs = desc->shared_ffn, L->r = desc->rank, L->fmt = desc->fmt, L->max_tokens = max_tokens;
  L->Gd = L->d / 128, L->GF = L->F / 128;
  L->Kdense = L->Fs + L->r;
  L->Kd = (L->Kdense + 63) / 64 * 64;
  L->stream_min_tokens = 16;  // below this the few active experts spread better over the split-K kernels
  L->tc_decode = 0;
  L->deterministic = 1;
  cudaStream_t s = as_stream(stream);
  const int tb = scion::tile_bytes(L->fmt);
  const int TD = SCION_TDEC;
  std::vector<scion::XUnit> units;
  int64_t bad_host = 0;

  if (!desc->router_fp32)
    for (int e0 = 0; e0 < L->E; e0 += 16) units.push_back({scion::kUnitRouter, e0});
  for (int f0 = 0; f0 < L->Fs; f0 += 16) units.push_back({scion::kUnitSwiglu, f0});
  for (int q0 = 0; q0 < L->r; q0 += 16) units.push_back({scion::kUnitPlain, q0});
  L->n_xunits = int(units.size());
  L->n_xrouter = desc->router_fp32 ? 0 : (L->E + 15) / 16;
  L->n_xchunks = (L->d + SCION_XPROJ_KC - 1) / SCION_XPROJ_KC;

  SCION_TRY(scion::configure_kernels());
  SCION_TRY(dev_alloc(L, &L->gu_bank, size_t(L->El) * (L->F / 128) * L->Gd * 2 * 8 * tb));
  SCION_TRY(dev_alloc(L, &L->dn_bank, size_t(L->El) * (L->d / 128) * L->GF * 8 * tb));
  SCION_TRY(dev_alloc(L, &L->dense_down, size_t(L->d) * L->Kd * sizeof(__half)));
  SCION_TRY(dev_alloc(L, &L->xunits, sizeof(scion::XUnit) * (units.size() ? units.size() : 1)));
  SCION_TRY(dev_alloc(L, &L->logits, sizeof(float) * TD * L->E));
  SCION_TRY(dev_alloc(L, &L->ids, sizeof(int32_t) * TD * L->k));
  SCION_TRY(dev_alloc(L, &L->gates, sizeof(float) * TD * L->k));
  SCION_TRY(dev_alloc(L, &L->counts, sizeof(int32_t) * L->El));
  SCION_TRY(dev_alloc(L, &L->offsets, sizeof(int32_t) * (L->El + 1)));
  SCION_TRY(dev_alloc(L, &L->perm, sizeof(int32_t) * TD * L->k));
  SCION_TRY(dev_alloc(L, &L->gperm, sizeof(float) * TD * L->k));
  SCION_TRY(dev_alloc(L, &L->active, sizeof(int32_t) * L->El));
  SCION_TRY(dev_alloc(L, &L->n_active, sizeof(int32_t)));
  SCION_TRY(dev_alloc(L, reinterpret_cast<uint8_t**>(&L->slot_info), sizeof(int4) * L->El));
  SCION_TRY(dev_alloc(L, &L->route_done, sizeof(unsigned)));
  SCION_TRY(cudaMemsetAsync(L->route_done, 0, sizeof(unsigned), s));
  SCION_TRY(dev_alloc(L, &L->h, sizeof(__half) * TD * L->k * L->GF * SCION_BROW));
  SCION_TRY(dev_alloc(L, &L->hz, sizeof(__half) * TD * (L->Kd ? L->Kd : 1)));
  SCION_TRY(dev_alloc(L, &L->xfrag, sizeof(__half) * TD * L->Gd * SCION_BROW));
  SCION_TRY(dev_alloc(L, &L->xexp, sizeof(int32_t) * TD));
  SCION_TRY(dev_alloc(L, &L->pexp, sizeof(int32_t) * TD * L->k));
  SCION_TRY(dev_alloc(L, reinterpret_cast<uint8_t**>(&L->dtiles),
                      sizeof(int4) * (size_t(TD) * L->k / scion::kDecTile + L->El + 1)));
  SCION_TRY(dev_alloc(L, &L->n_dtiles, sizeof(int32_t)));
  SCION_TRY(dev_alloc(L, &L->any_scaled, sizeof(int32_t)));
  SCION_TRY(dev_alloc(L, &L->xsum, sizeof(float) * TD * L->Gd));
  SCION_TRY(dev_alloc(L, &L->hsum, sizeof(float) * TD * L->k * L->GF));
  SCION_TRY(dev_alloc(L, &L->x16d, sizeof(__half) * TD * L->d));
  SCION_TRY(dev_alloc(L, &L->hp, sizeof(__half) * TD * L->k * L->F));
  SCION_TRY(dev_alloc(L, &L->x_stage, sizeof(__nv_bfloat16) * size_t(max_tokens) * L->d));
  SCION_TRY(dev_alloc(L, &L->out_stage, sizeof(float) * size_t(max_tokens) * L->d));
  SCION_TRY(dev_alloc(L, &L->bad, sizeof(int64_t)));
  SCION_TRY(dev_alloc(L, &L->err, sizeof(int)));
  SCION_TRY(cudaStreamCreateWithFlags(&L->side, cudaStreamNonBlocking));
  SCION_TRY(cudaEventCreateWithFlags(&L->ev_start, cudaEventDisableTiming));
  SCION_TRY(cudaEventCreateWithFlags(&L->ev_x, cudaEventDisableTiming));
  SCION_TRY(cudaEventCreateWithFlags(&L->ev_dense, cudaEventDisableTiming));
  SCION_TRY(cudaMemsetAsync(L->err, 0, sizeof(int), s));

  if (!units.empty())
    SCION_TRY(cudaMemcpyAsync(L->xunits, units.data(), sizeof(scion::XUnit) * units.size(), cudaMemcpyHostToDevice, s));
  SCION_TRY(cudaMemsetAsync(L->hz, 0, sizeof(__half) * TD * (L->Kd ? L->Kd : 1), s));
  SCION_TRY(cudaMemsetAsync(L->bad, 0, sizeof(int64_t), s));
  if (L->Kd) {
    SCION_TRY(cudaMemsetAsync(L->dense_down, 0, size_t(L->d) * L->Kd * sizeof(__half), s));
    if (L->Fs)
      SCION_TRY(scion::launch_bf16_to_f16_rows(static_cast<const __nv_bfloat16*>(desc->sh_down), L->d, L->Fs,
                                               L->dense_down, L->Kd, s));
    if (L->r && !desc->corr_packed)
      SCION_TRY(scion::launch_bf16_to_f16_rows(static_cast<const __nv_bfloat16*>(desc->corr_b), L->d, L->r,
                                               L->dense_down + L->Fs, L->Kd, s));
    if (L->r && desc->corr_packed) {
      // ternary correction factors: B as its exact fp16 values beside the shared down weights;
      // A's codes checked here (decode reads its blocks in place)
      SCION_TRY(scion::launch_dequant_corr(static_cast<const uint8_t*>(desc->corr_b), L->d, L->r,
                                           L->dense_down + L->Fs, L->Kd, -1, L->bad, s));
      SCION_TRY(scion::launch_dequant_corr(static_cast<const uint8_t*>(desc->corr_a), L->r, L->d, nullptr, 0, -1,
                                           L->bad, s));
    }
  }
  SCION_TRY(scion::launch_retile(L->fmt, static_cast<const uint8_t*>(desc->gate_exps), L->El, L->F, L->Gd, 2, 0,
                                 L->gu_bank, L->bad, s));
  SCION_TRY(scion::launch_retile(L->fmt, static_cast<const uint8_t*>(desc->up_exps), L->El, L->F, L->Gd, 2, 1,
                                 L->gu_bank, L->bad, s));
  SCION_TRY(scion::launch_retile(L->fmt, static_cast<const uint8_t*>(desc->down_exps), L->El, L->d, L->GF, 1, 0,
                                 L->dn_bank, L->bad, s));
  // B operand of the tcgen05 decode down projection: the hidden rows, 16-row TMA boxes
  if ((st = scion::make_tmap_2d(&L->hp_map, L->hp, 0, int64_t(TD) * L->k, L->F, 16)) != SCION_OK) goto fail;
  if (max_tokens > SCION_TDEC) {
    st = create_prefill(L, s);
    if (st != SCION_OK) goto fail;
  }
  SCION_TRY(cudaMemcpyAsync(&bad_host, L->bad, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
  SCION_TRY(cudaStreamSynchronize(s));
  if (bad_host != 0) {
    st = SCION_EFORMAT;
    goto fail;
  }
  *out = L;
  return SCION_OK;
fail:
  free_layer(L);
  return st;
}

extern "C" void scion_layer_destroy(scion_layer* layer) {
  if (!layer) return;
  cudaDeviceSynchronize();
  free_layer(layer);
}

extern "C" size_t scion_layer_device_bytes(const scion_layer* layer) { return layer ? layer->device_bytes : 0; }

namespace {
int forward_any(const void* x, int T, const scion_layer* L, const float* resid, float* out, void* stream) {
  if (!L || T < 0 || T > L->max_tokens) return SCION_EINVAL;
  if (T == 0) return SCION_OK;
  if (!x || !out) return SCION_EINVAL;
  // 16-byte accesses
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(resid)) & 15)
    return SCION_EINVAL;
  cudaStream_t s = as_stream(stream);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  // a layer built for more than one decode pass (max_tokens > SCION_TDEC) has the tensor-core
  // path, so every batch is either one decode pass or one prefill
  if (T > SCION_TDEC) return forward_prefill(L, xb, T, out, resid, s);
  return forward_pass(L, xb, T, out, resid, s);
}
}  // namespace

extern "C" int scion_moe_forward(const void* x, int T, const scion_layer* L, float* out, void* stream) {
  return forward_any(x, T, L, nullptr, out, stream);
}

extern "C" int scion_moe_forward_residual(const void* x, int T, const scion_layer* L, const float* resid, float* out,
                                          void* stream) {
  if (!resid) return SCION_EINVAL;
  return forward_any(x, T, L, resid, out, stream);
}

extern "C" int scion_moe_forward_host(const void* x_host, int T, const scion_layer* L, float* out_host, void* stream) {
  if (!L || T < 0 || T > L->max_tokens) return SCION_EINVAL;
  if (T == 0) return SCION_OK;
  if (!x_host || !out_host) return SCION_EINVAL;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = cudaMemcpyAsync(L->x_stage, x_host, sizeof(__nv_bfloat16) * size_t(T) * L->d,
                                  cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_status(e);
  int st = scion_moe_forward(L->x_stage, T, L, L->out_stage, stream);
  if (st != SCION_OK) return st;
  e = cudaMemcpyAsync(out_host, L->out_stage, sizeof(float) * size_t(T) * L->d, cudaMemcpyDeviceToHost, s);
  return cuda_status(e);
}

extern "C" int scion_moe_forward_debug(const void* x, int T, const scion_layer* L, float* out,
                                       const scion_debug_out* dbg, void* stream) {
  if (!L || !dbg || T < 0 || T > L->max_tokens) return SCION_EINVAL;
  const bool pre = T > SCION_TDEC;
  if (pre && !L->pre) return SCION_EINVAL;
  int st = scion_moe_forward(x, T, L, out, stream);
  if (st != SCION_OK || T == 0) return st;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = cudaSuccess;
  auto cp = [&](void* dst, const void* src, size_t bytes) {
    if (dst && e == cudaSuccess) e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s);
  };
  const scion::PrefillState* P = L->pre;
  cp(dbg->logits, pre ? P->logits : L->logits, sizeof(float) * size_t(T) * L->E);
  cp(dbg->ids, pre ? P->ids : L->ids, sizeof(int32_t) * size_t(T) * L->k);
  cp(dbg->gates, pre ? P->gates : L->gates, sizeof(float) * size_t(T) * L->k);
  cp(dbg->counts, pre ? P->counts : L->counts, sizeof(int32_t) * size_t(L->El));
  cp(dbg->offsets, pre ? P->offsets : L->offsets, sizeof(int32_t) * size_t(L->El + 1));
  cp(dbg->perm, pre ? P->perm : L->perm, sizeof(int32_t) * size_t(T) * L->k);
  if (dbg->h && e == cudaSuccess)
    e = pre ? scion::launch_unperm_prefill(L->fmt, 0, P->h, int64_t(T) * L->k * L->F, reinterpret_cast<__half*>(dbg->h), s)
        : (T >= L->stream_min_tokens && L->tc_decode && L->E <= 512)
            ? scion::launch_unperm_prefill(L->fmt, 1, L->hp, int64_t(T) * L->k * L->F, reinterpret_cast<__half*>(dbg->h), s)
            : scion::launch_unfrag(L->fmt, L->h, T * L->k, L->GF, reinterpret_cast<__half*>(dbg->h), s);
  if (dbg->hz && e == cudaSuccess && L->Kdense)
    e = cudaMemcpy2DAsync(dbg->hz, sizeof(__half) * L->Kdense, pre ? P->hz : L->hz, sizeof(__half) * L->Kd,
                          sizeof(__half) * L->Kdense, T, cudaMemcpyDeviceToDevice, s);
  return cuda_status(e);
}

extern "C" int scion_debug_route(const void* x, int T, const scion_layer* L, int32_t* ids, float* gates,
                                 int32_t* offsets, int32_t* perm, void* stream) {
  if (!L) return SCION_EINVAL;
  scion_debug_out dbg;
  memset(&dbg, 0, sizeof(dbg));
  dbg.ids = ids, dbg.gates = gates, dbg.offsets = offsets, dbg.perm = perm;
  return scion_moe_forward_debug(x, T, L, L->out_stage, &dbg, stream);
}

// ------------------------------------------------ correction branch on the attention output
namespace {
template <typename T>
cudaError_t corr_alloc(scion::CorrState* C, T** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return cudaSuccess;
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), bytes);
  if (e == cudaSuccess) C->device_bytes += bytes;
  return e;
}

void free_corr(scion_corr* H) {
  if (!H) return;
  scion::CorrState& C = H->c;
  void* ptrs[] = {C.b16, C.xunits, C.hz, C.xexp, C.v16, C.a16, C.units_z, C.units_o, C.err};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  delete H;
}
}  // namespace

extern "C" int scion_corr_create(const scion_corr_desc* D, int max_tokens, void* stream, scion_corr** out) {
  if (!out) return SCION_EINVAL;
  *out = nullptr;
  if (!D || max_tokens < 1 || !D->corr_a || !D->corr_b) return SCION_EINVAL;
  if (D->d_in <= 0 || D->d_in % 128 || D->d_in > 8 * SCION_XPROJ_KC || D->d_out <= 0 || D->d_out % 128) return SCION_EINVAL;
  if (D->packed != 0 && D->packed != 1) return SCION_EINVAL;
  if (D->rank <= 0 || D->rank % 16 || D->rank > 4096 || (D->packed && D->rank % 128)) return SCION_EINVAL;
  if (D->packed && ((reinterpret_cast<uintptr_t>(D->corr_a) | reinterpret_cast<uintptr_t>(D->corr_b)) & 1))
    return SCION_EINVAL;  // blocks are read with 2-byte loads
  if (!D->packed && ((reinterpret_cast<uintptr_t>(D->corr_a) | reinterpret_cast<uintptr_t>(D->corr_b)) & 15))
    return SCION_EINVAL;  // rows are read with 16-byte loads
  scion_corr* H = new (std::nothrow) scion_corr;
  if (!H) return SCION_ENOMEM;
  memset(H, 0, sizeof(*H));
  scion::CorrState& C = H->c;
  C.d_in = D->d_in, C.d_out = D->d_out, C.r = D->rank, C.packed = D->packed, C.max_tokens = max_tokens;
  C.Kd = (C.r + 63) / 64 * 64;
  C.a = D->corr_a, C.b = D->corr_b;
  C.n_xunits = (C.r + 15) / 16, C.n_xchunks = (C.d_in + SCION_XPROJ_KC - 1) / SCION_XPROJ_KC;
  cudaStream_t s = as_stream(stream);
  int st = SCION_OK;
  int64_t* bad = nullptr;
  int64_t bad_host = 0;
  std::vector<scion::XUnit> units;
  for (int q0 = 0; q0 < C.r; q0 += 16) units.push_back({scion::kUnitPlain, q0});
  const int T = max_tokens > SCION_TDEC ? max_tokens : SCION_TDEC;
  SCION_TRY(scion::configure_kernels());
  SCION_TRY(corr_alloc(&C, &C.b16, sizeof(__half) * size_t(C.d_out) * C.Kd));
  SCION_TRY(corr_alloc(&C, &C.xunits, sizeof(scion::XUnit) * units.size()));
  SCION_TRY(corr_alloc(&C, &C.hz, sizeof(__half) * size_t(T) * C.Kd));
  SCION_TRY(corr_alloc(&C, &C.xexp, sizeof(int32_t) * T));
  SCION_TRY(corr_alloc(&C, &C.err, sizeof(int)));
  SCION_TRY(cudaMalloc(&bad, sizeof(int64_t)));
  SCION_TRY(cudaMemsetAsync(bad, 0, sizeof(int64_t), s));
  SCION_TRY(cudaMemsetAsync(C.err, 0, sizeof(int), s));
  SCION_TRY(cudaMemsetAsync(C.hz, 0, sizeof(__half) * size_t(T) * C.Kd, s));  // pad columns stay 0
  SCION_TRY(cudaMemsetAsync(C.b16, 0, sizeof(__half) * size_t(C.d_out) * C.Kd, s));
  SCION_TRY(cudaMemcpyAsync(C.xunits, units.data(), sizeof(scion::XUnit) * units.size(), cudaMemcpyHostToDevice, s));
  if (C.packed) {
    // B's exact fp16 values (code * scale); A's codes are checked here and read in place by decode
    SCION_TRY(scion::launch_dequant_corr(static_cast<const uint8_t*>(C.b), C.d_out, C.r, C.b16, C.Kd, -1, bad, s));
    SCION_TRY(scion::launch_dequant_corr(static_cast<const uint8_t*>(C.a), C.r, C.d_in, nullptr, 0, -1, bad, s));
  } else {
    SCION_TRY(scion::launch_bf16_to_f16_rows(static_cast<const __nv_bfloat16*>(C.b), C.d_out, C.r, C.b16, C.Kd, s));
  }
  if (max_tokens > SCION_TDEC) {
    SCION_TRY(corr_alloc(&C, &C.v16, sizeof(__half) * size_t(max_tokens) * C.d_in));
    if (C.packed) {
      SCION_TRY(corr_alloc(&C, &C.a16, sizeof(__half) * size_t(C.r) * C.d_in));
      // in the column order of v16 (the PTQ1_0 order carries no per-position factors)
      SCION_TRY(scion::launch_dequant_corr(static_cast<const uint8_t*>(C.a), C.r, C.d_in, C.a16, C.d_in, SCION_PTQ1_0,
                                           bad, s));
    }
    if ((st = scion::corr_prefill_setup(&C, s)) != SCION_OK) goto fail;
  }
  SCION_TRY(cudaMemcpyAsync(&bad_host, bad, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
  SCION_TRY(cudaStreamSynchronize(s));
  cudaFree(bad);
  bad = nullptr;
  if (bad_host) {
    st = SCION_EFORMAT;
    goto fail;
  }
  *out = H;
  return SCION_OK;
fail:
  if (bad) cudaFree(bad);
  free_corr(H);
  return st;
}

extern "C" void scion_corr_destroy(scion_corr* H) {
  if (!H) return;
  cudaDeviceSynchronize();
  free_corr(H);
}

extern "C" int scion_corr_forward(const void* v, int T, const scion_corr* H, const float* base, float* out,
                                  void* stream) {
  if (!H || T < 0 || T > H->c.max_tokens) return SCION_EINVAL;
  if (T == 0) return SCION_OK;
  if (!v || !out) return SCION_EINVAL;
  if ((reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(base)) & 15)
    return SCION_EINVAL;
  const scion::CorrState& C = H->c;
  cudaStream_t s = as_stream(stream);
  if (T > SCION_TDEC) {
    g_launches.fetch_add(2, std::memory_order_relaxed);  // three kernels, the scope counts one
    StageScope scope_(SCION_STAGE_XPROJ, s);
    return cuda_status(scion::launch_corr_prefill(&C, static_cast<const __nv_bfloat16*>(v), T, base, out, s));
  }
  // out starts at base (or zero); the B z product is added with fp32 reductions
  cudaError_t e = base ? (base != out ? cudaMemcpyAsync(out, base, sizeof(float) * size_t(T) * C.d_out,
                                                        cudaMemcpyDeviceToDevice, s)
                                      : cudaSuccess)
                       : cudaMemsetAsync(out, 0, sizeof(float) * size_t(T) * C.d_out, s);
  if (e != cudaSuccess) return cuda_status(e);
  SCION_STAGE(SCION_STAGE_XPROJ, scion::launch_corr_z(&C, static_cast<const __nv_bfloat16*>(v), T, s));
  SCION_STAGE(SCION_STAGE_DOWN_DENSE, scion::launch_corr_out(&C, T, out, s));
  return SCION_OK;
}

extern "C" size_t scion_corr_device_bytes(const scion_corr* H) { return H ? H->c.device_bytes : 0; }

extern "C" int scion_corr_check(const scion_corr* H, void* stream) {
  if (!H) return SCION_EINVAL;
  cudaStream_t s = as_stream(stream);
  int err = 0;
  cudaError_t e = cudaMemcpyAsync(&err, H->c.err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  if (err != 0) {
    const int zero = 0;
    e = cudaMemcpyAsync(H->c.err, &zero, sizeof(int), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return err;
  }
  return SCION_OK;
}

extern "C" int scion_layer_check(const scion_layer* L, void* stream) {
  if (!L) return SCION_EINVAL;
  cudaStream_t s = as_stream(stream);
  int err = 0;
  cudaError_t e = cudaMemcpyAsync(&err, L->err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  if (err != 0) {
    const int zero = 0;
    e = cudaMemcpyAsync(L->err, &zero, sizeof(int), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return err;
  }
  return SCION_OK;
}

extern "C" int scion_profile_begin(int max_launches) {
  if (g_prof.on || max_launches < 1) return SCION_EINVAL;
  g_prof.ev.assign(size_t(2) * max_launches, nullptr);
  g_prof.stage.assign(size_t(max_launches), -1);
  for (auto& e : g_prof.ev) {
    cudaError_t err = cudaEventCreate(&e);
    if (err != cudaSuccess) {
      for (auto& f : g_prof.ev)
        if (f) cudaEventDestroy(f);
      g_prof.ev.clear();
      g_prof.stage.clear();
      return cuda_status(err);
    }
  }
  g_prof.used = 0;
  g_prof.on = true;
  return SCION_OK;
}

extern "C" int scion_profile_end(int n_stages, double* ms_total, int64_t* launches) {
  if (!g_prof.on || n_stages < 0 || (n_stages > 0 && (!ms_total || !launches))) return SCION_EINVAL;
  g_prof.on = false;
  for (int i = 0; i < n_stages; ++i) ms_total[i] = 0.0, launches[i] = 0;
  cudaError_t err = cudaSuccess;
  if (g_prof.used > 0) err = cudaEventSynchronize(g_prof.ev[2 * g_prof.used - 1]);
  for (int i = 0; i < g_prof.used && err == cudaSuccess; ++i) {
    float ms = 0.f;
    err = cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]);
    int st = g_prof.stage[i];
    if (err == cudaSuccess && st >= 0 && st < n_stages) ms_total[st] += ms, launches[st] += 1;
  }
  for (auto& e : g_prof.ev) cudaEventDestroy(e);
  g_prof.ev.clear();
  g_prof.stage.clear();
  g_prof.used = 0;
  return cuda_status(err);
}

extern "C" int64_t scion_kernel_launches(void) { return g_launches.load(); }

extern "C" int scion_layer_set_option(scion_layer* L, int option, int value) {
  if (!L) return SCION_EINVAL;
  switch (option) {
    case SCION_OPT_STREAM_MIN_TOKENS:
      if (value < 1) return SCION_EINVAL;
      L->stream_min_tokens = value;
      return SCION_OK;
    case SCION_OPT_DECODE_TC:
      if (value != 0 && value != 1) return SCION_EINVAL;
      L->tc_decode = value;
      return SCION_OK;
    case SCION_OPT_DETERMINISTIC:
      if (value != 0 && value != 1) return SCION_EINVAL;
      L->deterministic = value;
      return SCION_OK;
    case SCION_OPT_PARTS:
      if (value < 1 || value > (SCION_PART_ROUTED | SCION_PART_DENSE)) return SCION_EINVAL;
      L->parts = value;
      return SCION_OK;
    default:
      return SCION_EINVAL;
  }
}
