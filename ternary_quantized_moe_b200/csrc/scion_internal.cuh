// scion_internal.cuh -- shared internals of libscion (not part of the ABI).
//
// Device layout of the ternary expert banks (built once by scion_layer_create):
// every expert matrix [R rows][K] is cut into 16-row x 128-column tiles ("sub-tile
// blocks").  A sub-tile block holds exactly the bytes of its sixteen 128-weight
// container blocks, regrouped so that lane L = 4*r + c of a warp (r = L/4 in 0..7,
// c = L%4) finds what it needs for rows r and r+8 in one contiguous run:
//
//   PQ2_0, 544 B = 16 x 34:
//     [16L + j]        row r,   code byte 8c + j   (j < 8)
//     [16L + 8 + j]    row r+8, code byte 8c + j
//     [512 + 4r + 0/2] fp16 scale of row r / row r+8
//   PTQ1_0, 448 B = 16 x 28:
//     [12L + m]        row r,   quintet byte 6c + m (m < 6)
//     [12L + 6 + m]    row r+8, quintet byte 6c + m
//     [384 + 4r + 0/1] even remainder trits of row r / row r+8
//     [384 + 4r + 2/3] odd remainder trits of row r / row r+8
//   The 8 remainder trits of a row (digits 0..4 of quintet byte 24, digits 0..2 of tail byte
//   25: columns 120..127) are re-encoded as 2-bit fields (trit value 0..2): trit 2i at bits
//   2i..2i+1 of the "even" byte, trit 2i+1 at bits 2i..2i+1 of the "odd" byte.  The same 16
//   bits per row; lane c then takes its columns 120+2c, 121+2c with one shift and one mask.
//     [416 + 4r + 0/2] fp16 scale of row r / row r+8
//
// Sub-tile blocks are ordered [expert][row/128][group][matrix][row%128/16] with
// matrix = {gate, up} interleaved for the gate/up bank and a single matrix for the
// down bank, so a 128-row x 128-column stage of either bank is one contiguous run.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/scion.h"

#define SCION_TDEC 64         // tokens of the decode path (larger batches take the tensor-core path)
#define SCION_XPROJ_KC 512    // K columns per x-projection CTA (4 warps x 128)
namespace scion {
constexpr int kDecTile = 16;  // tokens per tile of the tensor-core decode kernels (one MMA N)
}

// Fragment-ordered B operands of the decode expert kernels (x for gate/up, h for down) are
// stored per 128-column group as 128 fp16 values followed by a 16-byte tail; the first 4
// bytes of the tail hold  -2^-24 * sum_k B_k * 4^f(k)  in fp32 (the start value of the PQ2_0
// subnormal unpack's accumulators, see tern_tile.cuh).
#define SCION_BROW 136        // halves per group row (128 + 8)

namespace scion {

constexpr int kPq2Block = 34;
constexpr int kPtq1Block = 28;
constexpr int kPq2Tile = 544;   // 16 rows x 34 B
constexpr int kPtq1Tile = 448;  // 16 rows x 28 B

__host__ __device__ inline int tile_bytes(int fmt) { return fmt == SCION_PQ2_0 ? kPq2Tile : kPtq1Tile; }
__host__ __device__ inline int block_bytes(int fmt) { return fmt == SCION_PQ2_0 ? kPq2Block : kPtq1Block; }

// x-projection work unit: 16 output rows of one kind.
enum UnitKind : int { kUnitRouter = 0, kUnitSwiglu = 1, kUnitPlain = 2 };
struct XUnit {
  int kind;
  int row0;  // first row of the unit within its matrices
};

// Buffers and tensor maps of the tensor-core (prefill) path, present when the layer
// accepts batches above one decode pass.
struct PrefillState {
  CUtensorMap maps[6];  // A operands: router, delta, sh_gate, sh_up, corr_a, dense_down
  CUtensorMap hz_map;   // B operand of the dense down GEMM
  void* xunits;         // DenseUnit[] (device): router units, shared gate/up units, correction units
  int n_xunits;
  int n_xrouter;        // router units at the front of xunits
  void* dunits;
  int n_dunits;
  CUtensorMap x16_map;  // B operand of the ternary correction A's units (fp16 GEMM against x16)
  __half* corr_a16;     // [r][d] exact fp16 copy of the ternary correction A in x16's column order
  float* logits;        // [maxT][E]
  int32_t* ids;         // [maxT][k]
  float* gates;         // [maxT][k]
  int32_t* counts;      // [E]
  int32_t* offsets;     // [E+1]
  int32_t* perm;        // [maxT*k]
  int32_t* inv;         // [maxT*k] position of entry t*k+j in perm
  int32_t* cursor;      // [E] next free position of each expert's segment (grouping scratch)
  __half* y;            // [maxT*k][d] expert down outputs in fp16 (gate not yet applied), one row per routed entry
  void* tiles;          // token tiles of the ternary GEMMs (128 or 160 tokens), [maxT*k/128 + E]
  int32_t* n_tiles;
  __half* x16;          // [maxT][d]   x 2^s_t in the container column order (fp16)
  int32_t* xexp;        // [maxT] per-token range exponent s_t (see token_shift)
  int32_t* pexp;        // [maxT*k] s_t of the token of each routed position
  float* gperm;         // [maxT*k] gate of the entry at each routed position, times 2^(-2 s_t)
  __half* h;            // [maxT*k][F] expert SwiGLU hidden, container column order
  __half* hz;           // [maxT][Kd]
};

// The correction branch on the attention output (scion_corr_*): z = A v, out = base + B z.
struct CorrState {
  int d_in, d_out, r, Kd, packed, max_tokens;
  const void* a;       // bf16 [r][d_in] or PQ2_0 blocks [r][d_in/128] (read in place)
  const void* b;       // bf16 [d_out][r] or PQ2_0 blocks [d_out][r/128] (packed: read in place by decode)
  __half* b16;         // [d_out][Kd] exact fp16 copy of B (bf16 decode and the tensor-core path)
  XUnit* xunits;       // decode: one kind-Plain unit per 16 rows of A
  int n_xunits, n_xchunks;
  __half* hz;          // [max_tokens][Kd] z times 2^s_t
  int32_t* xexp;       // [max_tokens] range exponent of each token
  // tensor-core path (max_tokens > SCION_TDEC)
  __half* v16;         // [max_tokens][d_in] v 2^s_t in the PTQ1_0 column order (fp16)
  __half* a16;         // packed A: [r][d_in] exact fp16 in the same column order
  void* units_z;       // dense-GEMM units: rows of A, then rows of B
  void* units_o;
  int n_units_z, n_units_o;
  CUtensorMap map_a, map_b16, map_v16, map_hz;
  int* err;            // device status word (a bounded wait of the tensor-core path that gave up)
  size_t device_bytes;
};

}  // namespace scion

struct scion_corr {
  scion::CorrState c;
};

struct scion_layer {
  scion_layer_desc desc;
  int d, E, k, F, Fs, r, fmt, max_tokens;
  int elo, El;      // local experts [elo, elo + El) of the E the router scores (banks and grouping hold El)
  int parts;        // SCION_PART_ROUTED | SCION_PART_DENSE: what a forward computes
  int Gd, GF;       // 128-groups along d and along F
  int Kdense;       // Fs + r
  int Kd;           // Kdense rounded up to 64: row stride of dense_down and hz (pad = 0)
  // owned device memory
  uint8_t* gu_bank;    // [E][F/128][Gd][2][8][tile]
  uint8_t* dn_bank;    // [E][d/128][GF][8][tile]
  __half* dense_down;  // [d][Kd] fp16: sh_down | corr_b | 0
  scion::XUnit* xunits;
  int n_xunits;
  int n_xrouter;     // router units (the first n_xrouter entries of xunits)
  int n_xchunks;
  // workspace (sized for SCION_TDEC tokens per pass, max_tokens for staging)
  float* logits;     // [TDEC][E]
  int32_t* ids;      // [TDEC][k]
  float* gates;      // [TDEC][k]
  int32_t* counts;   // [E]
  int32_t* offsets;  // [E+1]
  int32_t* perm;     // [TDEC*k]
  float* gperm;      // [TDEC*k] gate of the entry at each routed position, times 2^(-2 s_t)
  int32_t* active;   // [E]
  int32_t* n_active; // [1]
  void* slot_info;    // int4 [E]: {expert, first position, token count, 0} per active slot
  unsigned* route_done;  // [1] arrival counter of the multi-CTA decode route kernel (zero between calls)
  __half* h;         // [TDEC*k][GF][SCION_BROW] fragment order + group-sum tails
  __half* hz;        // [TDEC][Kd] (pad columns stay 0)
  __half* xfrag;     // [TDEC][Gd][SCION_BROW] x in fragment order (fp16) + group-sum tails
  int32_t* xexp;     // [TDEC] per-token range exponent s_t (see token_shift)
  int32_t* pexp;     // [TDEC*k] s_t of the token of each routed position (written by the routing)
  int32_t* any_scaled;  // [1] nonzero when some token of the pass has s_t != 0 (written by the routing)
  void* dtiles;      // int4 [TDEC*k/kDecTile + E]: tiles of <= kDecTile tokens per active expert (routing)
  int32_t* n_dtiles; // [1]
  float* xsum;       // [TDEC][Gd] per-group sums of the tensor-core decode's B values times 4^f (x)
  float* hsum;       // [TDEC*k][GF] the same for the expert hidden
  // tensor-core decode (batches on the ring threshold and above, tc_decode = 1): x 2^s_t in the
  // tcgen05 column order, the expert hidden one row per routed position, and its TMA map (16-row boxes)
  __half* x16d;      // [TDEC][d]
  __half* hp;        // [TDEC*k][F]
  CUtensorMap hp_map;
  int tc_decode;     // 1 (default): decode batches of stream_min_tokens and more run the tcgen05 expert GEMMs
  int deterministic; // 1: the prefill down projection writes one row per routed entry and a combine sums them in slot order
  void* x_stage;     // [max_tokens][d] bf16 (host-buffer forward)
  float* out_stage;  // [max_tokens][d]
  int64_t* bad;      // [1] invalid-code counter used at create
  int* err;          // [1] device status word (a bounded wait that gave up writes ETIMEOUT)
  scion::PrefillState* pre;  // tensor-core path (nullptr when max_tokens <= SCION_TDEC)
  int stream_min_tokens;     // decode batches of at least this many tokens use the bulk-copy ring kernels
  cudaStream_t side;         // the dense down projection of ring-kernel batches runs here
  cudaEvent_t ev_start, ev_x, ev_dense;  // fork (x ready) / out cleared / dense down done (join)
  size_t device_bytes;
};

namespace scion {

// ---------------------------------------------------------------- launchers
// k_format.cu
cudaError_t launch_pack(int fmt, const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out,
                        int64_t* bad, cudaStream_t s);
cudaError_t launch_unpack(int fmt, const uint8_t* in, int64_t n_groups, int8_t* codes, uint16_t* scales,
                          int64_t* bad, cudaStream_t s);
// Re-tile a packed bank [E][R][G] blocks into sub-tile blocks; `nmat`/`mat` select
// the matrix slot of the interleaved gate/up bank (nmat = 1 for the down bank).
cudaError_t launch_retile(int fmt, const uint8_t* src, int E, int R, int G, int nmat, int mat, uint8_t* dst,
                          int64_t* bad, cudaStream_t s);
cudaError_t launch_bf16_to_f16_rows(const __nv_bfloat16* src, int rows, int cols, __half* dst, int ld_dst,
                                    cudaStream_t s);

// k_route.cu
cudaError_t launch_router_f32(const scion_layer* L, const __nv_bfloat16* x, int T, float* logits, cudaStream_t s);
cudaError_t launch_route(const scion_layer* L, int T, cudaStream_t s);
cudaError_t configure_route_kernels();
cudaError_t launch_slot_info(const scion_layer* L, cudaStream_t s);

// k_decode.cu
// Units [unit0, unit0 + n_units) of the layer's x-projection table (router units first, then
// shared gate/up, then correction A); `aux` adds the CTAs that write x's fragment rows and
// clear out and the hidden's group-sum tails.
// x16 = true: the aux CTAs write x for the tcgen05 decode kernels (L->x16d) instead of the
// fragment-ordered rows of the register kernels.
cudaError_t launch_xproj(const scion_layer* L, const __nv_bfloat16* x, int T, float* out, const float* resid,
                         int unit0, int n_units, bool aux, bool x16, cudaStream_t s);
cudaError_t launch_gateup(const scion_layer* L, const __nv_bfloat16* x, int T, cudaStream_t s);
cudaError_t launch_down_routed(const scion_layer* L, int T, float* out, cudaStream_t s);
cudaError_t launch_down_dense(const scion_layer* L, int T, float* out, cudaStream_t s);
bool gateup_merges_dense(const scion_layer* L, int T);
cudaError_t launch_gateup_dense(const scion_layer* L, int T, float* out, cudaStream_t s);
// fragment-ordered rows [rows][G][SCION_BROW] -> natural order [rows][G*128]
cudaError_t launch_unfrag(int fmt, const __half* src, int rows, int G, __half* dst, cudaStream_t s);
cudaError_t configure_kernels();

// k_stream.cu (bulk-copy-ring expert kernels for decode batches)
cudaError_t configure_stream_kernels();
cudaError_t launch_stream_gateup(const scion_layer* L, int T, cudaStream_t s);
cudaError_t launch_stream_down(const scion_layer* L, int T, float* out, cudaStream_t s);

// correction branch on the attention output: decode kernels (k_decode.cu) and the tensor-core
// path with its unit tables (k_prefill.cu)
cudaError_t launch_corr_z(const CorrState* C, const __nv_bfloat16* v, int T, cudaStream_t s);
cudaError_t launch_corr_out(const CorrState* C, int T, float* out, cudaStream_t s);
int corr_prefill_setup(CorrState* C, cudaStream_t s);
cudaError_t launch_corr_prefill(const CorrState* C, const __nv_bfloat16* v, int T, const float* base, float* out,
                                cudaStream_t s);

// k_prefill.cu
int make_tmap_2d(CUtensorMap* map, const void* ptr, int bf16, int64_t rows, int64_t K, int box_rows = 128);
// k_tdec.cu: expert gate/up (na = 2) or down (na = 1, gate-weighted fp32 reductions into out) of
// a decode batch on the tensor cores, tiles of up to kDecTile tokens listed by the routing.
cudaError_t configure_tdec_kernels();
cudaError_t launch_tdec(int na, const scion_layer* L, int T, float* out, cudaStream_t s);
cudaError_t configure_prefill_kernels();
size_t prefill_unit_bytes();
size_t prefill_tile_bytes();
int prefill_max_units(const scion_layer* L);
void prefill_units(const scion_layer* L, void* xunits_host, int* n_x, void* dunits_host, int* n_d);
cudaError_t launch_dequant_corr(const uint8_t* blocks, int rows, int K, __half* dst, int ld, int order,
                                int64_t* bad, cudaStream_t s);
cudaError_t launch_unperm_prefill(int fmt, int pos_scaled, const __half* src, int64_t n, __half* dst, cudaStream_t s);
cudaError_t launch_prefill_stage(int stage, const scion_layer* L, const __nv_bfloat16* x, int T, float* out,
                                 const float* resid, cudaStream_t s);
// Whether a prefill forward runs the dense down projection (shared expert / correction selected
// and present).
bool prefill_dense_down(const scion_layer* L);

// Launch with programmatic dependent launch: the kernel may start while its predecessor
// on the stream drains; it must execute pdl_wait() before touching anything the
// predecessor (or anything earlier on the stream) writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Same with a thread-block cluster of `cluster` CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, dim3 cluster, size_t smem,
                               cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster.x;
  attr[1].val.clusterDim.y = cluster.y;
  attr[1].val.clusterDim.z = cluster.z;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------ device helpers
// Wait until the preceding grid on the stream has completed and its writes are visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next grid on the stream to be scheduled (it still waits in pdl_wait()).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// Thread-block cluster: full barrier of all threads of the cluster (release / acquire), the
// shared-window address of a variable, its address in the CTA of cluster rank `rank`, and a
// load through that address.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t smem_addr(const void* p) { return uint32_t(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ uint32_t map_cluster_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t magic) {
  // (a & mask) | magic in one LOP3
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(r) : "r"(a), "r"(mask), "r"(magic));
  return r;
}

// ---------------------------------------------------- per-token range scaling
// The expert GEMMs and the stored hidden values run in fp16, whose range (2^-14 .. 65504 for
// full precision) is far narrower than bf16's.  Every token t gets an exponent s_t from the
// largest magnitude of its activations: s_t = 0 while max|x_t| lies in [2^-3, 2^6) (the usual
// case: nothing changes), otherwise s_t = 2 - floor(log2 max|x_t|) clamped to [-40, 40], which
// brings max|x_t 2^s_t| into [4, 8).  All factors are powers of two, so every scaling is exact:
//   expert input     x 2^s                  (fp16 operand of the expert gate/up GEMMs)
//   expert hidden    h 2^(2s)               (silu(g 2^-s) * (u 2^s) from the scaled sums g, u;
//                                            |silu(y)| <= |y| keeps it within the range of the
//                                            hidden of the scaled token)
//   expert output    gate 2^(-2s) y         (applied where the weighted sum enters out)
//   shared / z rows  hz 2^p, the dense down projection multiplies its output by 2^-p:
//                    p = s on a layer without a shared expert (z alone, which grows like x),
//                    p = 2s on a layer without a correction (the shared hidden, like x^2), and
//                    with both p = s for s > 0, else 2s (for s < 0 the x^2 terms dominate the
//                    output, for s > 0 the correction does, so the term whose stored value may
//                    leave the fp16 range is the one too small to matter).
constexpr int kShiftLo = -3, kShiftHi = 5, kShiftTarget = 2, kShiftMax = 40;
// s_t from the largest bf16 magnitude of the token (its bit pattern with the sign cleared)
__host__ __device__ __forceinline__ int token_shift(uint32_t max_mag_bits) {
  if (max_mag_bits == 0) return 0;
  const int e = int(max_mag_bits >> 7) - 127;  // floor(log2 |x|) for normal values; subnormals -> -127
  if (e >= kShiftLo && e <= kShiftHi) return 0;
  const int s = kShiftTarget - e;
  return s < -kShiftMax ? -kShiftMax : (s > kShiftMax ? kShiftMax : s);
}
// 2^n as fp32 for |n| <= 126, built from its exponent field
__host__ __device__ __forceinline__ float pow2i(int n) {
  union {
    uint32_t u;
    float f;
  } v;
  v.u = uint32_t(n + 127) << 23;
  return v.f;
}
// exponent p of the shared / z rows' factor (see above)
__host__ __device__ __forceinline__ int hz_shift(int s, int has_shared, int has_corr) {
  if (!has_shared) return s;
  return (has_corr && s > 0) ? s : 2 * s;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// PTQ1_0 remainder trits in the sub-tile layout (2-bit fields, trit value 0..2): the low two
// bits of each half of (rem >> shift), OR-ed into fp16 1024 and less 1025, give the half2
// (trit - 1) exactly.
__device__ __forceinline__ uint32_t ptq1_rem_pair(uint32_t rem, int shift) {
  const __half2 v = u32_as_h2(lop3_and_or(rem >> shift, 0x00030003u, 0x64006400u));
  return h2_as_u32(__hsub2(v, u32_as_h2(0x64016401u)));
}

// x * sigmoid(x) with the fast exponential and division (a few ulp of fp32; the result is
// rounded to fp16 or multiplied into an fp32 accumulation well above that error).
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

}  // namespace scion
