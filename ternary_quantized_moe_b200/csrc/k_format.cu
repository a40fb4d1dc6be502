// k_format.cu -- device-side container work: pack, unpack, validate and re-tile.
//
// Containers: PQ2_0 ("Scion-35B-A3B" model card, Weight Representation) and PTQ1_0
// ("Scion-FlashNext-176B-A6B" model card, Weight Representation); bit orders as in
// include/scion.h.  None of these kernels is on the per-token hot path: they run
// when banks are built or loaded.
#include "scion_internal.cuh"

namespace scion {
namespace {

__device__ __forceinline__ unsigned long long count_bad_add(int64_t* bad, unsigned long long n) {
  if (bad && n) atomicAdd(reinterpret_cast<unsigned long long*>(bad), n);
  return n;
}

// One thread per 128-weight group.
__global__ void pack_kernel(int fmt, const int8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                            int64_t n_groups, uint8_t* __restrict__ out, int64_t* bad) {
  int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= n_groups) return;
  const int8_t* c = codes + g * 128;
  unsigned nbad = 0;
  auto code_at = [&](int i) -> int {
    int v = c[i];
    if (v < -1 || v > 1) {
      ++nbad;
      v = 0;
    }
    return v + 1;  // field / trit value
  };
  uint16_t s = scales[g];
  if (fmt == SCION_PQ2_0) {
    uint8_t* o = out + g * kPq2Block;
    for (int i = 0; i < 32; ++i) {
      unsigned b = 0;
      for (int j = 0; j < 4; ++j) b |= unsigned(code_at(4 * i + j)) << (2 * j);
      o[i] = uint8_t(b);
    }
    o[32] = uint8_t(s & 0xff);
    o[33] = uint8_t(s >> 8);
  } else {
    uint8_t* o = out + g * kPtq1Block;
    for (int q = 0; q < 26; ++q) {
      int n = q < 25 ? 5 : 3, v = 0;
      for (int j = n - 1; j >= 0; --j) v = v * 3 + code_at(5 * q + j);
      o[q] = uint8_t(v);
    }
    o[26] = uint8_t(s & 0xff);
    o[27] = uint8_t(s >> 8);
  }
  count_bad_add(bad, nbad);
}

__global__ void unpack_kernel(int fmt, const uint8_t* __restrict__ in, int64_t n_groups, int8_t* __restrict__ codes,
                              uint16_t* __restrict__ scales, int64_t* bad) {
  int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= n_groups) return;
  int8_t* c = codes + g * 128;
  unsigned nbad = 0;
  if (fmt == SCION_PQ2_0) {
    const uint8_t* b = in + g * kPq2Block;
    for (int i = 0; i < 32; ++i) {
      unsigned byte = b[i];
      for (int j = 0; j < 4; ++j) {
        int f = (byte >> (2 * j)) & 3;
        nbad += (f == 3);
        c[4 * i + j] = int8_t(f == 3 ? 0 : f - 1);
      }
    }
    scales[g] = uint16_t(b[32] | (b[33] << 8));
  } else {
    const uint8_t* b = in + g * kPtq1Block;
    for (int q = 0; q < 26; ++q) {
      int n = q < 25 ? 5 : 3, v = b[q];
      bool isbad = v >= (q < 25 ? 243 : 27);
      nbad += isbad;
      for (int j = 0; j < n; ++j) {
        c[5 * q + j] = int8_t(isbad ? 0 : v % 3 - 1);
        v /= 3;
      }
    }
    scales[g] = uint16_t(b[26] | (b[27] << 8));
  }
  count_bad_add(bad, nbad);
}

// One thread per source block (e, row, g).  Writes the block's bytes to their places
// in the sub-tile layout (see scion_internal.cuh) and counts invalid fields.
__global__ void retile_kernel(int fmt, const uint8_t* __restrict__ src, int E, int R, int G, int nmat, int mat,
                              uint8_t* __restrict__ dst, int64_t* bad) {
  int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  int64_t total = int64_t(E) * R * G;
  if (idx >= total) return;
  int g = int(idx % G);
  int row = int((idx / G) % R);
  int e = int(idx / (int64_t(G) * R));
  const int bb = block_bytes(fmt), tb = tile_bytes(fmt);
  const uint8_t* s = src + idx * bb;
  int rt = row >> 7, sub = (row & 127) >> 4, rho = row & 15, r8 = rho & 7, hi = rho >> 3;
  int64_t tile_off = ((((int64_t(e) * (R >> 7) + rt) * G + g) * nmat + mat) * 8 + sub) * tb;
  uint8_t* t = dst + tile_off;
  unsigned nbad = 0;
  if (fmt == SCION_PQ2_0) {
    for (int i = 0; i < 32; ++i) {
      unsigned b = s[i];
      for (int j = 0; j < 4; ++j) nbad += (((b >> (2 * j)) & 3) == 3);
      int lane = 4 * r8 + (i >> 3);
      t[16 * lane + 8 * hi + (i & 7)] = uint8_t(b);
    }
    t[512 + 4 * r8 + 2 * hi] = s[32];
    t[512 + 4 * r8 + 2 * hi + 1] = s[33];
  } else {
    for (int q = 0; q < 24; ++q) {
      nbad += (s[q] > 242);
      int lane = 4 * r8 + q / 6;
      t[12 * lane + 6 * hi + q % 6] = s[q];
    }
    nbad += (s[24] > 242) + (s[25] > 26);
    // the row's 8 remainder trits (digits 0..4 of byte 24, 0..2 of the tail byte) as 2-bit
    // fields: even trits 2i at bits 2i of byte L, odd trits 2i+1 at bits 2i of byte H
    unsigned v24 = s[24], vt = s[25], L = 0, H = 0;
    for (int j = 0; j < 8; ++j) {
      unsigned dgt;
      if (j < 5) dgt = v24 % 3, v24 /= 3;
      else dgt = vt % 3, vt /= 3;
      if (j & 1) H |= dgt << (j - 1);
      else L |= dgt << j;
    }
    t[384 + 4 * r8 + hi] = uint8_t(L);
    t[384 + 4 * r8 + 2 + hi] = uint8_t(H);
    t[416 + 4 * r8 + 2 * hi] = s[26];
    t[416 + 4 * r8 + 2 * hi + 1] = s[27];
  }
  count_bad_add(bad, nbad);
}

// dst[r][c] = fp16(src[r][c]) (round to nearest; exact for bf16 values in fp16's normal range).
__global__ void bf16_to_f16_kernel(const __nv_bfloat16* __restrict__ src, int rows, int cols, __half* __restrict__ dst,
                                   int ld_dst) {
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= int64_t(rows) * cols) return;
  int r = int(i / cols), c = int(i % cols);
  dst[int64_t(r) * ld_dst + c] = __float2half_rn(__bfloat162float(src[i]));
}

inline unsigned grid_for(int64_t n, int block) { return unsigned((n + block - 1) / block); }

}  // namespace

cudaError_t launch_pack(int fmt, const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out,
                        int64_t* bad, cudaStream_t s) {
  if (n_groups == 0) return cudaSuccess;
  pack_kernel<<<grid_for(n_groups, 256), 256, 0, s>>>(fmt, codes, scales, n_groups, out, bad);
  return cudaGetLastError();
}

cudaError_t launch_unpack(int fmt, const uint8_t* in, int64_t n_groups, int8_t* codes, uint16_t* scales, int64_t* bad,
                          cudaStream_t s) {
  if (n_groups == 0) return cudaSuccess;
  unpack_kernel<<<grid_for(n_groups, 256), 256, 0, s>>>(fmt, in, n_groups, codes, scales, bad);
  return cudaGetLastError();
}

cudaError_t launch_retile(int fmt, const uint8_t* src, int E, int R, int G, int nmat, int mat, uint8_t* dst,
                          int64_t* bad, cudaStream_t s) {
  int64_t n = int64_t(E) * R * G;
  if (n == 0) return cudaSuccess;
  retile_kernel<<<grid_for(n, 256), 256, 0, s>>>(fmt, src, E, R, G, nmat, mat, dst, bad);
  return cudaGetLastError();
}

cudaError_t launch_bf16_to_f16_rows(const __nv_bfloat16* src, int rows, int cols, __half* dst, int ld_dst,
                                    cudaStream_t s) {
  int64_t n = int64_t(rows) * cols;
  if (n == 0) return cudaSuccess;
  bf16_to_f16_kernel<<<grid_for(n, 256), 256, 0, s>>>(src, rows, cols, dst, ld_dst);
  return cudaGetLastError();
}

}  // namespace scion
