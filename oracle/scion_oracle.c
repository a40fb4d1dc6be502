/*
 * scion_oracle.c -- plain, slow, fp64 CPU oracle for one ternary MoE block.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header or table with the CUDA
 * library: every decoder below (fp16, bf16, PQ2_0, PTQ1_0) is written here
 * from its definition.
 *
 * What it computes, per token t (each token is independent):
 *   1. logits   l[e] = x.W_r[e] + x.D[e]          (router plus router delta)
 *   2. top-k    the k largest logits, ties -> lower expert index
 *   3. gates    softmax over the k selected logits (norm_topk = 1), or the
 *               selected entries of a softmax over all E (norm_topk = 0)
 *   4. experts  y_e = W_d,e (silu(W_g,e x) * (W_u,e x)), W = code * scale
 *   5. shared   y_s = same SwiGLU with the bf16 shared-expert weights
 *               (times sigmoid(x.v) when a shared gate vector v is given)
 *   6. corr     c = B (A in), in = x (default) or the MoE output
 *   7. out      sum_j g_j y_{e_j} + y_s + c
 *
 * Sources (titles and sections of the pages this follows):
 *  - "Scion: ternary MoE quantization with trained corrections", The idea:
 *    ternary expert banks, rank-512 corrections on the MoE block output,
 *    router deltas.
 *  - "Scion-35B-A3B" model card, Model Overview (256 experts, top-8 plus
 *    shared) and Weight Representation (codes in {-1,0,+1}, one fp16 scale
 *    per 128 weights, 2.125 bpw; routers stay F32).
 *  - "Scion-FlashNext-176B-A6B" model card, Highlights and Weight
 *    Representation (base-3 PTQ1_0, 28 bytes per 128 weights, 1.75 bpw;
 *    512 experts, top-10 routed + 1 shared).
 * The bit orders inside the two containers are not on the pages; the ones
 * used here are the library's container specification:
 *  - PQ2_0 (34 B / 128): byte i < 32 holds weights 4i..4i+3, weight 4i+j in
 *    bits 2j..2j+1 (low bits first); field value 0 -> -1, 1 -> 0, 2 -> +1,
 *    3 invalid; bytes 32..33 hold the fp16 scale, little-endian.
 *  - PTQ1_0 (28 B / 128): byte q < 25 holds trits 5q..5q+4 as
 *    sum_j t_{5q+j} 3^j (lowest weight in the least significant digit);
 *    byte 25 holds t125 + 3 t126 + 9 t127; trit value t -> code t - 1;
 *    bytes 26..27 hold the fp16 scale, little-endian.
 * Readings taken where the pages are silent: gates renormalised over the
 * top-k; correction input = block input x, scale 1; no shared-expert gate
 * unless one is given; groups of 128 run along each row's reduction axis.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)
#define ORACLE_EFORMAT (-4)

#define ORACLE_PQ2_0 0
#define ORACLE_PTQ1_0 1

/* ---------------------------------------------------------------- scalars */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 31;
  int frac = h & 1023;
  double v;
  if (expo == 0)
    v = ldexp((double)frac, -24); /* subnormal: frac * 2^-24 */
  else if (expo == 31)
    v = frac ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + frac), expo - 25); /* (1 + frac/1024) 2^(expo-15) */
  return sign ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE 754 binary32. */
double oracle_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }
static double silu(double v) { return v / (1.0 + exp(-v)); }

/* ------------------------------------------------------------- containers */

long oracle_block_bytes(int fmt) {
  if (fmt == ORACLE_PQ2_0) return 34;
  if (fmt == ORACLE_PTQ1_0) return 28;
  return -1;
}

/* codes: n_groups*128 values in {-1,0,+1}; scales: n_groups fp16 bit patterns. */
int oracle_pq2_pack(const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out) {
  for (int64_t g = 0; g < n_groups; g++) {
    const int8_t* c = codes + g * 128;
    uint8_t* blk = out + g * 34;
    for (int i = 0; i < 32; i++) {
      unsigned byte = 0;
      for (int j = 0; j < 4; j++) {
        int code = c[4 * i + j];
        if (code < -1 || code > 1) return ORACLE_EINVAL;
        byte |= (unsigned)(code + 1) << (2 * j);
      }
      blk[i] = (uint8_t)byte;
    }
    blk[32] = (uint8_t)(scales[g] & 0xff);
    blk[33] = (uint8_t)(scales[g] >> 8);
  }
  return ORACLE_OK;
}

/* Returns ORACLE_EFORMAT if any 2-bit field holds 3 (codes still written, 0 there). */
int oracle_pq2_unpack(const uint8_t* in, int64_t n_groups, int8_t* codes, uint16_t* scales) {
  int status = ORACLE_OK;
  for (int64_t g = 0; g < n_groups; g++) {
    const uint8_t* blk = in + g * 34;
    int8_t* c = codes + g * 128;
    for (int i = 0; i < 32; i++) {
      for (int j = 0; j < 4; j++) {
        int field = (blk[i] >> (2 * j)) & 3;
        if (field == 3) {
          status = ORACLE_EFORMAT;
          c[4 * i + j] = 0;
        } else {
          c[4 * i + j] = (int8_t)(field - 1);
        }
      }
    }
    scales[g] = (uint16_t)(blk[32] | (blk[33] << 8));
  }
  return status;
}

int oracle_ptq1_pack(const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out) {
  for (int64_t g = 0; g < n_groups; g++) {
    const int8_t* c = codes + g * 128;
    uint8_t* blk = out + g * 28;
    for (int i = 0; i < 128; i++)
      if (c[i] < -1 || c[i] > 1) return ORACLE_EINVAL;
    for (int q = 0; q < 25; q++) {
      int v = 0, p = 1;
      for (int j = 0; j < 5; j++) {
        v += (c[5 * q + j] + 1) * p;
        p *= 3;
      }
      blk[q] = (uint8_t)v;
    }
    blk[25] = (uint8_t)((c[125] + 1) + 3 * (c[126] + 1) + 9 * (c[127] + 1));
    blk[26] = (uint8_t)(scales[g] & 0xff);
    blk[27] = (uint8_t)(scales[g] >> 8);
  }
  return ORACLE_OK;
}

/* Returns ORACLE_EFORMAT if a quintet byte exceeds 242 or the tail byte 26. */
int oracle_ptq1_unpack(const uint8_t* in, int64_t n_groups, int8_t* codes, uint16_t* scales) {
  int status = ORACLE_OK;
  for (int64_t g = 0; g < n_groups; g++) {
    const uint8_t* blk = in + g * 28;
    int8_t* c = codes + g * 128;
    for (int q = 0; q < 25; q++) {
      int v = blk[q];
      if (v > 242) {
        status = ORACLE_EFORMAT;
        for (int j = 0; j < 5; j++) c[5 * q + j] = 0;
        continue;
      }
      for (int j = 0; j < 5; j++) {
        c[5 * q + j] = (int8_t)(v % 3 - 1);
        v /= 3;
      }
    }
    int v = blk[25];
    if (v > 26) {
      status = ORACLE_EFORMAT;
      c[125] = c[126] = c[127] = 0;
    } else {
      for (int j = 0; j < 3; j++) {
        c[125 + j] = (int8_t)(v % 3 - 1);
        v /= 3;
      }
    }
    scales[g] = (uint16_t)(blk[26] | (blk[27] << 8));
  }
  return status;
}

/* Dequantize one row of K weights stored as K/128 consecutive blocks: w = code * scale. */
int oracle_dequant_row(int fmt, const uint8_t* blocks, int K, double* w) {
  int8_t codes[128];
  uint16_t scale;
  long bb = oracle_block_bytes(fmt);
  int status = ORACLE_OK;
  for (int g = 0; g < K / 128; g++) {
    int s = (fmt == ORACLE_PQ2_0) ? oracle_pq2_unpack(blocks + g * bb, 1, codes, &scale)
                                  : oracle_ptq1_unpack(blocks + g * bb, 1, codes, &scale);
    if (s != ORACLE_OK) status = s;
    double sc = oracle_f16_to_f64(scale);
    for (int i = 0; i < 128; i++) w[g * 128 + i] = (double)codes[i] * sc;
  }
  return status;
}

/* ------------------------------------------------------------------ layer */

typedef struct {
  int d, n_experts, top_k, ffn, shared_ffn, rank;
  int fmt;            /* ORACLE_PQ2_0 or ORACLE_PTQ1_0 */
  int router_f32;     /* 1: router and delta are fp32 [E][d]; 0: bf16 */
  int norm_topk;      /* 1: softmax over the k selected logits */
  int corr_on_output; /* 0: correction reads x; 1: it reads the MoE output */
  const void* w_router;
  const void* w_delta;
  const uint8_t* gate_exps; /* [E][ffn][d/128] blocks */
  const uint8_t* up_exps;   /* [E][ffn][d/128] blocks */
  const uint8_t* down_exps; /* [E][d][ffn/128] blocks */
  const uint16_t* sh_gate;  /* bf16 [shared_ffn][d] */
  const uint16_t* sh_up;    /* bf16 [shared_ffn][d] */
  const uint16_t* sh_down;  /* bf16 [d][shared_ffn] */
  const uint16_t* sh_gate_vec; /* bf16 [d] or NULL */
  const uint16_t* corr_a;   /* bf16 [rank][d] (or PQ2_0 blocks, see corr_packed) */
  const uint16_t* corr_b;   /* bf16 [d][rank] (or PQ2_0 blocks) */
  int corr_packed;          /* 1: corr_a = PQ2_0 blocks [rank][d/128], corr_b = [d][rank/128]: ternary
                               correction factors, w = code * scale ("Scion-35B-A3B" model card, Weight
                               Representation: 2-bit codes plus one fp16 scale per 128, q1_0_g128) */
} oracle_layer;

static double router_weight(const oracle_layer* L, const void* w, long idx) {
  if (L->router_f32) return (double)((const float*)w)[idx];
  return oracle_bf16_to_f64(((const uint16_t*)w)[idx]);
}

/* x: bf16 [d] -> xv: fp64 (exact). */
static void load_x(const uint16_t* x, int d, double* xv) {
  for (int i = 0; i < d; i++) xv[i] = oracle_bf16_to_f64(x[i]);
}

/* Step 1: l[e] = sum_i x_i W_r[e,i] + sum_i x_i D[e,i]. */
void oracle_router_logits_one(const oracle_layer* L, const double* xv, double* logits) {
  for (int e = 0; e < L->n_experts; e++) {
    double a = 0.0, b = 0.0;
    for (int i = 0; i < L->d; i++) {
      a += xv[i] * router_weight(L, L->w_router, (long)e * L->d + i);
      b += xv[i] * router_weight(L, L->w_delta, (long)e * L->d + i);
    }
    logits[e] = a + b;
  }
}

/* Step 2: the k largest logits in descending order; equal values -> lower index first. */
void oracle_topk(const double* logits, int E, int k, int32_t* ids) {
  char* taken = (char*)calloc((size_t)E, 1);
  for (int j = 0; j < k; j++) {
    int best = -1;
    for (int e = 0; e < E; e++) {
      if (taken[e]) continue;
      if (best < 0 || logits[e] > logits[best]) best = e;
    }
    ids[j] = best;
    taken[best] = 1;
  }
  free(taken);
}

/* Step 3: gate weights of the selected experts. */
void oracle_gates(const double* logits, int E, int k, const int32_t* ids, int norm_topk, double* gates) {
  if (norm_topk) {
    double m = logits[ids[0]];
    for (int j = 1; j < k; j++)
      if (logits[ids[j]] > m) m = logits[ids[j]];
    double z = 0.0;
    for (int j = 0; j < k; j++) z += exp(logits[ids[j]] - m);
    for (int j = 0; j < k; j++) gates[j] = exp(logits[ids[j]] - m) / z;
  } else {
    double m = logits[0];
    for (int e = 1; e < E; e++)
      if (logits[e] > m) m = logits[e];
    double z = 0.0;
    for (int e = 0; e < E; e++) z += exp(logits[e] - m);
    for (int j = 0; j < k; j++) gates[j] = exp(logits[ids[j]] - m) / z;
  }
}

/* Token-to-expert grouping: histogram of the T*k ids, exclusive scan, stable scatter
 * (token order, then slot order).  perm[pos] = t*k + j. */
void oracle_group(const int32_t* ids, int T, int k, int E, int32_t* counts, int32_t* offsets, int32_t* perm) {
  for (int e = 0; e < E; e++) counts[e] = 0;
  for (long i = 0; i < (long)T * k; i++) counts[ids[i]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  for (int e = 0; e < E; e++) cursor[e] = offsets[e];
  for (int t = 0; t < T; t++)
    for (int j = 0; j < k; j++) {
      int e = ids[(long)t * k + j];
      perm[cursor[e]++] = t * k + j;
    }
  free(cursor);
}

/* Dense dequantized expert e: wg, wu [ffn][d]; wd [d][ffn]. */
static int dequant_expert(const oracle_layer* L, int e, double* wg, double* wu, double* wd) {
  long bb = oracle_block_bytes(L->fmt);
  long gate_row = (long)(L->d / 128) * bb, down_row = (long)(L->ffn / 128) * bb;
  int status = ORACLE_OK, s;
  for (int f = 0; f < L->ffn; f++) {
    long row = (long)e * L->ffn + f;
    if ((s = oracle_dequant_row(L->fmt, L->gate_exps + row * gate_row, L->d, wg + (long)f * L->d))) status = s;
    if ((s = oracle_dequant_row(L->fmt, L->up_exps + row * gate_row, L->d, wu + (long)f * L->d))) status = s;
  }
  for (int i = 0; i < L->d; i++) {
    long row = (long)e * L->d + i;
    if ((s = oracle_dequant_row(L->fmt, L->down_exps + row * down_row, L->ffn, wd + (long)i * L->ffn))) status = s;
  }
  return status;
}

/* SwiGLU MLP on dense fp64 weights: h = silu(Wg x) * (Wu x); y = Wd h. */
static void swiglu_mlp(const double* wg, const double* wu, const double* wd, int d, int ffn, const double* xv,
                       double* h, double* y) {
  for (int f = 0; f < ffn; f++) {
    double g = 0.0, u = 0.0;
    for (int i = 0; i < d; i++) {
      g += wg[(long)f * d + i] * xv[i];
      u += wu[(long)f * d + i] * xv[i];
    }
    h[f] = silu(g) * u;
  }
  for (int i = 0; i < d; i++) {
    double a = 0.0;
    for (int f = 0; f < ffn; f++) a += wd[(long)i * ffn + f] * h[f];
    y[i] = a;
  }
}

/* Step 4 for one (expert, token): y and (optionally) the SwiGLU hidden h. */
int oracle_expert_one(const oracle_layer* L, int e, const uint16_t* x, double* h_out, double* y) {
  long n = (long)L->ffn * L->d;
  double* wg = (double*)malloc(sizeof(double) * n);
  double* wu = (double*)malloc(sizeof(double) * n);
  double* wd = (double*)malloc(sizeof(double) * n);
  double* xv = (double*)malloc(sizeof(double) * L->d);
  double* h = (double*)malloc(sizeof(double) * L->ffn);
  if (!wg || !wu || !wd || !xv || !h) {
    free(wg), free(wu), free(wd), free(xv), free(h);
    return ORACLE_ENOMEM;
  }
  int status = dequant_expert(L, e, wg, wu, wd);
  load_x(x, L->d, xv);
  swiglu_mlp(wg, wu, wd, L->d, L->ffn, xv, h, y);
  if (h_out) memcpy(h_out, h, sizeof(double) * L->ffn);
  free(wg), free(wu), free(wd), free(xv), free(h);
  return status;
}

/* Step 5: shared expert on one token (bf16 weights), plus its optional sigmoid gate. */
static void shared_one(const oracle_layer* L, const double* xv, double* h, double* y) {
  int d = L->d, fs = L->shared_ffn;
  for (int f = 0; f < fs; f++) {
    double g = 0.0, u = 0.0;
    for (int i = 0; i < d; i++) {
      g += oracle_bf16_to_f64(L->sh_gate[(long)f * d + i]) * xv[i];
      u += oracle_bf16_to_f64(L->sh_up[(long)f * d + i]) * xv[i];
    }
    h[f] = silu(g) * u;
  }
  double gate = 1.0;
  if (L->sh_gate_vec) {
    double a = 0.0;
    for (int i = 0; i < d; i++) a += oracle_bf16_to_f64(L->sh_gate_vec[i]) * xv[i];
    gate = sigmoid(a);
  }
  for (int i = 0; i < d; i++) {
    double a = 0.0;
    for (int f = 0; f < fs; f++) a += oracle_bf16_to_f64(L->sh_down[(long)i * fs + f]) * h[f];
    y[i] = gate * a;
  }
}

/* Step 6: rank-r correction c = B (A in). */
static void corr_one(const oracle_layer* L, const double* in, double* z, double* y) {
  int d = L->d, r = L->rank;
  if (L->corr_packed) {
    /* dequantize one row at a time with the container decoder above */
    const uint8_t* A = (const uint8_t*)L->corr_a;
    const uint8_t* B = (const uint8_t*)L->corr_b;
    double* w = (double*)malloc(sizeof(double) * (d > r ? d : r));
    for (int q = 0; q < r; q++) {
      oracle_dequant_row(ORACLE_PQ2_0, A + (long)q * (d / 128) * 34, d, w);
      double a = 0.0;
      for (int i = 0; i < d; i++) a += w[i] * in[i];
      z[q] = a;
    }
    for (int i = 0; i < d; i++) {
      oracle_dequant_row(ORACLE_PQ2_0, B + (long)i * (r / 128) * 34, r, w);
      double a = 0.0;
      for (int q = 0; q < r; q++) a += w[q] * z[q];
      y[i] = a;
    }
    free(w);
    return;
  }
  for (int q = 0; q < r; q++) {
    double a = 0.0;
    for (int i = 0; i < d; i++) a += oracle_bf16_to_f64(L->corr_a[(long)q * d + i]) * in[i];
    z[q] = a;
  }
  for (int i = 0; i < d; i++) {
    double a = 0.0;
    for (int q = 0; q < r; q++) a += oracle_bf16_to_f64(L->corr_b[(long)i * r + q]) * z[q];
    y[i] = a;
  }
}

/* Routing for T tokens: logits [T][E] (optional), ids [T][k], gates [T][k]. */
int oracle_route(const oracle_layer* L, const uint16_t* x, int T, double* logits_out, int32_t* ids, double* gates) {
  int d = L->d, E = L->n_experts, k = L->top_k;
  int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; t++) {
    double* xv = (double*)malloc(sizeof(double) * d);
    double* l = (double*)malloc(sizeof(double) * E);
    if (!xv || !l) {
      status = ORACLE_ENOMEM;
    } else {
      load_x(x + (long)t * d, d, xv);
      oracle_router_logits_one(L, xv, l);
      oracle_topk(l, E, k, ids + (long)t * k);
      oracle_gates(l, E, k, ids + (long)t * k, L->norm_topk, gates + (long)t * k);
      if (logits_out) memcpy(logits_out + (long)t * E, l, sizeof(double) * E);
    }
    free(xv), free(l);
  }
  return status;
}

static int check_layer(const oracle_layer* L) {
  if (!L || L->d <= 0 || L->d % 128 || L->ffn <= 0 || L->ffn % 128) return ORACLE_EINVAL;
  if (L->n_experts <= 0 || L->top_k <= 0 || L->top_k > L->n_experts) return ORACLE_EINVAL;
  if (L->fmt != ORACLE_PQ2_0 && L->fmt != ORACLE_PTQ1_0) return ORACLE_EINVAL;
  if (L->shared_ffn < 0 || L->rank < 0) return ORACLE_EINVAL;
  if (L->corr_packed && L->rank % 128) return ORACLE_EINVAL; /* groups of 128 along B's rank axis */
  return ORACLE_OK;
}

/*
 * The block forward.  x: bf16 [T][d]; out: fp64 [T][d]; ids/gates: [T][k] (may be NULL).
 * y_e(x_t) for every routed pair is computed by the same code whatever the loop
 * order; the pairs are visited expert by expert so each expert is dequantized once,
 * and the per-token sums then run in slot order.
 */
/*
 * The block forward, or the part of it that one rank of an expert-parallel layout computes:
 * routed terms only for experts e in [expert_lo, expert_lo + n_local) (parts & 1), the shared
 * expert and the correction (parts & 2).  Disjoint expert ranges covering all E, plus the dense
 * part once, sum to the block output.  (Expert parallelism is not on the pages; "Scion: ternary
 * MoE quantization with trained corrections", Serving notes, places the experts of one large
 * model on more than one device, and this is the plainest such split: by expert.)
 */
static int moe_forward_impl(const oracle_layer* L, const uint16_t* x, int T, double* out, int32_t* ids_out,
                            double* gates_out, int expert_lo, int n_local, int parts) {
  int st = check_layer(L);
  if (st) return st;
  if (T <= 0) return ORACLE_OK;
  int d = L->d, E = L->n_experts, k = L->top_k, F = L->ffn;
  long Tk = (long)T * k;
  int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * Tk);
  double* gates = (double*)malloc(sizeof(double) * Tk);
  double* y = (double*)malloc(sizeof(double) * Tk * d);
  int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * E);
  int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * (E + 1));
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * Tk);
  if (!ids || !gates || !y || !counts || !offsets || !perm) {
    st = ORACLE_ENOMEM;
    goto done;
  }
  st = oracle_route(L, x, T, NULL, ids, gates);
  if (st) goto done;
  oracle_group(ids, T, k, E, counts, offsets, perm);

  /* Step 4: y[t][j] = expert e_{t,j} applied to x_t (for the experts of this part). */
#pragma omp parallel for schedule(dynamic, 1)
  for (int e = 0; e < E; e++) {
    if (counts[e] == 0 || !(parts & 1) || e < expert_lo || e >= expert_lo + n_local) continue;
    long n = (long)F * d;
    double* wg = (double*)malloc(sizeof(double) * n);
    double* wu = (double*)malloc(sizeof(double) * n);
    double* wd = (double*)malloc(sizeof(double) * n);
    double* xv = (double*)malloc(sizeof(double) * d);
    double* h = (double*)malloc(sizeof(double) * F);
    if (!wg || !wu || !wd || !xv || !h) {
      st = ORACLE_ENOMEM;
    } else {
      int s = dequant_expert(L, e, wg, wu, wd);
      if (s) st = s;
      for (int p = offsets[e]; p < offsets[e + 1]; p++) {
        int t = perm[p] / k;
        load_x(x + (long)t * d, d, xv);
        swiglu_mlp(wg, wu, wd, d, F, xv, h, y + (long)perm[p] * d);
      }
    }
    free(wg), free(wu), free(wd), free(xv), free(h);
  }
  if (st) goto done;

  /* Steps 5-7 per token. */
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; t++) {
    double* xv = (double*)malloc(sizeof(double) * d);
    double* acc = (double*)malloc(sizeof(double) * d);
    double* ys = (double*)malloc(sizeof(double) * d);
    double* hs = (double*)malloc(sizeof(double) * (L->shared_ffn > 0 ? L->shared_ffn : 1));
    double* z = (double*)malloc(sizeof(double) * (L->rank > 0 ? L->rank : 1));
    if (!xv || !acc || !ys || !hs || !z) {
      st = ORACLE_ENOMEM;
    } else {
      load_x(x + (long)t * d, d, xv);
      for (int i = 0; i < d; i++) acc[i] = 0.0;
      for (int j = 0; j < k; j++) {
        const int e = ids[(long)t * k + j];
        if (!(parts & 1) || e < expert_lo || e >= expert_lo + n_local) continue;
        const double* yj = y + ((long)t * k + j) * d;
        double g = gates[(long)t * k + j];
        for (int i = 0; i < d; i++) acc[i] += g * yj[i];
      }
      if (!(parts & 2)) {
        /* no dense terms in this part */
      } else if (L->shared_ffn > 0) {
        shared_one(L, xv, hs, ys);
        for (int i = 0; i < d; i++) acc[i] += ys[i];
      }
      if (L->rank > 0 && (parts & 2)) {
        const double* in = L->corr_on_output ? acc : xv;
        double* in_copy = (double*)malloc(sizeof(double) * d);
        memcpy(in_copy, in, sizeof(double) * d);
        corr_one(L, in_copy, z, ys);
        free(in_copy);
        for (int i = 0; i < d; i++) acc[i] += ys[i];
      }
      memcpy(out + (long)t * d, acc, sizeof(double) * d);
    }
    free(xv), free(acc), free(ys), free(hs), free(z);
  }
  if (ids_out) memcpy(ids_out, ids, sizeof(int32_t) * Tk);
  if (gates_out) memcpy(gates_out, gates, sizeof(double) * Tk);
done:
  free(ids), free(gates), free(y), free(counts), free(offsets), free(perm);
  return st;
}

/*
 * Cross-form: out[t] = sum over ALL experts e < E of m_e y_e(x_t) + shared + corr,
 * with m_e = the gate of e if e is among the top-k of t, else 0.  Same result as
 * oracle_moe_forward; used on tiny sizes to check that the sparse form drops nothing.
 */
int oracle_moe_forward(const oracle_layer* L, const uint16_t* x, int T, double* out, int32_t* ids_out,
                       double* gates_out) {
  return moe_forward_impl(L, x, T, out, ids_out, gates_out, 0, L ? L->n_experts : 0, 3);
}

int oracle_moe_forward_part(const oracle_layer* L, const uint16_t* x, int T, int expert_lo, int n_local, int parts,
                            double* out) {
  if (!L || expert_lo < 0 || n_local < 0 || expert_lo + n_local > L->n_experts || parts < 0 || parts > 3)
    return ORACLE_EINVAL;
  return moe_forward_impl(L, x, T, out, NULL, NULL, expert_lo, n_local, parts);
}

int oracle_moe_forward_dense(const oracle_layer* L, const uint16_t* x, int T, double* out) {
  int st = check_layer(L);
  if (st) return st;
  int d = L->d, E = L->n_experts, k = L->top_k, F = L->ffn;
  long n = (long)F * d;
  double* wg = (double*)malloc(sizeof(double) * n);
  double* wu = (double*)malloc(sizeof(double) * n);
  double* wd = (double*)malloc(sizeof(double) * n);
  double* xv = (double*)malloc(sizeof(double) * d);
  double* h = (double*)malloc(sizeof(double) * F);
  double* ye = (double*)malloc(sizeof(double) * d);
  double* l = (double*)malloc(sizeof(double) * E);
  double* m = (double*)malloc(sizeof(double) * E);
  double* hs = (double*)malloc(sizeof(double) * (L->shared_ffn > 0 ? L->shared_ffn : 1));
  double* z = (double*)malloc(sizeof(double) * (L->rank > 0 ? L->rank : 1));
  int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * k);
  double* g = (double*)malloc(sizeof(double) * k);
  if (!wg || !wu || !wd || !xv || !h || !ye || !l || !m || !hs || !z || !ids || !g) {
    st = ORACLE_ENOMEM;
    goto done;
  }
  for (int t = 0; t < T; t++) {
    double* acc = out + (long)t * d;
    load_x(x + (long)t * d, d, xv);
    oracle_router_logits_one(L, xv, l);
    oracle_topk(l, E, k, ids);
    oracle_gates(l, E, k, ids, L->norm_topk, g);
    for (int e = 0; e < E; e++) m[e] = 0.0;
    for (int j = 0; j < k; j++) m[ids[j]] = g[j];
    for (int i = 0; i < d; i++) acc[i] = 0.0;
    for (int e = 0; e < E; e++) {
      int s = dequant_expert(L, e, wg, wu, wd);
      if (s) st = s;
      swiglu_mlp(wg, wu, wd, d, F, xv, h, ye);
      for (int i = 0; i < d; i++) acc[i] += m[e] * ye[i];
    }
    if (L->shared_ffn > 0) {
      shared_one(L, xv, hs, ye);
      for (int i = 0; i < d; i++) acc[i] += ye[i];
    }
    if (L->rank > 0) {
      double* in_copy = (double*)malloc(sizeof(double) * d);
      memcpy(in_copy, L->corr_on_output ? acc : xv, sizeof(double) * d);
      corr_one(L, in_copy, z, ye);
      free(in_copy);
      for (int i = 0; i < d; i++) acc[i] += ye[i];
    }
  }
done:
  free(wg), free(wu), free(wd), free(xv), free(h), free(ye), free(l), free(m), free(hs), free(z), free(ids), free(g);
  return st;
}

/* Shared-expert SwiGLU hidden and output for T tokens (stage-wise checks). */
int oracle_shared(const oracle_layer* L, const uint16_t* x, int T, double* h_out, double* y_out) {
  int d = L->d, fs = L->shared_ffn;
  if (fs <= 0) return ORACLE_EINVAL;
  double* xv = (double*)malloc(sizeof(double) * d);
  if (!xv) return ORACLE_ENOMEM;
  for (int t = 0; t < T; t++) {
    load_x(x + (long)t * d, d, xv);
    shared_one(L, xv, h_out + (long)t * fs, y_out + (long)t * d);
  }
  free(xv);
  return ORACLE_OK;
}

/* Correction z = A x and c = B z for T tokens whose input is the block input x. */
int oracle_corr(const oracle_layer* L, const uint16_t* x, int T, double* z_out, double* y_out) {
  int d = L->d;
  if (L->rank <= 0) return ORACLE_EINVAL;
  double* xv = (double*)malloc(sizeof(double) * d);
  if (!xv) return ORACLE_ENOMEM;
  for (int t = 0; t < T; t++) {
    load_x(x + (long)t * d, d, xv);
    corr_one(L, xv, z_out + (long)t * L->rank, y_out + (long)t * d);
  }
  free(xv);
  return ORACLE_OK;
}

/* ------------------------------------------------------------- quantizers */
/* Float -> ternary quantizers of groups of 128 consecutive weights ("Scion: ternary MoE
 * quantization with trained corrections", Findings: the deployable Lloyd quantizer against
 * one-shot absmean; "Scion-35B-A3B" model card, Highlights: ternary Lloyd g128).  Each group
 * gets codes in {-1, 0, +1} and one scale s, w ~ code * s.
 *   absmean: s = mean |w| over the group; code = w / s rounded half away from zero and
 *            clamped to [-1, 1], i.e. sign(w) where 2|w| >= s, else 0.
 *   Lloyd:   Lloyd's algorithm for the levels {-s, 0, +s}: starting from the absmean codes,
 *            alternately set s to the centroid of the nonzero cells (mean |w| over codes != 0)
 *            and re-partition to the nearest level (the same rule as above), until the codes
 *            stop changing or `iters` rounds have run; the stored s is the centroid of the
 *            final codes.
 * Decisions are taken in fp64; the scale is stored as the nearest binary16. */

/* Nearest binary16 (ties to even) of a finite v >= 0, as its bit pattern (+inf at >= 65520). */
uint16_t oracle_f64_to_f16_nonneg(double v) {
  if (!(v > 0.0)) return 0;
  if (v >= 65520.0) return 0x7c00;
  int e;
  frexp(v, &e);                              /* v = m 2^e with 0.5 <= m < 1: v in [2^(e-1), 2^e) */
  const int E = e - 1;                       /* unbiased exponent of v */
  const int q = E >= -14 ? E - 10 : -24;     /* weight of the last fraction bit (normal / subnormal) */
  double r = nearbyint(ldexp(v, -q));        /* v in units of that bit, rounded half to even */
  if (q == -24) return (uint16_t)r;          /* subnormal (r = 1024 is the smallest normal) */
  int Eo = E;
  if (r >= 2048.0) r /= 2.0, Eo += 1;        /* rounding carried into the next binade */
  if (Eo > 15) return 0x7c00;
  return (uint16_t)(((Eo + 15) << 10) | ((int)r - 1024));
}

static int quant_finite(const float* w) {
  for (int i = 0; i < 128; i++)
    if (!isfinite(w[i])) return 0;
  return 1;
}

/* sign(w) where 2|w| >= s, else 0; returns how many codes differ from c_old (if given). */
static int quant_partition(const float* w, double s, int8_t* c) {
  int changed = 0;
  for (int i = 0; i < 128; i++) {
    const double a = fabs((double)w[i]);
    const int8_t v = (w[i] != 0.0f && 2.0 * a >= s) ? (w[i] > 0.0f ? 1 : -1) : 0;
    changed += v != c[i];
    c[i] = v;
  }
  return changed;
}

static double quant_centroid(const float* w, const int8_t* c) {
  double sum = 0.0;
  int n = 0;
  for (int i = 0; i < 128; i++)
    if (c[i]) sum += fabs((double)w[i]), n++;
  return n ? sum / n : 0.0;
}

int oracle_quantize(int method, const float* w, int64_t n_groups, int iters, int8_t* codes, uint16_t* scales) {
  if ((method != 0 && method != 1) || n_groups < 0 || iters < 0) return ORACLE_EINVAL;
  for (int64_t g = 0; g < n_groups; g++)
    if (!quant_finite(w + g * 128)) return ORACLE_EINVAL;
#pragma omp parallel for schedule(static)
  for (int64_t g = 0; g < n_groups; g++) {
    const float* wg = w + g * 128;
    int8_t* c = codes + g * 128;
    double s = 0.0;
    for (int i = 0; i < 128; i++) s += fabs((double)wg[i]);
    s /= 128.0;
    for (int i = 0; i < 128; i++) c[i] = 0;
    quant_partition(wg, s, c);
    if (method == 1) {
      for (int it = 0; it < iters; it++) {
        s = quant_centroid(wg, c);
        if (quant_partition(wg, s, c) == 0) break;
      }
      s = quant_centroid(wg, c);
    }
    scales[g] = oracle_f64_to_f16_nonneg(s);
  }
  return ORACLE_OK;
}

/*
 * The correction branch on the attention output ("Scion: ternary MoE quantization with trained
 * corrections", The idea: rank-512 branches on the attention output and on the MoE block output;
 * Findings: the attention-output branch ships as a standard low-rank adapter on the attention
 * output projection).  Reading: the branch takes that projection's input v (d_in wide) and adds
 * its low-rank product to the projection's output (d_out wide), scale 1 (any alpha / r folded into
 * B), on top of a given base (the projection's output, or the residual stream it joins):
 *   z = A v,   out[t] = base[t] + B z
 * v: bf16 [T][d_in]; A, B: bf16 [r][d_in] and [d_out][r], or (packed = 1) PQ2_0 blocks
 * [r][d_in/128] and [d_out][r/128] decoded by oracle_dequant_row; base: fp64 [T][d_out] or NULL
 * (zero); out: fp64 [T][d_out]; z_out: fp64 [T][r] or NULL.
 */
int oracle_attn_corr(int d_in, int d_out, int r, int packed, const void* A, const void* B, const uint16_t* v, int T,
                     const double* base, double* out, double* z_out) {
  if (d_in <= 0 || d_out <= 0 || r <= 0 || T < 0 || !A || !B || !out) return ORACLE_EINVAL;
  if (packed && (d_in % 128 || r % 128)) return ORACLE_EINVAL;
  double* a = (double*)malloc(sizeof(double) * (size_t)r * d_in);
  double* b = (double*)malloc(sizeof(double) * (size_t)d_out * r);
  if (!a || !b) {
    free(a), free(b);
    return ORACLE_ENOMEM;
  }
  int status = ORACLE_OK;
  for (int q = 0; q < r && status == ORACLE_OK; q++) {
    if (packed)
      status = oracle_dequant_row(ORACLE_PQ2_0, (const uint8_t*)A + (long)q * (d_in / 128) * 34, d_in, a + (long)q * d_in);
    else
      for (int i = 0; i < d_in; i++) a[(long)q * d_in + i] = oracle_bf16_to_f64(((const uint16_t*)A)[(long)q * d_in + i]);
  }
  for (int i = 0; i < d_out && status == ORACLE_OK; i++) {
    if (packed)
      status = oracle_dequant_row(ORACLE_PQ2_0, (const uint8_t*)B + (long)i * (r / 128) * 34, r, b + (long)i * r);
    else
      for (int q = 0; q < r; q++) b[(long)i * r + q] = oracle_bf16_to_f64(((const uint16_t*)B)[(long)i * r + q]);
  }
  if (status == ORACLE_OK) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; t++) {
      double* vv = (double*)malloc(sizeof(double) * d_in);
      double* z = (double*)malloc(sizeof(double) * r);
      if (!vv || !z) {
        status = ORACLE_ENOMEM;
      } else {
        for (int i = 0; i < d_in; i++) vv[i] = oracle_bf16_to_f64(v[(long)t * d_in + i]);
        for (int q = 0; q < r; q++) {
          double s = 0.0;
          for (int i = 0; i < d_in; i++) s += a[(long)q * d_in + i] * vv[i];
          z[q] = s;
          if (z_out) z_out[(long)t * r + q] = s;
        }
        for (int i = 0; i < d_out; i++) {
          double s = 0.0;
          for (int q = 0; q < r; q++) s += b[(long)i * r + q] * z[q];
          out[(long)t * d_out + i] = (base ? base[(long)t * d_out + i] : 0.0) + s;
        }
      }
      free(vv), free(z);
    }
  }
  free(a), free(b);
  return status;
}
