/*
 * moe_q4 oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU restatement of what the routed-expert
 * MoE hot path over 4-bit codebook weights computes.  Only the tests, the
 * package's smoke check and the benchmark's CPU-baseline leg may load this
 * library.  It shares no code, header, table or constant with the CUDA
 * library; it is written from the pages' definitions directly:
 *
 *   [NF4-Lloyd]  "aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ"
 *                sections "Contents", "Codes are indices into the per-layer
 *                grid -- not E2M1", "What this is", "Known defect".
 *   [ROUND7]     "Round 7 -- Rewrite the GLM-5.2 routed-expert encoder"
 *                (CODEX_ROUND7.md), "Owner-locked decisions" items 4, 6, 7
 *                and "Ground truth and corrections" (model geometry).
 *   [TR3v4]      "GLM-5.2 EXL3 TR3 v4 -- 3.5 bpw mixed experts" README,
 *                "Shared residual rotations, private intermediate rotations"
 *                (routing-weighted sum of expert outputs).
 *   [DENSE6]     "GLM-5.2-EXL3-DENSE6-MTP78", section "Quant recipe" (the
 *                router mlp.gate is held in BF16).
 *
 * Precision: every floating-point value of the MoE is carried in fp64.  The
 * dequantisation entry point produces bf16 bit patterns under the rule
 * "fp32 multiply, then round-to-nearest-even to bf16" (see oq_decode_bf16).
 * Build without -ffast-math and with -ffp-contract=off so that float
 * products are single IEEE multiplies with subnormals kept.
 *
 * Parity pins (all in tests/, marked "not gpu"): hand-computed decodes of
 * all 16 codes x edge scale bytes x both nibble positions; the E2M1 table
 * against the closed-form OCP E2M1 decode; brute-force signed-level search
 * for pack; library (numpy) sort for routing/grouping; dense-FFN reductions
 * and the intermediate-channel permutation invariant for the MoE; for the
 * grid fit, the uniform quantiser of U(0,1), a closed-form weighted step,
 * decoded weights as a fixed point and power-of-two scale invariance.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OQ_OK 0
#define OQ_EINVAL 1

int oq_abi_version(void) { return 1; }

/* ---- bf16 helpers ------------------------------------------------------ */

static float bf16_bits_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* IEEE round-to-nearest-even from fp32 to bf16 (NaN -> quiet 0x7FC0 with the
 * input's sign). */
static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)(0x7fc0u | ((u >> 16) & 0x8000u));
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* A table is 8 fp32 magnitudes.  Accepted: all finite, none with the sign
 * bit set (a magnitude is >= 0; -0.0 is not a magnitude), max > 0 (the pack
 * rule divides the block amax by the largest level). */
static int table_ok(const float* t) {
  float mx = 0.0f;
  for (int i = 0; i < 8; ++i) {
    if (!isfinite(t[i]) || signbit(t[i])) return 0;
    if (t[i] > mx) mx = t[i];
  }
  return mx > 0.0f;
}

static int tables_ok(const float* tables, int n_tables, const uint8_t* table_id, int E) {
  if (!tables || n_tables < 1 || n_tables > 255 || !table_id) return 0;
  for (int i = 0; i < n_tables; ++i)
    if (!table_ok(tables + 8 * i)) return 0;
  for (int e = 0; e < E; ++e)
    if (table_id[e] >= n_tables) return 0;
  return 1;
}

/* ---- decode ------------------------------------------------------------ */

/* One weight, as the bf16 the dequantisation emits.
 * [NF4-Lloyd, "Codes are indices into the per-layer grid"]:
 *   mag = code & 0x07 indexes the grid, code & 0x08 is the sign,
 *   w = sign * grid[mag] * 2^(scale_byte - 127).
 * Readings (the pages give no rounding rule for a 16-bit output):
 *   - the multiplier 2^(s-127) is an exact fp32 (subnormal for s = 0);
 *   - grid[mag] * multiplier is one fp32 multiply, rounded to nearest even;
 *   - that fp32 is rounded to bf16 to nearest even;
 *   - the sign is applied last by flipping bit 15, so a zero level with the
 *     sign bit set decodes to -0.0;
 *   - scale byte 0xFF is the E8M0 NaN encoding: the result is the quiet NaN
 *     0x7FC0 with the code's sign bit. */
uint16_t oq_decode_bf16(uint8_t code, uint8_t scale, const float* table8) {
  uint16_t bits;
  if (scale == 0xFF) {
    bits = 0x7fc0u;
  } else {
    volatile float mult = ldexpf(1.0f, (int)scale - 127);
    volatile float v = table8[code & 7] * mult;
    bits = f32_to_bf16_rne(v);
  }
  if (code & 8) bits ^= 0x8000u;
  return bits;
}

/* The exact value of one weight in fp64 (no bf16 rounding): the level as
 * stored (fp32) times 2^(s-127), which fp64 holds exactly. */
static double decode_f64(uint8_t code, uint8_t scale, const float* table8) {
  if (scale == 0xFF) return NAN;
  double v = ldexp((double)table8[code & 7], (int)scale - 127);
  return (code & 8) ? -v : v;
}

/* Code for K index k of a packed row: two codes per byte, the low nibble
 * holds the even K index ([NF4-Lloyd, "Contents"]). */
static uint8_t code_at(const uint8_t* packed_row, int k) {
  uint8_t byte = packed_row[k >> 1];
  return (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0x0f);
}

/* Full dequantisation of E stacked [N][K] projections.
 * weight: [E][N][K/2] bytes; weight_scale: [E][N][K/32] E8M0 bytes (one per
 * 32 weights along K); expert e decodes with tables[table_id[e]].
 * out: [E][N][K] bf16 bit patterns. */
int oq_dequant(const uint8_t* weight, const uint8_t* weight_scale, const float* tables,
               int n_tables, const uint8_t* table_id, int E, int N, int K, uint16_t* out) {
  if (E < 0 || N < 0 || K < 0 || (K % 32) != 0) return OQ_EINVAL;
  if (E == 0 || N == 0 || K == 0) return OQ_OK;
  if (!weight || !weight_scale || !out || !tables_ok(tables, n_tables, table_id, E)) return OQ_EINVAL;
  for (int e = 0; e < E; ++e) {
    const float* t = tables + 8 * table_id[e];
    for (int n = 0; n < N; ++n) {
      size_t row = (size_t)e * N + n;
      const uint8_t* wr = weight + row * (size_t)(K / 2);
      const uint8_t* sr = weight_scale + row * (size_t)(K / 32);
      for (int k = 0; k < K; ++k)
        out[row * (size_t)K + k] = oq_decode_bf16(code_at(wr, k), sr[k / 32], t);
    }
  }
  return OQ_OK;
}

/* Exact fp64 values of one [N][K] projection (for the tests' dense
 * references). out: [N][K] doubles. */
int oq_decode_matrix_f64(const uint8_t* weight, const uint8_t* weight_scale, const float* table8,
                         int N, int K, double* out) {
  if (N < 0 || K < 0 || (K % 32) != 0 || !weight || !weight_scale || !out) return OQ_EINVAL;
  if (!table_ok(table8)) return OQ_EINVAL;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      out[(size_t)n * K + k] = decode_f64(code_at(weight + (size_t)n * (K / 2), k),
                                          weight_scale[(size_t)n * (K / 32) + k / 32], table8);
  return OQ_OK;
}

/* ---- pack -------------------------------------------------------------- */

/* Block exponent.  [NF4-Lloyd, "Codes are indices..."]: codes were packed
 * against gmax * 2^e >= amax, the grid not amax-normalised.  Reading: e is the
 * smallest integer with gmax * 2^e >= amax, clamped to the E8M0 range
 * [-127, 127] (scale byte e + 127, never 0xFF); an all-zero block has no
 * smallest e and takes -127.  fp64 holds every gmax * 2^e exactly. */
static int block_exponent(double amax, double gmax) {
  if (amax == 0.0) return -127;
  int ea, eg;
  frexp(amax, &ea);
  frexp(gmax, &eg);
  int e = ea - eg;
  while (ldexp(gmax, e) < amax) ++e;
  while (ldexp(gmax, e - 1) >= amax) --e;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* Round-to-nearest level: index of the table entry closest (fp64 distance) to
 * r; on a tie the lower index wins. */
static int nearest_level(double r, const float* t) {
  int best = 0;
  double bd = fabs(r - (double)t[0]);
  for (int i = 1; i < 8; ++i) {
    double d = fabs(r - (double)t[i]);
    if (d < bd) {
      bd = d;
      best = i;
    }
  }
  return best;
}

/* Pack bf16 weights [E][N][K] into codes [E][N][K/2] and E8M0 bytes
 * [E][N][K/32], expert e against tables[table_id[e]]: per 32-block along K,
 * e by block_exponent(amax, max level), then each weight rounds to the nearest
 * level of |x| / 2^e with sign bit = (x < 0) (so -0.0 packs as +).  A NaN or
 * Inf input is an error. */
int oq_pack(const uint16_t* src, int E, int N, int K, const float* tables, int n_tables,
            const uint8_t* table_id, uint8_t* weight, uint8_t* weight_scale) {
  if (E < 0 || N < 0 || K < 0 || (K % 32) != 0) return OQ_EINVAL;
  if (E == 0 || N == 0 || K == 0) return OQ_OK;
  if (!src || !weight || !weight_scale || !tables_ok(tables, n_tables, table_id, E)) return OQ_EINVAL;
  for (int e = 0; e < E; ++e) {
    const float* t = tables + 8 * table_id[e];
    double gmax = 0.0;
    for (int i = 0; i < 8; ++i)
      if ((double)t[i] > gmax) gmax = (double)t[i];
    for (int n = 0; n < N; ++n) {
      size_t row = (size_t)e * N + n;
      for (int b = 0; b < K / 32; ++b) {
        const uint16_t* blk = src + row * (size_t)K + (size_t)b * 32;
        double amax = 0.0;
        for (int i = 0; i < 32; ++i) {
          double v = (double)bf16_bits_to_f32(blk[i]);
          if (!isfinite(v)) return OQ_EINVAL;
          if (fabs(v) > amax) amax = fabs(v);
        }
        int ex = block_exponent(amax, gmax);
        weight_scale[row * (size_t)(K / 32) + b] = (uint8_t)(ex + 127);
        uint8_t* wr = weight + row * (size_t)(K / 2) + (size_t)b * 16;
        for (int i = 0; i < 32; i += 2) {
          uint8_t c[2];
          for (int q = 0; q < 2; ++q) {
            double v = (double)bf16_bits_to_f32(blk[i + q]);
            int idx = nearest_level(ldexp(fabs(v), -ex), t);
            c[q] = (uint8_t)((v < 0.0 ? 8 : 0) | idx);
          }
          wr[i / 2] = (uint8_t)(c[0] | (c[1] << 4));
        }
      }
    }
  }
  return OQ_OK;
}

/* ---- router logits ----------------------------------------------------- */

/* Router logits of T tokens: logits[t][e] = sum over h of x[t][h] * w[e][h],
 * the router gate ("mlp.gate", held in BF16 per [DENSE6, "Quant recipe"])
 * applied to the hidden states, with the geometry of [ROUND7, "Ground truth
 * and corrections"] (hidden 6144, 256 routed experts).  x and w are bf16 bit
 * patterns; each product is exact in fp64 and the sum runs over h in order.
 * absdot[t][e] (optional) = sum of |x[t][h] * w[e][h]|, the scale of the
 * rounding error a finite-precision evaluation may make.
 * x: [T][H]; w: [E][H]; logits, absdot: [T][E]. */
int oq_router_logits(const uint16_t* x, const uint16_t* w, int T, int H, int E, double* logits, double* absdot) {
  if (T < 0 || H < 0 || E < 1) return OQ_EINVAL;
  if (T == 0) return OQ_OK;
  if (!x || !w || !logits) return OQ_EINVAL;
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0, mag = 0.0;
      for (int h = 0; h < H; ++h) {
        const double p = (double)bf16_bits_to_f32(x[(size_t)t * H + h]) * (double)bf16_bits_to_f32(w[(size_t)e * H + h]);
        acc += p;
        mag += fabs(p);
      }
      logits[(size_t)t * E + e] = acc;
      if (absdot) absdot[(size_t)t * E + e] = mag;
    }
  return OQ_OK;
}

/* ---- shared expert ----------------------------------------------------- */

/* The shared expert ([TR3v4] README, "Checkpoint layout update": the
 * shared-expert MLP is kept as its original BF16 weights, gate and up
 * concatenated into one payload): for every token,
 *   g = Wg x, u = Wu x, h = silu(g) * u, y = Wd h,
 * with Wgu = [Wg; Wu] ([2 I][H], rows 0..I-1 the gate, I..2I-1 the up, the
 * order in which the page concatenates them) and Wd [H][I], all in fp64 from
 * the bf16 values.  Readings: the shared expert sees every token with weight
 * 1 and its output is added to the routed experts' weighted sum (the pages
 * describe the shared expert beside the routed ones, with no gate of its own).
 * x: [T][H] bf16; out: [T][H] fp64 (the shared expert's output alone). */
int oq_shared_ffn(const uint16_t* x, int T, int H, const uint16_t* wgu, const uint16_t* wd, int I, double* out) {
  if (T < 0 || H <= 0 || I <= 0) return OQ_EINVAL;
  if (T == 0) return OQ_OK;
  if (!x || !wgu || !wd || !out) return OQ_EINVAL;
  double* xv = (double*)malloc(sizeof(double) * H);
  double* hv = (double*)malloc(sizeof(double) * I);
  if (!xv || !hv) {
    free(xv);
    free(hv);
    return OQ_EINVAL;
  }
  for (int t = 0; t < T; ++t) {
    for (int c = 0; c < H; ++c) xv[c] = (double)bf16_bits_to_f32(x[(size_t)t * H + c]);
    for (int i = 0; i < I; ++i) {
      double g = 0.0, u = 0.0;
      for (int c = 0; c < H; ++c) {
        g += (double)bf16_bits_to_f32(wgu[(size_t)i * H + c]) * xv[c];
        u += (double)bf16_bits_to_f32(wgu[(size_t)(I + i) * H + c]) * xv[c];
      }
      hv[i] = g / (1.0 + exp(-g)) * u;
    }
    for (int c = 0; c < H; ++c) {
      double y = 0.0;
      for (int i = 0; i < I; ++i) y += (double)bf16_bits_to_f32(wd[(size_t)c * I + i]) * hv[i];
      out[(size_t)t * H + c] = y;
    }
  }
  free(xv);
  free(hv);
  return OQ_OK;
}

/* ---- routing ----------------------------------------------------------- */

/* Top-k of E logits per token, then softmax over the k kept.
 * Geometry from [ROUND7, "Ground truth and corrections"] (256 routed experts,
 * top-8).  The pages give no router formula; the reading taken: order by
 * logit descending, equal logits by lower expert id; weights
 * exp(l_j - l_max) / sum_i exp(l_i - l_max) over the k kept, in fp64; no bias
 * and no scaling factor.  A non-finite logit is an error.
 * ids: [T][k] int32 (descending logit); w: [T][k] fp64. */
int oq_route(const float* logits, int T, int E, int k, int32_t* ids, double* w) {
  if (T < 0 || E < 1 || k < 1 || k > E) return OQ_EINVAL;
  if (T == 0) return OQ_OK;
  if (!logits || !ids || !w) return OQ_EINVAL;
  char* taken = (char*)malloc((size_t)E);
  if (!taken) return OQ_EINVAL;
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    for (int e = 0; e < E; ++e)
      if (!isfinite(l[e])) {
        free(taken);
        return OQ_EINVAL;
      }
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
      taken[best] = 1;
      ids[(size_t)t * k + j] = best;
    }
    double lmax = (double)l[ids[(size_t)t * k]];
    double sum = 0.0;
    for (int j = 0; j < k; ++j) sum += exp((double)l[ids[(size_t)t * k + j]] - lmax);
    for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = exp((double)l[ids[(size_t)t * k + j]] - lmax) / sum;
  }
  free(taken);
  return OQ_OK;
}

/* Group (token, slot) rows by expert: counts[e]; offsets[0..E] the exclusive
 * scan; rows of expert e are offsets[e]..offsets[e+1]-1 in ascending token
 * order; row_token[row] = token; inv[t][j] = row of (t, j).  This is a stable
 * counting sort by expert id (the pages' fused kernel walks "route blocks" of
 * rows per expert: [TR3v4, "Tuning: prefill route block size"]). */
int oq_group(const int32_t* ids, int T, int E, int k, int32_t* counts, int32_t* offsets,
             int32_t* row_token, int32_t* inv) {
  if (T < 0 || E < 1 || k < 1 || k > E) return OQ_EINVAL;
  if (!counts || !offsets) return OQ_EINVAL;
  if (T > 0 && (!ids || !row_token || !inv)) return OQ_EINVAL;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (size_t r = 0; r < (size_t)T * k; ++r) {
    if (ids[r] < 0 || ids[r] >= E) return OQ_EINVAL;
    counts[ids[r]]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  if (!cursor) return OQ_EINVAL;
  for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int e = ids[(size_t)t * k + j];
      int r = cursor[e]++;
      row_token[r] = t;
      inv[(size_t)t * k + j] = r;
    }
  free(cursor);
  return OQ_OK;
}

/* ---- the MoE layer ------------------------------------------------------ */

/* Packed layer, one pointer per expert per tensor (NULL for experts the
 * caller did not load; touching one is an error).
 *   gate_w[e], up_w[e]: [I][H/2]   gate_s[e], up_s[e]: [I][H/32]
 *   down_w[e]: [H][I/2]            down_s[e]: [H][I/32]
 * Shapes from [ROUND7, "Owner-locked decisions" 6] (down is [K=I, N=H]). */
typedef struct {
  int E, H, I;
  const uint8_t* const* gate_w;
  const uint8_t* const* gate_s;
  const uint8_t* const* up_w;
  const uint8_t* const* up_s;
  const uint8_t* const* down_w;
  const uint8_t* const* down_s;
  const float* tables;
  int n_tables;
  const uint8_t* table_id;
} oq_layer;

/* y = W v for one packed [N][K] projection, all in fp64. */
static void matvec_f64(const uint8_t* w, const uint8_t* s, const float* t, int N, int K,
                       const double* v, double* y) {
  for (int n = 0; n < N; ++n) {
    const uint8_t* wr = w + (size_t)n * (K / 2);
    const uint8_t* sr = s + (size_t)n * (K / 32);
    double acc = 0.0;
    for (int k = 0; k < K; ++k) acc += decode_f64(code_at(wr, k), sr[k / 32], t) * v[k];
    y[n] = acc;
  }
}

/* MoE output for n_tokens independent tokens.
 * x: [n][H] bf16 bits; logits: [n][E] fp32; out: [n][H] fp64;
 * ids_out/w_out (optional, may be NULL): [n][k].
 * For each token: route (oq_route); for each kept expert e in slot order,
 *   g = Wg_e x, u = Wu_e x, h = silu(g) * u = g / (1 + e^-g) * u
 *   ([ROUND7, "Owner-locked decisions" 4]: I_e = silu(X Wg^T) * (X Wu^T)),
 *   y = Wd_e h,
 *   out += w_j * y  ([TR3v4]: expert outputs are routing-weighted and summed).
 * Nothing is rounded: x is exact from bf16, weights exact from the codes. */
int oq_moe_tokens(const oq_layer* L, const uint16_t* x, const float* logits, int n, int k,
                  double* out, int32_t* ids_out, double* w_out) {
  if (!L || n < 0 || L->E < 1 || L->H <= 0 || L->I <= 0 || (L->H % 32) || (L->I % 32)) return OQ_EINVAL;
  if (k < 1 || k > L->E) return OQ_EINVAL;
  if (n == 0) return OQ_OK;
  if (!x || !logits || !out || !tables_ok(L->tables, L->n_tables, L->table_id, L->E)) return OQ_EINVAL;
  const int H = L->H, I = L->I;
  double* xv = (double*)malloc(sizeof(double) * H);
  double* g = (double*)malloc(sizeof(double) * I);
  double* u = (double*)malloc(sizeof(double) * I);
  double* y = (double*)malloc(sizeof(double) * H);
  int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * k);
  double* wts = (double*)malloc(sizeof(double) * k);
  int rc = OQ_OK;
  if (!xv || !g || !u || !y || !ids || !wts) {
    rc = OQ_EINVAL;
    goto done;
  }
  for (int t = 0; t < n; ++t) {
    if (oq_route(logits + (size_t)t * L->E, 1, L->E, k, ids, wts) != OQ_OK) {
      rc = OQ_EINVAL;
      goto done;
    }
    if (ids_out)
      for (int j = 0; j < k; ++j) ids_out[(size_t)t * k + j] = ids[j];
    if (w_out)
      for (int j = 0; j < k; ++j) w_out[(size_t)t * k + j] = wts[j];
    for (int h = 0; h < H; ++h) xv[h] = (double)bf16_bits_to_f32(x[(size_t)t * H + h]);
    double* o = out + (size_t)t * H;
    for (int h = 0; h < H; ++h) o[h] = 0.0;
    for (int j = 0; j < k; ++j) {
      int e = ids[j];
      if (!L->gate_w[e] || !L->gate_s[e] || !L->up_w[e] || !L->up_s[e] || !L->down_w[e] || !L->down_s[e]) {
        rc = OQ_EINVAL;
        goto done;
      }
      const float* tb = L->tables + 8 * L->table_id[e];
      matvec_f64(L->gate_w[e], L->gate_s[e], tb, I, H, xv, g);
      matvec_f64(L->up_w[e], L->up_s[e], tb, I, H, xv, u);
      for (int i = 0; i < I; ++i) g[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
      matvec_f64(L->down_w[e], L->down_s[e], tb, H, I, g, y);
      for (int h = 0; h < H; ++h) o[h] += wts[j] * y[h];
    }
  }
done:
  free(xv);
  free(g);
  free(u);
  free(y);
  free(ids);
  free(wts);
  return rc;
}

/* One expert's output for one token restricted to intermediate channels
 * [i0, i1):  y[n] = sum_{i0 <= i < i1} Wd_e[n][i] * silu(g_i) * u_i, with
 * g = Wg_e x and u = Wu_e x as in oq_moe_tokens.  The expert's full output is
 * the sum of these over any partition of [0, I); the benchmark's CPU
 * baseline times such pieces as bounded samples of the layer.
 * x: [H] bf16 bits; y: [H] fp64 (out). */
int oq_expert_partial(const oq_layer* L, int e, const uint16_t* x, int i0, int i1, double* y) {
  if (!L || e < 0 || e >= L->E || i0 < 0 || i1 > L->I || i0 > i1 || !x || !y) return OQ_EINVAL;
  if (!tables_ok(L->tables, L->n_tables, L->table_id, L->E)) return OQ_EINVAL;
  if (!L->gate_w[e] || !L->gate_s[e] || !L->up_w[e] || !L->up_s[e] || !L->down_w[e] || !L->down_s[e])
    return OQ_EINVAL;
  const int H = L->H, I = L->I;
  const float* tb = L->tables + 8 * L->table_id[e];
  double* xv = (double*)malloc(sizeof(double) * H);
  if (!xv) return OQ_EINVAL;
  for (int h = 0; h < H; ++h) xv[h] = (double)bf16_bits_to_f32(x[h]);
  for (int n = 0; n < H; ++n) y[n] = 0.0;
  for (int i = i0; i < i1; ++i) {
    double g = 0.0, u = 0.0;
    const uint8_t* gw = L->gate_w[e] + (size_t)i * (H / 2);
    const uint8_t* gs = L->gate_s[e] + (size_t)i * (H / 32);
    const uint8_t* uw = L->up_w[e] + (size_t)i * (H / 2);
    const uint8_t* us = L->up_s[e] + (size_t)i * (H / 32);
    for (int k = 0; k < H; ++k) {
      g += decode_f64(code_at(gw, k), gs[k / 32], tb) * xv[k];
      u += decode_f64(code_at(uw, k), us[k / 32], tb) * xv[k];
    }
    const double hi = g / (1.0 + exp(-g)) * u;
    for (int n = 0; n < H; ++n)
      y[n] += decode_f64(code_at(L->down_w[e] + (size_t)n * (I / 2), i),
                         L->down_s[e][(size_t)n * (I / 32) + i / 32], tb) * hi;
  }
  free(xv);
  return OQ_OK;
}

/* ---- weighted Lloyd-Max grid fit ---------------------------------------- */

/* Index of the level closest (fp64 distance) to r; on a tie the lower index
 * wins (the same rule as the pack's nearest_level). */
static int nearest_level_f64(double r, const double* m) {
  int best = 0;
  double bd = fabs(r - m[0]);
  for (int i = 1; i < 8; ++i) {
    double d = fabs(r - m[i]);
    if (d < bd) {
      bd = d;
      best = i;
    }
  }
  return best;
}

/* The per-layer grid fit of [NF4-Lloyd, "What this is"]: 8 magnitudes fitted
 * by weighted Lloyd-Max over the pooled ratios |W / 2^e| of all the layer's
 * weights, each ratio weighted by (2^e)^2 so that it counts in proportion to
 * its weight-space squared error.  Readings (the page names the objective,
 * not the procedure around it):
 *   - e is each 32-block's exponent under the pack rule ([NF4-Lloyd], "Codes
 *     are indices...": gmax * 2^e >= amax) with gmax the largest level of the
 *     starting grid, fixed for the whole fit;
 *   - a Lloyd step assigns every ratio to its nearest level (tie -> lower
 *     index) and moves each level to the weighted mean sum(w r) / sum(w) of
 *     its ratios; a level with no ratio keeps its value;
 *   - steps repeat until no level moves by more than tol, or max_iter steps;
 *   - the result is each fp64 level rounded to fp32.
 * src: n_blocks x 32 bf16 bit patterns (each run of 32 one block along K);
 * grid0: 8 fp32 magnitudes, strictly ascending, finite, >= 0, max > 0;
 * grid: [8] fp32 (out); *iters: steps taken (out). */
int oq_lloyd_fit(const uint16_t* src, long long n_blocks, const float* grid0, int max_iter, double tol,
                 float* grid, int* iters) {
  if (n_blocks < 0 || !grid0 || !grid || !iters || max_iter < 0 || !(tol >= 0.0)) return OQ_EINVAL;
  if (n_blocks > 0 && !src) return OQ_EINVAL;
  if (!table_ok(grid0)) return OQ_EINVAL;
  for (int i = 1; i < 8; ++i)
    if (!(grid0[i] > grid0[i - 1])) return OQ_EINVAL;
  const double gmax = (double)grid0[7];
  int* ex = (int*)malloc(sizeof(int) * (size_t)(n_blocks > 0 ? n_blocks : 1));
  if (!ex) return OQ_EINVAL;
  for (long long b = 0; b < n_blocks; ++b) {
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) {
      double v = (double)bf16_bits_to_f32(src[b * 32 + i]);
      if (!isfinite(v)) {
        free(ex);
        return OQ_EINVAL;
      }
      if (fabs(v) > amax) amax = fabs(v);
    }
    ex[b] = block_exponent(amax, gmax);
  }
  double m[8];
  for (int i = 0; i < 8; ++i) m[i] = (double)grid0[i];
  int it = 0;
  while (it < max_iter) {
    double sw[8] = {0}, swr[8] = {0};
    for (long long b = 0; b < n_blocks; ++b) {
      const double wgt = ldexp(1.0, 2 * ex[b]);
      for (int i = 0; i < 32; ++i) {
        const double r = ldexp(fabs((double)bf16_bits_to_f32(src[b * 32 + i])), -ex[b]);
        const int j = nearest_level_f64(r, m);
        sw[j] += wgt;
        swr[j] += wgt * r;
      }
    }
    double moved = 0.0;
    for (int j = 0; j < 8; ++j) {
      if (sw[j] > 0.0) {
        const double nm = swr[j] / sw[j];
        if (fabs(nm - m[j]) > moved) moved = fabs(nm - m[j]);
        m[j] = nm;
      }
    }
    ++it;
    if (moved <= tol) break;
  }
  for (int j = 0; j < 8; ++j) grid[j] = (float)m[j];
  *iters = it;
  free(ex);
  return OQ_OK;
}
