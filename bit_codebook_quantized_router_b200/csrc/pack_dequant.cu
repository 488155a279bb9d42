// Pack (bf16 -> 4-bit codes + E8M0 scales) and dequantisation (codes -> bf16)
// kernels and their C-ABI entry points.
//
// Format and rules: "aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", sections
// "Contents" (block 32 along K, low nibble = even K) and "Codes are indices
// into the per-layer grid -- not E2M1" (w = sign * grid[code & 7] *
// 2^(scale - 127); codes packed against gmax * 2^e >= amax).
#include <math.h>

#include "q4_api_internal.h"
#include "q4_common.cuh"

namespace q4 {

// ---------------------------------------------------------------------------
// Pack: one thread per 32-weight block (a setup step, not on the hot path).
// The exponent and the nearest-level choice follow the reference definition
// exactly: fp64 distances (exact for fp32 levels and power-of-two scaled
// bf16 inputs), first minimum wins, sign bit = (x < 0).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_exponent(double amax, double gmax) {
  if (amax == 0.0) return -127;
  int ea, eg;
  frexp(amax, &ea);
  frexp(gmax, &eg);
  int e = ea - eg;
  while (ldexp(gmax, e) < amax) ++e;
  while (ldexp(gmax, e - 1) >= amax) --e;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

__global__ void __launch_bounds__(256) pack_kernel(const uint16_t* __restrict__ w, int64_t n_blocks,
                                                   int N, int K, const __grid_constant__ TableParams tp,
                                                   uint8_t* __restrict__ codes,
                                                   uint8_t* __restrict__ scales, int32_t* status) {
  const int bpr = K / kBlockK;  // blocks per row
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < n_blocks;
       b += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = b / bpr;
    const int e = (int)(row / N);
    const float* t = tp.t[tp.id[e]];
    double lev[8], gmax = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lev[i] = (double)t[i];
      gmax = fmax(gmax, lev[i]);
    }
    const uint4* src = reinterpret_cast<const uint4*>(w + b * kBlockK);
    uint32_t v[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u = src[q];
      v[4 * q + 0] = u.x;
      v[4 * q + 1] = u.y;
      v[4 * q + 2] = u.z;
      v[4 * q + 3] = u.w;
    }
    double amax = 0.0;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const uint32_t bits = (v[i >> 1] >> ((i & 1) * 16)) & 0xffffu;
      if ((bits & 0x7f80u) == 0x7f80u) bad = true;  // Inf or NaN
      amax = fmax(amax, (double)__uint_as_float((bits & 0x7fffu) << 16));
    }
    if (bad) record_error(status, MOE_Q4_EDEVICE);
    const int ex = block_exponent(amax, gmax);
    uint32_t out[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const uint32_t bits = (v[i >> 1] >> ((i & 1) * 16)) & 0xffffu;
      const double r = ldexp((double)__uint_as_float((bits & 0x7fffu) << 16), -ex);
      int best = 0;
      double bd = fabs(r - lev[0]);
#pragma unroll
      for (int j = 1; j < 8; ++j) {
        const double d = fabs(r - lev[j]);
        if (d < bd) {
          bd = d;
          best = j;
        }
      }
      // x < 0: sign bit set and not -0.0 (NaN excluded above).
      const bool neg = (bits & 0x8000u) && (bits & 0x7fffu);
      const uint32_t code = (neg ? 8u : 0u) | (uint32_t)best;
      out[i >> 3] |= code << ((i & 7) * 4);
    }
    reinterpret_cast<uint4*>(codes)[b] = make_uint4(out[0], out[1], out[2], out[3]);
    scales[b] = (uint8_t)(ex + 127);
  }
}

// ---------------------------------------------------------------------------
// Dequantisation: one thread per 32-bit code word (8 weights, 16 bytes of
// bf16 out), so a warp's loads cover 128 contiguous code bytes and its stores
// 512 contiguous output bytes; each thread takes kDqWords words a grid stride
// apart, loads first, so several loads are in flight per thread.
// Fast path (the block's scale keeps every non-zero level a normal bf16):
// PRMT byte-plane lookups of the bf16-rounded levels decode the 8 codes, then
// one bf16x2 multiply per pair by the scale 2^e (an exact bf16; the products
// are normal, so exact too).  Rounding commutes with a power-of-two scale in
// the normal range, so this equals "fp32 multiply, then RNE to bf16" bit for
// bit.  Otherwise (subnormal / overflowing results, scale bytes 0 and 0xFF)
// every weight takes the literal fp32 path.
// ---------------------------------------------------------------------------
struct DequantTable {
  uint32_t b[8];     // bf16 bits of each level (RNE)
  int emin, emax;    // exponent fields over non-zero levels
  int has_sub;       // a non-zero level that is a bf16 subnormal
  Planes pl;         // byte planes of b[] for the PRMT lookup
};

constexpr int kDqWords = 8;

__device__ __forceinline__ void dequant_word(uint32_t cw, uint32_t s, const DequantTable& d, const float* t,
                                             uint32_t res[4]) {
  const int e = (int)s - 127;
  // emin + e >= 2 keeps even the unrounded fp32 level times 2^e normal.
  if (!d.has_sub && s != 0u && s != 255u && d.emin + e >= 2 && d.emax + e <= 254) {
    decode8(cw, d.pl, res);
    const uint32_t s2 = (s << 7) | (s << 23);  // 2^e in both bf16 halves
#pragma unroll
    for (int i = 0; i < 4; ++i) res[i] = bf16x2_mul(res[i], s2);
  } else {
    const float mult = __uint_as_float(s == 0u ? 0x00400000u : (s << 23));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t code = (cw >> (4 * i)) & 0xfu;
      uint32_t bits = (s == 255u) ? 0x7fc0u : (uint32_t)bf16_bits_rn(__fmul_rn(t[code & 7], mult));
      if (code & 8u) bits ^= 0x8000u;
      if (i & 1)
        res[i >> 1] |= bits << 16;
      else
        res[i >> 1] = bits;
    }
  }
}

__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ codes,
                                                      const uint8_t* __restrict__ scales,
                                                      int64_t n_words, int N, int K,
                                                      const __grid_constant__ TableParams tp,
                                                      uint16_t* __restrict__ out) {
  __shared__ DequantTable st[kMaxTables];
  if (threadIdx.x < tp.n) {
    DequantTable d;
    d.emin = 255;
    d.emax = 0;
    d.has_sub = 0;
    for (int i = 0; i < 8; ++i) {
      const float lv = tp.t[threadIdx.x][i];
      d.b[i] = bf16_bits_rn(lv);
      const int ef = (d.b[i] >> 7) & 0xff;
      if (lv != 0.0f) {
        // a positive level whose bf16 is zero or subnormal cannot take the
        // fast path
        if (ef == 0) d.has_sub = 1;
        d.emin = min(d.emin, ef);
        d.emax = max(d.emax, ef);
      }
    }
    const uint32_t w01 = d.b[0] | (d.b[1] << 16), w23 = d.b[2] | (d.b[3] << 16);
    const uint32_t w45 = d.b[4] | (d.b[5] << 16), w67 = d.b[6] | (d.b[7] << 16);
    d.pl.l0 = prmt(w01, w23, 0x6420);
    d.pl.h0 = prmt(w01, w23, 0x7531);
    d.pl.l1 = prmt(w45, w67, 0x6420);
    d.pl.h1 = prmt(w45, w67, 0x7531);
    st[threadIdx.x] = d;
  }
  __syncthreads();
  const uint64_t words_per_expert = (uint64_t)N * (uint64_t)(K / 8);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t w0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w0 < n_words; w0 += stride * kDqWords) {
    uint32_t cw[kDqWords], sc[kDqWords];
#pragma unroll
    for (int u = 0; u < kDqWords; ++u) {
      const int64_t w = w0 + u * stride;
      if (w < n_words) {
        cw[u] = __ldcs(reinterpret_cast<const unsigned int*>(codes) + w);
        sc[u] = __ldg(scales + (w >> 2));  // 4 words per 32-weight block
      }
    }
#pragma unroll
    for (int u = 0; u < kDqWords; ++u) {
      const int64_t w = w0 + u * stride;
      if (w >= n_words) break;
      const int tid = tp.n == 1 ? 0 : tp.id[(int)((uint64_t)w / words_per_expert)];
      uint32_t res[4];
      dequant_word(cw[u], sc[u], st[tid], tp.t[tid], res);
      __stcs(reinterpret_cast<uint4*>(out) + w, make_uint4(res[0], res[1], res[2], res[3]));
    }
  }
}

}  // namespace q4

using namespace q4;

extern "C" int moe_q4_pack(const void* w, int E, int N, int K, const float* tables, int n_tables,
                           const uint8_t* table_id, uint8_t* weight, uint8_t* weight_scale,
                           int32_t* status, void* stream) {
  if (E < 0 || N < 0 || K < 0 || (K % kBlockK) != 0 || E > kMaxExperts) return MOE_Q4_EINVAL;
  if ((int64_t)E * N * K == 0) return MOE_Q4_OK;
  if (!w || !weight || !weight_scale || !status) return MOE_Q4_EINVAL;
  TableParams tp;
  int rc = q4_fill_tables(&tp, tables, n_tables, table_id, E);
  if (rc != MOE_Q4_OK) return rc;
  if (((uintptr_t)w & 15) || ((uintptr_t)weight & 15)) return MOE_Q4_EINVAL;
  const int64_t n_blocks = (int64_t)E * N * (K / kBlockK);
  const int threads = 256;
  const int64_t want = (n_blocks + threads - 1) / threads;
  const int grid = (int)(want < 148 * 64 ? want : 148 * 64);
  pack_kernel<<<grid, threads, 0, (cudaStream_t)stream>>>((const uint16_t*)w, n_blocks, N, K, tp,
                                                           weight, weight_scale, status);
  return cudaGetLastError() == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}

extern "C" int moe_q4_dequant(const uint8_t* weight, const uint8_t* weight_scale,
                              const float* tables, int n_tables, const uint8_t* table_id, int E,
                              int N, int K, void* out, void* stream) {
  if (E < 0 || N < 0 || K < 0 || (K % kBlockK) != 0 || E > kMaxExperts) return MOE_Q4_EINVAL;
  if ((int64_t)E * N * K == 0) return MOE_Q4_OK;
  if (!weight || !weight_scale || !out) return MOE_Q4_EINVAL;
  TableParams tp;
  int rc = q4_fill_tables(&tp, tables, n_tables, table_id, E);
  if (rc != MOE_Q4_OK) return rc;
  if (((uintptr_t)weight & 15) || ((uintptr_t)out & 15)) return MOE_Q4_EINVAL;
  const int64_t n_words = (int64_t)E * N * (K / 8);
  const int threads = 256;
  const int64_t want = (n_words + threads * kDqWords - 1) / (threads * kDqWords);
  const int grid = (int)(want < 148 * 8 ? want : 148 * 8);
  dequant_kernel<<<grid, threads, 0, (cudaStream_t)stream>>>(weight, weight_scale, n_words, N, K,
                                                              tp, (uint16_t*)out);
  return cudaGetLastError() == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}
