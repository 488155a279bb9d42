// Weighted Lloyd-Max fit of a layer's 8-level magnitude grid on the GPU
// ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", "What this is": the 8 levels
// are fitted by Lloyd-Max over the pooled ratios |W / 2^e| of the layer's
// weights, each ratio weighted by (2^e)^2).
//
// Readings (the page names the objective, not the procedure around it):
//   - e is each 32-block's exponent under the pack rule (the smallest e with
//     gmax * 2^e >= amax, clamped to [-127, 127]) for the largest level of
//     the starting grid, fixed for the whole fit;
//   - a step assigns every ratio to its nearest level (fp64 distance, a tie
//     to the lower index) and moves each level to the weighted mean of its
//     ratios; a level with no ratio keeps its value;
//   - steps repeat until no level moves by more than tol, or max_iter steps;
//     the levels are then rounded to fp32.
//
// Three kernels:
//   lloyd_hist_kernel   one pass over the bf16 weights.  Every ratio of a
//                       bf16 weight to a power of two is itself a bf16 value
//                       (exactly, unless it falls below the bf16 range), so
//                       the ratios are binned by their bf16 bit pattern, bins
//                       0 .. bits(gmax) (at most 16,768 for gmax < 16).  The
//                       weight (2^e)^2 of a ratio depends only on its block's
//                       exponent, so a CTA counts ratios per (exponent slot,
//                       bin) in 32-bit shared-memory counters (integer
//                       atomics; three slots, the exponents e0 - 1, e0, e0 + 1
//                       around its first block's), and writes the counts to
//                       its own slice of the workspace (no global atomics on
//                       the hot path).  A block whose exponent falls outside
//                       the slots adds (2^e)^2 per ratio straight into an fp64
//                       side histogram (rare: a layer's block exponents
//                       cluster within a step or two).
//   lloyd_sum_kernel    W[r] = sum over CTAs and slots of count * (2^e)^2,
//                       plus the side histogram, added in a fixed order.
//                       The terms are powers of four times integers: while a
//                       bin's sum stays within 2^53 of its smallest term
//                       (block exponents spanning less than about 9 steps at
//                       the GLM layer's size) the sum is exact.
//   lloyd_solve_kernel  one CTA runs the Lloyd steps on W: each thread takes
//                       a fixed set of bins, finds each bin's nearest level,
//                       and sums W and W * r per level; the per-thread sums
//                       are added in a fixed tree order, so the result is
//                       deterministic.
#include <math.h>

#include "q4_api_internal.h"
#include "q4_common.cuh"

namespace q4 {

constexpr int kLloydMaxBins = 16768;  // bf16 bit patterns 0 .. 0x417f: gmax < 16
constexpr int kLloydHistThreads = 512;
constexpr int kLloydSolveThreads = 1024;

struct LloydParams {
  double lev0[8];  // starting grid (fp32 values)
  double gmax;     // its largest level
  int n_bins;      // bits(gmax) + 1
};

// Block exponent under the pack rule: the smallest e with gmax * 2^e >= amax,
// clamped to [-127, 127]; an all-zero block takes -127.
__device__ __forceinline__ int lloyd_block_exponent(double amax, double gmax) {
  if (amax == 0.0) return -127;
  int ea, eg;
  frexp(amax, &ea);
  frexp(gmax, &eg);
  int e = ea - eg;
  while (ldexp(gmax, e) < amax) ++e;
  while (ldexp(gmax, e - 1) >= amax) --e;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// bf16 bit pattern of |x| * 2^-e for the magnitude bits m of a bf16 value
// (exact when the result is a bf16 value; below the bf16 range the result is
// rounded to nearest even, the one case the binning is not exact).
__device__ __forceinline__ uint32_t lloyd_ratio_bits(uint32_t m, int e) {
  const int E = (int)(m >> 7);
  if (m == 0u) return 0u;
  if (E >= 1 && E - e >= 1 && E - e <= 254) return m - (uint32_t)(e * 128);  // normal -> normal: exponent shift
  const double r = ldexp((double)__uint_as_float(m << 16), -e);
  return (uint32_t)bf16_bits_rn((float)r) & 0x7fffu;
}

// Block exponent from the bf16 bit pattern of amax (integers; the rare
// subnormal cases take the fp64 loop of the pack rule).
__device__ __forceinline__ int lloyd_block_exponent_bits(uint32_t amx, uint32_t gbits, double gmax) {
  if (amx == 0u) return -127;
  const int ae = (int)(amx >> 7), ge = (int)(gbits >> 23);
  if (ae == 0 || ge == 0) return lloyd_block_exponent((double)__uint_as_float(amx << 16), gmax);
  // gmax * 2^e >= amax  <=>  e >= (ae - ge) + [mantissa of amax > mantissa of gmax]
  int e = (ae - 127) - (ge - 127) + (((amx & 0x7fu) << 16) > (gbits & 0x7fffffu) ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

constexpr int kLloydSlots = 3;   // exponent slots per CTA
constexpr int kLloydUnroll = 8;  // 512-byte groups in flight per warp

// One pass: 4 lanes per 32-weight block (16 bytes = 8 weights each), a warp
// covers 8 consecutive blocks (512 contiguous bytes) per group, and loads
// kLloydUnroll groups before it bins any of them.
__global__ void __launch_bounds__(kLloydHistThreads, 1)
    lloyd_hist_kernel(const uint16_t* __restrict__ w, int64_t n_blocks, const __grid_constant__ LloydParams p,
                      uint32_t* __restrict__ counts, int32_t* __restrict__ slot_e, double* __restrict__ side,
                      int32_t* status) {
  extern __shared__ uint32_t cnt[];  // [kLloydSlots][n_bins]
  __shared__ int e0_s;
  const int nb = p.n_bins;
  for (int i = threadIdx.x; i < kLloydSlots * nb; i += blockDim.x) cnt[i] = 0u;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t n_groups = (n_blocks + 7) / 8;  // 8 blocks per group
  uint32_t gbits;
  {
    const float g = (float)p.gmax;
    gbits = __float_as_uint(g);
  }
  // the slots are centred on the exponent of the CTA's first block
  if (threadIdx.x == 0) {
    const int64_t blk = (int64_t)blockIdx.x * (blockDim.x >> 5) * 8;
    uint32_t amx = 0u;
    if (blk < n_blocks)
      for (int i = 0; i < 32; ++i) {
        const uint32_t m = w[blk * 32 + i] & 0x7fffu;
        if (m < 0x7f80u) amx = max(amx, m);
      }
    e0_s = lloyd_block_exponent_bits(amx, gbits, p.gmax);
  }
  __syncthreads();
  const int e0 = e0_s;
  bool bad = false, over = false;
  for (int64_t g0 = gw; g0 < n_groups; g0 += warps * kLloydUnroll) {
    uint4 v[kLloydUnroll];
#pragma unroll
    for (int u = 0; u < kLloydUnroll; ++u) {
      const int64_t blk = (g0 + u * warps) * 8 + (lane >> 2);
      v[u] = blk < n_blocks ? ldg_stream(w + blk * 32 + (lane & 3) * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kLloydUnroll; ++u) {
      const int64_t blk = (g0 + u * warps) * 8 + (lane >> 2);
      const uint32_t wd[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      // block amax over the 4 lanes of the block (bf16 magnitudes compare as integers)
      uint32_t amx = 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t lo = wd[q] & 0x7fffu, hi = (wd[q] >> 16) & 0x7fffu;
        if (lo >= 0x7f80u || hi >= 0x7f80u) bad = true;  // Inf or NaN
        amx = max(amx, max(lo, hi));
      }
      amx = max(amx, __shfl_xor_sync(0xffffffffu, amx, 1));
      amx = max(amx, __shfl_xor_sync(0xffffffffu, amx, 2));
      if (blk >= n_blocks) continue;
      const int e = lloyd_block_exponent_bits(amx, gbits, p.gmax);
      const int slot = e - e0 + 1;
      const bool in_slot = (unsigned)slot < (unsigned)kLloydSlots;
      uint32_t* c = cnt + (in_slot ? slot : 0) * nb;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t m = (wd[q >> 1] >> (16 * (q & 1))) & 0x7fffu;
        if (m >= 0x7f80u) continue;
        const uint32_t rb = lloyd_ratio_bits(m, e);
        if (rb >= (uint32_t)nb) {
          over = true;  // a ratio above gmax: only with the exponent clamped at 127
          continue;
        }
        if (in_slot)
          atomicAdd(&c[rb], 1u);
        else
          atomicAdd(&side[rb], ldexp(1.0, 2 * e));
      }
    }
  }
  if (bad) record_error(status, MOE_Q4_EDEVICE);
  if (over) record_error(status, MOE_Q4_ENOTSUP);
  __syncthreads();
  // this CTA's slice: counts [slot][bin] and the slots' exponents
  uint32_t* mine = counts + (size_t)blockIdx.x * kLloydSlots * nb;
  for (int i = threadIdx.x; i < kLloydSlots * nb; i += blockDim.x) mine[i] = cnt[i];
  if (threadIdx.x < kLloydSlots) slot_e[blockIdx.x * kLloydSlots + threadIdx.x] = e0 - 1 + (int)threadIdx.x;
}

// W[r] = side[r] + sum over CTAs c (in order) and slots j (in order) of
// counts[c][j][r] * 4^slot_e[c][j], one thread per bin; the CTAs of every
// earlier call on the same workspace were added already (acc).
__global__ void __launch_bounds__(256) lloyd_sum_kernel(const uint32_t* __restrict__ counts,
                                                        const int32_t* __restrict__ slot_e, int n_cta, int nb,
                                                        double* __restrict__ W) {
  const int r = blockIdx.x * 256 + threadIdx.x;
  if (r >= nb) return;
  double acc = W[r];
  for (int c = 0; c < n_cta; ++c)
    for (int j = 0; j < kLloydSlots; ++j) {
      const uint32_t n = counts[((size_t)c * kLloydSlots + j) * nb + r];
      if (n) acc += (double)n * ldexp(1.0, 2 * slot_e[c * kLloydSlots + j]);
    }
  W[r] = acc;
}

// The Lloyd steps on the histogram, one CTA.
__global__ void __launch_bounds__(kLloydSolveThreads, 1)
    lloyd_solve_kernel(const double* __restrict__ hist, const __grid_constant__ LloydParams p, int max_iter,
                       double tol, float* grid, int32_t* iters) {
  __shared__ double lev[8];
  __shared__ double red[kLloydSolveThreads / 32][16];
  __shared__ int done;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < 8) lev[tid] = p.lev0[tid];
  if (tid == 0) done = 0;
  __syncthreads();
  int it = 0;
  while (it < max_iter) {
    double m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = lev[j];
    double sw[8], swr[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sw[j] = swr[j] = 0.0;
    for (int b = tid; b < p.n_bins; b += kLloydSolveThreads) {
      const double W = hist[b];
      if (W == 0.0) continue;
      const double r = (double)__uint_as_float((uint32_t)b << 16);
      int best = 0;
      double bd = fabs(r - m[0]);
#pragma unroll
      for (int j = 1; j < 8; ++j) {
        const double d = fabs(r - m[j]);
        if (d < bd) {
          bd = d;
          best = j;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j == best) {
          sw[j] += W;
          swr[j] += W * r;
        }
    }
    // fixed-order reduction: butterfly within the warp, then warps in order
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sw[j] += __shfl_xor_sync(0xffffffffu, sw[j], off);
        swr[j] += __shfl_xor_sync(0xffffffffu, swr[j], off);
      }
    }
    if (lane == 0)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        red[warp][j] = sw[j];
        red[warp][8 + j] = swr[j];
      }
    __syncthreads();
    if (tid == 0) {
      double moved = 0.0;
      for (int j = 0; j < 8; ++j) {
        double a = 0.0, c = 0.0;
        for (int q = 0; q < kLloydSolveThreads / 32; ++q) {
          a += red[q][j];
          c += red[q][8 + j];
        }
        if (a > 0.0) {
          const double nm = c / a;
          if (fabs(nm - lev[j]) > moved) moved = fabs(nm - lev[j]);
          lev[j] = nm;
        }
      }
      done = moved <= tol;
    }
    __syncthreads();
    ++it;
    if (done) break;
  }
  if (tid < 8) grid[tid] = (float)lev[tid];
  if (tid == 0) *iters = it;
}

}  // namespace q4

using namespace q4;

namespace {

// Starting grid: finite, >= 0 (no sign bit), strictly ascending, gmax < 16.
int lloyd_params(const float* grid0, LloydParams* p) {
  if (!grid0) return MOE_Q4_EINVAL;
  for (int i = 0; i < 8; ++i) {
    if (!isfinite(grid0[i]) || signbit(grid0[i])) return MOE_Q4_EINVAL;
    if (i > 0 && !(grid0[i] > grid0[i - 1])) return MOE_Q4_EINVAL;
    p->lev0[i] = (double)grid0[i];
  }
  p->gmax = (double)grid0[7];
  if (!(p->gmax > 0.0)) return MOE_Q4_EINVAL;
  uint32_t bits;
  memcpy(&bits, &grid0[7], 4);
  p->n_bins = (int)(bits >> 16) + 1;
  if (p->n_bins > kLloydMaxBins) return MOE_Q4_ENOTSUP;
  return MOE_Q4_OK;
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

// Workspace: status int32 (256 bytes) | W fp64[n_bins] (the weighted
// histogram, accumulated over calls) | per-CTA counts uint32[kLloydMaxCta][3]
// [n_bins] | their slots' exponents int32[kLloydMaxCta][3].
constexpr int kLloydMaxCta = 160;

struct LloydWs {
  size_t W, counts, slot_e, end;
};

static LloydWs lloyd_ws(int n_bins) {
  LloydWs o;
  o.W = 256;
  o.counts = o.W + align256(sizeof(double) * (size_t)n_bins);
  o.slot_e = o.counts + align256(sizeof(uint32_t) * (size_t)kLloydMaxCta * kLloydSlots * n_bins);
  o.end = o.slot_e + align256(sizeof(int32_t) * (size_t)kLloydMaxCta * kLloydSlots);
  return o;
}

extern "C" size_t moe_q4_lloyd_workspace(const float* grid0) {
  LloydParams p;
  if (lloyd_params(grid0, &p) != MOE_Q4_OK) return 0;
  return lloyd_ws(p.n_bins).end;
}

extern "C" int moe_q4_lloyd_hist(const void* w, long long n_blocks, const float* grid0, int reset, void* ws,
                                 size_t ws_bytes, void* stream) {
  LloydParams p;
  int rc = lloyd_params(grid0, &p);
  if (rc != MOE_Q4_OK) return rc;
  if (n_blocks < 0 || (n_blocks > 0 && (!w || ((uintptr_t)w & 15)))) return MOE_Q4_EINVAL;
  if (!ws || ((uintptr_t)ws & 255) || ws_bytes < moe_q4_lloyd_workspace(grid0)) return MOE_Q4_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const LloydWs o = lloyd_ws(p.n_bins);
  char* base = (char*)ws;
  double* W = (double*)(base + o.W);
  if (reset && cudaMemsetAsync(ws, 0, o.counts, s) != cudaSuccess) return MOE_Q4_ECUDA;
  if (n_blocks == 0) return MOE_Q4_OK;
  const size_t smem = sizeof(uint32_t) * kLloydSlots * (size_t)p.n_bins;
  if (cudaFuncSetAttribute(lloyd_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MOE_Q4_ECUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms > kLloydMaxCta) sms = kLloydMaxCta;
  const long long groups = (n_blocks + 7) / 8;
  const long long need = (groups + kLloydHistThreads / 32 - 1) / (kLloydHistThreads / 32);
  const int grid = (int)(need < sms ? need : sms);
  lloyd_hist_kernel<<<grid, kLloydHistThreads, smem, s>>>((const uint16_t*)w, (int64_t)n_blocks, p,
                                                          (uint32_t*)(base + o.counts), (int32_t*)(base + o.slot_e),
                                                          W, (int32_t*)ws);
  if (cudaGetLastError() != cudaSuccess) return MOE_Q4_ECUDA;
  lloyd_sum_kernel<<<(p.n_bins + 255) / 256, 256, 0, s>>>((const uint32_t*)(base + o.counts),
                                                          (const int32_t*)(base + o.slot_e), grid, p.n_bins, W);
  return cudaGetLastError() == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}

extern "C" int moe_q4_lloyd_solve(const float* grid0, int max_iter, double tol, float* grid, int32_t* iters,
                                  const void* ws, size_t ws_bytes, void* stream) {
  LloydParams p;
  int rc = lloyd_params(grid0, &p);
  if (rc != MOE_Q4_OK) return rc;
  if (max_iter < 0 || !(tol >= 0.0) || !grid || !iters) return MOE_Q4_EINVAL;
  if (!ws || ((uintptr_t)ws & 255) || ws_bytes < moe_q4_lloyd_workspace(grid0)) return MOE_Q4_EWORKSPACE;
  lloyd_solve_kernel<<<1, kLloydSolveThreads, 0, (cudaStream_t)stream>>>(
      (const double*)((const char*)ws + lloyd_ws(p.n_bins).W), p, max_iter, tol, grid, iters);
  return cudaGetLastError() == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}
