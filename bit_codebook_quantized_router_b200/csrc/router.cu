// Router logits: logits[t][e] = sum over h of x[t][h] * w[e][h] for bf16
// hidden states x [T][H] and the bf16 router gate w [E][H] (the "mlp.gate"
// linear that "GLM-5.2-EXL3-DENSE6-MTP78", "Quant recipe", holds in BF16),
// fp32 accumulation on the tensor cores (mma.sync m16n8k16).
//
// A warp computes 16 gate rows x 32 tokens over a range of K.  Per 32 K, lane
// (g, t) loads 16 bytes (8 bf16, K offsets 8t .. 8t + 7) of gate rows g and
// g + 8 and of token rows g, 8 + g, 16 + g, 24 + g; the two MMAs of the step
// take pairs 0, 1 and 2, 3 of those loads.  K is thereby permuted the same
// way for both operands (a sum over K does not depend on its order), and
// every load is a whole 16-byte run.  With few tokens the K range is split
// over warps so that every SM streams part of the gate; the partial sums are
// added afterwards in a fixed order, so the result does not depend on
// scheduling.
#include "q4_api_internal.h"
#include "q4_common.cuh"

namespace q4 {

namespace rt {
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kRows = 16;               // gate rows per warp unit (MMA M)
constexpr int kNT = 4;                  // 8-token MMA columns per warp unit
constexpr int kTokens = 8 * kNT;        // tokens per warp unit
constexpr int kKStep = 32;              // K per step: two MMAs per column tile
constexpr int kTargetWarps = 2 * 148 * kWarps;  // units aimed for before splitting K
}  // namespace rt

// How the work is cut: K split into `chunks` ranges of `steps` 32-K steps.
struct RouterPlan {
  int e_tiles, t_tiles, chunks, steps;
};

// With one token tile (decode sizes) each warp unit takes exactly kFewSteps
// steps of K, a compile-time count, so that all its loads are issued before
// its first MMA waits; the K range is then cut into H / (32 kFewSteps) chunks.
constexpr int kFewSteps = 4;

static bool router_few(int T, int H) { return T <= rt::kTokens && H % (rt::kKStep * kFewSteps) == 0; }

static RouterPlan router_plan(int T, int H, int E) {
  RouterPlan p;
  p.e_tiles = (E + rt::kRows - 1) / rt::kRows;
  p.t_tiles = (T + rt::kTokens - 1) / rt::kTokens;
  const int ksteps = H / rt::kKStep;
  if (router_few(T, H)) {
    p.steps = kFewSteps;
    p.chunks = ksteps / kFewSteps;
    return p;
  }
  const long long base = (long long)p.e_tiles * p.t_tiles;
  long long want = base > 0 ? rt::kTargetWarps / base : 1;
  if (want < 1) want = 1;
  if (want > ksteps) want = ksteps;
  p.steps = (int)((ksteps + want - 1) / want);
  p.chunks = (ksteps + p.steps - 1) / p.steps;
  return p;
}

// FEW: every unit takes exactly kFewSteps steps (plan.steps == kFewSteps).
template <bool FEW>
__global__ void __launch_bounds__(rt::kThreads) router_kernel(const uint16_t* __restrict__ x,
                                                              const uint16_t* __restrict__ w, int T, int H, int E,
                                                              RouterPlan plan, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const long long units = (long long)plan.e_tiles * plan.t_tiles * plan.chunks;
  const size_t TE = (size_t)T * E;
  for (long long u = (long long)blockIdx.x * rt::kWarps + (threadIdx.x >> 5); u < units;
       u += (long long)gridDim.x * rt::kWarps) {
    const int c = (int)(u % plan.chunks);
    const long long rest = u / plan.chunks;
    const int et = (int)(rest % plan.e_tiles), tt = (int)(rest / plan.e_tiles);
    const int e_a = et * rt::kRows + g, e_b = e_a + 8;
    const int k_begin = c * plan.steps * rt::kKStep;
    const int k_end = min(H, k_begin + plan.steps * rt::kKStep);
    // rows past E or T read row 0 (always valid); their results are not written
    const uint16_t* wa = w + (size_t)(e_a < E ? e_a : 0) * H + 8 * tq;
    const uint16_t* wb = w + (size_t)(e_b < E ? e_b : 0) * H + 8 * tq;
    const uint16_t* xr[rt::kNT];
#pragma unroll
    for (int nt = 0; nt < rt::kNT; ++nt) {
      const int t = tt * rt::kTokens + 8 * nt + g;
      xr[nt] = x + (size_t)(t < T ? t : 0) * H + 8 * tq;
    }
    float acc[rt::kNT][4];
#pragma unroll
    for (int nt = 0; nt < rt::kNT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
    if constexpr (FEW) {
      // all loads of the unit first, then the MMAs (one token tile: the x rows
      // of the four column tiles repeat, so only distinct rows are loaded)
      uint4 a[kFewSteps], b[kFewSteps], v[kFewSteps][rt::kNT];
#pragma unroll
      for (int j = 0; j < kFewSteps; ++j) {
        const int k = k_begin + j * rt::kKStep;
        a[j] = ldg_nc(wa + k);
        b[j] = ldg_nc(wb + k);
#pragma unroll
        for (int nt = 0; nt < rt::kNT; ++nt) v[j][nt] = ldg_nc(xr[nt] + k);
      }
#pragma unroll
      for (int j = 0; j < kFewSteps; ++j)
#pragma unroll
        for (int nt = 0; nt < rt::kNT; ++nt) {
          mma_16816(acc[nt], a[j].x, b[j].x, a[j].y, b[j].y, v[j][nt].x, v[j][nt].y);
          mma_16816(acc[nt], a[j].z, b[j].z, a[j].w, b[j].w, v[j][nt].z, v[j][nt].w);
        }
    } else {
#pragma unroll 4
      for (int k = k_begin; k < k_end; k += rt::kKStep) {
        const uint4 a = ldg_nc(wa + k), b = ldg_nc(wb + k);
#pragma unroll
        for (int nt = 0; nt < rt::kNT; ++nt) {
          const uint4 v = ldg_nc(xr[nt] + k);
          mma_16816(acc[nt], a.x, b.x, a.y, b.y, v.x, v.y);
          mma_16816(acc[nt], a.z, b.z, a.w, b.w, v.z, v.w);
        }
      }
    }
    // D fragment: rows g / g + 8 (gate rows e_a / e_b), columns 2 tq, 2 tq + 1
    float* dst = out + (plan.chunks > 1 ? (size_t)c * TE : 0);
#pragma unroll
    for (int nt = 0; nt < rt::kNT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = tt * rt::kTokens + 8 * nt + 2 * tq + (i & 1);
        const int e = (i >> 1) ? e_b : e_a;
        if (t < T && e < E) dst[(size_t)t * E + e] = acc[nt][i];
      }
  }
}

// logits = the chunks' partial sums, added in a fixed order: one thread per
// logit in chunk order, or (many chunks) one warp per logit, lane l adding
// chunks l, l + 32, ... and the lanes' sums combined by a fixed butterfly.
__global__ void router_reduce_kernel(const float* __restrict__ part, int chunks, size_t n, float* __restrict__ out) {
  if (chunks <= 8) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
      float s = 0.0f;
      for (int c = 0; c < chunks; ++c) s += part[(size_t)c * n + i];
      out[i] = s;
    }
    return;
  }
  const int lane = threadIdx.x & 31;
  const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
  for (size_t i = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < n; i += warps) {
    float s = 0.0f;
    for (int c = lane; c < chunks; c += 32) s += part[(size_t)c * n + i];
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
    if (lane == 0) out[i] = s;
  }
}

}  // namespace q4

using namespace q4;

static bool router_args_ok(int T, int H, int E) {
  return T >= 0 && H > 0 && E > 0 && H % rt::kKStep == 0 && (long long)T * H < (1ll << 40) &&
         (long long)T * E < (1ll << 31);
}

extern "C" size_t moe_q4_router_workspace(int T, int H, int E) {
  if (!router_args_ok(T, H, E) || T == 0) return 0;
  const RouterPlan p = router_plan(T, H, E);
  return p.chunks > 1 ? sizeof(float) * (size_t)p.chunks * T * E : 0;
}

extern "C" int moe_q4_router(const void* x, const void* w, int T, int H, int E, float* logits, void* ws,
                             size_t ws_bytes, void* stream) {
  if (!router_args_ok(T, H, E)) return MOE_Q4_EINVAL;
  if (T == 0) return MOE_Q4_OK;
  if (!x || !w || !logits) return MOE_Q4_EINVAL;
  if (((uintptr_t)x & 15) || ((uintptr_t)w & 15)) return MOE_Q4_EINVAL;
  const RouterPlan p = router_plan(T, H, E);
  const size_t need = moe_q4_router_workspace(T, H, E);
  if (need > 0 && (!ws || ws_bytes < need || ((uintptr_t)ws & 15))) return MOE_Q4_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const long long units = (long long)p.e_tiles * p.t_tiles * p.chunks;
  const long long want = (units + rt::kWarps - 1) / rt::kWarps;
  const int grid = (int)(want < 148 * 8 ? want : 148 * 8);
  float* dst = p.chunks > 1 ? reinterpret_cast<float*>(ws) : logits;
  if (router_few(T, H))
    router_kernel<true><<<grid, rt::kThreads, 0, s>>>(static_cast<const uint16_t*>(x),
                                                       static_cast<const uint16_t*>(w), T, H, E, p, dst);
  else
    router_kernel<false><<<grid, rt::kThreads, 0, s>>>(static_cast<const uint16_t*>(x),
                                                        static_cast<const uint16_t*>(w), T, H, E, p, dst);
  if (cudaGetLastError() != cudaSuccess) return MOE_Q4_ECUDA;
  if (p.chunks > 1) {
    const size_t n = (size_t)T * E;
    const size_t per_block = p.chunks <= 8 ? 256 : 8;  // logits per 256-thread block
    const size_t rgrid = (n + per_block - 1) / per_block;
    router_reduce_kernel<<<(int)(rgrid < 148 * 8 ? rgrid : 148 * 8), 256, 0, s>>>(dst, p.chunks, n, logits);
    if (cudaGetLastError() != cudaSuccess) return MOE_Q4_ECUDA;
  }
  return MOE_Q4_OK;
}
