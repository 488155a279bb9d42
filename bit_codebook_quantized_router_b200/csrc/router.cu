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
#include <cooperative_groups.h>

#include "q4_api_internal.h"
#include "q4_common.cuh"
#include "route_small.cuh"

namespace cg = cooperative_groups;

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

// One warp unit's loads and MMAs over `steps` 32-K steps from k_begin:
// acc[nt] (16 gate rows x 8 tokens each) += w[rows] . x[tokens]^T.
// FEW_STEPS > 0: exactly that many steps, all loads issued before the first
// MMA, and only the first NT 8-token column tiles (the tokens present).
template <int FEW_STEPS, int NT = rt::kNT>
__device__ __forceinline__ void router_unit(const uint16_t* wa, const uint16_t* wb, const uint16_t* const xr[rt::kNT],
                                            int k_begin, int k_end, float acc[rt::kNT][4]) {
  if constexpr (FEW_STEPS > 0) {
    uint4 a[FEW_STEPS], b[FEW_STEPS], v[FEW_STEPS][NT];
#pragma unroll
    for (int j = 0; j < FEW_STEPS; ++j) {
      const int k = k_begin + j * rt::kKStep;
      a[j] = ldg_nc(wa + k);
      b[j] = ldg_nc(wb + k);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) v[j][nt] = ldg_nc(xr[nt] + k);
    }
#pragma unroll
    for (int j = 0; j < FEW_STEPS; ++j)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
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
}

// General sizes: one warp per (gate tile, token tile, K chunk) unit; with
// more than one chunk the partial sums go to the workspace for
// router_reduce_kernel.
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
    router_unit<0>(wa, wb, xr, k_begin, k_end, acc);
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

// Decode sizes (one token tile, H a multiple of 32 kFewSteps): one kernel,
// NT = ceil(T / 8) column tiles computed (the others stay zero).
// A cluster of C CTAs owns one 16-row gate tile; warp w of cluster rank r
// takes the K chunks w C + r, w C + r + 8 C, ...  Each CTA adds its warps'
// partial tiles in warp order in shared memory; after a cluster barrier rank
// r finishes logits [r 512 / C, (r + 1) 512 / C) of the tile's 16 x 32,
// adding the C CTA sums in rank order through distributed shared memory.  The order of every sum is
// fixed by (H, C), so the result does not depend on scheduling.
template <int NT>
__device__ __forceinline__ void router_few_body(const uint16_t* __restrict__ x, const uint16_t* __restrict__ w, int T,
                                                int H, int E, int chunks, float* __restrict__ logits) {
  constexpr int kTile = rt::kRows * rt::kTokens;  // 512 logits: [gate row][token]
  __shared__ float part[rt::kWarps][kTile];
  __shared__ float cta_sum[kTile];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int et = blockIdx.x / C;
  const int e_a = et * rt::kRows + g, e_b = e_a + 8;
  const uint16_t* wa = w + (size_t)(e_a < E ? e_a : 0) * H + 8 * tq;
  const uint16_t* wb = w + (size_t)(e_b < E ? e_b : 0) * H + 8 * tq;
  const uint16_t* xr[rt::kNT];
#pragma unroll
  for (int nt = 0; nt < rt::kNT; ++nt) {
    const int t = 8 * nt + g;
    xr[nt] = x + (size_t)(t < T ? t : 0) * H + 8 * tq;
  }
  float acc[rt::kNT][4];
#pragma unroll
  for (int nt = 0; nt < rt::kNT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
  for (int c = warp * C + rank; c < chunks; c += rt::kWarps * C) {
    const int k0 = c * kFewSteps * rt::kKStep;
    router_unit<kFewSteps, NT>(wa, wb, xr, k0, k0 + kFewSteps * rt::kKStep, acc);
  }
#pragma unroll
  for (int nt = 0; nt < rt::kNT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = g + 8 * (i >> 1), t = 8 * nt + 2 * tq + (i & 1);
      part[warp][row * rt::kTokens + t] = acc[nt][i];
    }
  __syncthreads();
  for (int i = threadIdx.x; i < kTile; i += rt::kThreads) {
    float s = 0.0f;
#pragma unroll
    for (int q = 0; q < rt::kWarps; ++q) s += part[q][i];
    cta_sum[i] = s;
  }
  cluster.sync();  // every CTA's sums are complete and visible cluster-wide
  const int lo = rank * kTile / C, hi = (rank + 1) * kTile / C;
  for (int i = lo + threadIdx.x; i < hi; i += rt::kThreads) {
    const int row = i / rt::kTokens, t = i % rt::kTokens;
    const int e = et * rt::kRows + row;
    float s = 0.0f;
    for (int q = 0; q < C; ++q) s += *cluster.map_shared_rank(&cta_sum[i], q);
    if (t < T && e < E) logits[(size_t)t * E + e] = s;
  }
  cluster.sync();  // no CTA leaves while another still reads its shared memory
}

template <int NT>
__global__ void __launch_bounds__(rt::kThreads, 1) router_few_kernel(const uint16_t* __restrict__ x,
                                                                  const uint16_t* __restrict__ w, int T, int H, int E,
                                                                  int chunks, float* __restrict__ logits) {
  router_few_body<NT>(x, w, T, H, E, chunks, logits);
}

// The same with the routing fused behind it ("GLM-5.2-EXL3-DENSE6-MTP78",
// "Quant recipe": the BF16 mlp.gate in front of the routed experts): every
// CTA writes its share of the logits, makes it visible device-wide and takes
// a ticket; the CTA holding the last ticket (no CTA waits for another) reads
// all the logits through L2 and routes and groups the T tokens (route_small),
// then clears the ticket for the next call.  One launch from hidden states
// to the grouped rows; the logits stay in L2.
template <int NT>
__global__ void __launch_bounds__(rt::kThreads, 1) router_route_kernel(const __grid_constant__ FwdArgs a,
                                                                    const uint16_t* __restrict__ w, int chunks) {
  extern __shared__ int route_sm[];
  __shared__ int last;
  pdl_trigger();  // scheduling only: the next kernel's wait covers this whole grid
  router_few_body<NT>(reinterpret_cast<const uint16_t*>(a.x), w, a.T, a.H, a.E, chunks, const_cast<float*>(a.logits));
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(a.hdr + kRouterTicket, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  route_small<rt::kThreads, true>(a, route_sm);
  if (threadIdx.x == 0) a.hdr[kRouterTicket] = 0;
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

// Cluster size of the decode-size kernel: just enough CTAs for one K chunk
// per warp (8 at most, the portable limit; beyond that warps loop).  Sizes
// that are not powers of two keep the cluster count of a 256-expert gate
// (16 clusters) within what the GPU holds at once: clusters of 8 fit only 15
// times on 148 SMs, and a 16th would run as a second wave.
static int router_few_cluster(int chunks) {
  const int c = (chunks + rt::kWarps - 1) / rt::kWarps;
  return c < 1 ? 1 : (c > 8 ? 8 : c);
}

// Above the decode sizes, with E a multiple of 128 and H of 64, the gate runs
// as a dense GEMM on the tensor cores (q4_launch_dense: tcgen05, fp32
// accumulators in TMEM, K split over the SMs when there are few token tiles,
// the split partial sums added in a fixed order).  Its workspace: a status
// word (256 bytes) then the split partial sums.
static bool router_dense(int T, int H, int E) { return !router_few(T, H) && T > 32 && E % 128 == 0 && H % 64 == 0; }

size_t q4_router_partial_bytes(int T, int H, int E) {
  if (T == 0 || router_few(T, H)) return 0;
  if (router_dense(T, H, E)) return q4_dense_partial_bytes(T, E, H, 1);
  const RouterPlan p = router_plan(T, H, E);
  return p.chunks > 1 ? sizeof(float) * (size_t)p.chunks * T * E : 0;
}

// Cluster launch of a decode-size kernel over the gate tiles.
template <typename... Args>
static cudaError_t launch_few(void (*kern)(Args...), const RouterPlan& p, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  const int C = router_few_cluster(p.chunks);
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.e_tiles * C);
  cfg.blockDim = dim3(rt::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

int q4_launch_router(const void* x, const void* w, int T, int H, int E, float* logits, void* part, int32_t* status,
                     cudaStream_t s) {
  if (T == 0) return MOE_Q4_OK;
  const RouterPlan p = router_plan(T, H, E);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  const uint16_t* wb = static_cast<const uint16_t*>(w);
  if (router_few(T, H)) {
    const int nt = (T + 7) / 8;
    cudaError_t e;
    if (nt == 1)
      e = launch_few(router_few_kernel<1>, p, 0, s, xb, wb, T, H, E, p.chunks, logits);
    else if (nt == 2)
      e = launch_few(router_few_kernel<2>, p, 0, s, xb, wb, T, H, E, p.chunks, logits);
    else if (nt == 3)
      e = launch_few(router_few_kernel<3>, p, 0, s, xb, wb, T, H, E, p.chunks, logits);
    else
      e = launch_few(router_few_kernel<4>, p, 0, s, xb, wb, T, H, E, p.chunks, logits);
    return e == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
  }
  if (router_dense(T, H, E))
    return q4_launch_dense(w, 1, 0, E, H, x, T, nullptr, logits, E, static_cast<float*>(part), status, s);
  const long long units = (long long)p.e_tiles * p.t_tiles * p.chunks;
  const long long want = (units + rt::kWarps - 1) / rt::kWarps;
  const int grid = (int)(want < 148 * 8 ? want : 148 * 8);
  float* dst = p.chunks > 1 ? static_cast<float*>(part) : logits;
  router_kernel<<<grid, rt::kThreads, 0, s>>>(xb, wb, T, H, E, p, dst);
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

bool q4_router_route_fused(int T, int H, int k) { return T >= 1 && router_few(T, H) && T * k <= 4096; }

int q4_launch_router_route(const FwdArgs& a, const void* w, cudaStream_t s) {
  const RouterPlan p = router_plan(a.T, a.H, a.E);
  const size_t smem = route_small_smem_bytes(a.E, a.T, a.k);
  const uint16_t* wb = static_cast<const uint16_t*>(w);
  const int nt = (a.T + 7) / 8;
  cudaError_t e;
  if (nt == 1)
    e = launch_few(router_route_kernel<1>, p, smem, s, a, wb, p.chunks);
  else if (nt == 2)
    e = launch_few(router_route_kernel<2>, p, smem, s, a, wb, p.chunks);
  else if (nt == 3)
    e = launch_few(router_route_kernel<3>, p, smem, s, a, wb, p.chunks);
  else
    e = launch_few(router_route_kernel<4>, p, smem, s, a, wb, p.chunks);
  return e == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}

extern "C" size_t moe_q4_router_workspace(int T, int H, int E) {
  if (!router_args_ok(T, H, E) || T == 0 || router_few(T, H)) return 0;
  const size_t part = q4_router_partial_bytes(T, H, E);
  return router_dense(T, H, E) ? 256 + part : part;
}

extern "C" int moe_q4_router(const void* x, const void* w, int T, int H, int E, float* logits, void* ws,
                             size_t ws_bytes, void* stream) {
  if (!router_args_ok(T, H, E)) return MOE_Q4_EINVAL;
  if (T == 0) return MOE_Q4_OK;
  if (!x || !w || !logits) return MOE_Q4_EINVAL;
  if (((uintptr_t)x & 15) || ((uintptr_t)w & 15)) return MOE_Q4_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t need = moe_q4_router_workspace(T, H, E);
  if (need > 0 && (!ws || ws_bytes < need || ((uintptr_t)ws & 15))) return MOE_Q4_EWORKSPACE;
  if (router_dense(T, H, E)) {
    // the dense GEMM's status word at the workspace start, its partial sums after it
    if ((uintptr_t)ws & 255) return MOE_Q4_EWORKSPACE;
    int32_t* status = reinterpret_cast<int32_t*>(ws);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_Q4_ECUDA;
    void* part = need > 256 ? reinterpret_cast<char*>(ws) + 256 : nullptr;
    return q4_launch_router(x, w, T, H, E, logits, part, status, s);
  }
  return q4_launch_router(x, w, T, H, E, logits, ws, nullptr, s);
}
