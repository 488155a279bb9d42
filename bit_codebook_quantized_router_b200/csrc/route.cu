// Router top-k + softmax-over-k, and the grouping of (token, slot) rows by
// expert (counts, exclusive-scan offsets, stable token order, inverse map,
// per-path expert lists).
//
// Geometry: "Round 7 -- Rewrite the GLM-5.2 routed-expert encoder", "Ground
// truth and corrections" (256 routed experts, top-8).  Rows per expert form
// the "route blocks" of "GLM-5.2 EXL3 TR3 v4" README, "Tuning: prefill route
// block size".  The pages give no router formula; the reading implemented:
// top-k by logit (equal logits -> lower expert id), softmax over the k kept.
#include <math.h>

#include "q4_api_internal.h"
#include "q4_common.cuh"
#include "route_small.cuh"

namespace q4 {

constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kFusedMaxT = 256;  // above this, top-k runs on many CTAs first

// Block-wide exclusive scan of one value per thread (kRouteThreads threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int wv = warp_tot[lane];
    int winc = wv;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, winc, off);
      if (lane >= off) winc += o;
    }
    warp_tot[lane] = winc - wv;  // exclusive prefix of warp totals
    if (lane == 31) warp_tot[32] = winc;
  }
  __syncthreads();
  const int res = warp_tot[warp] + inc - v;
  total = warp_tot[32];
  __syncthreads();
  return res;
}

// Grouping by one CTA of kRouteThreads threads, ids already in a.ids.
// Shared memory: counts[E] | offs[E+1] | running[E] | mask[32][E] | pre[32][E].
__device__ void group_rows(const FwdArgs& a, int* sm) {
  const int E = a.E, T = a.T, k = a.k;
  int* counts = sm;
  int* offs = counts + E;
  int* running = offs + E + 1;
  int* mask = running + E;
  int* pre = mask + kRouteWarps * E;
  __shared__ int warp_tot[33];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += kRouteThreads) {
    counts[e] = 0;
    running[e] = 0;
  }
  // per-tile arrival counters of the small-M kernels start at zero every call
  for (int i = tid; i < a.dk_counter_n; i += kRouteThreads) a.dk_counter[i] = 0;
  __syncthreads();
  // ids come from topk_warp and are always < E; a value out of range would be
  // a library bug: record it and leave the row out rather than index past smem.
  for (int r = tid; r < T * k; r += kRouteThreads) {
    const int e = a.ids[r];
    if ((unsigned)e < (unsigned)E)
      atomicAdd(&counts[e], 1);
    else
      record_error(a.hdr + kStatus, MOE_Q4_EDEVICE);
  }
  __syncthreads();
  // offsets and per-path expert lists (E <= kRouteThreads)
  const int c = tid < E ? counts[tid] : 0;
  int total;
  const int off = block_exclusive_scan(c, warp_tot, total);
  const int wmax = a.mid_list ? a.wide_max : a.dec_max;
  const bool fd = c > 0 && c <= a.dec_max, fm = c > a.dec_max && c <= wmax, fp = c > wmax;
  int nd, nm, np;
  const int pd = block_exclusive_scan(fd ? 1 : 0, warp_tot, nd);
  const int pm = block_exclusive_scan(fm ? 1 : 0, warp_tot, nm);
  const int pp = block_exclusive_scan(fp ? 1 : 0, warp_tot, np);
  // token tiles of each tensor-core-path expert, as an exclusive scan in
  // pre_list order (tiles[p] .. tiles[p+1]-1 are expert pre_list[p]'s)
  int ntot;
  const int ntl = fp ? (c + a.tile_n - 1) / a.tile_n : 0;
  const int ntoff = block_exclusive_scan(ntl, warp_tot, ntot);
  if (tid < E) {
    offs[tid] = off;
    a.offsets[tid] = off;
    a.counts[tid] = c;
    if (a.user_counts) a.user_counts[tid] = c;
    if (fd) a.dec_list[pd] = tid;
    if (fm) a.mid_list[pm] = tid;
    if (fp) a.pre_list[pp] = tid;
    if (fp && a.tiles) a.tiles[pp] = ntoff;
  }
  if (tid == 0) {
    offs[E] = total;
    a.offsets[E] = total;
    a.hdr[kNumDecode] = nd;
    a.hdr[kNumMid] = nm;
    a.hdr[kNumPrefill] = np;
    a.hdr[kNumTiles] = ntot;
    if (a.tiles) a.tiles[np] = ntot;
  }
  __syncthreads();
  // stable placement, kRouteThreads tokens per round
  for (int base = 0; base < T; base += kRouteThreads) {
    for (int i = tid; i < kRouteWarps * E; i += kRouteThreads) mask[i] = 0;
    __syncthreads();
    const int t = base + tid;
    if (t < T)
      for (int j = 0; j < k; ++j) {
        const int e = a.ids[t * k + j];
        if ((unsigned)e < (unsigned)E) atomicOr(&mask[warp * E + e], 1 << lane);
      }
    __syncthreads();
    for (int e = tid; e < E; e += kRouteThreads) {
      int acc = running[e];
      for (int w2 = 0; w2 < kRouteWarps; ++w2) {
        pre[w2 * E + e] = acc;
        acc += __popc(mask[w2 * E + e]);
      }
      running[e] = acc;
    }
    __syncthreads();
    if (t < T) {
      const uint32_t below = (1u << lane) - 1u;
      for (int j = 0; j < k; ++j) {
        const int e = a.ids[t * k + j];
        if ((unsigned)e >= (unsigned)E) continue;
        const int pos = offs[e] + pre[warp * E + e] + __popc(mask[warp * E + e] & below);
        a.row_token[pos] = t;
        a.inv[t * k + j] = pos;
      }
    }
    __syncthreads();
  }
}

// Small T (<= kFusedMaxT): one CTA routes every token and groups
// (route_small, ids kept in shared memory).
__global__ void __launch_bounds__(kRouteThreads) route_fused_kernel(const __grid_constant__ FwdArgs a) {
  extern __shared__ int sm[];
  pdl_wait();
  // The next kernel may be scheduled now.  Its own wait still covers this
  // kernel's results; what it reads before that wait (the layer's inputs x
  // and logits, the weights) is complete once this kernel's wait returned.
  pdl_trigger();
  route_small<kRouteThreads, false>(a, sm);
}

// Large T: top-k on many CTAs (one warp per token; the host clears the
// status word before this launch) ...
__global__ void __launch_bounds__(256) route_topk_kernel(const __grid_constant__ FwdArgs a) {
  pdl_trigger();  // scheduling only: the next kernel's wait covers this one
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t < a.T) {
    int id;
    float w;
    topk_warp(a.logits + (size_t)t * a.E, a.E, a.k, lane, a.hdr + kStatus, id, w);
    store_route(a, t, lane, id, w);
  }
}

// ... then one CTA groups.
__global__ void __launch_bounds__(kRouteThreads) route_group_kernel(const __grid_constant__ FwdArgs a) {
  extern __shared__ int sm[];
  pdl_trigger();  // scheduling only: the next kernel's wait covers this one
  pdl_wait();
  group_rows(a, sm);
}

// Gather the activation rows in expert-grouped order for the tensor-core
// GEMMs (both paths read activations by TMA from contiguous rows):
// xg[row] = x[row_token[row]] for all T*k rows.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __grid_constant__ FwdArgs a) {
  pdl_trigger();  // scheduling only: the next kernel's wait covers this one
  pdl_wait();
  const int vec_per_row = a.H / 8;  // 16-byte vectors
  const int64_t n = (int64_t)a.T * a.k * vec_per_row;
  for (int64_t v = blockIdx.x * 256 + threadIdx.x; v < n; v += (int64_t)gridDim.x * 256) {
    const int r = (int)(v / vec_per_row);
    const int q = (int)(v % vec_per_row);
    if (!q4_check((unsigned)a.row_token[r] < (unsigned)a.T, a.hdr + kStatus)) continue;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)a.row_token[r] * a.H) + q;
    reinterpret_cast<uint4*>(a.xg + (size_t)r * a.H)[q] = *src;
  }
}

}  // namespace q4

using namespace q4;

static size_t group_smem_bytes(int E) { return sizeof(int) * ((size_t)3 * E + 1 + (size_t)2 * kRouteWarps * E); }

int q4_launch_route(const FwdArgs& a, cudaStream_t s) {
  const size_t smem = a.T <= kFusedMaxT ? route_small_smem_bytes(a.E, a.T, a.k) : group_smem_bytes(a.E);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.T <= kFusedMaxT) {
    if (cudaFuncSetAttribute(route_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOE_Q4_ECUDA;
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = smem;
    if (cudaLaunchKernelEx(&cfg, route_fused_kernel, a) != cudaSuccess) return MOE_Q4_ECUDA;
  } else {
    if (cudaFuncSetAttribute(route_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOE_Q4_ECUDA;
    if (!a.keep_status && cudaMemsetAsync(a.hdr + kStatus, 0, sizeof(int32_t), s) != cudaSuccess)
      return MOE_Q4_ECUDA;
    cfg.gridDim = dim3((a.T + 7) / 8);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    if (cudaLaunchKernelEx(&cfg, route_topk_kernel, a) != cudaSuccess) return MOE_Q4_ECUDA;
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = smem;
    if (cudaLaunchKernelEx(&cfg, route_group_kernel, a) != cudaSuccess) return MOE_Q4_ECUDA;
  }
  return MOE_Q4_OK;
}

int q4_launch_gather(const FwdArgs& a, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const long long vecs = (long long)a.T * a.k * (a.H / 8);
  const long long blocks = (vecs + 255) / 256;
  cfg.gridDim = dim3((unsigned)(blocks < 148 * 8 ? blocks : 148 * 8));
  cfg.blockDim = dim3(256);
  return cudaLaunchKernelEx(&cfg, gather_rows_kernel, a) == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}
