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
constexpr int kFusedMaxT = 256;  // above this, the chunked three-kernel grouping

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

// Large T: chunks of kChunkT tokens.
// (1) route_topk_kernel, one warp per token (8 tokens per CTA, the host clears
//     the status word and chunk_cnt before it): top-k of each token, and each
//     chosen expert's row count in the token's chunk (global atomics);
// (2) route_scan_kernel, one CTA: each expert's rows over all chunks, the
//     exclusive-scan offsets, the per-path expert lists and tile offsets, and
//     every chunk's first row inside each expert (the rows of earlier chunks
//     come first: token order is row order within an expert);
// (3) route_place_kernel, one CTA per chunk: a row's place is its chunk's
//     base for the expert plus the number of earlier tokens of the chunk that
//     chose the expert (per-expert token bitmasks, as route_small).
// Every result is an integer: the same as one CTA grouping all rows.
constexpr int kChunkT = 256;
constexpr int kChunkThreads = 256;

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
    if (lane < a.k) {
      // ids come from topk_warp and are always < E; a value out of range
      // would be a library bug: record it and leave the row out
      if ((unsigned)id < (unsigned)a.E)
        atomicAdd(a.chunk_cnt + (size_t)(t / kChunkT) * a.E + id, 1);
      else
        record_error(a.hdr + kStatus, MOE_Q4_EDEVICE);
    }
  }
}

__global__ void __launch_bounds__(kRouteThreads) route_scan_kernel(const __grid_constant__ FwdArgs a,
                                                                    int n_chunks) {
  __shared__ int warp_tot[33];
  pdl_trigger();  // scheduling only: the next kernel's wait covers this one
  pdl_wait();
  const int E = a.E, tid = threadIdx.x;
  // per-tile arrival counters of the small-M kernels start at zero every call
  for (int i = tid; i < a.dk_counter_n; i += kRouteThreads) a.dk_counter[i] = 0;
  int c = 0;
  if (tid < E) {
#pragma unroll 4
    for (int ch = 0; ch < n_chunks; ++ch) c += a.chunk_cnt[(size_t)ch * E + tid];
  }
  // offsets and per-path expert lists (E <= kRouteThreads)
  int total;
  const int off = block_exclusive_scan(c, warp_tot, total);
  const int wmax = a.mid_list ? a.wide_max : a.dec_max;
  const bool fd = c > 0 && c <= a.dec_max, fm = c > a.dec_max && c <= wmax, fp = c > wmax;
  int nd, nm, np;
  const int pd = block_exclusive_scan(fd ? 1 : 0, warp_tot, nd);
  const int pm = block_exclusive_scan(fm ? 1 : 0, warp_tot, nm);
  const int pp = block_exclusive_scan(fp ? 1 : 0, warp_tot, np);
  // token tiles of each swap-AB expert, as an exclusive scan in pre_list order
  int ntot;
  const int ntl = fp ? (c + a.tile_n - 1) / a.tile_n : 0;
  const int ntoff = block_exclusive_scan(ntl, warp_tot, ntot);
  if (tid < E) {
    a.offsets[tid] = off;
    a.counts[tid] = c;
    if (a.user_counts) a.user_counts[tid] = c;
    if (fd) a.dec_list[pd] = tid;
    if (fm) a.mid_list[pm] = tid;
    if (fp) a.pre_list[pp] = tid;
    if (fp && a.tiles) a.tiles[pp] = ntoff;
    // each chunk's first row inside this expert
    int run = off;
    for (int ch = 0; ch < n_chunks; ++ch) {
      const size_t i = (size_t)ch * E + tid;
      const int n = a.chunk_cnt[i];
      a.chunk_base[i] = run;
      run += n;
    }
  }
  if (tid == 0) {
    a.offsets[E] = total;
    a.hdr[kNumDecode] = nd;
    a.hdr[kNumMid] = nm;
    a.hdr[kNumPrefill] = np;
    a.hdr[kNumTiles] = ntot;
    if (a.tiles) a.tiles[np] = ntot;
  }
}

__global__ void __launch_bounds__(kChunkThreads) route_place_kernel(const __grid_constant__ FwdArgs a) {
  extern __shared__ uint32_t tokmask[];  // [E][kChunkT / 32]
  constexpr int W = kChunkT / 32;
  pdl_trigger();  // scheduling only: the next kernel's wait covers this one
  pdl_wait();
  const int E = a.E, k = a.k;
  const int t0 = blockIdx.x * kChunkT, t1 = t0 + kChunkT < a.T ? t0 + kChunkT : a.T;
  const int n_rows = (t1 - t0) * k;
  for (int i = threadIdx.x; i < E * W; i += kChunkThreads) tokmask[i] = 0u;
  __syncthreads();
  for (int r = threadIdx.x; r < n_rows; r += kChunkThreads) {
    const int lt = r / k, e = a.ids[(size_t)t0 * k + r];
    if ((unsigned)e < (unsigned)E) atomicOr(&tokmask[e * W + (lt >> 5)], 1u << (lt & 31));
  }
  __syncthreads();
  const int32_t* base = a.chunk_base + (size_t)blockIdx.x * E;
  for (int r = threadIdx.x; r < n_rows; r += kChunkThreads) {
    const int lt = r / k, e = a.ids[(size_t)t0 * k + r];
    if ((unsigned)e >= (unsigned)E) continue;
    const uint32_t* m = tokmask + e * W;
    int rank = __popc(m[lt >> 5] & ((1u << (lt & 31)) - 1u));
    for (int q = 0; q < (lt >> 5); ++q) rank += __popc(m[q]);
    const int pos = base[e] + rank;
    if (!q4_check((unsigned)pos < (unsigned)(a.T * k), a.hdr + kStatus)) continue;
    a.row_token[pos] = t0 + lt;
    a.inv[(size_t)t0 * k + r] = pos;
  }
}

// Gather the activation rows in expert-grouped order for the tensor-core
// GEMMs (both paths read activations by TMA from contiguous rows):
// xg[row] = x[row_token[row]] for all T*k rows, taken token by token: each
// 16-byte vector of x[t] is read once and stored to the k grouped rows
// inv[t][0..k-1] (a row-ordered gather would read every x row k times).
__global__ void __launch_bounds__(256) gather_rows_kernel(const __grid_constant__ FwdArgs a) {
  pdl_trigger();  // scheduling only: the next kernel's wait covers this one
  pdl_wait();
  const int vec_per_row = a.H / 8;  // 16-byte vectors
  const int k = a.k, R = a.T * a.k;
  const int64_t n = (int64_t)a.T * vec_per_row;
  const uint4* x = reinterpret_cast<const uint4*>(a.x);
  uint4* xg = reinterpret_cast<uint4*>(a.xg);
  for (int64_t v = blockIdx.x * 256 + threadIdx.x; v < n; v += (int64_t)gridDim.x * 256) {
    const int t = (int)(v / vec_per_row);
    const int q = (int)(v % vec_per_row);
    const uint4 val = x[v];
    for (int j = 0; j < k; ++j) {
      const int pos = a.inv[t * k + j];
      if (q4_check((unsigned)pos < (unsigned)R, a.hdr + kStatus)) xg[(size_t)pos * vec_per_row + q] = val;
    }
  }
}

}  // namespace q4

using namespace q4;

int q4_route_chunks(int T) { return T > kFusedMaxT ? (T + kChunkT - 1) / kChunkT : 0; }

int q4_launch_route(const FwdArgs& a, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.T <= kFusedMaxT) {
    const size_t smem = route_small_smem_bytes(a.E, a.T, a.k);
    if (cudaFuncSetAttribute(route_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOE_Q4_ECUDA;
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = smem;
    return cudaLaunchKernelEx(&cfg, route_fused_kernel, a) == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
  }
  if (!a.chunk_cnt || !a.chunk_base) return MOE_Q4_ECUDA;
  if (!a.keep_status && cudaMemsetAsync(a.hdr + kStatus, 0, sizeof(int32_t), s) != cudaSuccess)
    return MOE_Q4_ECUDA;
  const int n_chunks = q4_route_chunks(a.T);
  if (cudaMemsetAsync(a.chunk_cnt, 0, sizeof(int32_t) * (size_t)n_chunks * a.E, s) != cudaSuccess)
    return MOE_Q4_ECUDA;
  cfg.gridDim = dim3((a.T + 7) / 8);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  if (cudaLaunchKernelEx(&cfg, route_topk_kernel, a) != cudaSuccess) return MOE_Q4_ECUDA;
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = 0;
  if (cudaLaunchKernelEx(&cfg, route_scan_kernel, a, n_chunks) != cudaSuccess) return MOE_Q4_ECUDA;
  cfg.gridDim = dim3(n_chunks);
  cfg.blockDim = dim3(kChunkThreads);
  cfg.dynamicSmemBytes = sizeof(uint32_t) * (size_t)a.E * (kChunkT / 32);
  return cudaLaunchKernelEx(&cfg, route_place_kernel, a) == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}

int q4_launch_gather(const FwdArgs& a, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const long long vecs = (long long)a.T * (a.H / 8);
  const long long blocks = (vecs + 255) / 256;
  cfg.gridDim = dim3((unsigned)(blocks < 148 * 8 ? blocks : 148 * 8));
  cfg.blockDim = dim3(256);
  return cudaLaunchKernelEx(&cfg, gather_rows_kernel, a) == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}
