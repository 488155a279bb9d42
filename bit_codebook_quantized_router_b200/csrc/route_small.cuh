// Routing and grouping of a small batch (T <= 256 tokens) by one CTA:
// per token the top-k by logit (equal logits -> lower expert id) and the
// softmax over the k kept, then the (token, slot) rows grouped by expert:
// counts, exclusive-scan offsets, stable token order within an expert, the
// inverse map, the per-path expert lists and the tensor-core tile offsets.
// Expert geometry: "Round 7 -- Rewrite the GLM-5.2 routed-expert encoder",
// "Ground truth and corrections" (256 routed experts, top-8); rows per
// expert are the "route blocks" of "GLM-5.2 EXL3 TR3 v4" README, "Tuning:
// prefill route block size".  The pages give no router formula; the reading
// implemented is top-k then softmax over the k kept.
//
// A row's place within its expert is the number of earlier tokens that chose
// the same expert, read from a per-expert bitmask of tokens (a token picks an
// expert at most once, so token order is row order within an expert).  One
// packed scan over experts gives the offsets, both expert lists and the tile
// offsets; thread i owns experts [i*per, (i+1)*per), per = ceil(E / NTH).
// Every result is an integer or a per-token softmax: the same for any NTH.
#pragma once

#include "q4_api_internal.h"
#include "q4_common.cuh"

namespace q4 {

__device__ __forceinline__ void store_route(const FwdArgs& a, int t, int lane, int id, float w) {
  if (lane < a.k) {
    const int r = t * a.k + lane;
    a.ids[r] = id;
    a.w[r] = w;
    if (a.user_ids) a.user_ids[r] = id;
    if (a.user_w) a.user_w[r] = w;
  }
}

// Dynamic shared memory of route_small, in bytes.
__host__ __device__ inline size_t route_small_smem_bytes(int E, int T, int k) {
  return sizeof(int) * ((size_t)T * k + 2 * (size_t)E + (size_t)E * ((T + 31) / 32));
}

// One CTA of NTH threads (NTH a multiple of 32, at most 1024).
// Shared memory: ids[T*k] | counts[E] | offs[E] | tokmask[E][W], W = ceil(T/32).
// L2_ONLY: the logits were written by other CTAs of this grid.
template <int NTH, bool L2_ONLY>
__device__ void route_small(const FwdArgs& a, int* sm) {
  constexpr int NW = NTH / 32;
  const int E = a.E, T = a.T, k = a.k;
  const int W = (T + 31) >> 5;
  int* ids_s = sm;
  int* counts = ids_s + T * k;
  int* offs = counts + E;
  uint32_t* tokmask = reinterpret_cast<uint32_t*>(offs + E);
  __shared__ unsigned long long warp_tot[33];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += NTH) counts[e] = 0;
  for (int i = tid; i < E * W; i += NTH) tokmask[i] = 0u;
  if (tid == 0 && !a.keep_status) a.hdr[kStatus] = MOE_Q4_OK;
  // per-tile arrival counters of the small-M kernels start at zero every call
  for (int i = tid; i < a.dk_counter_n; i += NTH) a.dk_counter[i] = 0;
  __syncthreads();
  for (int t = warp; t < T; t += NW) {
    int id;
    float w;
    topk_warp<L2_ONLY>(a.logits + (size_t)t * E, E, k, lane, a.hdr + kStatus, id, w);
    store_route(a, t, lane, id, w);
    if (lane < k) {
      ids_s[t * k + lane] = id;
      if ((unsigned)id < (unsigned)E) {
        atomicAdd(&counts[id], 1);
        atomicOr(&tokmask[id * W + (t >> 5)], 1u << (t & 31));
      } else {
        record_error(a.hdr + kStatus, MOE_Q4_EDEVICE);
      }
    }
  }
  __syncthreads();
  // one exclusive scan over experts of five packed fields:
  //   rows [0,13) | small-M experts [13,23) | wide experts [23,33) |
  //   swap-AB experts [33,43) | their tiles [43,55)
  // (T*k <= 4096 rows, E <= 512 experts, tiles <= E + T*k/16: no field overflows)
  const int wmax = a.mid_list ? a.wide_max : a.dec_max;
  const auto pack = [&](int c) -> unsigned long long {
    const bool fd = c > 0 && c <= a.dec_max, fm = c > a.dec_max && c <= wmax, fp = c > wmax;
    const int ntl = fp ? (c + a.tile_n - 1) / a.tile_n : 0;
    return (unsigned long long)c | ((unsigned long long)(fd ? 1 : 0) << 13) |
           ((unsigned long long)(fm ? 1 : 0) << 23) | ((unsigned long long)(fp ? 1 : 0) << 33) |
           ((unsigned long long)ntl << 43);
  };
  const int per = (E + NTH - 1) / NTH;
  const int e0 = tid * per, e1 = e0 + per < E ? e0 + per : E;
  unsigned long long v = 0;
  for (int e = e0; e < e1; ++e) v += pack(counts[e]);
  unsigned long long inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const unsigned long long wv = lane < NW ? warp_tot[lane] : 0ull;
    unsigned long long winc = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long u = __shfl_up_sync(0xffffffffu, winc, o);
      if (lane >= o) winc += u;
    }
    warp_tot[lane] = winc - wv;
    if (lane == 31) warp_tot[32] = winc;
  }
  __syncthreads();
  unsigned long long ex = warp_tot[warp] + inc - v;
  const unsigned long long tot = warp_tot[32];
  const auto field = [](unsigned long long x, int lo, int bits) -> int {
    return (int)((x >> lo) & ((1ull << bits) - 1));
  };
  for (int e = e0; e < e1; ++e) {
    const int c = counts[e];
    const unsigned long long pe = pack(c);
    offs[e] = field(ex, 0, 13);
    a.offsets[e] = field(ex, 0, 13);
    a.counts[e] = c;
    if (a.user_counts) a.user_counts[e] = c;
    if (field(pe, 13, 10)) a.dec_list[field(ex, 13, 10)] = e;
    if (field(pe, 23, 10)) a.mid_list[field(ex, 23, 10)] = e;
    if (field(pe, 33, 10)) {
      a.pre_list[field(ex, 33, 10)] = e;
      if (a.tiles) a.tiles[field(ex, 33, 10)] = field(ex, 43, 12);
    }
    ex += pe;
  }
  if (tid == 0) {
    const int np = field(tot, 33, 10), ntot = field(tot, 43, 12);
    a.offsets[E] = field(tot, 0, 13);
    a.hdr[kNumDecode] = field(tot, 13, 10);
    a.hdr[kNumMid] = field(tot, 23, 10);
    a.hdr[kNumPrefill] = np;
    a.hdr[kNumTiles] = ntot;
    if (a.tiles) a.tiles[np] = ntot;
  }
  __syncthreads();
  // stable placement: rank of token t among the tokens that chose expert e
  for (int r = tid; r < T * k; r += NTH) {
    const int t = r / k, e = ids_s[r];
    if ((unsigned)e >= (unsigned)E) continue;
    const uint32_t* m = tokmask + e * W;
    int rank = __popc(m[t >> 5] & ((1u << (t & 31)) - 1u));
    for (int q = 0; q < (t >> 5); ++q) rank += __popc(m[q]);
    const int pos = offs[e] + rank;
    a.row_token[pos] = t;
    a.inv[r] = pos;
  }
}

}  // namespace q4
