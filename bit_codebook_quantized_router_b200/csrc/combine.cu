// Weighted combine of the routed experts' outputs back into token order:
//   out[t] = sum_{j=0..k-1} w[t][j] * y[inv[t][j]]
// ("GLM-5.2 EXL3 TR3 v4" README, "Shared residual rotations, private
// intermediate rotations": expert outputs are routing-weighted and summed
// back into the residual space), plus the shared expert's output when the
// layer has one.  Each output element is summed by one
// thread in slot order in fp32, then rounded to bf16: deterministic, no
// atomics.
#include <string.h>

#include "q4_api_internal.h"
#include "q4_common.cuh"

namespace q4 {

// BATCH (few tokens, where the combine is latency-bound): the slots are taken
// kCombineSlots per round, their row indices and weights loaded first and
// every y load of the round issued before the first one is used, so a thread
// waits for one round trip per round instead of two per slot.  Without BATCH
// (many tokens, bandwidth-bound) one slot at a time in fewer registers, so
// more CTAs stay resident.  Both add the same products in the same order.
constexpr int kCombineSlots = 8;
constexpr int kCombineBatchMaxT = 64;

template <bool BATCH>
__global__ void __launch_bounds__(256) combine_kernel(const __grid_constant__ FwdArgs a) {
  pdl_wait();
  pdl_trigger();
  const int n4 = (blockIdx.x * 256 + threadIdx.x) * 4;
  if (n4 >= a.H) return;
  const int k = a.k, R = a.T * a.k;
  int32_t* status = a.hdr ? a.hdr + kStatus : nullptr;
  for (int t = blockIdx.y; t < a.T; t += gridDim.y) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!BATCH) {
      for (int j = 0; j < k; ++j) {
        // (no inverse map: the rows are in (token, slot) order)
        const int r = a.inv ? a.inv[t * k + j] : t * k + j;
        const float wj = a.w[t * k + j];
        if (!q4_check((unsigned)r < (unsigned)R, status)) continue;
        const float4 v = *reinterpret_cast<const float4*>(a.y + (size_t)r * a.H + n4);
        acc.x = fmaf(wj, v.x, acc.x);
        acc.y = fmaf(wj, v.y, acc.y);
        acc.z = fmaf(wj, v.z, acc.z);
        acc.w = fmaf(wj, v.w, acc.w);
      }
    }
    for (int j0 = 0; BATCH && j0 < k; j0 += kCombineSlots) {
      int r[kCombineSlots];
      float wj[kCombineSlots];
#pragma unroll
      for (int u = 0; u < kCombineSlots; ++u) {
        const int j = j0 + u < k ? j0 + u : k - 1;
        // (no inverse map: the rows are in (token, slot) order)
        r[u] = a.inv ? a.inv[t * k + j] : t * k + j;
        wj[u] = a.w[t * k + j];
      }
      bool ok[kCombineSlots];
#pragma unroll
      for (int u = 0; u < kCombineSlots; ++u)
        ok[u] = j0 + u < k && q4_check((unsigned)r[u] < (unsigned)R, status);
      float4 v[kCombineSlots];
#pragma unroll
      for (int u = 0; u < kCombineSlots; ++u)
        if (ok[u]) v[u] = *reinterpret_cast<const float4*>(a.y + (size_t)r[u] * a.H + n4);
      // slot order, one fmaf per slot: the same sum as taking the slots one by one
#pragma unroll
      for (int u = 0; u < kCombineSlots; ++u)
        if (ok[u]) {
          acc.x = fmaf(wj[u], v[u].x, acc.x);
          acc.y = fmaf(wj[u], v[u].y, acc.y);
          acc.z = fmaf(wj[u], v[u].z, acc.z);
          acc.w = fmaf(wj[u], v[u].w, acc.w);
        }
    }
    if (a.y_s) {
      // the shared expert's output, weight 1, after the routed slots
      const float4 v = *reinterpret_cast<const float4*>(a.y_s + (size_t)t * a.H + n4);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if (a.out_f32) *reinterpret_cast<float4*>(a.out_f32 + (size_t)t * a.H + n4) = acc;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(a.out + (size_t)t * a.H + n4) = pk;
  }
}

}  // namespace q4

using namespace q4;

int q4_launch_combine(const FwdArgs& a, cudaStream_t s) {
  if (a.T == 0) return MOE_Q4_OK;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.H / 4 + 255) / 256, a.T < 65535 ? a.T : 65535);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = a.T <= kCombineBatchMaxT ? cudaLaunchKernelEx(&cfg, combine_kernel<true>, a)
                                                 : cudaLaunchKernelEx(&cfg, combine_kernel<false>, a);
  return e == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}

// The combine alone: y fp32 [T*k][H] (rows in (token, slot) order, or placed
// by inv), w fp32 [T][k] -> out bf16 [T][H] and optionally out_f32.
extern "C" int moe_q4_combine(const float* y, const float* w, const int32_t* inv, int T, int k, int H, void* out,
                              float* out_f32, void* stream) {
  if (T < 0 || k < 1 || k > MOE_Q4_MAX_TOPK || H <= 0 || H % 4) return MOE_Q4_EINVAL;
  if (T == 0) return MOE_Q4_OK;
  if (!y || !w || !out || ((uintptr_t)y & 15) || ((uintptr_t)out & 7) || ((uintptr_t)out_f32 & 15) ||
      ((uintptr_t)w & 3))
    return MOE_Q4_EINVAL;
  FwdArgs a;
  memset(&a, 0, sizeof a);
  a.T = T;
  a.k = k;
  a.H = H;
  a.y = const_cast<float*>(y);
  a.w = const_cast<float*>(w);
  a.inv = const_cast<int32_t*>(inv);
  a.out = (__nv_bfloat16*)out;
  a.out_f32 = out_f32;
  return q4_launch_combine(a, (cudaStream_t)stream);
}
