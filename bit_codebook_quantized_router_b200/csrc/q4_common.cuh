// Device-side building blocks shared by the moe_q4 kernels (sm_100a).
//
// Weight format ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", "Contents",
// "Codes are indices into the per-layer grid -- not E2M1"): 4-bit codes,
// low nibble = even K, code & 7 indexes an 8-entry magnitude table, code & 8
// is the sign, one E8M0 byte per 32 weights along K scales by 2^(s - 127).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "moe_q4.h"

namespace q4 {

constexpr int kBlockK = 32;          // weights per E8M0 scale byte
constexpr int kMaxTables = MOE_Q4_MAX_TABLES;
constexpr int kMaxExperts = MOE_Q4_MAX_EXPERTS;
constexpr int kMaxTopK = MOE_Q4_MAX_TOPK;

// Magnitude tables and the per-expert table id, passed by value to kernels
// (read once per CTA from the constant parameter bank).
struct TableParams {
  float t[kMaxTables][8];
  uint8_t id[kMaxExperts];
  int n;
};

// Workspace header words (int32, at the start of the workspace).
enum HeaderWord : int {
  kStatus = 0,     // MOE_Q4_OK or the first error code recorded
  kNumDecode = 1,  // experts on the small-M streaming path
  kNumPrefill = 2, // experts on the tensor-core path
  kNumTiles = 3,   // tensor-core path work tiles
  kRouterTicket = 4,  // CTAs of the fused router + routing kernel done with their logits
  kNumMid = 5,     // experts on the wide tensor-core kernel
  kHeaderWords = 64,
};

__device__ __forceinline__ void record_error(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

// Device-side index check of the debug build (MOE_Q4_DEBUG): true when `ok`;
// else records MOE_Q4_EBOUNDS and the caller skips the access.  The release
// build compiles it to `true`.
#ifdef MOE_Q4_DEBUG
__device__ __forceinline__ bool q4_check(bool ok, int32_t* status) {
  if (!ok) record_error(status, MOE_Q4_EBOUNDS);
  return ok;
}
#else
__device__ __forceinline__ constexpr bool q4_check(bool, int32_t*) { return true; }
#endif

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

// The 8 table levels, rounded to bf16, split into byte planes so that one
// PRMT looks up four codes: l0/l1 hold the low bytes of levels 0-3 / 4-7,
// h0/h1 the high bytes (sign bit clear: magnitudes are >= 0).
struct Planes {
  uint32_t l0, l1, h0, h1;
};

__device__ __forceinline__ Planes make_planes(const float* t) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = bf16_bits_rn(t[i]);
  Planes p;
  p.l0 = (b[0] & 0xff) | ((b[1] & 0xff) << 8) | ((b[2] & 0xff) << 16) | ((b[3] & 0xff) << 24);
  p.l1 = (b[4] & 0xff) | ((b[5] & 0xff) << 8) | ((b[6] & 0xff) << 16) | ((b[7] & 0xff) << 24);
  p.h0 = (b[0] >> 8) | ((b[1] >> 8) << 8) | ((b[2] >> 8) << 16) | ((b[3] >> 8) << 24);
  p.h1 = (b[4] >> 8) | ((b[5] >> 8) << 8) | ((b[6] >> 8) << 16) | ((b[7] >> 8) << 24);
  return p;
}

// Decode one 32-bit word of packed codes (nibble i = K index i within the
// word, since the low nibble of each byte is the even K) into four bf16x2
// words: out[q] = (K 2q, K 2q+1), unscaled, sign applied.
//   m = w & 0x77777777 gives PRMT selectors 0..7 (byte index into a plane);
//   the sign of nibble i (bit 4i+3) is moved to bit 7 of the high byte by a
//   byte shuffle of (w << 4, w): bytes [ws.b0, w.b0, ws.b1, w.b1] carry the
//   signs of nibbles 0..3 in their top bits.
__device__ __forceinline__ void decode8(uint32_t w, const Planes& p, uint32_t out[4]) {
  const uint32_t m = w & 0x77777777u;
  const uint32_t mh = m >> 16;
  const uint32_t ws = w << 4;
  const uint32_t la = prmt(p.l0, p.l1, m);
  uint32_t ha = prmt(p.h0, p.h1, m);
  const uint32_t lb = prmt(p.l0, p.l1, mh);
  uint32_t hb = prmt(p.h0, p.h1, mh);
  ha |= prmt(ws, w, 0x5140) & 0x80808080u;
  hb |= prmt(ws, w, 0x7362) & 0x80808080u;
  out[0] = prmt(la, ha, 0x5140);
  out[1] = prmt(la, ha, 0x7362);
  out[2] = prmt(lb, hb, 0x5140);
  out[3] = prmt(lb, hb, 0x7362);
}

// bf16 bit pattern of 2^(s - 127) duplicated in both halves: s = 0 is the bf16
// subnormal 2^-127 (0x0040), s = 255 the E8M0 NaN (0x7FC0).
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t s) {
  uint32_t b = (s == 0u) ? 0x0040u : ((s == 255u) ? 0x7fc0u : (s << 7));
  return b | (b << 16);
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a);
  __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&b);
  __nv_bfloat162 z = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&z);
}

// D += A(16x16, bf16, row) * B(16x8, bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Streaming 16-byte load of packed weights (read once: no L1 allocation).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_nc(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ldg_u8(const uint8_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

// The same with the hardware approximations (__expf, and __fdividef, which
// returns 0 once 1 + e^-g overflows, as the exact form does in the limit):
// a few ulp of fp32, far below the bf16 rounding of h that follows.
__device__ __forceinline__ float silu_mul_fast(float g, float u) {
  return g * u * __fdividef(1.0f, 1.0f + __expf(-g));
}

constexpr int kMaxLogitsPerLane = kMaxExperts / 32;

// One warp routes one token: lane l holds logits of experts l, l+32, ...
// Each of the k rounds takes the best remaining (value, then lower id) by a
// warp argmax; lane j ends up holding slot j.  Non-finite logits are
// treated as -inf and recorded as a device error (unless status is null).
// L2_ONLY: read the logits through L2 only (ld.global.cg), for logits that
// other CTAs of the same grid wrote.
template <bool L2_ONLY = false>
__device__ __forceinline__ void topk_warp(const float* __restrict__ row, int E, int k, int lane,
                                          int32_t* status, int& my_id, float& my_w) {
  float v[kMaxLogitsPerLane];
  uint32_t avail = 0;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kMaxLogitsPerLane; ++i) {
    const int id = lane + 32 * i;
    v[i] = -INFINITY;
    if (id < E) {
      float x = L2_ONLY ? __ldcg(row + id) : row[id];
      if (!isfinite(x)) {
        bad = true;
        x = -INFINITY;
      }
      v[i] = x;
      avail |= 1u << i;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0 && status) record_error(status, MOE_Q4_EDEVICE);
  float mine = -INFINITY;
  my_id = -1;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < kMaxLogitsPerLane; ++i)
      if (((avail >> i) & 1u) && (bi < 0 || v[i] > bv)) {
        bv = v[i];
        bi = i;
      }
    int bid = bi < 0 ? 0x7fffffff : lane + 32 * bi;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oid = __shfl_xor_sync(0xffffffffu, bid, off);
      if (ov > bv || (ov == bv && oid < bid)) {
        bv = ov;
        bid = oid;
      }
    }
    if ((bid & 31) == lane) avail &= ~(1u << (bid >> 5));
    if (lane == j) {
      my_id = bid;
      mine = bv;
    }
  }
  const float m = __shfl_sync(0xffffffffu, mine, 0);
  float ex = (lane < k) ? expf(mine - m) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  my_w = ex / sum;
}

// Programmatic dependent launch: wait for the previous kernel's results /
// let the next kernel start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace q4
