// Small-M ("decode") expert GEMMs over 4-bit codebook weights, streaming the
// packed bytes from HBM once per token tile.
//
//   gate/up: h[row] = silu(W_gate x) * (W_up x)   for each row of an expert
//   down:    y[row] = W_down h[row]
// ("Round 7 -- Rewrite the GLM-5.2 routed-expert encoder", "Owner-locked
// decisions" 4: I_e = silu(X Wg^T) * (X Wu^T); item 6: down is [K=I, N=H].)
//
// Decode of the format ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", "Codes
// are indices into the per-layer grid -- not E2M1", "Contents"): the expert's
// 8 levels live in registers as bf16 byte planes; one PRMT looks up four
// codes, so a 32-bit word of 8 codes becomes four bf16x2 pairs in 15 integer
// ops; the block's E8M0 scale is applied by one bf16x2 multiply per pair
// (exact: a power of two).  The products run on the tensor cores
// (mma.sync m16n8k16, fp32 accumulate), which costs far fewer instructions
// per weight than scalar FMAs and makes up to 8 tokens per n-tile free.
//
// Work decomposition.  A warp owns two 16-row m-tiles (gate+up rows r..r+15
// for gate/up; rows r..r+31 for down) and a contiguous range of 128-wide K
// steps.  In each step, lane (g = lane/4, c = lane%4) loads the 16 code bytes
// of 32-block 4j+c for rows g and g+8 of each tile (one 128-bit load each:
// each group of 4 lanes reads 64 contiguous bytes of a row) and the 32
// activations of the same block for token g.  Because both MMA operands of
// logical k = 2c.. come from the lane with the same c, the K order inside the
// MMA is a permutation of the block's K order, applied to both operands: the
// product is unchanged and no data is reshuffled.  S warps of a CTA split K;
// their partial tiles are summed in shared memory in warp order.
#include "q4_api_internal.h"
#include "q4_common.cuh"

namespace q4 {

struct Stage {
  uint4 a0, a1, b0, b1;  // codes: tile A rows g, g+8; tile B rows g, g+8
  uint32_t sa0, sa1, sb0, sb1;
};

template <bool GATEUP>
__device__ __forceinline__ void load_stage(Stage& st, const uint8_t* wa, const uint8_t* sa,
                                           const uint8_t* wb, const uint8_t* sb, size_t rb, size_t sbytes,
                                           int g, int kb) {
  st.a0 = ldg_stream(wa + (size_t)g * rb + (size_t)kb * 16);
  st.a1 = ldg_stream(wa + (size_t)(g + 8) * rb + (size_t)kb * 16);
  st.b0 = ldg_stream(wb + (size_t)g * rb + (size_t)kb * 16);
  st.b1 = ldg_stream(wb + (size_t)(g + 8) * rb + (size_t)kb * 16);
  st.sa0 = ldg_u8(sa + (size_t)g * sbytes + kb);
  st.sa1 = ldg_u8(sa + (size_t)(g + 8) * sbytes + kb);
  st.sb0 = ldg_u8(sb + (size_t)g * sbytes + kb);
  st.sb1 = ldg_u8(sb + (size_t)(g + 8) * sbytes + kb);
}

// 16 codes-bytes (32 codes) of one row, scaled: 16 bf16x2 words, word m holds
// K = 2m, 2m+1 of the block.
__device__ __forceinline__ void decode_block(const uint4& c, uint32_t s, const Planes& P, uint32_t out[16]) {
  const uint32_t s2 = scale_bf16x2(s);
  decode8(c.x, P, &out[0]);
  decode8(c.y, P, &out[4]);
  decode8(c.z, P, &out[8]);
  decode8(c.w, P, &out[12]);
#pragma unroll
  for (int i = 0; i < 16; ++i) out[i] = bf16x2_mul(out[i], s2);
}

// acc[nt] += tile(16 rows) x block(32 K) x tokens(8) for the n-tiles in use.
__device__ __forceinline__ void mma_block(float acc[2][4], const uint32_t r0[16], const uint32_t r1[16],
                                          const uint32_t xw[2][16], bool two) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mma_16816(acc[0], r0[2 * i], r1[2 * i], r0[2 * i + 1], r1[2 * i + 1], xw[0][2 * i], xw[0][2 * i + 1]);
    if (two)
      mma_16816(acc[1], r0[2 * i], r1[2 * i], r0[2 * i + 1], r1[2 * i + 1], xw[1][2 * i],
                xw[1][2 * i + 1]);
  }
}

// 32 bf16 activations of block kb for the n-tiles in use (zeros past n_e).
__device__ __forceinline__ void load_act(uint32_t xw[2][16], const __nv_bfloat16* const xr[2], int kb,
                                         bool two) {
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    if (xr[nt] && (nt == 0 || two)) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = ldg_nc(xr[nt] + (size_t)kb * 32 + q * 8);
        xw[nt][4 * q] = v.x;
        xw[nt][4 * q + 1] = v.y;
        xw[nt][4 * q + 2] = v.z;
        xw[nt][4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 16; ++q) xw[nt][q] = 0u;
    }
  }
}

template <bool GATEUP, int S>
__global__ void __launch_bounds__(32 * S) decode_kernel(const __grid_constant__ FwdArgs a,
                                                        const __grid_constant__ TableParams tp) {
  __shared__ float red[S > 1 ? S - 1 : 1][32][16];
  const int rows_total = GATEUP ? a.I : a.H;
  const int K = GATEUP ? a.H : a.I;
  const int units_per_e = GATEUP ? (rows_total >> 4) : (rows_total >> 5);
  const int slot = blockIdx.x / units_per_e;
  const int unit = blockIdx.x - slot * units_per_e;
  pdl_wait();
  pdl_trigger();
  if (slot >= a.hdr[kNumDecode]) return;
  const int e = a.dec_list[slot];
  const int row0 = a.offsets[e];
  const int n_e = a.counts[e];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const Planes P = make_planes(tp.t[tp.id[e]]);
  const size_t rb = (size_t)K / 2, sbytes = (size_t)K / 32;
  // tile A / tile B first rows
  const int rowA = GATEUP ? unit * 16 : unit * 32;
  const int rowB = GATEUP ? unit * 16 : unit * 32 + 16;
  const size_t eb = (size_t)e * rows_total;
  const uint8_t* wa = (GATEUP ? a.gate_w : a.down_w) + (eb + rowA) * rb;
  const uint8_t* sa = (GATEUP ? a.gate_s : a.down_s) + (eb + rowA) * sbytes;
  const uint8_t* wb = (GATEUP ? a.up_w : a.down_w) + (eb + rowB) * rb;
  const uint8_t* sb = (GATEUP ? a.up_s : a.down_s) + (eb + rowB) * sbytes;
  const int nsteps = K >> 7;
  const int s0 = (warp * nsteps) / S, s1 = ((warp + 1) * nsteps) / S;

  for (int tt = 0; tt < n_e; tt += 16) {
    float accA[2][4], accB[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) accA[i][q] = accB[i][q] = 0.0f;
    // activation rows of this lane's B-fragment tokens (tt + g, tt + 8 + g);
    // the down projection reads h as its bf16 pair (h, h_lo): two MMAs
    const __nv_bfloat16* xr[2];
    const __nv_bfloat16* xl[2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int n = tt + nt * 8 + g;
      xr[nt] = nullptr;
      xl[nt] = nullptr;
      if (n < n_e) {
        if (GATEUP) {
          xr[nt] = a.x + (size_t)a.row_token[row0 + n] * a.H;
        } else {
          xr[nt] = a.h + (size_t)(row0 + n) * a.I;
          xl[nt] = a.h_lo + (size_t)(row0 + n) * a.I;
        }
      }
    }
    const bool two = (tt + 8) < n_e;
    Stage cur, nxt;
    if (s0 < s1) load_stage<GATEUP>(cur, wa, sa, wb, sb, rb, sbytes, g, 4 * s0 + c);
    for (int j = s0; j < s1; ++j) {
      if (j + 1 < s1) load_stage<GATEUP>(nxt, wa, sa, wb, sb, rb, sbytes, g, 4 * (j + 1) + c);
      const int kb = 4 * j + c;
      uint32_t xw[2][16];
      load_act(xw, xr, kb, two);
      uint32_t p0[16], p1[16], q0[16], q1[16];
      decode_block(cur.a0, cur.sa0, P, p0);
      decode_block(cur.a1, cur.sa1, P, p1);
      decode_block(cur.b0, cur.sb0, P, q0);
      decode_block(cur.b1, cur.sb1, P, q1);
      mma_block(accA, p0, p1, xw, two);
      mma_block(accB, q0, q1, xw, two);
      if (!GATEUP) {
        load_act(xw, xl, kb, two);
        mma_block(accA, p0, p1, xw, two);
        mma_block(accB, q0, q1, xw, two);
      }
      cur = nxt;
    }
    if (S > 1) {
      if (warp > 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            red[warp - 1][lane][i * 4 + q] = accA[i][q];
            red[warp - 1][lane][8 + i * 4 + q] = accB[i][q];
          }
      }
      __syncthreads();
      if (warp == 0) {
        for (int w2 = 0; w2 < S - 1; ++w2)
#pragma unroll
          for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              accA[i][q] += red[w2][lane][i * 4 + q];
              accB[i][q] += red[w2][lane][8 + i * 4 + q];
            }
      }
      __syncthreads();
    }
    if (warp == 0) {
      // C fragment: acc[nt][rr*2 + cc] = (row g + 8 rr, token tt + 8 nt + 2c + cc)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int n = tt + nt * 8 + 2 * c + cc;
          if (n >= n_e) continue;
          const size_t r = (size_t)row0 + n;
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const float va = accA[nt][rr * 2 + cc], vb = accB[nt][rr * 2 + cc];
            if (GATEUP) {
              const float hv = silu_mul(va, vb);
              const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
              const size_t o = r * a.I + rowA + g + 8 * rr;
              a.h[o] = hi;
              a.h_lo[o] = __float2bfloat16_rn(hv - __bfloat162float(hi));
            } else {
              a.y[r * a.H + rowA + g + 8 * rr] = va;
              a.y[r * a.H + rowB + g + 8 * rr] = vb;
            }
          }
        }
    }
  }
}

template <bool GATEUP, int S>
static int launch_decode_t(const FwdArgs& a, const TableParams& tp, int grid, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(32 * S);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<GATEUP, S>, a, tp) == cudaSuccess ? MOE_Q4_OK
                                                                                  : MOE_Q4_ECUDA;
}

}  // namespace q4

using namespace q4;

int q4_launch_decode(const FwdArgs& a, const TableParams& tp, bool gateup, cudaStream_t s) {
  // Upper bound on experts that can be on this path: distinct experts <= T*k.
  const int max_exp = a.T * a.k < a.E ? a.T * a.k : a.E;
  if (max_exp == 0) return MOE_Q4_OK;
  const int units_per_e = gateup ? a.I / 16 : a.H / 32;
  const long long units = (long long)max_exp * units_per_e;
  // Enough warps to keep ~16 per SM streaming: split K across warps when the
  // unit count alone is small.
  const long long target = 148LL * 16;
  int S = 1;
  if (units * 4 <= target)
    S = 4;
  else if (units * 2 <= target)
    S = 2;
  const int grid = (int)units;
  if (gateup) {
    if (S == 4) return launch_decode_t<true, 4>(a, tp, grid, s);
    if (S == 2) return launch_decode_t<true, 2>(a, tp, grid, s);
    return launch_decode_t<true, 1>(a, tp, grid, s);
  }
  if (S == 4) return launch_decode_t<false, 4>(a, tp, grid, s);
  if (S == 2) return launch_decode_t<false, 2>(a, tp, grid, s);
  return launch_decode_t<false, 1>(a, tp, grid, s);
}
