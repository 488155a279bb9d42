// Dense BF16 GEMMs on the 5th-generation tensor cores: the shared expert that
// runs beside the routed experts, and the router gate at prefill sizes.
//
// Shared expert ("GLM-5.2 EXL3 TR3 v4" README, "Checkpoint layout update":
// mlp.shared_experts.{gate,up,down}_proj kept as the original BF16 weights,
// gate and up concatenated into one [2 I][H] payload so that one launch
// computes both; HF discussion #2, "Store shared experts in BF16"):
//   gate/up: h_s[t] = silu(W_g x_t) * (W_u x_t)   (W_gu = [W_g; W_u], [2 I][H])
//   down:    y_s[t] = W_d h_s[t]                  (W_d [H][I])
// every token, weight 1, added to the routed experts' weighted sum.
//
// Router gate at prefill sizes ("GLM-5.2-EXL3-DENSE6-MTP78", "Quant recipe":
// mlp.gate held in BF16): logits[t] = W_r x_t, fp32 out.
//
// One kernel template: the MMA's M = 128 weight rows, N = up to 256 tokens
// (the last tile rounded up to 16; rows past T are zero-filled by the TMA), K
// in steps of 64.  The weight tile comes by TMA straight into the canonical
// 128-byte-swizzle K-major layout the MMA reads (no decode: these weights are
// BF16).  Work items (m-tile, K split, token tile) are walked by persistent
// CTAs; at decode sizes the K range of every m-tile is split so that every SM
// streams weights, each split writing fp32 partial sums that a second kernel
// adds in split order (deterministic) before the SwiGLU / the output.
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocation + MMA issue (one
// thread), warps 2..9 epilogue (two per 32-lane TMEM quarter, each draining
// half of the token tile).  Every mbarrier wait is bounded; a timeout sets
// MOE_Q4_ETIMEOUT in the status word.
#include <cuda.h>

#include "q4_api_internal.h"
#include "q4_common.cuh"
#include "sm100.cuh"

namespace q4 {

using namespace sm100;

namespace sx {
constexpr int kBN = 256;  // token tile (largest MMA N)
constexpr int kBM = 128;  // weight rows per tile (MMA M)
constexpr int kBK = 64;   // K per stage (128 bytes of bf16)
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kEpiWarp0 = 2;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
}  // namespace sx

template <int MATS>
struct SxCfg {
  static constexpr int kMaxStages = 8;
  static constexpr int kATile = sx::kBM * sx::kBK * 2;  // 16 KB bf16 per matrix
  static constexpr int kAccBufs = MATS == 2 ? 1 : 2;  // TMEM holds 512 columns
  static constexpr int kTmemCols = kAccBufs * MATS * sx::kBN;
};

// shared memory of a launch: `stages` ring stages of the weight tiles and a
// token tile of bn rows (bn = T rounded up to 16, at most 256: small T does
// not pay for a 256-row tile of zeros), the alignment pad and the barriers
__host__ __device__ constexpr int sx_stage_bytes(int mats, int bn) { return mats * sx::kBM * sx::kBK * 2 + bn * 128; }
constexpr int kSxSmemLimit = 227 * 1024;

// What the epilogue writes.
enum SxOut : int {
  kSxSwiGLU = 0,   // bf16 silu(acc0) * acc1 into out_bf16 [T][ld]
  kSxF32 = 1,      // fp32 acc0 into out_f32 [T][ld]
  kSxPartial = 2,  // fp32 raw accumulators into partial [split][mats][T][rows]
};

struct SxParams {
  int T;            // tokens
  int bn;           // token tile (rows of the B tile): T rounded up to 16, at most 256
  int stages;       // ring stages
  int rows;         // output rows per matrix (I of the shared expert, H, or E)
  int K;            // reduction length
  int mat1_off;     // row offset of the second matrix in the weight array (gate/up: I)
  int splits;       // K splits per m-tile
  int ksteps_split; // k-steps of 64 per split
  int out_mode;     // SxOut
  int ld;           // row length of the output (elements)
  __nv_bfloat16* out_bf16;
  float* out_f32;
  float* partial;
  int32_t* status;
};

// item -> (m-tile, split, token tile); items ordered (m, split, nt) so the
// token tiles of one weight tile run back to back and re-read it from L2
__device__ __forceinline__ void sx_item(int item, int n_tiles, int splits, int& m, int& sp, int& nt) {
  nt = item % n_tiles;
  const int q = item / n_tiles;
  sp = q % splits;
  m = q / splits;
}

template <int MATS>
__global__ void __launch_bounds__(sx::kThreads, 1)
    sx_gemm_kernel(const __grid_constant__ SxParams P, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_b) {
  using C = SxCfg<MATS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = P.stages;
  const int b_tile = P.bn * 128;
  uint8_t* sA = smem;                         // [S][mats][128][128 B]
  uint8_t* sB = sA + S * MATS * C::kATile;    // [S][bn][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * b_tile);
  uint64_t* full = bars;                        // [S] weight + token tiles landed
  uint64_t* empty = full + C::kMaxStages;       // [S] stage consumed by the MMAs
  uint64_t* acc_full = empty + C::kMaxStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* drain = acc_empty + 2;          // [1] final MMA completion
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], sx::kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // the activations may come from the previous kernel
  pdl_wait();
  const int m_tiles = P.rows / sx::kBM;
  const int n_tiles = (P.T + P.bn - 1) / P.bn;
  const int total = m_tiles * P.splits * n_tiles;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      for (int item = blockIdx.x; item < total && !*abort_flag; item += gridDim.x) {
        int m, sp, nt;
        sx_item(item, n_tiles, P.splits, m, sp, nt);
        const int k0 = sp * P.ksteps_split;
        for (int ks = k0; ks < k0 + P.ksteps_split; ++ks, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, sx::kWaitNs)) break;
          mbar_arrive_expect_tx(&full[s], MATS * C::kATile + b_tile);
          tma_load_2d(sA + (s * MATS) * C::kATile, &tm_w, &full[s], ks * sx::kBK, m * sx::kBM);
          if (MATS == 2)
            tma_load_2d(sA + (s * MATS + 1) * C::kATile, &tm_w, &full[s], ks * sx::kBK, P.mat1_off + m * sx::kBM);
          tma_load_2d(sB + s * b_tile, &tm_b, &full[s], ks * sx::kBK, nt * P.bn);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      for (int item = blockIdx.x; item < total && !*abort_flag; item += gridDim.x, ++tcount) {
        int m, sp, nt;
        sx_item(item, n_tiles, P.splits, m, sp, nt);
        const int left = P.T - nt * P.bn;
        const int n_cols = left >= P.bn ? P.bn : ((left + 15) & ~15);
        const uint32_t idesc = umma_idesc_bf16(sx::kBM, n_cols);
        const int buf = (int)(tcount % C::kAccBufs);
        const uint32_t use = tcount / C::kAccBufs;  // earlier uses of this buffer
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, sx::kWaitNs)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * (MATS * sx::kBN);
        bool ok = true;
        for (int j = 0; j < P.ksteps_split; ++j, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag, sx::kWaitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t db = umma_desc_sw128(smem_u32(sB + s * b_tile));
#pragma unroll
          for (int mat = 0; mat < MATS; ++mat) {
            const uint64_t da = umma_desc_sw128(smem_u32(sA + (s * MATS + mat) * C::kATile));
#pragma unroll
            for (int kk = 0; kk < sx::kBK / 16; ++kk)  // +32 bytes of K per MMA (>> 4 -> +2)
              umma_bf16(d0 + mat * sx::kBN, da + 2 * kk, db + 2 * kk, idesc, (j | kk) != 0);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
      }
      // all MMAs issued by this thread complete before TMEM is released
      umma_commit(drain);
      mbar_wait(drain, 0, abort_flag, sx::kWaitNs);
    }
  } else {
    // ---------------- epilogue ----------------
    const int quad = warp & 3;                        // TMEM lanes 32 quad .. +31
    const int ehalf = (warp - sx::kEpiWarp0) >> 2;    // tokens 128 ehalf .. + 127 of the tile
    const int row = quad * 32 + lane;                 // weight row in the tile
    uint32_t tcount = 0;
    for (int item = blockIdx.x; item < total && !warp_aborted(abort_flag); item += gridDim.x, ++tcount) {
      int m, sp, nt;
      sx_item(item, n_tiles, P.splits, m, sp, nt);
      const int buf = (int)(tcount % C::kAccBufs);
      const uint32_t use = tcount / C::kAccBufs;
      if (!mbar_wait_warp(&acc_full[buf], use & 1, abort_flag, sx::kWaitNs)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16) + buf * (MATS * sx::kBN);
      const int orow = m * sx::kBM + row;  // output row of this thread
      const int n_hi = P.T - nt * P.bn < P.bn ? P.T - nt * P.bn : P.bn;
      const int c_lo = (P.bn / 2) * ehalf;
      const int c_hi = n_hi < c_lo + P.bn / 2 ? n_hi : c_lo + P.bn / 2;
      for (int c0 = c_lo; c0 < c_hi; c0 += 8) {
        uint32_t v[MATS][8];
#pragma unroll
        for (int mt = 0; mt < MATS; ++mt) tmem_ld8_nowait(tb + mt * sx::kBN + c0, v[mt]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int t = nt * P.bn + c0 + j;
          if (c0 + j >= c_hi) break;
          if (P.out_mode == kSxPartial) {
#pragma unroll
            for (int mt = 0; mt < MATS; ++mt)
              P.partial[(((size_t)sp * MATS + mt) * P.T + t) * P.rows + orow] = __uint_as_float(v[mt][j]);
          } else if (P.out_mode == kSxSwiGLU) {
            P.out_bf16[(size_t)t * P.ld + orow] =
                __float2bfloat16_rn(silu_mul(__uint_as_float(v[0][j]), __uint_as_float(v[MATS - 1][j])));
          } else {
            P.out_f32[(size_t)t * P.ld + orow] = __uint_as_float(v[0][j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  // ---------------- teardown ----------------
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) record_error(P.status, MOE_Q4_ETIMEOUT);
  if (warp == 0 && lane == 0 && *abort_flag) {
    // let any copy still in flight land before the CTA's smem goes away
    for (int s = 0; s < S; ++s)
      for (uint32_t par = 0; par < 2; ++par) {
        volatile int quick = 0;
        mbar_wait(&full[s], par, &quick, 50000000ull);
      }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  pdl_trigger();
}

// Split-K partial sums added in split order, then the SwiGLU (two matrices,
// bf16 out) or the fp32 output.  One thread per (token, row).
template <int MATS>
__global__ void __launch_bounds__(256) sx_reduce_kernel(const __grid_constant__ SxParams P) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)P.T * P.rows;
  for (int64_t i = blockIdx.x * 256 + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256) {
    float acc[MATS];
#pragma unroll
    for (int mt = 0; mt < MATS; ++mt) {
      float v = 0.0f;
      for (int sp = 0; sp < P.splits; ++sp) v += P.partial[((size_t)sp * MATS + mt) * n + i];
      acc[mt] = v;
    }
    const int64_t t = i / P.rows, r = i % P.rows;
    if (MATS == 2)
      P.out_bf16[t * P.ld + r] = __float2bfloat16_rn(silu_mul(acc[0], acc[1]));
    else
      P.out_f32[t * P.ld + r] = acc[0];
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn sx_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 row-major [rows][cols], boxes of 64 columns x box_rows rows, 128-byte swizzle
static bool sx_map(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = sx_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)sx::kBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace q4

using namespace q4;

static int sx_bn(int T) { return T >= sx::kBN ? sx::kBN : ((T + 15) & ~15); }

// Bytes of split-K partial sums a dense GEMM of this shape may need (the
// split count is planned for 148 SMs, the same on every device).
size_t q4_dense_partial_bytes(int T, int rows, int K, int mats) {
  if (T <= 0) return 0;
  const int m_tiles = rows / sx::kBM;
  const int n_tiles = (T + sx_bn(T) - 1) / sx_bn(T);
  const int ksteps = K / sx::kBK;
  int splits = 1;
  // split K until every SM has an item (as long as a split keeps >= 4 k-steps)
  while (m_tiles * n_tiles * splits * 2 <= 148 && ksteps % (splits * 2) == 0 && ksteps / (splits * 2) >= 4)
    splits *= 2;
  return splits > 1 ? sizeof(float) * (size_t)splits * mats * T * rows : 0;
}

// out = W act^T for bf16 weights [rows (x mats)][K] and bf16 activations
// [T][K]; two matrices (mat1 at row offset mat1_off): bf16 silu(W0 a) * (W1 a)
// into out_bf16 [T][ld]; one matrix: fp32 into out_f32 [T][ld].  partial:
// workspace of q4_dense_partial_bytes (NULL when that is 0).
int q4_launch_dense(const void* w, int mats, int mat1_off, int rows, int K, const void* act, int T,
                    __nv_bfloat16* out_bf16, float* out_f32, int ld, float* partial, int32_t* status,
                    cudaStream_t s) {
  if (T <= 0) return MOE_Q4_OK;
  if (rows % sx::kBM || K % sx::kBK) return MOE_Q4_EINVAL;
  SxParams P;
  P.T = T;
  P.bn = sx_bn(T);
  const int sb = sx_stage_bytes(mats, P.bn);
  P.stages = (kSxSmemLimit - 2048) / sb;
  if (P.stages > SxCfg<1>::kMaxStages) P.stages = SxCfg<1>::kMaxStages;
  if (P.stages < 2) return MOE_Q4_ECUDA;
  const int smem = P.stages * sb + 2048;
  P.rows = rows;
  P.K = K;
  P.mat1_off = mat1_off;
  P.ld = ld;
  P.out_bf16 = out_bf16;
  P.out_f32 = out_f32;
  P.status = status;
  const int ksteps = K / sx::kBK;
  P.splits = 1;
  const size_t pb = q4_dense_partial_bytes(T, rows, K, mats);
  if (pb) P.splits = (int)(pb / (sizeof(float) * (size_t)mats * T * rows));
  P.ksteps_split = ksteps / P.splits;
  P.partial = partial;
  P.out_mode = P.splits > 1 ? kSxPartial : (mats == 2 ? kSxSwiGLU : kSxF32);
  if (P.splits > 1 && !partial) return MOE_Q4_EWORKSPACE;
  CUtensorMap tw, tb;
  // (the weight map covers both matrices: rows of the second start at mat1_off)
  if (!sx_map(&tw, w, K, mats == 2 ? (uint64_t)mat1_off + rows : (uint64_t)rows, sx::kBM) ||
      !sx_map(&tb, act, K, T, P.bn))
    return MOE_Q4_ECUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int total = (rows / sx::kBM) * P.splits * ((T + P.bn - 1) / P.bn);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(total < sms ? total : sms);
  cfg.blockDim = dim3(sx::kThreads);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err;
  if (mats == 2) {
    cfg.dynamicSmemBytes = smem;
    if (cudaFuncSetAttribute(sx_gemm_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return MOE_Q4_ECUDA;
    err = cudaLaunchKernelEx(&cfg, sx_gemm_kernel<2>, P, tw, tb);
  } else {
    cfg.dynamicSmemBytes = smem;
    if (cudaFuncSetAttribute(sx_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return MOE_Q4_ECUDA;
    err = cudaLaunchKernelEx(&cfg, sx_gemm_kernel<1>, P, tw, tb);
  }
  if (err != cudaSuccess) return MOE_Q4_ECUDA;
  if (P.splits == 1) return MOE_Q4_OK;
  P.out_mode = mats == 2 ? kSxSwiGLU : kSxF32;
  const int64_t n = (int64_t)T * rows;
  const int64_t blocks = (n + 255) / 256;
  cfg.gridDim = dim3((unsigned)(blocks < 4 * sms ? blocks : 4 * sms));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  err = mats == 2 ? cudaLaunchKernelEx(&cfg, sx_reduce_kernel<2>, P) : cudaLaunchKernelEx(&cfg, sx_reduce_kernel<1>, P);
  return err == cudaSuccess ? MOE_Q4_OK : MOE_Q4_ECUDA;
}
