// Large-M ("prefill") expert GEMMs on the 5th-generation tensor cores.
//
//   gate/up: h[row] = silu(W_gate x) * (W_up x)     (fused SwiGLU epilogue)
//   down:    y[row] = W_down h[row]
// ("Round 7 -- Rewrite the GLM-5.2 routed-expert encoder", "Owner-locked
// decisions" 4 and 6), for the experts whose row count exceeds the streaming
// path's limit.
//
// Two tile orientations of one kernel template:
// * swap-AB (experts with more than 128 rows): the MMA's M = 128 weight rows,
//   N = a tile of up to 256 tokens of one expert (the expert's last tile takes
//   N = its remaining rows rounded up to 16), K streamed in steps of 64.  A
//   persistent CTA per SM walks tiles ordered (expert, weight m-tile, token
//   tile) so the token tiles of one weight tile run back to back and re-read
//   it from L2.
// * WIDE (experts with 17..128 rows, layers whose I and H are multiples of
//   256): M = the expert's (padded) 128 token rows, N = 256 weight rows; tiles
//   (expert, 256-row weight tile).  See TcCfg.
//
// Warp roles:
//   warp 0       TMA producer: packed codes of the weight tile (128-row boxes
//                x 32 B per k-step, 32-byte swizzle) and the token tile (128
//                bytes of K per row, 128-byte swizzle) into the copy ring;
//   warp 1       allocates TMEM and issues tcgen05.mma (one thread): for each
//                k-step, 4 MMAs of K=16 per weight matrix into fp32 TMEM
//                accumulators (gate + up fill all 512 columns: one buffer;
//                down: double-buffered across tiles);
//   next 8 or 16 dequantise: codes -> bf16 through the PRMT byte-plane lookup
//                of the expert's table, E8M0 scale by an exact bf16x2
//                multiply, stored to the decoded-weight ring in the canonical
//                128-byte-swizzle K-major layout the MMA reads ("aidendle94/
//                GLM-5.2-NF4-Lloyd-Experts-GPTQ", "Codes are indices into the
//                per-layer grid"); with single-buffered accumulators they also
//                help drain them while the MMA waits for that drain;
//   last 8       epilogue: tcgen05.ld of the accumulators (one TMEM lane = one
//                weight row, or one token for WIDE tiles), SwiGLU in fp32,
//                bf16 stores of h (or fp32 stores of y).
// Every mbarrier wait is bounded; on a timeout the CTA sets the status word
// to MOE_Q4_ETIMEOUT, drains its own copies and MMAs (bounded), frees TMEM
// and exits.
#include <cuda.h>

#include "q4_api_internal.h"
#include "q4_common.cuh"
#include "sm100.cuh"

namespace q4 {

using namespace sm100;

constexpr int kBN = 256;          // token tile (largest MMA N)
constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBK = 64;           // K per pipeline stage (128 bytes of bf16)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// WIDE: the orientation for experts with few rows (up to 128): the tokens are
// the MMA's M = 128 rows (the expert's rows, padded) and 256 weight rows its N,
// so one instruction covers twice the weight rows of the swap-AB tile (a
// tcgen05.mma costs about the same whatever its N: a 48-token swap-AB tile
// would use a fifth of it).  The decoded weights are the B operand
// (K-major, 128-byte swizzle, like the token tile of the swap-AB kernel), the
// token tile the A operand; the accumulator's TMEM lanes are tokens and its
// columns weight rows, so each thread stores 8 contiguous outputs of its token.
template <bool GATEUP, bool WIDE>
struct TcCfg {
  static constexpr int kMats = GATEUP ? 2 : 1;
  static constexpr int kWRows = WIDE ? 256 : kBM;     // weight rows per tile
  static constexpr int kTRows = WIDE ? 128 : kBN;     // token rows per tile
  // dequant warps: per k-step one 16-byte code chunk (32 weights) of a row per
  // thread (swap-AB: 128 rows x 2 chunks per matrix) or both chunks of a row
  // (WIDE: 256 rows per matrix)
  static constexpr int kDequantThreads = kMats * 256;
  static constexpr int kEpiWarp0 = 2 + kDequantThreads / 32;
  // epilogue: two warps per 32-lane TMEM quarter, each finishing half the columns
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
  static constexpr int kATile = kWRows * kBK * 2;     // bf16 weights per matrix
  static constexpr int kBTile = kTRows * kBK * 2;     // bf16 token tile
  static constexpr int kCTile = kWRows * kBK / 2;     // codes per matrix
  // Two rings: the TMA copies (token tile + codes) and the decoded weights.
  // Swap-AB: as many weight stages as copy stages; WIDE (weight stages of 32
  // KB per matrix): a short weight ring and a deeper copy ring, so the copies'
  // latency stays hidden behind the decode.
  static constexpr int kWStageBytes = kMats * kATile;
  static constexpr int kTStageBytes = kBTile + kMats * kCTile;
  static constexpr int kBudget = 227 * 1024 - 2048;
  static constexpr int kFitBoth = kBudget / (kWStageBytes + kTStageBytes);
  static constexpr int kStagesW = WIDE ? (GATEUP ? 2 : 3) : (kFitBoth > 4 ? 4 : kFitBoth);
  static constexpr int kFitT = (kBudget - kStagesW * kWStageBytes) / kTStageBytes;
  static constexpr int kStagesT = WIDE ? (kFitT > 4 ? 4 : kFitT) : kStagesW;
  static_assert(kStagesW >= 2 && kStagesT >= kStagesW, "pipeline stages");
  static constexpr int kAccCols = 256;                // accumulator columns per matrix
  static constexpr int kAccBufs = GATEUP ? 1 : 2;     // TMEM holds 512 columns
  // single-buffered accumulators (gate/up): the dequant warps, idle while the
  // MMA waits for the drain, drain beside the epilogue warps
  static constexpr bool kHelp = kAccBufs == 1;
  static constexpr int kDrainWarps = kEpiWarps + (kHelp ? kDequantThreads / 32 : 0);
  static constexpr int kWorkersPerQuad = kDrainWarps / 4;
  static constexpr int kTmemCols = kAccBufs * kMats * kAccCols;
  static constexpr int kSmem = kStagesW * kWStageBytes + kStagesT * kTStageBytes + 1024 /*align*/ + 1024 /*barriers*/;
  static_assert(kSmem <= 227 * 1024, "shared memory plan exceeds 227 KB");
};

struct TcParams {
  FwdArgs a;
  int m_tiles;  // weight rows / rows per tile
  int k_steps;  // K / 64
  int early_trigger;  // swap-AB followed by the WIDE kernel: let it launch once this one's inputs are complete
};

// Tile id -> (prefill slot p, m-tile, token tile) with tiles ordered
// (expert, m, n); ntile_off[p] = token tiles of the prefill experts before p.
__device__ __forceinline__ void tile_coords(const FwdArgs& a, int m_tiles, int np, int tile, int& p, int& m,
                                            int& nt) {
  int lo = 0, hi = np - 1;
  while (lo < hi) {  // last p with m_tiles * ntile_off[p] <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (m_tiles * a.tiles[mid] <= tile)
      lo = mid;
    else
      hi = mid - 1;
  }
  p = lo;
  const int n_tiles_p = a.tiles[p + 1] - a.tiles[p];
  const int local = tile - m_tiles * a.tiles[p];
  m = local / n_tiles_p;
  nt = local - m * n_tiles_p;
}

template <bool GATEUP, bool WIDE>
__global__ void __launch_bounds__(TcCfg<GATEUP, WIDE>::kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ TcParams P, const __grid_constant__ TableParams tp,
                   const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_wa,
                   const __grid_constant__ CUtensorMap tm_wb) {
  using C = TcCfg<GATEUP, WIDE>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                        // [S][mats][weight rows][128 B]
  uint8_t* sB = sA + C::kStagesW * C::kMats * C::kATile;     // [T][token rows][128 B]
  uint8_t* sC = sB + C::kStagesT * C::kBTile;                // [T][mats][weight rows][32 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sC + C::kStagesT * C::kMats * C::kCTile);
  uint64_t* full_c = bars;                       // [T] codes landed
  uint64_t* full_b = full_c + C::kStagesT;       // [T] token tile landed
  uint64_t* empty = full_b + C::kStagesT;        // [T] copy stage consumed (codes decoded, tokens by the MMAs)
  uint64_t* a_ready = empty + C::kStagesT;       // [W] decoded weights written
  uint64_t* a_empty = a_ready + C::kStagesW;     // [W] decoded weights consumed by the MMAs
  uint64_t* acc_full = a_empty + C::kStagesW;    // [2]
  uint64_t* acc_empty = acc_full + 2;            // [2]
  uint64_t* mma_done = acc_empty + 2;            // [1] final MMA completion
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const FwdArgs& a = P.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStagesT; ++s) {
      mbar_init(&full_c[s], 1);
      mbar_init(&full_b[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int w = 0; w < C::kStagesW; ++w) {
      mbar_init(&a_ready[w], C::kDequantThreads / 32);  // one arrival per dequant warp
      mbar_init(&a_empty[w], 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::kDrainWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_wa);
    if (GATEUP) prefetch_tmap(&tm_wb);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // The WIDE kernel follows the swap-AB kernel of the same projection and
  // reads nothing that kernel writes: its inputs (routing tables, activation
  // rows) were complete before the swap-AB kernel's own wait returned, which
  // precedes that kernel's early trigger, so its CTAs start as the swap-AB
  // CTAs leave their SMs (filling that grid's last wave); it waits for the
  // swap-AB grid only before it exits, so the kernels after it still find
  // both complete.
  if (!WIDE) pdl_wait();
  if (!WIDE && P.early_trigger) pdl_trigger();
  // routing tables: the WIDE kernel reads them through L2 only (no L1 line of
  // an earlier call can be stale there)
  const auto rt = [&](const int32_t* q) -> int { return WIDE ? __ldcg(q) : *q; };
  const int np = WIDE ? rt(a.hdr + kNumMid) : a.hdr[kNumPrefill];
  const int total = np > 0 ? P.m_tiles * (WIDE ? np : a.tiles[np]) : 0;
  const int rows_total = GATEUP ? a.I : a.H;
  const int K = GATEUP ? a.H : a.I;
  // tile -> (expert slot p, weight tile m, token tile nt) and the expert;
  // WIDE: tiles ordered (expert, weight tile), one token tile per expert
  const auto coords = [&](int tile, int& p, int& m, int& nt) -> int {
    if (WIDE) {
      p = tile / P.m_tiles;
      m = tile - p * P.m_tiles;
      nt = 0;
      return rt(a.mid_list + p);
    }
    tile_coords(a, P.m_tiles, np, tile, p, m, nt);
    return a.pre_list[p];
  };

  // Drain of the accumulators of the tcount-th tile of this CTA by one warp:
  // worker `wk` of the C::kWorkersPerQuad warps of its TMEM lane quarter takes
  // a contiguous range of 8-column chunks; tcgen05.ld of the fp32 sums (one
  // lane = one weight row), SwiGLU (gate/up) or fp32 y (down), stores, then
  // the warp signs off on acc_empty.  False when a wait gave up.
  const auto drain = [&](int tile, uint32_t tcount, int wk) -> bool {
    const int quad = warp & 3;          // TMEM lanes 32*quad .. +31
    const int row = quad * 32 + lane;   // weight row (swap-AB) or token (WIDE) in the tile
    int p, m, nt;
    int e = coords(tile, p, m, nt);
    if (!q4_check((unsigned)e < (unsigned)a.E, a.hdr + kStatus)) e = 0;
    int n_e = rt(a.counts + e);
    const int row0 = rt(a.offsets + e);
    // (a failed check leaves the tile's rows unwritten)
    if (!q4_check(row0 >= 0 && n_e >= 0 && row0 + n_e <= a.T * a.k, a.hdr + kStatus)) n_e = nt * kBN;
    const int buf = (int)(tcount % C::kAccBufs);
    const uint32_t use = tcount / C::kAccBufs;
    if (!mbar_wait_warp(&acc_full[buf], use & 1, abort_flag, kWaitLimitNs)) return false;
    tc_fence_after();
    const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16) + buf * (C::kMats * C::kAccCols);
    const int wrow = m * C::kWRows + row;
    const int n_hi = n_e - nt * kBN < kBN ? n_e - nt * kBN : kBN;  // tokens of this tile (swap-AB)
    // 8 token columns of every matrix per chunk; the next chunk's TMEM loads
    // are in flight while this chunk is finished (one wait per chunk)
    constexpr int kCw = 8;
    uint32_t va[C::kMats][kCw], vb[C::kMats][kCw];
    const auto issue = [&](uint32_t (*v)[kCw], int c0) {
#pragma unroll
      for (int mt = 0; mt < C::kMats; ++mt) tmem_ld8_nowait(tb + mt * C::kAccCols + c0, v[mt]);
    };
    // swap-AB: this thread's row in the output rows of the tile's tokens, token
    // c of the tile at out_off + c * stride; WIDE: this thread's token, its
    // outputs m * 256 + c contiguous from out_off
    const size_t stride = GATEUP ? (size_t)a.I : (size_t)a.H;
    const size_t out_off = WIDE ? (size_t)(row0 + row) * stride + (size_t)m * C::kWRows
                                : (size_t)(row0 + nt * kBN) * stride + (size_t)wrow;
    const bool tok_ok = !WIDE || row < n_e;  // WIDE: lanes past the expert's rows store nothing
    const auto finish_wide = [&](uint32_t (*v)[kCw], int c0) {
      if (!tok_ok) return;
      if (GATEUP) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __nv_bfloat162 hv = __floats2bfloat162_rn(
              silu_mul_fast(__uint_as_float(v[0][2 * j]), __uint_as_float(v[1][2 * j])),
              silu_mul_fast(__uint_as_float(v[0][2 * j + 1]), __uint_as_float(v[1][2 * j + 1])));
          w[j] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(a.h + out_off + c0) = make_uint4(w[0], w[1], w[2], w[3]);
      } else {
        float4* yo = reinterpret_cast<float4*>(a.y + out_off + c0);
        yo[0] = make_float4(__uint_as_float(v[0][0]), __uint_as_float(v[0][1]), __uint_as_float(v[0][2]),
                            __uint_as_float(v[0][3]));
        yo[1] = make_float4(__uint_as_float(v[0][4]), __uint_as_float(v[0][5]), __uint_as_float(v[0][6]),
                            __uint_as_float(v[0][7]));
      }
    };
    const auto finish = [&](uint32_t (*v)[kCw], int c0) {
      if (WIDE) {
        finish_wide(v, c0);
        return;
      }
      const int valid = n_hi - c0;  // tokens of this chunk that exist (>= 1)
      size_t o = out_off + (size_t)c0 * stride;
#pragma unroll
      for (int j = 0; j < kCw; ++j, o += stride) {
        if (valid < kCw && j >= valid) break;
        if (GATEUP)
          a.h[o] = __float2bfloat16_rn(silu_mul_fast(__uint_as_float(v[0][j]), __uint_as_float(v[C::kMats - 1][j])));
        else
          a.y[o] = __uint_as_float(v[0][j]);
      }
    };
    // this warp's columns (tokens; WIDE: weight rows): chunks [wk n / W,
    // (wk + 1) n / W) of the n = 256 / 8
    constexpr int kChunks = C::kAccCols / kCw;
    const int c_lo = kCw * (wk * kChunks / C::kWorkersPerQuad);
    const int c_end = kCw * ((wk + 1) * kChunks / C::kWorkersPerQuad);
    const int c_hi = WIDE ? c_end : (n_hi < c_end ? n_hi : c_end);
    if (c_lo < c_hi) {
      issue(va, c_lo);
      tmem_wait_ld();
#pragma unroll 1
      for (int c0 = c_lo; c0 < c_hi; c0 += 2 * kCw) {
        if (c0 + kCw < c_hi) issue(vb, c0 + kCw);
        finish(va, c0);
        tmem_wait_ld();
        if (c0 + kCw >= c_hi) break;
        if (c0 + 2 * kCw < c_hi) issue(va, c0 + 2 * kCw);
        finish(vb, c0 + kCw);
        tmem_wait_ld();
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&acc_empty[buf]);
    return true;
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        int p, m, nt;
        int e = coords(tile, p, m, nt);
        if (!q4_check((unsigned)e < (unsigned)a.E, a.hdr + kStatus)) e = 0;
        const int wrow = e * rows_total + m * C::kWRows;
        const int brow = rt(a.offsets + e) + nt * C::kTRows;
        for (int ks = 0; ks < P.k_steps; ++ks, ++it) {
          const int s = it % C::kStagesT;
          const uint32_t ph = (it / C::kStagesT) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, kWaitLimitNs)) break;
          mbar_arrive_expect_tx(&full_c[s], C::kMats * C::kCTile);
          // codes: boxes of 128 rows (two per matrix for a 256-row WIDE tile)
#pragma unroll
          for (int h = 0; h < C::kWRows / kBM; ++h) {
            tma_load_2d(sC + (s * C::kMats) * C::kCTile + h * (kBM * kBK / 2), &tm_wa, &full_c[s], ks * (kBK / 2),
                        wrow + h * kBM);
            if (GATEUP)
              tma_load_2d(sC + (s * C::kMats + 1) * C::kCTile + h * (kBM * kBK / 2), &tm_wb, &full_c[s],
                          ks * (kBK / 2), wrow + h * kBM);
          }
          mbar_arrive_expect_tx(&full_b[s], C::kBTile);
          tma_load_2d(sB + s * C::kBTile, &tm_b, &full_b[s], ks * kBK, brow);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x, ++tcount) {
        int p, m, nt;
        const int e = coords(tile, p, m, nt);
        // swap-AB: M = 128 weight rows, N = the tile's tokens rounded up to 16;
        // WIDE: M = 128 token rows (padded), N = 256 weight rows
        const int left = rt(a.counts + e) - nt * kBN;  // tokens in this tile and after
        const int n_cols = left >= kBN ? kBN : ((left + 15) & ~15);
        const uint32_t idesc = WIDE ? umma_idesc_bf16(128, 256) : umma_idesc_bf16(kBM, n_cols);
        const int buf = (int)(tcount % C::kAccBufs);
        const uint32_t use = tcount / C::kAccBufs;  // earlier uses of this buffer
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, kWaitLimitNs)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * (C::kMats * C::kAccCols);
        bool ok = true;
        for (int ks = 0; ks < P.k_steps; ++ks, ++it) {
          const int s = it % C::kStagesT;
          const uint32_t ph = (it / C::kStagesT) & 1;
          const int w = it % C::kStagesW;
          const uint32_t wph = (it / C::kStagesW) & 1;
          if (!mbar_wait(&full_b[s], ph, abort_flag, kWaitLimitNs) ||
              !mbar_wait(&a_ready[w], wph, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t db = umma_desc_sw128(smem_u32(sB + s * C::kBTile));
#pragma unroll
          for (int mat = 0; mat < C::kMats; ++mat) {
            const uint64_t da = umma_desc_sw128(smem_u32(sA + (w * C::kMats + mat) * C::kATile));
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {  // +32 bytes of K per MMA (>> 4 -> +2)
              if (WIDE)  // A: the token tile, B: the weights
                umma_bf16(d0 + mat * C::kAccCols, db + 2 * kk, da + 2 * kk, idesc, (ks | kk) != 0);
              else
                umma_bf16(d0 + mat * C::kAccCols, da + 2 * kk, db + 2 * kk, idesc, (ks | kk) != 0);
            }
          }
          umma_commit(&a_empty[w]);
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
      }
      // all MMAs issued by this thread complete before TMEM is released
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, abort_flag, kWaitLimitNs);
    }
  } else if (warp < C::kEpiWarp0) {
    // ---------------- dequantise ----------------
    const int d = threadIdx.x - 64;           // 0 .. kDequantThreads - 1
    const int r = d & (C::kWRows - 1);        // weight row in the tile
    const int my_half = WIDE ? -1 : (d >> 7) & 1;  // 32-weight half of the row's 64 K (WIDE: both)
    const int mat = GATEUP ? (d >> 8) : 0;    // gate / up
    // drain worker index of this warp in its TMEM lane quarter (after the
    // epilogue warps'); it helps drain tile n while working on tile n + 1,
    // once the ring is full and the MMA waits for that drain
    const int help_wk = C::kEpiWarps / 4 + ((warp - 2) >> 2);
    const int help_at = P.k_steps - 1 < C::kStagesW ? P.k_steps - 1 : C::kStagesW;
    int prev_tile = -1;
    uint32_t it = 0, tcount = 0;
    for (int tile = blockIdx.x; tile < total && !warp_aborted(abort_flag); tile += gridDim.x, ++tcount) {
      int p, m, nt;
      int e = coords(tile, p, m, nt);
      if (!q4_check((unsigned)e < (unsigned)a.E, a.hdr + kStatus)) e = 0;
      const Planes PL = make_planes(tp.t[tp.id[e]]);
      const uint8_t* srow = (GATEUP ? (mat ? a.up_s : a.gate_s) : a.down_s) +
                            ((size_t)e * rows_total + m * C::kWRows + r) * (size_t)(K / 32);
      // scale bytes of blocks 2ks .. 2ks+3 (k-steps ks, ks+1) as one 4-byte word
      // (K % 128 == 0 keeps every word inside the row and aligned), loaded three
      // words ahead of use so the loads' latency hides behind the decode
      const uint32_t* sw32 = reinterpret_cast<const uint32_t*>(srow);
      const int n_sw = P.k_steps / 2;
      uint32_t q0 = sw32[0], q1 = n_sw > 1 ? sw32[1] : 0u, q2 = n_sw > 2 ? sw32[2] : 0u;
      uint32_t sc = 0;
      bool ok = true;
      for (int ks = 0; ks < P.k_steps; ++ks, ++it) {
        if (C::kHelp && ks == help_at && prev_tile >= 0 && !drain(prev_tile, tcount - 1, help_wk)) {
          ok = false;
          break;
        }
        if ((ks & 1) == 0) {
          sc = q0;
          q0 = q1;
          q1 = q2;
          q2 = (ks >> 1) + 3 < n_sw ? sw32[(ks >> 1) + 3] : 0u;
        }
        const int s = it % C::kStagesT;
        const uint32_t ph = (it / C::kStagesT) & 1;
        const int w = it % C::kStagesW;
        const uint32_t wph = (it / C::kStagesW) & 1;
        // the codes have landed and the weight stage is free (its previous
        // contents consumed by the MMAs)
        if (!mbar_wait_warp(&full_c[s], ph, abort_flag, kWaitLimitNs) ||
            !mbar_wait_warp(&a_empty[w], wph ^ 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        const uint8_t* ctile = sC + (s * C::kMats + mat) * C::kCTile;
        uint8_t* arow = sA + (w * C::kMats + mat) * C::kATile + r * 128;
        // 32-byte swizzle of the codes tile: chunk c of row r at c ^ ((r >> 2) & 1)
        const int sw = (r >> 2) & 1;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!WIDE && half != my_half) continue;
          const uint4 cv = *reinterpret_cast<const uint4*>(ctile + r * 32 + ((half ^ sw) << 4));
          const int blk = 2 * (ks & 1) + half;  // block within the 4 loaded
          const uint32_t sbyte = (sc >> (blk * 8)) & 0xffu;
          uint32_t w16[16];
          const uint32_t s2 = scale_bf16x2(sbyte);
          decode8(cv.x, PL, &w16[0]);
          decode8(cv.y, PL, &w16[4]);
          decode8(cv.z, PL, &w16[8]);
          decode8(cv.w, PL, &w16[12]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {  // 16-byte chunks 4*half + q of the row, 128-byte swizzle
            const int ch = 4 * half + q;
            uint4 v = make_uint4(bf16x2_mul(w16[4 * q], s2), bf16x2_mul(w16[4 * q + 1], s2),
                                 bf16x2_mul(w16[4 * q + 2], s2), bf16x2_mul(w16[4 * q + 3], s2));
            *reinterpret_cast<uint4*>(arow + ((ch ^ (r & 7)) << 4)) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_ready[w]);
      }
      if (!ok) break;
      prev_tile = tile;
    }
    // the CTA's last tile: no next tile to overlap with, drain it beside the epilogue
    if (C::kHelp && prev_tile >= 0 && !warp_aborted(abort_flag)) drain(prev_tile, tcount - 1, help_wk);
  } else {
    // ---------------- epilogue ----------------
    const int ehalf = (warp - C::kEpiWarp0) >> 2;  // drain worker 0 or 1 of its TMEM lane quarter
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < total && !warp_aborted(abort_flag); tile += gridDim.x, ++tcount)
      if (!drain(tile, tcount, ehalf)) break;
  }

  // ---------------- teardown ----------------
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) record_error(a.hdr + kStatus, MOE_Q4_ETIMEOUT);
  if (warp == 0 && lane == 0 && *abort_flag) {
    // let any copy still in flight land before the CTA's smem goes away
    for (int s = 0; s < C::kStagesT; ++s) {
      volatile int quick = 0;
      mbar_wait(&full_c[s], 0, &quick, 50000000ull);
      quick = 0;
      mbar_wait(&full_c[s], 1, &quick, 50000000ull);
      quick = 0;
      mbar_wait(&full_b[s], 0, &quick, 50000000ull);
      quick = 0;
      mbar_wait(&full_b[s], 1, &quick, 50000000ull);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  // the WIDE kernel completes only after the swap-AB grid before it
  if (WIDE) pdl_wait();
  // triggered at the end (unless early, above): the next kernel's CTAs (shared
  // memory near the SM's limit) could not share an SM with this one anyway, and
  // launching them while this persistent grid still runs measured slower
  pdl_trigger();
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
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

// 2-D map over a row-major [rows][cols] array.
static bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t cols,
                     uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool GATEUP, bool WIDE>
static int launch_tc(const FwdArgs& a, const TableParams& tp, cudaStream_t s, bool wide_next) {
  using C = TcCfg<GATEUP, WIDE>;
  TcParams P;
  P.a = a;
  P.m_tiles = (GATEUP ? a.I : a.H) / C::kWRows;
  P.k_steps = (GATEUP ? a.H : a.I) / kBK;
  P.early_trigger = !WIDE && wide_next;
  const int R = a.T * a.k;
  CUtensorMap tb, twa, twb;
  bool ok;
  if (GATEUP) {
    ok = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.xg, a.H, R, kBK, C::kTRows,
                  CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_map(&twa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.gate_w, a.H / 2, (uint64_t)a.E * a.I, kBK / 2, kBM,
                  CU_TENSOR_MAP_SWIZZLE_32B) &&
         make_map(&twb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.up_w, a.H / 2, (uint64_t)a.E * a.I, kBK / 2, kBM,
                  CU_TENSOR_MAP_SWIZZLE_32B);
  } else {
    ok = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.h, a.I, R, kBK, C::kTRows,
                  CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_map(&twa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.down_w, a.I / 2, (uint64_t)a.E * a.H, kBK / 2, kBM,
                  CU_TENSOR_MAP_SWIZZLE_32B);
    twb = twa;
  }
  if (!ok) return MOE_Q4_ECUDA;
  if (cudaFuncSetAttribute(tc_gemm_kernel<GATEUP, WIDE>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
      cudaSuccess)
    return MOE_Q4_ECUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_gemm_kernel<GATEUP, WIDE>, P, tp, tb, twa, twb) == cudaSuccess ? MOE_Q4_OK
                                                                                                      : MOE_Q4_ECUDA;
}

}  // namespace q4

using namespace q4;

int q4_prefill_tile_n() { return kBN; }

int q4_prefill_wide_max() { return 128; }

int q4_launch_prefill(const FwdArgs& a, const TableParams& tp, bool gateup, bool wide_next, cudaStream_t s) {
  return gateup ? launch_tc<true, false>(a, tp, s, wide_next) : launch_tc<false, false>(a, tp, s, wide_next);
}

int q4_launch_prefill_wide(const FwdArgs& a, const TableParams& tp, bool gateup, cudaStream_t s) {
  return gateup ? launch_tc<true, true>(a, tp, s, false) : launch_tc<false, true>(a, tp, s, false);
}
