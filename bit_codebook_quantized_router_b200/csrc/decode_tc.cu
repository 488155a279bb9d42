// Small-M ("decode") expert GEMMs on tcgen05 with the A operand in TMEM.
//
//   gate/up: h[row] = silu(W_gate x) * (W_up x)   (experts with <= 16 rows)
//   down:    y[row] = W_down h[row]
// ("Round 7 -- Rewrite the GLM-5.2 routed-expert encoder", "Owner-locked
// decisions" 4 and 6.)  The packed weights are streamed from HBM once per
// call; the rest is arranged so the stream never waits:
//
// * Work split.  A unit is (expert on this path, tile of 128 weight rows);
//   the units' stages (256 weights of K each, 128 if K % 256 != 0) form one
//   sequence that the persistent CTAs (one per SM) cut into equal contiguous
//   ranges, so every SM streams the same number of bytes.  A tile whose K
//   range spans several CTAs is finished by the last of them to arrive (a
//   per-tile counter): it adds the partial sums in K order (deterministic)
//   and writes the result.
// * Data movement: per stage and matrix one TMA brings 128 weight rows x 128
//   bytes of codes (a full 128-byte line per row: narrower boxes stream at a
//   fraction of HBM bandwidth) with the 128-byte swizzle; TMA brings the
//   activation rows (grouped by expert, 128 bytes per row per 64 K); the
//   producer warp's lanes copy each row's scale bytes for the stage with
//   cp.async, completing on the stage's barrier.
// * Decode ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", "Codes are indices
//   into the per-layer grid"): one thread per weight row.  Most code bytes
//   are looked up in a shared-memory table byte -> signed bf16 pair (256
//   entries, one copy per lane so a warp's 32 lookups hit 32 banks; the
//   entry address is one PRMT of the code word); a few words per sub-step
//   use the in-register PRMT byte-plane decode instead, to balance the
//   integer pipe against shared-memory bandwidth.  The E8M0 block scale is
//   one exact bf16x2 multiply.  Each 64-K sub-step goes to TMEM (tcgen05.st).
// * MMA: tcgen05.mma kind::f16, M = 128 weight rows (A from TMEM), N = 16
//   token columns (gate/up) or 2 x hrows (down: hrows rows of h, then the
//   same rows of its low part h_lo; hrows = 8 when no expert can hold more
//   than 8 rows), K = 16 per instruction, fp32 accumulators in TMEM
//   (double-buffered per segment).
//
// Warps: 0 producer, 1 TMEM allocation + MMA issue, 2..9 decode (two
// matrices or two K halves x four TMEM lane quarters), 10..13 epilogue.
// Every wait is bounded (a timeout sets MOE_Q4_ETIMEOUT in the status word and
// the CTA drains and exits); warps wait and leave together (vote).
#include <cuda.h>

#include "q4_api_internal.h"
#include "q4_common.cuh"
#include "sm100.cuh"

namespace q4 {

using namespace sm100;

namespace dk {
constexpr int kThreads = 448;
constexpr int kRows = 128;         // weight rows per tile = MMA M
constexpr int kSubK = 64;          // K per sub-step (one TMEM A stage)
constexpr int kTok = 16;           // token columns kept per expert
constexpr int kMaxRing = 6;        // shared-memory stages, at most
constexpr int kAStages = 4;        // TMEM A stages
constexpr int kDecWarps = 8;
constexpr int kEpiWarp0 = 10;
constexpr int kPrmtWords = 3;      // of every 8 code words, decoded in registers (rest: table)
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kLutBytes = 65536;  // 256 entries x (2 table slots x 32 lanes x 4 B)
constexpr uint32_t kScaleSlot = 8;     // scale bytes per row per stage (4 used when a stage is 128 K)
constexpr uint32_t kBarBytes = 1024;   // barriers and flags
}  // namespace dk

// Shared-memory placement (addresses in the CTA's shared window).  The table
// sits at a 64 KB boundary so its entry addresses can be formed by one PRMT;
// the activation and scale rings and the barriers go below it when the gap
// holds them, the code ring above it.  Host and device compute the same
// placement from the window's start `raw`.
struct DkLayout {
  uint32_t lut, codes, x, scales, bars, end;
};

__host__ __device__ inline DkLayout dk_layout(uint32_t raw, uint32_t code_stage, uint32_t x_stage,
                                              uint32_t scale_stage, int ring) {
  DkLayout L;
  L.lut = (raw + 65535u) & ~65535u;
  L.codes = L.lut + dk::kLutBytes;
  const uint32_t codes_end = L.codes + (uint32_t)ring * code_stage;
  const uint32_t others = (uint32_t)ring * (x_stage + scale_stage) + dk::kBarBytes;
  const uint32_t o = (raw + 1023u) & ~1023u;
  if (o + others <= L.lut) {
    L.x = o;
    L.end = codes_end;
  } else {
    L.x = codes_end;
    L.end = codes_end + others;
  }
  L.scales = L.x + (uint32_t)ring * x_stage;
  L.bars = L.scales + (uint32_t)ring * scale_stage;
  return L;
}

struct DkParams {
  FwdArgs a;
  int tiles_per_e;  // weight rows / 128
  int subs;         // 64-K sub-steps per stage: 4 (K % 256 == 0) or 2
  int stages;       // stages per tile: K / (64 * subs)
  int ring;         // shared-memory stages
  int hrows;        // rows per activation box: 16 (gate/up), 8 or 16 (down)
  int n_max;        // token columns kept in partial sums: min(16, T)
  uint32_t code_stage, x_stage, scale_stage;  // bytes per stage
  float* partial;   // [2 * gridDim.x][mats][n_max][128]
  int32_t* counter; // [units], zero at launch
};

__device__ __forceinline__ long long dk_range(int b, long long total, int G) { return (long long)b * total / G; }

// CTA whose range holds stage g.
__device__ __forceinline__ int dk_owner(long long g, long long total, int G) {
  int b = (int)((g * G) / total);
  while (b + 1 < G && dk_range(b + 1, total, G) <= g) ++b;
  while (b > 0 && dk_range(b, total, G) > g) --b;
  return b;
}

// CTAs holding part of [us, ue): the owners of its ends and every non-empty
// range between them (with fewer stages than CTAs some ranges are empty).
__device__ __forceinline__ int dk_contributors(long long us, long long ue, long long total, int G, int& c_first,
                                               int& c_last) {
  c_first = dk_owner(us, total, G);
  c_last = dk_owner(ue - 1, total, G);
  int n = 0;
  for (int c = c_first; c <= c_last; ++c) n += dk_range(c + 1, total, G) > dk_range(c, total, G);
  return n;
}

__device__ __forceinline__ void ring_next(int& s, uint32_t& ph, int n) {
  if (++s == n) {
    s = 0;
    ph ^= 1u;
  }
}

template <bool GATEUP>
__global__ void __launch_bounds__(dk::kThreads, 1)
    dk_kernel(const __grid_constant__ DkParams P, const __grid_constant__ TableParams tp,
              const __grid_constant__ CUtensorMap tm_wa, const __grid_constant__ CUtensorMap tm_wb,
              const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xl) {
  constexpr int kMats = GATEUP ? 2 : 1;
  constexpr int kACols = dk::kSubK / 2;  // TMEM columns per matrix per A stage
  constexpr uint32_t kTmemCols = GATEUP ? 512 : 256;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const DkLayout Ls = dk_layout(raw_s, P.code_stage, P.x_stage, P.scale_stage, P.ring);
  const FwdArgs& a = P.a;
  if (Ls.end > raw_s + dynamic_smem_size()) {  // launched with less shared memory than the layout needs
    if (threadIdx.x == 0) record_error(a.hdr + kStatus, MOE_Q4_ECUDA);
    return;
  }
  uint8_t* lut = smem_raw + (Ls.lut - raw_s);
  uint8_t* sCode = smem_raw + (Ls.codes - raw_s);    // [ring][mats][128 rows x row_bytes], swizzled
  uint8_t* sX = smem_raw + (Ls.x - raw_s);           // [ring][subs][N rows x 128 B], 128-byte swizzle
  uint8_t* sScale = smem_raw + (Ls.scales - raw_s);  // [ring][mats][128 rows][8 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + (Ls.bars - raw_s));
  uint64_t* full = bars;                             // [ring] codes + activations (TMA), scales (cp.async)
  uint64_t* stage_empty = full + dk::kMaxRing;       // [ring] decoders done with codes/scales, MMAs with x
  uint64_t* a_full = stage_empty + dk::kMaxRing;     // [AS] decoded sub-step in TMEM
  uint64_t* a_empty = a_full + dk::kAStages;         // [AS] MMAs done with the A stage
  uint64_t* acc_full = a_empty + dk::kAStages;       // [2]
  uint64_t* acc_empty = acc_full + 2;                // [2]
  uint64_t* drain = acc_empty + 2;
  uint64_t* lut_bar = drain + 1;                     // decoders rebuilding a table slot
  uint64_t* epi_bar = lut_bar + 1;                   // epilogue threads of a split tile
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;

  const int ring = P.ring;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < ring; ++s) {
      mbar_init(&full[s], 1 + 32);  // producer lane 0 (with the TMA bytes) + 32 cp.async arrivals
      mbar_init(&stage_empty[s], dk::kDecWarps + 1);
    }
    for (int q = 0; q < dk::kAStages; ++q) {
      mbar_init(&a_full[q], dk::kDecWarps);
      mbar_init(&a_empty[q], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    mbar_init(lut_bar, dk::kDecWarps * 32);
    mbar_init(epi_bar, 128);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_wa);
    if (GATEUP) prefetch_tmap(&tm_wb);
    prefetch_tmap(&tm_x);
    if (!GATEUP) prefetch_tmap(&tm_xl);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tA = tmem;                                      // A ring
  const uint32_t tAcc = tmem + dk::kAStages * kMats * kACols;    // accumulators

  pdl_wait();
  const int n_dec = a.hdr[kNumDecode];
  const int rows_total = GATEUP ? a.I : a.H;
  const int K = GATEUP ? a.H : a.I;
  const int subs = P.subs;
  const int row_bytes = 32 * subs;                 // code bytes per row per stage
  const int hrows = P.hrows;
  const int n_cols = GATEUP ? dk::kTok : 2 * hrows;  // MMA N
  const uint32_t x_sub = (uint32_t)n_cols * 128u;   // activation bytes per sub-step
  const long long total = (long long)n_dec * P.tiles_per_e * P.stages;
  const int G = gridDim.x, b = blockIdx.x;
  const long long k0 = dk_range(b, total, G), k1 = dk_range(b + 1, total, G);

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (long long g = k0; g < k1 && ok;) {
      const int unit = (int)(g / P.stages);
      const int st0 = (int)(g - (long long)unit * P.stages);
      const long long seg_end = min(k1, (long long)(unit + 1) * P.stages);
      const int e = a.dec_list[unit / P.tiles_per_e];
      const int t = unit % P.tiles_per_e;
      const int row0 = a.offsets[e];
      const int wrow = e * rows_total + t * dk::kRows;
      for (int st = st0; st < st0 + (int)(seg_end - g); ++st) {
        if (!mbar_wait_warp(&stage_empty[s], ph ^ 1, abort_flag, dk::kWaitNs)) {
          ok = false;
          break;
        }
        // scale bytes of the stage (2 per 64-K sub-step) for 4 rows per lane
#pragma unroll
        for (int m = 0; m < kMats; ++m) {
          const uint8_t* sbase = (GATEUP ? (m ? a.up_s : a.gate_s) : a.down_s) + (size_t)wrow * (K / 32) +
                                 (size_t)st * 2 * subs;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = lane + 32 * j;
            const uint32_t dst = Ls.scales + (uint32_t)s * P.scale_stage + (uint32_t)(m * dk::kRows + r) * dk::kScaleSlot;
            if (subs == 4)
              cp_async_small<8>(dst, sbase + (size_t)r * (K / 32));
            else
              cp_async_small<4>(dst, sbase + (size_t)r * (K / 32));
          }
        }
        cp_async_arrive_noinc(&full[s]);
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], kMats * dk::kRows * row_bytes + subs * x_sub);
          uint8_t* cdst = sCode + (size_t)s * P.code_stage;
          tma_load_2d(cdst, &tm_wa, &full[s], st * row_bytes, wrow);
          if (GATEUP) tma_load_2d(cdst + dk::kRows * row_bytes, &tm_wb, &full[s], st * row_bytes, wrow);
          // the expert's activation rows, grouped; rows past n_e belong to the next
          // expert or lie past the end: they only feed MMA columns the epilogue drops
          uint8_t* xdst = sX + (size_t)s * P.x_stage;
          for (int j = 0; j < subs; ++j) {
            const int kx = (st * subs + j) * dk::kSubK;
            tma_load_2d(xdst + j * x_sub, &tm_x, &full[s], kx, row0);
            if (!GATEUP) tma_load_2d(xdst + j * x_sub + hrows * 128, &tm_xl, &full[s], kx, row0);
          }
        }
        __syncwarp();
        ring_next(s, ph, ring);
      }
      g = seg_end;
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issue ------------------------------
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(dk::kRows, n_cols);
      int s = 0, q = 0;
      uint32_t ph = 0, qph = 0, seg = 0;
      bool ok = true;
      for (long long g = k0; g < k1 && ok; ++seg) {
        const int unit = (int)(g / P.stages);
        const long long seg_end = min(k1, (long long)(unit + 1) * P.stages);
        const int nst = (int)(seg_end - g);
        const int buf = seg & 1;
        if (!mbar_wait(&acc_empty[buf], ((seg >> 1) & 1) ^ 1, abort_flag, dk::kWaitNs)) break;
        tc_fence_after();
        for (int j = 0; j < nst && ok; ++j) {
          if (!mbar_wait(&full[s], ph, abort_flag, dk::kWaitNs)) {
            ok = false;
            break;
          }
          for (int u = 0; u < subs; ++u) {
            if (!mbar_wait(&a_full[q], qph, abort_flag, dk::kWaitNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t xd = umma_desc_sw128(smem_u32(sX + (size_t)s * P.x_stage + u * x_sub));
#pragma unroll
            for (int m = 0; m < kMats; ++m) {
              const uint32_t dacc = tAcc + (buf * kMats + m) * n_cols;
              const uint32_t da = tA + (q * kMats + m) * kACols;
#pragma unroll
              for (int kk = 0; kk < dk::kSubK / 16; ++kk)  // 16 K = 8 TMEM columns of A, 32 bytes of x
                umma_bf16_ts(dacc, da + kk * 8, xd + 2 * kk, idesc, (j | u | kk) != 0);
            }
            umma_commit(&a_empty[q]);
            ring_next(q, qph, dk::kAStages);
          }
          if (!ok) break;
          umma_commit(&stage_empty[s]);
          ring_next(s, ph, ring);
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
        g = seg_end;
      }
      // every MMA issued has finished before TMEM is released
      umma_commit(drain);
      volatile int own = 0;
      mbar_wait(drain, 0, &own, dk::kWaitNs);
    }
  } else if (warp < dk::kEpiWarp0) {
    // ------------------------------ decode ------------------------------
    const int dw = warp - 2;           // 0..7
    const int part = dw >> 2;          // gate/up: matrix; down: K half of a sub-step
    const int quad = warp & 3;         // TMEM lane quarter
    const int r = quad * 32 + lane;    // weight row in the tile
    const int dtid = threadIdx.x - 64; // 0..255
    const int mat = GATEUP ? part : 0;
    // 128-byte rows: chunk c at c ^ (r & 7); 64-byte rows: c ^ ((r >> 1) & 3)
    const int swz = subs == 4 ? (r & 7) : ((r >> 1) & 3);
    // table slots: which table each of the 2 slots holds (the same decisions in
    // every decoder thread: they walk the same segments)
    int slot_tab0 = -1, slot_tab1 = -1, victim = 0;
    uint32_t lgen = 0;
    const uint32_t lane_k = (Ls.lut & 0xffff0000u) | ((uint32_t)lane << 2);
    int s = 0, q = 0;
    uint32_t ph = 0, qph = 0;
    bool ok = true;
    for (long long g = k0; g < k1 && ok;) {
      const int unit = (int)(g / P.stages);
      const long long seg_end = min(k1, (long long)(unit + 1) * P.stages);
      const int nst = (int)(seg_end - g);
      const int e = a.dec_list[unit / P.tiles_per_e];
      const int tid = tp.id[e];
      int slot = tid == slot_tab0 ? 0 : (tid == slot_tab1 ? 1 : -1);
      if (slot < 0) {
        // (re)build a slot: entry c -> bf16 pair of codes (c & 15, c >> 4), signed,
        // unscaled, copied for all 32 lanes.  Bounded barriers on both sides: every
        // decoder is done with the old contents before any write, and all writes
        // land before anyone reads.
        mbar_arrive(lut_bar);
        if (!mbar_wait_warp(lut_bar, lgen & 1, abort_flag, dk::kWaitNs)) break;
        ++lgen;
        slot = victim;
        victim ^= 1;
        if (slot == 0)
          slot_tab0 = tid;
        else
          slot_tab1 = tid;
        const float* tv = tp.t[tid];
        const uint32_t lo = dtid & 15, hi = dtid >> 4;
        const uint32_t blo = (uint32_t)bf16_bits_rn(tv[lo & 7]) ^ ((lo & 8) ? 0x8000u : 0u);
        const uint32_t bhi = (uint32_t)bf16_bits_rn(tv[hi & 7]) ^ ((hi & 8) ? 0x8000u : 0u);
        const uint32_t word = blo | (bhi << 16);
        uint4* dst = reinterpret_cast<uint4*>(lut + dtid * 256 + slot * 128);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_uint4(word, word, word, word);
        mbar_arrive(lut_bar);
        if (!mbar_wait_warp(lut_bar, lgen & 1, abort_flag, dk::kWaitNs)) break;
        ++lgen;
      }
      const uint32_t kreg = lane_k | ((uint32_t)slot << 7);
      const Planes PL = make_planes(tp.t[tid]);
      for (int j = 0; j < nst && ok; ++j) {
        if (!mbar_wait_warp(&full[s], ph, abort_flag, dk::kWaitNs)) {
          ok = false;
          break;
        }
        // this row's scale bytes for the stage (2 per sub-step)
        const uint2 scs = *reinterpret_cast<const uint2*>(sScale + (size_t)s * P.scale_stage +
                                                          (size_t)(mat * dk::kRows + r) * dk::kScaleSlot);
        const uint8_t* crow = sCode + (size_t)s * P.code_stage + (size_t)(mat * dk::kRows + r) * row_bytes;
        for (int u = 0; u < subs; ++u) {
          // code chunks 2u, 2u+1 of the row (down: this thread's chunk 2u + part)
          uint32_t cw[8];
          if (GATEUP) {
            const uint4 c0 = *reinterpret_cast<const uint4*>(crow + (((2 * u) ^ swz) << 4));
            const uint4 c1 = *reinterpret_cast<const uint4*>(crow + (((2 * u + 1) ^ swz) << 4));
            cw[0] = c0.x; cw[1] = c0.y; cw[2] = c0.z; cw[3] = c0.w;
            cw[4] = c1.x; cw[5] = c1.y; cw[6] = c1.z; cw[7] = c1.w;
          } else {
            const uint4 c0 = *reinterpret_cast<const uint4*>(crow + (((2 * u + part) ^ swz) << 4));
            cw[0] = c0.x; cw[1] = c0.y; cw[2] = c0.z; cw[3] = c0.w;
            cw[4] = cw[5] = cw[6] = cw[7] = 0u;
          }
          constexpr int kWords = GATEUP ? 8 : 4;
          constexpr int kPrmt = GATEUP ? dk::kPrmtWords : (dk::kPrmtWords + 1) / 2;
          uint32_t v[32];
#pragma unroll
          for (int wi = 0; wi < kWords; ++wi) {
            const uint32_t w = cw[wi];
            if (wi < kPrmt) {
              decode8(w, PL, &v[4 * wi]);
            } else {
              // table entry address = table | byte << 8 | slot << 7 | lane << 2
              v[4 * wi + 0] = lds32(prmt(w, kreg, 0x7604));
              v[4 * wi + 1] = lds32(prmt(w, kreg, 0x7614));
              v[4 * wi + 2] = lds32(prmt(w, kreg, 0x7624));
              v[4 * wi + 3] = lds32(prmt(w, kreg, 0x7634));
            }
          }
          // E8M0 scales: sub-step u covers blocks 2u (gate/up words 0-3; down part 0)
          // and 2u+1 (gate/up words 4-7; down part 1): bytes 2u, 2u+1 of the stage
          const uint32_t sw2 = u < 2 ? scs.x : scs.y;
          const int sh = (u & 1) * 16;
          const uint32_t s_lo = scale_bf16x2((sw2 >> (sh + (GATEUP ? 0 : 8 * part))) & 0xffu);
          const uint32_t s_hi = scale_bf16x2((sw2 >> (sh + 8)) & 0xffu);
#pragma unroll
          for (int i = 0; i < 4 * kWords; ++i) v[i] = bf16x2_mul(v[i], (GATEUP && i >= 16) ? s_hi : s_lo);
          if (!mbar_wait_warp(&a_empty[q], qph ^ 1, abort_flag, dk::kWaitNs)) {
            ok = false;
            break;
          }
          const uint32_t ta = tA + (q * kMats + mat) * kACols + ((uint32_t)(quad * 32) << 16);
          if (GATEUP)
            tmem_st32(ta, v);
          else
            tmem_st16(ta + part * 16, v);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[q]);
          ring_next(q, qph, dk::kAStages);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&stage_empty[s]);
        ring_next(s, ph, ring);
      }
      g = seg_end;
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int etid = threadIdx.x - dk::kEpiWarp0 * 32;  // 0..127
    uint32_t seg = 0, egen = 0;
    for (long long g = k0; g < k1 && !warp_aborted(abort_flag); ++seg) {
      const int unit = (int)(g / P.stages);
      const long long ustart = (long long)unit * P.stages, uend = ustart + P.stages;
      const long long seg_end = min(k1, uend);
      const int e = a.dec_list[unit / P.tiles_per_e];
      const int t = unit % P.tiles_per_e;
      const int row0 = a.offsets[e], n_e = a.counts[e];
      const int buf = seg & 1;
      if (!mbar_wait_warp(&acc_full[buf], (seg >> 1) & 1, abort_flag, dk::kWaitNs)) break;
      tc_fence_after();
      const uint32_t tr = tAcc + buf * kMats * n_cols + ((uint32_t)(quad * 32) << 16);
      float acc[kMats][dk::kTok];
      if (GATEUP) {
        tmem_ld16(tr, acc[0]);
        tmem_ld16(tr + n_cols, acc[kMats - 1]);
      } else if (hrows == 16) {
        float lo[16];
        tmem_ld16(tr, acc[0]);
        tmem_ld16(tr + 16, lo);
#pragma unroll
        for (int n = 0; n < 16; ++n) acc[0][n] += lo[n];
      } else {  // columns 0..7 h, 8..15 h_lo
        float v[16];
        tmem_ld16(tr, v);
#pragma unroll
        for (int n = 0; n < 16; ++n) acc[0][n] = n < 8 ? v[n] + v[n + 8] : 0.0f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      const int wr = t * dk::kRows + r;  // row within the expert's matrix
      const bool final_here = (g == ustart && seg_end == uend);
      if (!final_here) {
        // partial: slot 2b (segment starts this CTA's range) or 2b+1 (its last)
        const int slot = (g == k0) ? 2 * b : 2 * b + 1;
        float* pp = P.partial + (size_t)slot * kMats * P.n_max * dk::kRows;
#pragma unroll
        for (int m = 0; m < kMats; ++m)
#pragma unroll
          for (int n = 0; n < dk::kTok; ++n)
            if (n < P.n_max) pp[(m * P.n_max + n) * dk::kRows + r] = acc[m][n];
        __threadfence();
        mbar_arrive(epi_bar);
        if (!mbar_wait_warp(epi_bar, egen & 1, abort_flag, dk::kWaitNs)) break;
        ++egen;
        if (etid == 0) {
          int c_first, c_last;
          const int n_contrib = dk_contributors(ustart, uend, total, G, c_first, c_last);
          const int old = atomicAdd(&P.counter[unit], 1);
          *last_flag = (old == n_contrib - 1) ? 1 : 0;
        }
        mbar_arrive(epi_bar);
        if (!mbar_wait_warp(epi_bar, egen & 1, abort_flag, dk::kWaitNs)) break;
        ++egen;
        if (!*last_flag) {
          g = seg_end;
          continue;
        }
        __threadfence();
        // last arrival: add the partials of every CTA on this tile in K order
        int c_first, c_last;
        dk_contributors(ustart, uend, total, G, c_first, c_last);
#pragma unroll
        for (int m = 0; m < kMats; ++m)
#pragma unroll
          for (int n = 0; n < dk::kTok; ++n) acc[m][n] = 0.0f;
        for (int c = c_first; c <= c_last; ++c) {
          if (dk_range(c + 1, total, G) == dk_range(c, total, G)) continue;  // empty range
          const int sl = (c == c_first && dk_range(c, total, G) != ustart) ? 2 * c + 1 : 2 * c;
          const float* qp = P.partial + (size_t)sl * kMats * P.n_max * dk::kRows;
#pragma unroll
          for (int m = 0; m < kMats; ++m)
#pragma unroll
            for (int n = 0; n < dk::kTok; ++n)
              if (n < P.n_max) acc[m][n] += __ldcg(qp + (m * P.n_max + n) * dk::kRows + r);
        }
      }
      // finished tile: h (gate/up, as the bf16 pair h, h_lo) or y (down)
#pragma unroll
      for (int n = 0; n < dk::kTok; ++n) {
        if (n >= n_e) break;
        const size_t row = (size_t)row0 + n;
        if (GATEUP) {
          const float hv = silu_mul(acc[0][n], acc[kMats - 1][n]);
          const __nv_bfloat16 hb = __float2bfloat16_rn(hv);
          a.h[row * a.I + wr] = hb;
          a.h_lo[row * a.I + wr] = __float2bfloat16_rn(hv - __bfloat162float(hb));
        } else {
          a.y[row * a.H + wr] = acc[0][n];
        }
      }
      g = seg_end;
    }
  }

  // ------------------------------ teardown ------------------------------
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) record_error(a.hdr + kStatus, MOE_Q4_ETIMEOUT);
  if (warp == 0 && *abort_flag) {
    // copies still in flight land before the CTA's shared memory goes away
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0)
      for (int s = 0; s < ring; ++s)
        for (uint32_t par = 0; par < 2; ++par) {
          volatile int quick = 0;
          mbar_wait(&full[s], par, &quick, 20000000ull);
        }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  pdl_trigger();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn dk_encode() {
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

static bool dk_map(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t cols,
                   uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = dk_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool GATEUP>
static int launch_dk(const FwdArgs& a, const TableParams& tp, float* partial, int32_t* counter, int grid,
                     cudaStream_t s) {
  constexpr int kMats = GATEUP ? 2 : 1;
  DkParams P;
  P.a = a;
  const int K = GATEUP ? a.H : a.I;
  P.tiles_per_e = (GATEUP ? a.I : a.H) / dk::kRows;
  P.subs = (K % 256 == 0) ? 4 : 2;  // K % 128 == 0 always
  P.stages = K / (dk::kSubK * P.subs);
  P.n_max = a.T < dk::kTok ? a.T : dk::kTok;
  // an expert holds at most T rows: with T <= 8 the down GEMM needs 8 h rows
  P.hrows = (GATEUP || a.T > 8) ? 16 : 8;
  const int n_cols = GATEUP ? dk::kTok : 2 * P.hrows;
  P.code_stage = (uint32_t)(kMats * dk::kRows * 32 * P.subs);
  P.x_stage = (uint32_t)(P.subs * n_cols * 128);
  P.scale_stage = (uint32_t)(kMats * dk::kRows * dk::kScaleSlot);
  P.partial = partial;
  P.counter = counter;

  // deepest ring that fits; the dynamic window starts after the reserved bytes
  // (the kernel has no static shared memory)
  int dev = 0, reserved = 1024, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  P.ring = 0;
  uint32_t smem = 0;
  for (int rs = dk::kMaxRing; rs >= 2 && !P.ring; --rs) {
    const DkLayout L = dk_layout((uint32_t)reserved, P.code_stage, P.x_stage, P.scale_stage, rs);
    if (L.end - (uint32_t)reserved <= (uint32_t)optin) {
      P.ring = rs;
      smem = L.end - (uint32_t)reserved;
    }
  }
  if (!P.ring) return MOE_Q4_ECUDA;

  const int R = a.T * a.k;
  const CUtensorMapSwizzle csw = P.subs == 4 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const uint32_t cbox = 32u * P.subs;
  CUtensorMap twa, twb, tx, txl;
  bool ok;
  if (GATEUP) {
    ok = dk_map(&twa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.gate_w, a.H / 2, (uint64_t)a.E * a.I, cbox, dk::kRows, csw) &&
         dk_map(&twb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.up_w, a.H / 2, (uint64_t)a.E * a.I, cbox, dk::kRows, csw) &&
         dk_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.xg, a.H, R, dk::kSubK, dk::kTok,
                CU_TENSOR_MAP_SWIZZLE_128B);
    txl = tx;
  } else {
    ok = dk_map(&twa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.down_w, a.I / 2, (uint64_t)a.E * a.H, cbox, dk::kRows,
                csw) &&
         dk_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.h, a.I, R, dk::kSubK, P.hrows,
                CU_TENSOR_MAP_SWIZZLE_128B) &&
         dk_map(&txl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.h_lo, a.I, R, dk::kSubK, P.hrows,
                CU_TENSOR_MAP_SWIZZLE_128B);
    twb = twa;
  }
  if (!ok) return MOE_Q4_ECUDA;
  if (cudaFuncSetAttribute(dk_kernel<GATEUP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MOE_Q4_ECUDA;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(dk::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dk_kernel<GATEUP>, P, tp, twa, twb, tx, txl) == cudaSuccess ? MOE_Q4_OK
                                                                                             : MOE_Q4_ECUDA;
}

}  // namespace q4

using namespace q4;

int q4_launch_decode_tc(const FwdArgs& a, const TableParams& tp, bool gateup, float* partial, int32_t* counter,
                        int grid, cudaStream_t s) {
  if (a.T * a.k == 0) return MOE_Q4_OK;
  return gateup ? launch_dk<true>(a, tp, partial, counter, grid, s) : launch_dk<false>(a, tp, partial, counter, grid, s);
}
