// Small-M ("decode") expert GEMMs: the packed weights of experts with at most
// 16 rows, streamed from HBM once per call and decoded straight into MMA
// operand registers.
//
//   gate/up: h[row] = silu(W_gate x) * (W_up x)
//   down:    y[row] = W_down h[row]
// ("Round 7 -- Rewrite the GLM-5.2 routed-expert encoder", "Owner-locked
// decisions" 4 and 6.)
//
// * Work split.  A unit is (expert on this path, 128 weight rows of gate and
//   of up, or 256 rows of down as two 128-row tiles), so a stage carries 256
//   rows of codes in both kernels and the fixed cost of a stage (barriers,
//   activation and scale reads) is spread over the same bytes; the units' stages (256 weights of K each, 128 if K % 256 != 0) form one
//   sequence that the persistent CTAs (one per SM) cut into equal contiguous
//   ranges, so every SM streams the same number of bytes.  A tile whose K
//   range spans several CTAs is finished by the last of them to arrive (a
//   per-tile counter): it adds the partial sums in K order (deterministic)
//   and writes the result.
// * Data movement (warp 0): per stage and 128-row tile one TMA brings 128
//   weight rows x 128 bytes of codes (a full 128-byte line per row: narrower
//   boxes stream at a fraction of HBM bandwidth) with the 128-byte swizzle;
//   the warp's lanes copy each row's scale bytes for the stage with cp.async
//   and the expert's activation rows (x through the row -> token map for
//   gate/up, h and h_lo for down) by untiled bulk copies, all completing on
//   the stage barrier.
// * Decode + MMA (warps 1..8): warp s owns weight rows 16s..16s+15 of the
//   tile.  In each 128-K half of a stage, lane (g, t) reads the 16-byte code
//   chunk t of rows g and g+8 (32 weights, one E8M0 block), decodes it to bf16 pairs ("aidendle94/GLM-5.2-NF4-Lloyd-
//   Experts-GPTQ", "Codes are indices into the per-layer grid") and feeds
//   them to mma.sync m16n8k16 as the A operand.  K is permuted inside each
//   128-K half, the same way for weights and activations (a sum over K does
//   not depend on its order): MMA m takes from lane t the pairs at K offsets
//   32t + 4m and 32t + 4m + 2, so every lane's operands come from its own
//   code chunk and one 64-byte run of each activation row, and each MMA's two
//   activation registers are adjacent words of one 16-byte load.  Decoding mixes a
//   shared-memory table byte -> signed bf16 pair (one copy per lane: a warp's
//   32 lookups hit 32 banks) with the in-register PRMT decode, balancing the
//   integer pipe against shared-memory bandwidth; the block scale is one
//   exact bf16x2 multiply.
//   With N <= 16 token columns tcgen05.mma (A in TMEM) passes 2048 weights
//   per instruction at about 50 cycles; mma.sync sustains 0.5 instructions
//   per cycle per SM, 128 weights per cycle, and needs no copy of the decoded
//   weights to TMEM or shared memory: this path is bound by HBM, not by
//   tensor math, so it takes the faster of the two.
// * Token columns: gate/up 8 per n-tile (NT = 1 or 2 tiles); down multiplies
//   by h and by its low part h_lo (y = W h + W h_lo): with T <= 4 one n-tile
//   holds h in columns 0..3 and h_lo in 4..7, else separate tiles accumulate
//   into the same registers.
// * At the end of a segment the warp finishes its rows: SwiGLU and h / h_lo,
//   or y, or a partial sum for a tile shared with other CTAs.
//
// Every wait is bounded (a timeout sets MOE_Q4_ETIMEOUT in the status word and
// the CTA drains and exits); warps wait and leave together (vote).
#include <cuda.h>

#include "q4_api_internal.h"
#include "q4_common.cuh"
#include "sm100.cuh"

namespace q4 {

using namespace sm100;

namespace dk {
constexpr int kComputeWarps = 8;                     // one 16-row slab each
constexpr int kThreads = 32 * (1 + kComputeWarps);   // + the producer warp
constexpr int kRows = 128;                           // weight rows per tile
constexpr int kMaxRing = 10;                         // shared-memory stages, at most
constexpr int kPrmtWords = 1;                        // of the 4 words of a chunk, decoded in registers
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kLutBytes = 65536;  // 256 entries x (2 table slots x 32 lanes x 4 B)
constexpr uint32_t kBarBytes = 1024;   // barriers and flags
}  // namespace dk

template <bool GATEUP, int NT>
struct DkCfg {
  // two 128-row weight tiles per unit and stage: gate and up of the same rows
  // (gate/up), or two consecutive row tiles of the down matrix (down), so a
  // stage carries 256 rows of codes either way
  static constexpr int kMats = 2;
  static constexpr int kUnitRows = GATEUP ? dk::kRows : 2 * dk::kRows;  // output rows per unit
  // activation row slots of a stage: 8 per n-tile; slot 8 nt + c feeds column
  // c of n-tile nt.  Gate/up: x of the expert's row n at slot n.  Down: h of
  // row n at slot n and h_lo of row n at slot kLoSlot + n (NT = 1: h in
  // columns 0..3, h_lo in 4..7 of one tile; else separate tiles)
  static constexpr int kXSlots = 8 * NT;
  static constexpr int kLoSlot = 4 * NT;
  // 8-token groups of the result
  static constexpr int kTT = GATEUP ? NT : (NT == 4 ? 2 : 1);
  // bytes of one ring stage of 64 * SUBS K: codes, activation slots, scales
  template <int SUBS>
  struct Geom {
    static constexpr uint32_t kRowBytes = 32 * SUBS;  // code bytes per weight row
    static constexpr uint32_t kCodeStage = kMats * dk::kRows * kRowBytes;
    static constexpr uint32_t kXPitch = SUBS * 128 + 16;  // stage bytes of a row + 16
    static constexpr uint32_t kXStage = kXSlots * kXPitch;
    static constexpr uint32_t kScaleSlot = 2 * SUBS;  // E8M0 bytes per weight row
    static constexpr uint32_t kScaleStage = kMats * dk::kRows * kScaleSlot;
  };
  // independent accumulators per (matrix, token group): MMA mm of K half J adds
  // into chain 2J + (mm & 1) (or J), so no MMA waits on the one before it for
  // long; the chains are added in a fixed order at the end
  static constexpr int kChains = (kMats * kTT <= 2 && NT <= 2) ? 4 : 2;
};

// Shared-memory placement, as offsets from the start of the CTA's dynamic
// window.  The table sits at a 64 KB boundary so its entry addresses can be
// formed by one PRMT; that leaves a region below it and one above.  The
// activation and scale rings and the barriers go low, the code stages high
// and, when the low region has room left, one or more of them low too (a
// deeper ring keeps more bytes in flight per SM).  The host computes it for
// the window start it expects; the kernel checks alignment and size.
struct DkLayout {
  uint32_t lut, code_hi, code_lo, x, scales, bars, end;
  int n_hi;  // code stages at code_hi; stages n_hi.. at code_lo
};

static bool dk_layout(uint32_t raw, uint32_t limit, uint32_t code_stage, uint32_t x_stage, uint32_t scale_stage,
                      int ring, DkLayout& L) {
  const uint32_t lut = (raw + 65535u) & ~65535u;
  const uint32_t o = (raw + 1023u) & ~1023u;
  const uint32_t hi = lut + dk::kLutBytes;
  if (hi > limit) return false;
  const uint32_t others = (uint32_t)ring * (x_stage + scale_stage) + dk::kBarBytes;
  const int fit_hi = (int)((limit - hi) / code_stage);
  uint32_t x;
  if (o + others <= lut) {
    // low: others, then the code stages that do not fit high
    const int n_hi = fit_hi < ring ? fit_hi : ring;
    const uint32_t lo = (o + others + 1023u) & ~1023u;
    if (lo + (uint32_t)(ring - n_hi) * code_stage > lut) return false;
    x = o;
    L.n_hi = n_hi;
    L.code_hi = hi;
    L.code_lo = lo;
    L.end = hi + (uint32_t)n_hi * code_stage;
  } else {
    // all high: code stages, then the others
    if (fit_hi < ring || hi + (uint32_t)ring * code_stage + others > limit) return false;
    L.n_hi = ring;
    L.code_hi = L.code_lo = hi;
    x = hi + (uint32_t)ring * code_stage;
    L.end = x + others;
  }
  L.lut = lut;
  L.x = x;
  L.scales = x + (uint32_t)ring * x_stage;
  L.bars = L.scales + (uint32_t)ring * scale_stage;
  // offsets from the window start
  L.lut -= raw;
  L.code_hi -= raw;
  L.code_lo -= raw;
  L.x -= raw;
  L.scales -= raw;
  L.bars -= raw;
  L.end -= raw;
  return true;
}

struct DkParams {
  FwdArgs a;
  int tiles_per_e;  // units per expert: I / 128 (gate/up), ceil(H / 256) (down)
  int subs;         // 64-K super-steps per stage: 4 (K % 256 == 0) or 2
  int stages;       // stages per tile: K / (64 * subs)
  int ring;         // shared-memory stages
  DkLayout lay;     // shared-memory placement (offsets)
  int n_max;        // token columns kept in partial sums: min(16, T)
  float* partial;   // [2 * gridDim.x][mats][n_max][128]
  int32_t* counter; // [units][8 slabs], zero at launch
  int self_k;       // gate/up at T = 1: top-k (the producer routes the token itself), else 0
};

// Start of CTA b's range of stages (the host keeps total below 2^31).
__device__ __forceinline__ int dk_range(int b, int total, int G) { return (int)((long long)b * total / G); }

// CTA whose range holds stage g.
__device__ __forceinline__ int dk_owner(int g, int total, int G) {
  int b = (int)(((long long)g * G) / total);
  while (b + 1 < G && dk_range(b + 1, total, G) <= g) ++b;
  while (b > 0 && dk_range(b, total, G) > g) --b;
  return b;
}

// CTAs holding part of [us, ue): the owners of its ends and every non-empty
// range between them (with fewer stages than CTAs some ranges are empty).
__device__ __forceinline__ int dk_contributors(int us, int ue, int total, int G, int& c_first, int& c_last) {
  c_first = dk_owner(us, total, G);
  c_last = dk_owner(ue - 1, total, G);
  int n = 0;
  for (int c = c_first; c <= c_last; ++c) n += dk_range(c + 1, total, G) > dk_range(c, total, G);
  return n;
}

// A unit shared by several CTAs: its contributors, and the partial-sum slot
// of the first (2c + 1 when the unit is not where that CTA's range starts).
struct DkSplit {
  int c_first, c_last, n_contrib, first_slot;
};

__device__ __forceinline__ DkSplit dk_split(int unit, int stages, int total, int G) {
  DkSplit d;
  const int us = unit * stages;
  d.n_contrib = dk_contributors(us, us + stages, total, G, d.c_first, d.c_last);
  d.first_slot = dk_range(d.c_first, total, G) != us ? 2 * d.c_first + 1 : 2 * d.c_first;
  return d;
}

__device__ __forceinline__ int atom_add_acq_rel(int32_t* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void ring_next(int& s, uint32_t& ph, int n) {
  if (++s == n) {
    s = 0;
    ph ^= 1u;
  }
}

// Shared-memory loads and MMAs of the inner loop are plain (not volatile)
// asm, so the compiler may interleave the independent chains of a stage.
// Their order against the stage barriers comes from data dependencies:
// every address is derived from `after_wait(base)`, issued after the wait,
// and the release takes the loaded words as inputs (`arrive_after`).
__device__ __forceinline__ uint32_t after_wait(uint32_t v) {
  uint32_t r;
  asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v) : "memory");
  return r;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// 16-byte shared load by the lanes with `pred` set; the others get zeros and
// touch no shared memory (a 16-byte load is served a quarter-warp at a time,
// so a quarter-warp with no active lane costs nothing).
__device__ __forceinline__ void lds128_if(uint32_t addr, uint32_t pred, uint32_t& x, uint32_t& y, uint32_t& z,
                                          uint32_t& w) {
  asm("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %5, 0;\n\t"
      "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
      "@p ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n\t}"
      : "=&r"(x), "=&r"(y), "=&r"(z), "=&r"(w)
      : "r"(addr), "r"(pred));
}

// bf16 of 2^(s - 127) for the E8M0 byte of row r0 (low half) and of row r1
// (high half), `p` = s0 | s1 << 16; s = 0 gives the bf16 subnormal 0x0040 and
// s = 255 the NaN 0x7FC0, as in the format's definition.
__device__ __forceinline__ uint32_t e8m0_pair_bf16(uint32_t p) {
  const uint32_t a = p << 7;                                  // s << 7 per half
  const uint32_t nan = ((a + 0x00800080u) >> 9) & 0x00400040u;  // bit 6 where s == 255
  uint32_t m;
  asm("max.u16x2 %0, %1, %2;" : "=r"(m) : "r"(a), "r"(0x00400040u));  // s == 0 -> 0x0040
  return m | nan;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds32_nv(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Arrive on `bar` once `dep` (a value computed from every shared-memory word
// the warp read from the stage) is available.
__device__ __forceinline__ void arrive_after(uint64_t* bar, uint32_t dep) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)), "r"(dep)
               : "memory");
}

// D += A(16x16, bf16, row) * B(16x8, bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Table slot `slot`: entry c -> bf16 pair of codes (c & 15, c >> 4), signed,
// unscaled, one copy per lane (entry c of lane l at c * 256 + slot * 128 +
// l * 4).  Thread ent (0..255) writes entry ent.
__device__ __forceinline__ void build_lut_slot(uint8_t* lut, const float* tv, int slot, int ent) {
  const uint32_t lo = ent & 15, hi = ent >> 4;
  const uint32_t blo = (uint32_t)bf16_bits_rn(tv[lo & 7]) ^ ((lo & 8) ? 0x8000u : 0u);
  const uint32_t bhi = (uint32_t)bf16_bits_rn(tv[hi & 7]) ^ ((hi & 8) ? 0x8000u : 0u);
  const uint32_t word = blo | (bhi << 16);
  uint4* dst = reinterpret_cast<uint4*>(lut + ent * 256 + slot * 128);
#pragma unroll
  for (int i = 0; i < 8; ++i) dst[i] = make_uint4(word, word, word, word);
}

// 16 bf16 pairs of one code chunk (4 words, pair 4w + b from byte b of word
// w), scaled: words below kPrmtWords by the PRMT decode, the rest by table.
__device__ __forceinline__ void decode_chunk(const uint4 c, const Planes& PL, uint32_t kreg, uint32_t scale2,
                                             uint32_t p[16]) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i < dk::kPrmtWords) {
      decode8(w[i], PL, &p[4 * i]);
    } else {
      // table entry address = table | byte << 8 | slot << 7 | lane << 2
      p[4 * i + 0] = lds32_nv(prmt(w[i], kreg, 0x7604));
      p[4 * i + 1] = lds32_nv(prmt(w[i], kreg, 0x7614));
      p[4 * i + 2] = lds32_nv(prmt(w[i], kreg, 0x7624));
      p[4 * i + 3] = lds32_nv(prmt(w[i], kreg, 0x7634));
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) p[i] = bf16x2_mul(p[i], scale2);
}

// SUBS (64-K super-steps per stage, 4 or 2) is a template argument so that a
// stage's two 128-K halves form one unrolled block the compiler can interleave.
// SELF: the one-token routing below is compiled in (only the gate/up kernel
// of a one-token call uses it; compiled into the others it cost 2.5 us per
// launch at T = 8 although never run).
template <bool GATEUP, int NT, int SUBS, bool SELF>
__global__ void __launch_bounds__(dk::kThreads, 1)
    dk_kernel(const __grid_constant__ DkParams P, const __grid_constant__ TableParams tp,
              const __grid_constant__ CUtensorMap tm_wa, const __grid_constant__ CUtensorMap tm_wb) {
  using C = DkCfg<GATEUP, NT>;
  constexpr int kMats = C::kMats;
  constexpr int kComputeW = dk::kComputeWarps;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  // absolute shared addresses of the placement
  DkLayout Ls = P.lay;
  Ls.lut += raw_s;
  Ls.code_hi += raw_s;
  Ls.code_lo += raw_s;
  Ls.x += raw_s;
  Ls.scales += raw_s;
  Ls.bars += raw_s;
  const FwdArgs& a = P.a;
  if (P.lay.end > dynamic_smem_size() || (Ls.lut & 0xffffu) != 0u) {
    // the window is smaller or starts elsewhere than the host planned for
    if (threadIdx.x == 0) record_error(a.hdr + kStatus, MOE_Q4_ECUDA);
    return;
  }
  using Geo = typename C::template Geom<SUBS>;
  const auto code_base = [&](int s) -> uint32_t {
    return s < Ls.n_hi ? Ls.code_hi + (uint32_t)s * Geo::kCodeStage
                       : Ls.code_lo + (uint32_t)(s - Ls.n_hi) * Geo::kCodeStage;
  };
  uint8_t* lut = smem_raw + (Ls.lut - raw_s);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + (Ls.bars - raw_s));
  uint64_t* full = bars;                          // [ring] codes (+ h: TMA), scales (+ x: cp.async)
  uint64_t* stage_empty = full + dk::kMaxRing;    // [ring] compute warps done with the stage
  uint64_t* lut_bar = stage_empty + dk::kMaxRing; // compute threads rebuilding a table slot
  volatile int* abort_flag = reinterpret_cast<volatile int*>(lut_bar + 1);

  const int ring = P.ring;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < ring; ++s) {
      mbar_init(&full[s], 1 + 32);  // producer lane 0 (with the TMA bytes) + 32 cp.async arrivals
      mbar_init(&stage_empty[s], kComputeW);
    }
    mbar_init(lut_bar, 32 * kComputeW);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_wa);
    if (GATEUP) prefetch_tmap(&tm_wb);
  }
  // Gate/up with one token (self_k > 0): its k experts are distinct and hold
  // one row each, so the routing tables follow from the token's top-k alone
  // (the expert list is the k ids in ascending order; expert j of it has row
  // j, of token 0).  Warp 0 computes that top-k with the routing kernel's own
  // warp routine on the same logits (hence the same ids) and the CTA runs on
  // it without waiting for the routing kernel.  That kernel lets this one
  // launch only after its own wait, so x and the logits are complete.  What
  // this kernel does need of it, the split-tile counters it zeroes, is used
  // only after a wait at the end of each unit; every thread waits again
  // before it exits, so the kernels after this one still find the routing
  // kernel complete.
  const bool self = SELF && GATEUP && P.self_k > 0;
  int* self_e = reinterpret_cast<int*>(bars) + 64;  // [k] expert list (bytes 256.. of the barrier block)
  if (self && warp == 0) {  // (while warps 1..8 build the table below)
    const int k = P.self_k;
    int id;
    float wt;
    topk_warp(a.logits, a.E, k, lane, nullptr, id, wt);
    int rank = 0;  // lane j < k: number of smaller ids among the k
    for (int j = 0; j < k; ++j) {
      const int o = __shfl_sync(0xffffffffu, id, j);
      rank += (lane < k && o < id) ? 1 : 0;
    }
    if (lane < k) self_e[rank] = id;
  }
  // with a single table every expert uses table 0: its table slot is built
  // before waiting for the previous kernel
  if (tp.n == 1 && warp >= 1) build_lut_slot(lut, tp.t[0], 0, threadIdx.x - 32);
  __syncthreads();

  const int rows_total = GATEUP ? a.I : a.H;
  const int K = GATEUP ? a.H : a.I;
  constexpr int subs = SUBS;
  constexpr int row_bytes = 32 * subs;  // code bytes per row per stage
  const int G = gridDim.x, b = blockIdx.x;

  // producer: one ring stage s of stage index st of a unit whose weight rows
  // start at wrow: the codes (one TMA per 128-row tile, lane 0 registering
  // their bytes), every row's scale bytes (cp.async, 4 rows per lane), this
  // lane's activation row (untiled bulk copy, adding its own bytes) and the
  // lanes' cp.async arrivals
  const auto issue_stage = [&](int s, int st, int wrow, bool two, int my_slot, const __nv_bfloat16* my_src) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&full[s], (two ? 2 : 1) * dk::kRows * row_bytes);
      uint8_t* cdst = smem_raw + (code_base(s) - raw_s);
      tma_load_2d(cdst, &tm_wa, &full[s], st * row_bytes, wrow);
      if (GATEUP)
        tma_load_2d(cdst + dk::kRows * row_bytes, &tm_wb, &full[s], st * row_bytes, wrow);
      else if (two)
        tma_load_2d(cdst + dk::kRows * row_bytes, &tm_wa, &full[s], st * row_bytes, wrow + dk::kRows);
    }
    __syncwarp();  // the expected bytes are registered before any row copy can land
    // scale bytes of the stage (2 per 64-K super-step) for 4 rows per lane
#pragma unroll
    for (int m = 0; m < kMats; ++m) {
      if (!two && m == 1) break;  // (a missing tile's rows are computed on stale bytes, never written)
      const uint8_t* sbase = GATEUP ? (m ? a.up_s : a.gate_s) + (size_t)wrow * (K / 32) + (size_t)st * 2 * subs
                                    : a.down_s + (size_t)(wrow + m * dk::kRows) * (K / 32) + (size_t)st * 2 * subs;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = lane + 32 * j;
        const uint32_t dst =
            Ls.scales + (uint32_t)s * Geo::kScaleStage + (uint32_t)(m * dk::kRows + r) * Geo::kScaleSlot;
        if constexpr (subs == 4)
          cp_async_small<8>(dst, sbase + (size_t)r * (K / 32));
        else
          cp_async_small<4>(dst, sbase + (size_t)r * (K / 32));
      }
    }
    if (my_slot >= 0) {
      // slot n at n * x_pitch (x_pitch = stage bytes + 16: 16-byte aligned,
      // and an odd number of 16-byte chunks spreads the slots over the banks)
      uint8_t* d = smem_raw + (Ls.x - raw_s) + (uint32_t)s * Geo::kXStage + (uint32_t)my_slot * Geo::kXPitch;
      mbar_expect_tx(&full[s], (uint32_t)(subs * 128));
      bulk_load(d, my_src + st * subs * 64, (uint32_t)(subs * 128), &full[s]);
    }
    cp_async_arrive_noinc(&full[s]);
    __syncwarp();
  };

  // routing tables of a unit: expert, its first row, its rows
  const auto unit_expert = [&](int unit) -> int {
    return self ? self_e[unit / P.tiles_per_e] : a.dec_list[unit / P.tiles_per_e];
  };
  const auto expert_row0 = [&](int unit, int e) -> int { return self ? unit / P.tiles_per_e : a.offsets[e]; };
  const auto expert_rows = [&](int e) -> int { return self ? 1 : a.counts[e]; };

  // down: the next kernel (the combine, small CTAs that fit beside this one)
  // may be scheduled now; its own wait still covers all of this kernel's work
  if (!GATEUP) pdl_trigger();
  if (!self) pdl_wait();
  const int n_dec = self ? P.self_k : a.hdr[kNumDecode];
  const int total = n_dec * P.tiles_per_e * P.stages;
  const int k0 = dk_range(b, total, G), k1 = dk_range(b + 1, total, G);

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int g = k0; g < k1 && ok;) {
      const int unit = g / P.stages;
      const int st0 = g - unit * P.stages;
      const int seg_end = min(k1, (unit + 1) * P.stages);
      int e = unit_expert(unit);
      if (!q4_check((unsigned)e < (unsigned)a.E, a.hdr + kStatus)) e = 0;
      const int t = unit % P.tiles_per_e;
      const int wrow = e * rows_total + t * C::kUnitRows;
      // down: the unit's second row tile exists unless H is an odd number of 128s
      const bool two = GATEUP || t * C::kUnitRows + dk::kRows < rows_total;
      const int row0 = expert_row0(unit, e);
      if (!q4_check(row0 >= 0 && row0 + expert_rows(e) <= a.T * a.k, a.hdr + kStatus)) break;
      // Activation rows by untiled bulk copies (a tiled TMA would need a
      // 128-byte-aligned destination), one per row and stage: the stage's
      // 32 * subs * 4 bytes of x[token] (gate/up, lane n: row n) or of h / h_lo
      // (down, lane n: h of row n; lane 16 + n: h_lo of row n).  Slots past
      // n_e are not written: they only feed columns nobody writes.
      const int n_e = expert_rows(e);  // <= 16
      int my_slot = -1;
      const __nv_bfloat16* my_src = nullptr;
      if (GATEUP) {
        if (lane < n_e) {
          const int tok = self ? 0 : a.row_token[row0 + lane];
          if (q4_check((unsigned)tok < (unsigned)a.T, a.hdr + kStatus)) {
            my_slot = lane;
            my_src = a.x + (size_t)tok * a.H;
          }
        }
      } else {
        const int n = lane & 15;
        if (n < n_e) {
          my_slot = lane < 16 ? n : C::kLoSlot + n;
          my_src = (lane < 16 ? a.h : a.h_lo) + (size_t)(row0 + n) * a.I;
        }
      }
      for (int st = st0; st < st0 + (int)(seg_end - g); ++st) {
        if (!mbar_wait_warp(&stage_empty[s], ph ^ 1, abort_flag, dk::kWaitNs)) {
          ok = false;
          break;
        }
        issue_stage(s, st, wrow, two, my_slot, my_src);
        ring_next(s, ph, ring);
      }
      g = seg_end;
    }
  } else {
    // ------------------------------ compute ------------------------------
    const int cw = warp - 1;
    const int slab = cw;           // rows 16 slab .. + 15 of the tile
    const int gq = lane >> 2;      // MMA group: rows gq, gq + 8; token column gq
    const int tq = lane & 3;       // code chunk of a half; token columns 2tq, 2tq + 1
    const int ctid = threadIdx.x - 32;
    constexpr int kJ = subs / 2;   // 128-K halves per stage
    constexpr int kCh = C::kChains;
    // MMA rows gq and gq + 8 of the slab are tile rows r0 and r1.  With the
    // 128-byte swizzle the rows of one quarter-warp (gq = 2q, 2q + 1) are
    // taken 4 apart (r0 & 7 = q and q + 4), so their code chunks, XOR-ed with
    // r & 7, fall in disjoint halves of the 8 bank groups: no conflict.  (The
    // 64-byte swizzle of 128-K stages puts consecutive rows in disjoint bank
    // groups already.)
    const int r0 = 16 * slab + (subs == 4 ? (((gq & 1) << 2) | (gq >> 1)) : gq), r1 = r0 + 8;
    const int swz0 = subs == 4 ? (r0 & 7) : ((r0 >> 1) & 3);
    const int swz1 = subs == 4 ? (r1 & 7) : ((r1 >> 1) & 3);
    // per-lane offsets inside a stage: code chunk 4J + tq of rows r0 / r1 for
    // each 128-K half J; the activation run of half J is bytes 256 J + 64 tq ..
    // + 63 of a slot, its scale byte tq of word J of the row
    uint32_t coff[kJ][2];
#pragma unroll
    for (int J = 0; J < kJ; ++J) {
      const int chunk = 4 * J + tq;
      coff[J][0] = (uint32_t)(r0 * row_bytes + ((chunk ^ swz0) << 4));
      coff[J][1] = (uint32_t)(r1 * row_bytes + ((chunk ^ swz1) << 4));
    }
    // PRMT selector: byte tq of the row-r0 word to byte 0, of the row-r1 word to byte 2
    const uint32_t psel = (uint32_t)tq | ((uint32_t)(4 + tq) << 8);
    int slot_tab0 = tp.n == 1 ? 0 : -1, slot_tab1 = -1, victim = tp.n == 1 ? 1 : 0;
    uint32_t lgen = 0;
    const uint32_t lane_k = (Ls.lut & 0xffff0000u) | ((uint32_t)lane << 2);
    // only the first and the last unit of the range can be shared with other
    // CTAs: their contributors are found now, while the first stage is in flight
    DkSplit sp_first = {0, 0, 1, 0}, sp_last = {0, 0, 1, 0};
    if (k0 < k1) {
      sp_first = dk_split(k0 / P.stages, P.stages, total, G);
      sp_last = (k1 - 1) / P.stages == k0 / P.stages ? sp_first : dk_split((k1 - 1) / P.stages, P.stages, total, G);
    }
    int s = 0;
    uint32_t ph = 0;
    // shared addresses of ring slot s, advanced with it (no per-stage multiplies)
    const uint32_t c_first = Ls.n_hi > 0 ? Ls.code_hi : Ls.code_lo;
    uint32_t cur_c = c_first, cur_s = Ls.scales, cur_x = Ls.x;
    const auto advance = [&]() {
      if (++s == ring) {
        s = 0;
        ph ^= 1u;
        cur_c = c_first;
        cur_s = Ls.scales;
        cur_x = Ls.x;
      } else {
        cur_c = s == Ls.n_hi ? Ls.code_lo : cur_c + Geo::kCodeStage;
        cur_s += Geo::kScaleStage;
        cur_x += Geo::kXStage;
      }
    };
    bool ok = true;
    for (int g = k0; g < k1 && ok;) {
      const int unit = g / P.stages;
      const int ustart = unit * P.stages, uend = ustart + P.stages;
      const int seg_end = min(k1, uend);
      const int nst = (int)(seg_end - g);
      const int e = unit_expert(unit);
      const int tile = unit % P.tiles_per_e;
      const int tid = tp.id[e];
      int slot = tid == slot_tab0 ? 0 : (tid == slot_tab1 ? 1 : -1);
      if (slot < 0) {
        // (re)build a slot: entry c -> bf16 pair of codes (c & 15, c >> 4), signed,
        // unscaled, one copy per lane.  Bounded barriers on both sides: every
        // compute thread is done with the old contents before any write, and all
        // writes land before anyone reads.
        mbar_arrive(lut_bar);
        if (!mbar_wait_warp(lut_bar, lgen & 1, abort_flag, dk::kWaitNs)) break;
        ++lgen;
        slot = victim;
        victim ^= 1;
        if (slot == 0)
          slot_tab0 = tid;
        else
          slot_tab1 = tid;
        if (ctid < 256) build_lut_slot(lut, tp.t[tid], slot, ctid);  // one table entry per thread
        mbar_arrive(lut_bar);
        if (!mbar_wait_warp(lut_bar, lgen & 1, abort_flag, dk::kWaitNs)) break;
        ++lgen;
      }
      const uint32_t kreg = lane_k | ((uint32_t)slot << 7);
      const Planes PL = make_planes(tp.t[tid]);
      // activation slot of this lane's column gq in each n-tile; columns of
      // absent tokens are not read (zero operands; their MMA columns are never
      // written)
      const int n_e_seg = expert_rows(e);
      uint32_t xrow[NT], col_ok[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        int tok;
        if (GATEUP)
          tok = 8 * nt + gq;
        else if (NT == 1)
          tok = gq & 3;
        else if (NT == 2)
          tok = gq;
        else
          tok = 8 * (nt & 1) + gq;
        col_ok[nt] = tok < n_e_seg ? 1u : 0u;
        xrow[nt] = (uint32_t)(8 * nt + gq) * Geo::kXPitch + (uint32_t)(64 * tq);
      }
      float accc[kMats][C::kTT][kCh][4];
#pragma unroll
      for (int m = 0; m < kMats; ++m)
#pragma unroll
        for (int tt = 0; tt < C::kTT; ++tt)
#pragma unroll
          for (int c = 0; c < kCh; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i) accc[m][tt][c][i] = 0.0f;

      for (int j = 0; j < nst && ok; ++j) {
        if (!mbar_wait_warp(&full[s], ph, abort_flag, dk::kWaitNs)) {
          ok = false;
          break;
        }
        const uint32_t cbase = after_wait(cur_c);
        const uint32_t sbase = after_wait(cur_s);
        const uint32_t xstage = after_wait(cur_x);
        uint32_t dep = 0;  // every word read from the stage, folded
#pragma unroll
        for (int J = 0; J < kJ; ++J) {
          // activation operands: 16 pairs per n-tile, pair p at K offset 32 tq + 2p
          uint32_t xr[NT][16];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              lds128_if(xstage + xrow[nt] + (uint32_t)(256 * J + 16 * c), col_ok[nt], xr[nt][4 * c + 0],
                        xr[nt][4 * c + 1], xr[nt][4 * c + 2], xr[nt][4 * c + 3]);
              dep ^= xr[nt][4 * c + 0];
            }
          }
#pragma unroll
          for (int m = 0; m < kMats; ++m) {
            const uint32_t mb = cbase + (uint32_t)(m * dk::kRows * row_bytes);
            const uint4 c0 = lds128(mb + coff[J][0]);
            const uint4 c1 = lds128(mb + coff[J][1]);
            // scale word of this half (4 E8M0 bytes, block 4J + tq in byte tq)
            uint32_t w0, w1;
            if constexpr (SUBS == 4) {
              const uint2 s0 = lds64(sbase + (uint32_t)((m * dk::kRows + r0) * Geo::kScaleSlot));
              const uint2 s1 = lds64(sbase + (uint32_t)((m * dk::kRows + r1) * Geo::kScaleSlot));
              w0 = J ? s0.y : s0.x;
              w1 = J ? s1.y : s1.x;
            } else {
              w0 = lds32_nv(sbase + (uint32_t)((m * dk::kRows + r0) * Geo::kScaleSlot));
              w1 = lds32_nv(sbase + (uint32_t)((m * dk::kRows + r1) * Geo::kScaleSlot));
            }
            dep ^= c0.x ^ c1.x ^ w0 ^ w1;
            // byte tq of each row's word (block 4J + tq), as bf16 scales for both rows
            const uint32_t sc = e8m0_pair_bf16(prmt(w0, w1, psel) & 0x00ff00ffu);
            uint32_t pa[16], pb[16];
            decode_chunk(c0, PL, kreg, prmt(sc, 0u, 0x1010u), pa);
            decode_chunk(c1, PL, kreg, prmt(sc, 0u, 0x3232u), pb);
#pragma unroll
            for (int mm = 0; mm < 8; ++mm) {
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const int tt = GATEUP ? nt : (NT == 4 ? (nt & 1) : 0);
                const int ch = C::kChains == 4 ? 2 * J + (mm & 1) : J;
                mma_bf16_16816(accc[m][tt][ch], pa[2 * mm], pb[2 * mm], pa[2 * mm + 1], pb[2 * mm + 1],
                               xr[nt][2 * mm], xr[nt][2 * mm + 1]);
              }
            }
          }
        }
        // the table lookups read only the table, not the stage: the stage is free
        // once the loads above have returned (their values feed `dep`)
        dep = __reduce_xor_sync(0xffffffffu, dep);
        if (lane == 0) arrive_after(&stage_empty[s], dep);
        advance();
      }
      if (!ok) break;

      float acc[kMats][C::kTT][4];
#pragma unroll
      for (int m = 0; m < kMats; ++m)
#pragma unroll
        for (int tt = 0; tt < C::kTT; ++tt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float v = accc[m][tt][0][i];
#pragma unroll
            for (int c = 1; c < kCh; ++c) v += accc[m][tt][c][i];
            acc[m][tt][i] = v;
          }
      if (!GATEUP && NT == 1) {
        // columns 4..7 hold W h_lo for tokens 0..3: add them to columns 0..3
#pragma unroll
        for (int m = 0; m < kMats; ++m)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[m][0][i] += __shfl_xor_sync(0xffffffffu, acc[m][0][i], 2);
      }

      // ---- the warp finishes its rows: token n = 8 tt + 2 tq + (i & 1), row r0 / r1 ----
      if (self) pdl_wait();  // (the routing kernel zeroed the split-tile counters; returns at once after the first)
      const int row0 = expert_row0(unit, e), n_e = expert_rows(e);
      const bool final_here = (g == ustart && seg_end == uend);
      if (!final_here) {
        // partial: slot 2b (segment starts this CTA's range) or 2b+1 (its last)
        const int pslot = (g == k0) ? 2 * b : 2 * b + 1;
        float* pp = P.partial + (size_t)pslot * kMats * P.n_max * dk::kRows;
#pragma unroll
        for (int m = 0; m < kMats; ++m)
#pragma unroll
          for (int tt = 0; tt < C::kTT; ++tt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int n = 8 * tt + 2 * tq + (i & 1);
              if (n < P.n_max) pp[(m * P.n_max + n) * dk::kRows + ((i >> 1) ? r1 : r0)] = acc[m][tt][i];
            }
        // each slab warp signs in on its own counter (release: its lanes' partial
        // stores, ordered before lane 0's atomic by the warp barrier); the last
        // warp of a slab to sign in (acquire) finishes those rows
        __syncwarp();
        // a shared segment is the first or the last of this CTA's range
        const DkSplit sp = g == k0 ? sp_first : sp_last;
        int last = 0;
        if (lane == 0) last = atom_add_acq_rel(&P.counter[(size_t)unit * 8 + slab], 1) == sp.n_contrib - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) {
          g = seg_end;
          continue;
        }
        __syncwarp();
        // last arrival: add the partials of every CTA on this tile in K order
#pragma unroll
        for (int m = 0; m < kMats; ++m)
#pragma unroll
          for (int tt = 0; tt < C::kTT; ++tt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[m][tt][i] = 0.0f;
        for (int c = sp.c_first; c <= sp.c_last; ++c) {
          // with fewer stages than CTAs some ranges are empty
          if (total < G && dk_range(c + 1, total, G) == dk_range(c, total, G)) continue;
          const int sl = c == sp.c_first ? sp.first_slot : 2 * c;
          const float* qp = P.partial + (size_t)sl * kMats * P.n_max * dk::kRows;
#pragma unroll
          for (int m = 0; m < kMats; ++m)
#pragma unroll
            for (int tt = 0; tt < C::kTT; ++tt)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int n = 8 * tt + 2 * tq + (i & 1);
                if (n < P.n_max) acc[m][tt][i] += __ldcg(qp + (m * P.n_max + n) * dk::kRows + ((i >> 1) ? r1 : r0));
              }
        }
      }
      // finished slab: h (gate/up, as the bf16 pair h, h_lo) or y (down)
#pragma unroll
      for (int tt = 0; tt < C::kTT; ++tt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int n = 8 * tt + 2 * tq + (i & 1);
          if (n >= n_e) continue;
          const size_t row = (size_t)row0 + n;
          if (!q4_check(row < (size_t)a.T * a.k, a.hdr + kStatus)) continue;
          const int wr = tile * C::kUnitRows + ((i >> 1) ? r1 : r0);
          if (GATEUP) {
            const float hv = silu_mul(acc[0][tt][i], acc[1][tt][i]);
            const __nv_bfloat16 hb = __float2bfloat16_rn(hv);
            a.h[row * a.I + wr] = hb;
            a.h_lo[row * a.I + wr] = __float2bfloat16_rn(hv - __bfloat162float(hb));
          } else {
            a.y[row * a.H + wr] = acc[0][tt][i];
            if (wr + dk::kRows < a.H) a.y[row * a.H + wr + dk::kRows] = acc[1][tt][i];
          }
        }
      g = seg_end;
    }
  }

  // ------------------------------ teardown ------------------------------
  if (self) pdl_wait();  // the routing kernel is complete before this CTA is (and its status reset precedes ours)
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
  if (GATEUP) pdl_trigger();
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

template <bool GATEUP, int NT, int SUBS, bool SELF>
static int launch_dk_subs(const FwdArgs& a, const TableParams& tp, float* partial, int32_t* counter, int grid,
                     cudaStream_t s) {
  using C = DkCfg<GATEUP, NT>;
  DkParams P;
  P.a = a;
  const int K = GATEUP ? a.H : a.I;
  P.tiles_per_e = GATEUP ? a.I / dk::kRows : (a.H + C::kUnitRows - 1) / C::kUnitRows;
  P.subs = SUBS;
  P.stages = K / (64 * P.subs);
  // stage indices are 32-bit on the device
  if ((uint64_t)a.E * (uint64_t)P.tiles_per_e * (uint64_t)P.stages >= (1ull << 31)) return MOE_Q4_EINVAL;
  P.n_max = a.T < 16 ? a.T : 16;
  using Geo = typename C::template Geom<SUBS>;
  P.partial = partial;
  P.counter = counter;
  // (one token routed by the kernel itself reads the logits before its
  // dependency wait: only when they are an input of the forward)
  P.self_k = SELF && GATEUP && a.T == 1 && !a.logits_in_forward ? a.k : 0;

  // deepest ring that fits; the dynamic window starts after the reserved bytes
  // (the kernel has no static shared memory)
  int dev = 0, reserved = 1024, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  P.ring = 0;
  for (int rs = dk::kMaxRing; rs >= 2 && !P.ring; --rs)
    if (dk_layout((uint32_t)reserved, (uint32_t)reserved + (uint32_t)optin, Geo::kCodeStage, Geo::kXStage,
                  Geo::kScaleStage,
                  rs, P.lay))
      P.ring = rs;
  if (!P.ring) return MOE_Q4_ECUDA;
  const uint32_t smem = P.lay.end;

  const CUtensorMapSwizzle csw = P.subs == 4 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const uint32_t cbox = 32u * P.subs;
  // activation rows come by untiled bulk copies: only the weight codes have maps
  CUtensorMap twa, twb;
  bool ok;
  if (GATEUP) {
    ok = dk_map(&twa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.gate_w, a.H / 2, (uint64_t)a.E * a.I, cbox, dk::kRows, csw) &&
         dk_map(&twb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.up_w, a.H / 2, (uint64_t)a.E * a.I, cbox, dk::kRows, csw);
  } else {
    ok = dk_map(&twa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.down_w, a.I / 2, (uint64_t)a.E * a.H, cbox, dk::kRows,
                csw);
    twb = twa;
  }
  if (!ok) return MOE_Q4_ECUDA;
  if (cudaFuncSetAttribute(dk_kernel<GATEUP, NT, SUBS, SELF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) !=
      cudaSuccess)
    return MOE_Q4_ECUDA;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  // one token: the routing kernel (one CTA) still runs while this kernel
  // starts, so this kernel leaves it its SM rather than have one CTA start late
  cfg.gridDim = dim3(P.self_k > 0 && grid > 1 ? grid - 1 : grid);
  cfg.blockDim = dim3(dk::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dk_kernel<GATEUP, NT, SUBS, SELF>, P, tp, twa, twb) == cudaSuccess ? MOE_Q4_OK
                                                                                                 : MOE_Q4_ECUDA;
}

// stages of 256 K when K allows, else 128 (K % 128 == 0 always)
template <bool GATEUP, int NT>
static int launch_dk(const FwdArgs& a, const TableParams& tp, float* partial, int32_t* counter, int grid,
                     cudaStream_t s) {
  const int K = GATEUP ? a.H : a.I;
  // one token routed by the gate/up kernel itself (logits given as input)
  if constexpr (GATEUP && NT == 1) {
    if (a.T == 1 && !a.logits_in_forward)
      return K % 256 == 0 ? launch_dk_subs<GATEUP, NT, 4, true>(a, tp, partial, counter, grid, s)
                          : launch_dk_subs<GATEUP, NT, 2, true>(a, tp, partial, counter, grid, s);
  }
  return K % 256 == 0 ? launch_dk_subs<GATEUP, NT, 4, false>(a, tp, partial, counter, grid, s)
                      : launch_dk_subs<GATEUP, NT, 2, false>(a, tp, partial, counter, grid, s);
}

}  // namespace q4

using namespace q4;

// Token columns per launch follow from T: an expert holds at most min(T, 16)
// rows on this path.
int q4_launch_decode(const FwdArgs& a, const TableParams& tp, bool gateup, float* partial, int32_t* counter,
                     int grid, cudaStream_t s) {
  if (a.T * a.k == 0) return MOE_Q4_OK;
  if (gateup)
    return a.T <= 8 ? launch_dk<true, 1>(a, tp, partial, counter, grid, s)
                    : launch_dk<true, 2>(a, tp, partial, counter, grid, s);
  if (a.T <= 4) return launch_dk<false, 1>(a, tp, partial, counter, grid, s);
  if (a.T <= 8) return launch_dk<false, 2>(a, tp, partial, counter, grid, s);
  return launch_dk<false, 4>(a, tp, partial, counter, grid, s);
}
