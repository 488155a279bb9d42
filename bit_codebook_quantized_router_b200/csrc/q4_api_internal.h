// Host/device interface between the moe_q4 C-ABI layer and its kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_q4.h"

namespace q4 {
struct TableParams;

// Everything a forward kernel needs, passed by value.  Workspace arrays are
// carved by q4_carve_workspace(); see the layout there.
struct FwdArgs {
  int T, k, E, H, I;
  int dec_max;     // experts with 1..dec_max rows take the streaming path
  int wide_max;    // experts with dec_max+1..wide_max rows take the wide tensor-core kernel
                   // (tokens as MMA M, 256 weight rows as N); more rows: swap-AB tiles
  int tile_n;      // token tile of the tensor-core path
  const __nv_bfloat16* x;  // [T][H]
  const float* logits;     // [T][E]
  __nv_bfloat16* out;      // [T][H]
  int32_t* hdr;            // header words (HeaderWord)
  int32_t* ids;            // [T*k]
  float* w;                // [T*k]
  int32_t* counts;         // [E]
  int32_t* offsets;        // [E+1]
  int32_t* row_token;      // [T*k]
  int32_t* inv;            // [T*k]
  int32_t* dec_list;       // [E]
  int32_t* pre_list;       // [E]
  int32_t* mid_list;       // [E] experts of the wide tensor-core kernel (nullptr: none)
  int32_t* tiles;          // [E+1] token-tile offsets of the tensor-core-path experts
  int32_t* chunk_cnt;      // [chunks][E] rows per expert of each 256-token chunk (T > 256)
  int32_t* chunk_base;     // [chunks][E] each chunk's first row inside each expert (T > 256)
  __nv_bfloat16* h;        // [T*k][I] bf16 rounding of silu(g)*u
  __nv_bfloat16* h_lo;     // [T*k][I] bf16 rounding of the remainder silu(g)*u - h
  float* y;                // [T*k][H]
  float* out_f32;          // optional [T][H] fp32 combine result
  const float* y_s;        // optional [T][H] shared-expert output, added by the combine
  __nv_bfloat16* xg;       // [T*k][H] expert-grouped activations
  int32_t* dk_counter;     // [dk_counter_n] split-tile arrival counters (small-M path)
  int dk_counter_n;
  int keep_status;         // the status word was cleared before this forward's first kernel
  int logits_in_forward;   // the logits are computed by this forward's first kernel
  int32_t* user_ids;
  float* user_w;
  int32_t* user_counts;
  const uint8_t *gate_w, *gate_s, *up_w, *up_s, *down_w, *down_s;
};
}  // namespace q4

// Validate host tables / table ids and fill the kernel parameter block.
int q4_fill_tables(q4::TableParams* tp, const float* tables, int n_tables, const uint8_t* table_id,
                   int E);

// Kernel launchers (return MOE_Q4_OK or MOE_Q4_ECUDA).
int q4_launch_route(const q4::FwdArgs& a, cudaStream_t s);
// Chunks of the large-T grouping (0 for T <= 256): chunk_cnt and chunk_base
// hold q4_route_chunks(T) * E int32 each.
int q4_route_chunks(int T);
int q4_launch_combine(const q4::FwdArgs& a, cudaStream_t s);
// Router gate (router.cu): logits = x . w^T at any T (part: the partial sums,
// q4_router_partial_bytes; status: the dense GEMM's status word), and at
// decode sizes the router with the routing fused behind it (a.logits is the
// logits buffer it writes; a.hdr[kRouterTicket] must be 0 at launch).
size_t q4_router_partial_bytes(int T, int H, int E);
int q4_launch_router(const void* x, const void* w, int T, int H, int E, float* logits, void* part, int32_t* status,
                     cudaStream_t s);
bool q4_router_route_fused(int T, int H, int k);
int q4_launch_router_route(const q4::FwdArgs& a, const void* w, cudaStream_t s);
int q4_launch_gather(const q4::FwdArgs& a, cudaStream_t s);
// wide_next: the WIDE kernel is launched right after (see prefill.cu)
int q4_launch_prefill(const q4::FwdArgs& a, const q4::TableParams& tp, bool gateup, bool wide_next, cudaStream_t s);
// the wide tensor-core kernel (experts with dec_max+1 .. q4_prefill_wide_max() rows)
int q4_prefill_wide_max();
int q4_launch_prefill_wide(const q4::FwdArgs& a, const q4::TableParams& tp, bool gateup, cudaStream_t s);
int q4_prefill_tile_n();
int q4_launch_decode(const q4::FwdArgs& a, const q4::TableParams& tp, bool gateup, float* partial,
                        int32_t* counter, int grid, cudaStream_t s);
// Dense bf16 GEMM on the tensor cores (shared.cu): see q4_launch_dense.
size_t q4_dense_partial_bytes(int T, int rows, int K, int mats);
int q4_launch_dense(const void* w, int mats, int mat1_off, int rows, int K, const void* act, int T,
                    __nv_bfloat16* out_bf16, float* out_f32, int ld, float* partial, int32_t* status,
                    cudaStream_t s);
int q4_forward_in_workspace(const moe_q4_layer* layer, const void* x, const float* logits, int T, int top_k,
                            void* out, float* out_f32, void* ws, size_t ws_bytes, cudaStream_t stream);
