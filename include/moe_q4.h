/*
 * moe_q4 -- routed-expert MoE feed-forward over 4-bit codebook weights,
 * for NVIDIA B200 (sm_100a).  C ABI.
 *
 * Weight format ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ", sections
 * "Contents" and "Codes are indices into the per-layer grid -- not E2M1"):
 *   - every weight is a 4-bit code: code & 0x7 indexes an 8-entry magnitude
 *     table (the layer's Lloyd-Max grid, or the E2M1 table), code & 0x8 is
 *     the sign;
 *   - two codes per byte, the LOW nibble holds the EVEN K index;
 *   - one E8M0 scale byte per 32 weights along K; the weight is
 *       w = sign * table[code & 7] * 2^(scale_byte - 127);
 *   - a projection W[N][K] is stored as `weight` uint8 [N][K/2] and
 *     `weight_scale` uint8 [N][K/32], K contiguous; E experts are stacked
 *     along a leading dimension.
 * The layer (shapes as in "Round 7 -- Rewrite the GLM-5.2 routed-expert
 * encoder", "Ground truth and corrections" and "Owner-locked decisions" 4, 6):
 *   route:   top-k of E router logits per token, softmax over the k kept;
 *   gate/up: g = W_gate x, u = W_up x          (W_gate, W_up: [I][H]);
 *   SwiGLU:  h = silu(g) * u;
 *   down:    y = W_down h                      (W_down: [H][I]);
 *   combine: out = sum_j w_j * y_j over the k routed experts, in slot order.
 *
 * Conventions for every entry point:
 *   - "device" pointers are CUDA device memory on the current device;
 *     "host" pointers are ordinary host memory read during the call.
 *   - The caller allocates and owns every buffer.  The library allocates
 *     nothing inside these calls (moe_q4_forward_host excepted: none either,
 *     it only stages through the caller's workspace).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without waiting, except where stated.
 *   - Argument errors are detected on the host before anything is launched
 *     and return MOE_Q4_EINVAL (or MOE_Q4_EWORKSPACE); nothing is written.
 *   - Errors that only the device can see (a NaN router logit, a non-finite
 *     weight given to pack) are recorded in a device status word; read it
 *     with moe_q4_forward_status / moe_q4_read_status.  Kernels never trap.
 *   - bf16 tensors are passed as `void*` holding IEEE bfloat16 values.
 */
#ifndef MOE_Q4_H
#define MOE_Q4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_Q4_API __attribute__((visibility("default")))
#else
#define MOE_Q4_API
#endif

#define MOE_Q4_ABI_VERSION 1

/* Status codes. */
#define MOE_Q4_OK 0
#define MOE_Q4_EINVAL 1      /* null pointer, bad shape, K % 32, top_k > E, bad table, bad table id */
#define MOE_Q4_ECUDA 2       /* a CUDA runtime/driver call or a launch failed */
#define MOE_Q4_EWORKSPACE 3  /* workspace null or smaller than moe_q4_forward_workspace() */
#define MOE_Q4_ETIMEOUT 4    /* a bounded device-side wait gave up */
#define MOE_Q4_EDEVICE 5     /* the device flagged bad data (non-finite logit / weight) */
#define MOE_Q4_ENOTSUP 6     /* a size beyond what this build supports */
#define MOE_Q4_EBOUNDS 7     /* a device-side index check failed (debug build only, see below) */

/* Debug build: libmoe_q4 compiled with MOE_Q4_DEBUG defined (the package's
 * build step writes it as libmoe_q4_debug.so beside the release library)
 * checks on the device every index it reads from a routing table or the
 * workspace before using it (token and row numbers, expert ids, grouped-row
 * offsets).  A failing check records MOE_Q4_EBOUNDS in the status word and
 * skips the access; no kernel traps.  The release build makes no such checks
 * and computes the same bits. */

/* Limits of this build. */
#define MOE_Q4_MAX_TABLES 16
#define MOE_Q4_MAX_EXPERTS 512
#define MOE_Q4_MAX_TOPK 16

/* Version of this ABI (MOE_Q4_ABI_VERSION of the built library).  A caller
 * compares it with the header it was built against before any other call. */
MOE_Q4_API int moe_q4_abi_version(void);

/* Static, NUL-terminated description of a status code (never NULL). */
MOE_Q4_API const char* moe_q4_status_string(int status);

/* ---------------------------------------------------------------------------
 * moe_q4_pack -- quantise bf16 weights into codes + E8M0 scales.
 *
 * Rule ("Codes are indices into the per-layer grid -- not E2M1": codes are
 * packed against gmax * 2^e >= amax, the grid is not amax-normalised), per
 * 32-weight block along K of expert e with table t = tables[table_id[e]]:
 *   e_blk = the smallest integer with max(t) * 2^e_blk >= max |x|, clamped to
 *           [-127, 127] (an all-zero block takes -127); scale byte = e_blk+127;
 *   code  = (x < 0 ? 8 : 0) | argmin_i |(|x| / 2^e_blk) - t[i]|, distances in
 *           fp64, a tie taking the lower index.
 * Arguments:
 *   w            device, bf16 [E][N][K] (K contiguous);
 *   E, N, K      E >= 0, N >= 0, K >= 0, K % 32 == 0;
 *   tables       host, fp32 [n_tables][8] magnitudes, each finite and >= 0
 *                with a positive maximum; 1 <= n_tables <= MOE_Q4_MAX_TABLES;
 *   table_id     host, uint8 [E], each < n_tables;
 *   weight       device, uint8 [E][N][K/2] (out);
 *   weight_scale device, uint8 [E][N][K/32] (out);
 *   status       device, one int32 (in/out): left unchanged when all inputs
 *                are finite, set to MOE_Q4_EDEVICE if any input is NaN/Inf
 *                (the affected block's bytes are then unspecified).
 * Bit-exact with the reference definition above.
 * ------------------------------------------------------------------------- */
MOE_Q4_API int moe_q4_pack(const void* w, int E, int N, int K, const float* tables, int n_tables,
                const uint8_t* table_id, uint8_t* weight, uint8_t* weight_scale,
                int32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * moe_q4_dequant -- materialise packed weights as bf16 (the "materialize once"
 * step of "GLM-5.2-EXL3-DENSE6-MTP78", "Serving stack" patch 2).
 *
 * out[e][n][k] = bf16(fp32(t[code & 7]) * 2^(s - 127)) with the fp32 multiply
 * and the bf16 conversion both rounding to nearest even, the sign then
 * applied by flipping bit 15 (a signed zero level gives -0.0), and scale byte
 * 0xFF (E8M0 NaN) giving 0x7FC0 with the code's sign.  Bit-exact.
 *   weight        device, uint8 [E][N][K/2];
 *   weight_scale  device, uint8 [E][N][K/32];
 *   tables, n_tables, table_id: as for moe_q4_pack (host);
 *   out           device, bf16 [E][N][K] (out).
 * ------------------------------------------------------------------------- */
MOE_Q4_API int moe_q4_dequant(const uint8_t* weight, const uint8_t* weight_scale, const float* tables,
                   int n_tables, const uint8_t* table_id, int E, int N, int K, void* out,
                   void* stream);

/* ---------------------------------------------------------------------------
 * moe_q4_router -- router logits of T tokens: the router gate ("mlp.gate",
 * held in BF16 per "GLM-5.2-EXL3-DENSE6-MTP78", "Quant recipe") applied to
 * the hidden states ahead of routing:
 *   logits[t][e] = sum over h of x[t][h] * w[e][h]   (fp32 accumulate)
 * Deterministic: the same inputs give the same bits (fixed summation order).
 *   x         device, bf16 [T][H], 16-byte aligned;
 *   w         device, bf16 [E][H], 16-byte aligned;
 *   T >= 0; H > 0, H % 32 == 0; E > 0;
 *   logits    device, fp32 [T][E] (out): the input of moe_q4_forward;
 *   ws        device workspace of at least moe_q4_router_workspace(T, H, E)
 *             bytes (16-byte aligned, 256-byte aligned above T = 32; may be
 *             NULL when that is 0, as it is for T <= 32 with H % 128 == 0),
 *             owned by the call until the enqueued work completes.  Above
 *             T = 32 with E % 128 == 0 and H % 64 == 0 the gate runs on the
 *             tensor cores (tcgen05) and the workspace's first int32 is a
 *             status word (MOE_Q4_ETIMEOUT if a bounded device wait gave up;
 *             read it with moe_q4_read_status);
 *   ws_bytes  size of ws.
 * Returns MOE_Q4_EINVAL for bad sizes or pointers, MOE_Q4_EWORKSPACE for a
 * missing or short workspace; no host synchronisation, no allocation.
 * ------------------------------------------------------------------------- */
MOE_Q4_API size_t moe_q4_router_workspace(int T, int H, int E);
MOE_Q4_API int moe_q4_router(const void* x, const void* w, int T, int H, int E, float* logits, void* ws,
                             size_t ws_bytes, void* stream);

/* A packed MoE layer.  Device pointers are borrowed for the duration of
 * each call; tables and table_id are host memory read during each call. */
typedef struct moe_q4_layer {
  int E;                    /* routed experts, 1..MOE_Q4_MAX_EXPERTS */
  int H;                    /* hidden size, % 128 == 0 */
  int I;                    /* expert intermediate size, % 128 == 0 */
  const uint8_t* gate_w;    /* device [E][I][H/2], 16-byte aligned */
  const uint8_t* gate_s;    /* device [E][I][H/32], 8-byte aligned */
  const uint8_t* up_w;      /* device [E][I][H/2], 16-byte aligned */
  const uint8_t* up_s;      /* device [E][I][H/32], 8-byte aligned */
  const uint8_t* down_w;    /* device [E][H][I/2], 16-byte aligned */
  const uint8_t* down_s;    /* device [E][H][I/32], 8-byte aligned */
  const float* tables;      /* host [n_tables][8] magnitudes */
  int n_tables;             /* 1..MOE_Q4_MAX_TABLES */
  const uint8_t* table_id;  /* host [E]: table of each expert */
} moe_q4_layer;

/* Bytes of device workspace moe_q4_forward needs for T tokens and top_k
 * (0 if the arguments are invalid).  Deterministic in (layer shape, T, top_k). */
MOE_Q4_API size_t moe_q4_forward_workspace(const moe_q4_layer* layer, int T, int top_k);

/* ---------------------------------------------------------------------------
 * moe_q4_forward -- one MoE layer for T tokens.
 *
 * Routing: per token the top_k largest logits (equal logits: lower expert id
 * first), ids in descending-logit order; weights softmax over the kept
 * logits in fp32.  Rows are grouped by expert (ascending id), tokens
 * ascending within an expert.  Each expert's rows go through the small-M
 * streaming path or the tensor-core path, chosen on the device from the
 * per-expert row count.  The intermediate h = silu(g)*u is computed in fp32
 * and stored as bf16; on the small-M path also the bf16 rounding of its
 * remainder, so that path's down GEMM sees h to ~16 significant bits.  y is
 * fp32; the combine sums the top_k slots in slot order in fp32
 * (deterministic, no atomics).
 * Arguments:
 *   layer      see moe_q4_layer;
 *   x          device, bf16 [T][H];
 *   logits     device, fp32 [T][E];
 *   T          0 <= T; T * top_k <= 2^24;
 *   top_k      1 <= top_k <= min(E, MOE_Q4_MAX_TOPK);
 *   out        device, bf16 [T][H] (out): out_f32 rounded to nearest even;
 *   out_f32    optional device fp32 [T][H] (out), NULL to skip: the combine's
 *              fp32 sum, before the bf16 rounding of `out`;
 *   topk_ids   optional device int32 [T][top_k] (out), NULL to skip;
 *   topk_w     optional device fp32 [T][top_k] (out), NULL to skip;
 *   counts     optional device int32 [E] rows per expert (out), NULL to skip;
 *   ws         device workspace, 256-byte aligned, at least
 *              moe_q4_forward_workspace(layer, T, top_k) bytes; the call owns
 *              it until the enqueued work completes;
 *   ws_bytes   size of ws.
 * Device-detected errors (a non-finite logit) set the workspace status word;
 * the output is then unspecified.  No host synchronisation, no allocation.
 * ------------------------------------------------------------------------- */
MOE_Q4_API int moe_q4_forward(const moe_q4_layer* layer, const void* x, const float* logits,
                              int T, int top_k, void* out, float* out_f32, int32_t* topk_ids,
                              float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                              void* stream);

/* ---------------------------------------------------------------------------
 * A shared expert beside the routed ones ("GLM-5.2 EXL3 TR3 v4" README,
 * "Checkpoint layout update"; HF discussion #2 "Store shared experts in
 * BF16"): the shared-expert MLP kept as its original BF16 weights, gate and
 * up concatenated into one payload so that one launch computes both.
 * Every token goes through it with weight 1:
 *   out[t] = sum_j w_j * y_j[t] + Wd (silu(Wg x_t) * (Wu x_t)).
 * ------------------------------------------------------------------------- */
typedef struct moe_q4_shared {
  int I;                 /* intermediate size of the shared expert, % 128 == 0 */
  const void* gate_up;   /* device bf16 [2I][H], 16-byte aligned: rows 0..I-1 the
                            gate, rows I..2I-1 the up projection */
  const void* down;      /* device bf16 [H][I], 16-byte aligned */
} moe_q4_shared;

/* Workspace of moe_q4_forward_ex (0 if the arguments are invalid); with
 * shared == NULL it equals moe_q4_forward_workspace. */
MOE_Q4_API size_t moe_q4_forward_ex_workspace(const moe_q4_layer* layer, const moe_q4_shared* shared, int T,
                                              int top_k);

/* moe_q4_forward plus the shared expert (shared may be NULL: then exactly
 * moe_q4_forward).  The shared expert runs on the tensor cores in two
 * launches (merged gate+up with the SwiGLU, then down; at decode sizes each
 * splits its K range over the SMs and adds the split partial sums in a fixed
 * order), and the combine adds its output after the k routed slots, in fp32:
 * deterministic.  Arguments and errors as for moe_q4_forward; the workspace
 * must hold moe_q4_forward_ex_workspace(layer, shared, T, top_k) bytes. */
MOE_Q4_API int moe_q4_forward_ex(const moe_q4_layer* layer, const moe_q4_shared* shared, const void* x,
                                 const float* logits, int T, int top_k, void* out, float* out_f32,
                                 int32_t* topk_ids, float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                                 void* stream);

/* ---------------------------------------------------------------------------
 * moe_q4_forward_gated -- the layer with its router gate in front: from the
 * hidden states alone ("GLM-5.2-EXL3-DENSE6-MTP78", "Quant recipe": the
 * mlp.gate linear kept in BF16, ahead of the routed experts).
 *   logits[t][e] = sum_h x[t][h] * router_w[e][h]   (fp32 accumulation, as
 *   moe_q4_router computes them, bit for bit), then moe_q4_forward_ex on those
 *   logits.
 * For T <= 32 (with T * top_k <= 4096) one launch computes the logits on
 * every SM and routes and groups the tokens: each CTA adds its logits'
 * partial sums in a fixed order, publishes them device-wide and takes a
 * ticket; the last CTA to finish routes (no CTA waits for another).  Larger
 * T runs moe_q4_router's kernels (tensor cores for E % 128 == 0), then the
 * routing kernels.
 * Arguments as for moe_q4_forward_ex, plus:
 *   router_w   device bf16 [E][H], 16-byte aligned;
 *   logits     optional device fp32 [T][E] (out), 4-byte aligned: the
 *              router's logits; NULL keeps them in the workspace;
 *   ws         at least moe_q4_forward_gated_workspace(layer, shared, T,
 *              top_k) bytes, 256-byte aligned.
 * Device errors (a non-finite logit, a timed-out wait of the tensor-core
 * router) set the workspace status word, as for moe_q4_forward.
 * ------------------------------------------------------------------------- */
MOE_Q4_API size_t moe_q4_forward_gated_workspace(const moe_q4_layer* layer, const moe_q4_shared* shared, int T,
                                                 int top_k);
MOE_Q4_API int moe_q4_forward_gated(const moe_q4_layer* layer, const moe_q4_shared* shared, const void* router_w,
                                    const void* x, int T, int top_k, void* out, float* out_f32, float* logits,
                                    int32_t* topk_ids, float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                                    void* stream);

/* Synchronise `stream`, then return the status recorded in the workspace by
 * the last moe_q4_forward on it (MOE_Q4_OK, MOE_Q4_EDEVICE, MOE_Q4_ETIMEOUT),
 * or MOE_Q4_ECUDA if the stream itself reports an error. */
MOE_Q4_API int moe_q4_forward_status(const void* ws, void* stream);

/* ---------------------------------------------------------------------------
 * moe_q4_forward_host -- the same layer with HOST activations and output.
 * Copies x and logits host->device into the workspace, runs moe_q4_forward,
 * copies out device->host and waits for the stream; returns the forward's
 * device status.  x, logits and out are host pointers (pinned memory gives
 * asynchronous copies); the weights stay on the device.  The workspace must
 * hold moe_q4_forward_host_workspace(layer, T, top_k) bytes.
 * ------------------------------------------------------------------------- */
MOE_Q4_API size_t moe_q4_forward_host_workspace(const moe_q4_layer* layer, int T, int top_k);
MOE_Q4_API int moe_q4_forward_host(const moe_q4_layer* layer, const void* x_host, const float* logits_host,
                        int T, int top_k, void* out_host, void* ws, size_t ws_bytes,
                        void* stream);

/* moe_q4_forward_host without the wait: the copies in, the forward and the
 * copy out are enqueued on `stream` and the call returns (MOE_Q4_OK or an
 * argument / launch error).  x_host and logits_host are read, and out_host
 * written, when the stream reaches the copies: with pinned memory the caller
 * keeps them untouched until then (a later moe_q4_forward_status on the
 * same stream waits for the work and returns its device status).  Calls
 * enqueued back to back on one stream and workspace run in order. */
MOE_Q4_API int moe_q4_forward_host_async(const moe_q4_layer* layer, const void* x_host, const float* logits_host,
                                         int T, int top_k, void* out_host, void* ws, size_t ws_bytes,
                                         void* stream);

/* ---------------------------------------------------------------------------
 * moe_q4_route -- the routing and grouping steps of moe_q4_forward alone,
 * into caller buffers (all device, all required):
 *   ids [T][top_k] int32, w [T][top_k] fp32: as moe_q4_forward's topk_ids/w;
 *   counts [E] int32; offsets [E+1] int32 (exclusive scan of counts);
 *   row_token [T*top_k] int32: token of each expert-grouped row (experts
 *     ascending, tokens ascending within an expert);
 *   inv [T][top_k] int32: grouped row of (token, slot).
 * logits: device fp32 [T][E].  ws: device workspace of at least
 * moe_q4_route_workspace(E, T, top_k) bytes, 256-byte aligned; its first
 * int32 is the status word (read with moe_q4_forward_status(ws, stream)).
 * Bit-exact: the grouping is unique given the ids, and the ids are unique
 * under the ordering above.
 * ------------------------------------------------------------------------- */
MOE_Q4_API size_t moe_q4_route_workspace(int E, int T, int top_k);
MOE_Q4_API int moe_q4_route(const float* logits, int T, int E, int top_k, int32_t* ids, float* w,
                            int32_t* counts, int32_t* offsets, int32_t* row_token, int32_t* inv,
                            void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_q4_forward_stages -- moe_q4_forward with cudaEvent_t records at the
 * kernel boundaries, for timing each kernel on the launching stream:
 *   events[0] before routing, [1] after routing/grouping, [2] after the
 *   gather of activation rows, [3] after the tensor-core gate/up + SwiGLU,
 *   [4] after the small-M gate/up + SwiGLU, [5] after the tensor-core down
 *   projection, [6] after the small-M down projection, [7] after the combine
 *   (a kernel with no rows to take, e.g. the tensor-core ones for T <= 16,
 *   is not launched: its two events are recorded back to back).
 * events: host array of n_events (>= 8) cudaEvent_t handles created by the
 * caller.  The records separate the stages (no programmatic overlap across
 * them), so throughput is measured with moe_q4_forward itself.
 * ------------------------------------------------------------------------- */
MOE_Q4_API int moe_q4_forward_stages(const moe_q4_layer* layer, const void* x,
                                     const float* logits, int T, int top_k, void* out,
                                     void* ws, size_t ws_bytes, void* stream,
                                     void* const* events, int n_events);

/* ---------------------------------------------------------------------------
 * moe_q4_forward_noalloc -- moe_q4_forward for callers that cannot allocate
 * device memory (no workspace argument).  The pages have no counterpart of
 * this entry point; it exists for callers such as a serving loop that may not
 * call cudaMalloc once running (an allocation can synchronise the device), or
 * code that only holds raw device pointers from another framework's allocator.
 *
 * The workspace lives in a static device array of the library, 8 MiB, held on
 * every GPU that loads the library until the process exits.  Sizes whose
 * workspace (moe_q4_forward_workspace) exceeds it are rejected with
 * MOE_Q4_ENOTSUP before anything is launched; at the GLM-5.2 layer shape
 * (H 6144, I 2048, 256 experts, top-8) that admits T <= 9.  The first call on
 * a device looks up the array's device address (cudaGetSymbolAddress) and
 * caches it: make that first call before any stream capture, and do not use
 * this entry point on a device after cudaDeviceReset of that device (the
 * cached address would be stale).  All calls share the array and it keeps
 * the last call's contents; calls that overlap on the GPU race on it, so
 * serialise them.
 * Arguments as for moe_q4_forward, plus:
 *   status   optional device int32 (out), NULL to skip: receives the
 *            forward's device status word (MOE_Q4_OK / MOE_Q4_EDEVICE /
 *            MOE_Q4_ETIMEOUT) by a stream-ordered device-to-device copy;
 *            with T == 0 it receives MOE_Q4_OK.
 * No allocation of any kind (no cudaMalloc/cudaFree, no allocating library
 * routine); the call returns without waiting for the GPU.
 * ------------------------------------------------------------------------- */
MOE_Q4_API int moe_q4_forward_noalloc(const moe_q4_layer* layer, const void* x,
                                      const float* logits, int T, int top_k, void* out,
                                      float* out_f32, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * moe_q4_lloyd_hist / moe_q4_lloyd_solve -- fit a layer's 8-level magnitude
 * grid by weighted Lloyd-Max ("aidendle94/GLM-5.2-NF4-Lloyd-Experts-GPTQ",
 * "What this is": Lloyd-Max over the pooled ratios |W / 2^e| of all the
 * layer's weights, each ratio weighted by (2^e)^2).
 *
 * Procedure (the page names the objective; the steps around it are this
 * library's reading):
 *   - e is each 32-weight block's exponent under the pack rule (the smallest
 *     e with gmax * 2^e >= max |w|, clamped to [-127, 127]), with gmax the
 *     largest level of grid0, fixed for the whole fit;
 *   - a step assigns every ratio |w| / 2^e to its nearest level (fp64
 *     distance, a tie to the lower index) and moves each level to the
 *     (2^e)^2-weighted mean of its ratios; a level with no ratio keeps its
 *     value;
 *   - steps repeat until no level moves by more than tol, or max_iter steps;
 *     the levels are then rounded to fp32.
 * moe_q4_lloyd_hist adds the ratios of n_blocks blocks of 32 bf16 weights
 * (device, 16-byte aligned, each run of 32 one block along K) into the
 * workspace's histogram (reset != 0 clears it first); call it once per array
 * to pool several arrays (a layer's projections).  moe_q4_lloyd_solve runs
 * the steps on the histogram and writes grid (device fp32 [8]) and iters
 * (device int32, the steps taken).
 *   grid0   host fp32 [8]: finite, no sign bit, strictly ascending, gmax < 16
 *           (MOE_Q4_EINVAL / MOE_Q4_ENOTSUP otherwise);
 *   ws      device workspace of moe_q4_lloyd_workspace(grid0) bytes, 256-byte
 *           aligned; its first int32 is a status word (read with
 *           moe_q4_read_status): MOE_Q4_EDEVICE if a weight is NaN or Inf
 *           (those weights are left out), MOE_Q4_ENOTSUP if a ratio exceeds
 *           gmax (only for blocks whose exponent is clamped at 127).
 * Deterministic: the histogram sums powers of four (exact while a bin's sum
 * stays within 2^53 of its smallest term) and the steps add the per-level
 * sums in a fixed order.  No allocation, no host synchronisation.
 * ------------------------------------------------------------------------- */
MOE_Q4_API size_t moe_q4_lloyd_workspace(const float* grid0);
MOE_Q4_API int moe_q4_lloyd_hist(const void* w, long long n_blocks, const float* grid0, int reset, void* ws,
                                 size_t ws_bytes, void* stream);
MOE_Q4_API int moe_q4_lloyd_solve(const float* grid0, int max_iter, double tol, float* grid, int32_t* iters,
                                  const void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_q4_combine -- the layer's weighted combine alone (used by the expert-
 * parallel forward, where the expert outputs come back from other ranks):
 *   out[t] = sum_{j<k} w[t][j] * y[r(t, j)],  r(t, j) = inv ? inv[t*k+j] : t*k+j,
 * summed in slot order in fp32, rounded to bf16 (the same arithmetic as the
 * forward's combine: deterministic).
 *   y        device fp32 [T*k][H], 16-byte aligned;   w  device fp32 [T][k];
 *   inv      optional device int32 [T][k] (NULL: rows in (token, slot) order);
 *   out      device bf16 [T][H] (out);  out_f32  optional device fp32 [T][H];
 *   H % 4 == 0, 1 <= k <= MOE_Q4_MAX_TOPK.
 * ------------------------------------------------------------------------- */
MOE_Q4_API int moe_q4_combine(const float* y, const float* w, const int32_t* inv, int T, int k, int H, void* out,
                              float* out_f32, void* stream);

/* ---------------------------------------------------------------------------
 * moe_q4_selftest_wait -- test support: checks that a bounded device wait
 * gives up and reports instead of hanging.  One CTA: a producer warp that
 * issues nothing and a consumer warp waiting on the stage barrier it would
 * have completed, with the same bounded wait and teardown as the layer's
 * kernels.  After limit_us microseconds (1 .. 2,000,000) the wait gives up
 * and MOE_Q4_ETIMEOUT is recorded in *status (device int32, left unchanged
 * otherwise; it records only over MOE_Q4_OK).  The kernel returns normally:
 * the context stays usable for the next call.  Not part of the layer; the
 * pages have no counterpart.
 * ------------------------------------------------------------------------- */
MOE_Q4_API int moe_q4_selftest_wait(int32_t* status, unsigned limit_us, void* stream);

/* Synchronise `stream` and return the int32 at device address `status`
 * (as written by moe_q4_pack), or MOE_Q4_ECUDA. */
MOE_Q4_API int moe_q4_read_status(const int32_t* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_Q4_H */
