// C-ABI layer of libmoe_q4: argument validation, workspace layout, and the
// launch sequence of one MoE forward (route -> gate/up+SwiGLU -> down ->
// combine).  Nothing here allocates; every launch goes on the caller's stream.
#include <math.h>
#include <string.h>

#include <climits>

#include "q4_api_internal.h"
#include "q4_common.cuh"

using namespace q4;

namespace {

constexpr size_t kAlign = 256;
// Experts with at most this many rows take the streaming (mma.sync) path;
// larger ones the tcgen05 path.
constexpr int kDecodeMaxRows = 16;

bool uses_prefill(int T) { return T > kDecodeMaxRows; }

// Persistent small-M kernels run at most this many CTAs (one per SM); the
// workspace holds two split-tile partial slots per CTA.
constexpr int kDkMaxGrid = 160;
constexpr int kDkSlabs = 8;  // small-M row slabs per 128-row tile (one split-tile counter each)

int dk_grid() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  return sms < kDkMaxGrid ? sms : kDkMaxGrid;
}

size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

bool layer_ok(const moe_q4_layer* L) {
  if (!L) return false;
  if (L->E < 1 || L->E > kMaxExperts) return false;
  if (L->H <= 0 || L->I <= 0 || (L->H % 128) || (L->I % 128)) return false;
  if (!L->gate_w || !L->gate_s || !L->up_w || !L->up_s || !L->down_w || !L->down_s) return false;
  const uint8_t* p[3] = {L->gate_w, L->up_w, L->down_w};
  for (auto q : p)
    if ((uintptr_t)q & 15) return false;
  const uint8_t* sc[3] = {L->gate_s, L->up_s, L->down_s};
  for (auto q : sc)
    if ((uintptr_t)q & 7) return false;
  return true;
}

bool shape_ok(const moe_q4_layer* L, int T, int top_k) {
  if (!layer_ok(L) || T < 0) return false;
  if (top_k < 1 || top_k > L->E || top_k > kMaxTopK) return false;
  if ((long long)T * top_k > (1LL << 24)) return false;
  return true;
}

// Workspace layout, every array 256-byte aligned:
//   header int32[64] | ids int32[T*k] | w f32[T*k] | counts int32[E] |
//   offsets int32[E+1] | row_token int32[T*k] | inv int32[T*k] |
//   dec_list int32[E] | pre_list int32[E] | mid_list int32[E] | tiles int32[E+1] |
//   chunk_cnt int32[chunks][E] | chunk_base int32[chunks][E] (256-token chunks
//   of the grouping, T > 256 only) | h bf16[T*k][I] |
//   h_lo bf16[T*k][I] | y f32[T*k][H] | xg bf16[T*k][H] (activation rows in
//   expert order, T > 16 only) | split-tile counters int32[units] | partial sums of the
//   small-M kernels f32[2*160][4][min(16,T)][128] (two 128-row tiles per unit,
//   gate/up then down) | with a shared expert: h_s | y_s | its split partial
//   sums | with the router gate in front: logits f32[T][E] | its partial sums
struct Layout {
  size_t hdr, ids, w, counts, offsets, row_token, inv, dec_list, pre_list, mid_list, tiles, chunk_cnt,
      chunk_base, h, h_lo, y, xg,
      dk_counter,
      dk_partial, h_s, y_s, sx_partial, logits, router_partial, end;
  int dk_units_gu, dk_units_dn, n_max;
};

bool shared_ok(const moe_q4_layer* L, const moe_q4_shared* S) {
  if (!S) return true;
  if (S->I <= 0 || (S->I % 128) || !S->gate_up || !S->down) return false;
  if (((uintptr_t)S->gate_up & 15) || ((uintptr_t)S->down & 15)) return false;
  return L->H % 64 == 0;
}

Layout layout(const moe_q4_layer* L, int T, int k, const moe_q4_shared* S = nullptr, bool gated = false) {
  const size_t R = (size_t)T * k;
  Layout o;
  size_t p = 0;
  o.hdr = p;
  p = align_up(p + sizeof(int32_t) * kHeaderWords);
  o.ids = p;
  p = align_up(p + sizeof(int32_t) * R);
  o.w = p;
  p = align_up(p + sizeof(float) * R);
  o.counts = p;
  p = align_up(p + sizeof(int32_t) * L->E);
  o.offsets = p;
  p = align_up(p + sizeof(int32_t) * (L->E + 1));
  o.row_token = p;
  p = align_up(p + sizeof(int32_t) * R);
  o.inv = p;
  p = align_up(p + sizeof(int32_t) * R);
  o.dec_list = p;
  p = align_up(p + sizeof(int32_t) * L->E);
  o.pre_list = p;
  p = align_up(p + sizeof(int32_t) * L->E);
  o.mid_list = p;
  p = align_up(p + sizeof(int32_t) * L->E);
  o.tiles = p;
  p = align_up(p + sizeof(int32_t) * (L->E + 1));
  const size_t chunk_words = (size_t)q4_route_chunks(T) * L->E;
  o.chunk_cnt = p;
  p = align_up(p + sizeof(int32_t) * chunk_words);
  o.chunk_base = p;
  p = align_up(p + sizeof(int32_t) * chunk_words);
  o.h = p;
  p = align_up(p + sizeof(__nv_bfloat16) * R * L->I);
  o.h_lo = p;
  p = align_up(p + sizeof(__nv_bfloat16) * R * L->I);
  o.y = p;
  p = align_up(p + sizeof(float) * R * L->H);
  // grouped activation rows: read by the tensor-core path only (T > 16)
  o.xg = 0;
  if (uses_prefill(T)) {
    o.xg = p;
    p = align_up(p + sizeof(__nv_bfloat16) * R * L->H);
  }
  const int max_exp = (int)(R < (size_t)L->E ? R : (size_t)L->E);
  o.dk_units_gu = max_exp * (L->I / 128);
  o.dk_units_dn = max_exp * ((L->H + 255) / 256);  // down units: two 128-row tiles
  o.n_max = T < 16 ? T : 16;
  o.dk_counter = p;
  p = align_up(p + sizeof(int32_t) * (size_t)(o.dk_units_gu + o.dk_units_dn) * kDkSlabs);
  o.dk_partial = p;
  p = align_up(p + sizeof(float) * (size_t)2 * kDkMaxGrid * 4 * o.n_max * 128);  // 2 tiles per unit, both kernels
  // shared expert: h_s bf16 [T][I_s] | y_s f32 [T][H] | split-K partial sums
  o.h_s = o.y_s = o.sx_partial = 0;
  if (S) {
    o.h_s = p;
    p = align_up(p + sizeof(__nv_bfloat16) * (size_t)T * S->I);
    o.y_s = p;
    p = align_up(p + sizeof(float) * (size_t)T * L->H);
    const size_t pa = q4_dense_partial_bytes(T, S->I, L->H, 2), pb = q4_dense_partial_bytes(T, L->H, S->I, 1);
    o.sx_partial = p;
    p = align_up(p + (pa > pb ? pa : pb));
  }
  // router gate in front (moe_q4_forward_gated): logits f32 [T][E] | its partial sums
  o.logits = o.router_partial = 0;
  if (gated) {
    o.logits = p;
    p = align_up(p + sizeof(float) * (size_t)T * L->E);
    o.router_partial = p;
    p = align_up(p + q4_router_partial_bytes(T, L->H, L->E));
  }
  o.end = p;
  return o;
}

// Extra staging for moe_q4_forward_host: x_in bf16[T][H] | logits_in f32[T][E] | out bf16[T][H].
struct HostStage {
  size_t x, logits, out, end;
};

HostStage host_stage(const moe_q4_layer* L, int T, size_t base) {
  HostStage s;
  size_t p = base;
  s.x = p;
  p = align_up(p + sizeof(__nv_bfloat16) * (size_t)T * L->H);
  s.logits = p;
  p = align_up(p + sizeof(float) * (size_t)T * L->E);
  s.out = p;
  p = align_up(p + sizeof(__nv_bfloat16) * (size_t)T * L->H);
  s.end = p;
  return s;
}

int run_forward(const moe_q4_layer* L, const TableParams& tp, const void* x, const float* logits,
                int T, int k, void* out, float* out_f32, int32_t* topk_ids, float* topk_w,
                int32_t* counts, char* ws, cudaStream_t s, void* const* events = nullptr,
                const moe_q4_shared* S = nullptr, const void* router_w = nullptr) {
  const Layout o = layout(L, T, k, S, router_w != nullptr);
  FwdArgs a;
  memset(&a, 0, sizeof a);
  a.T = T;
  a.k = k;
  a.E = L->E;
  a.H = L->H;
  a.I = L->I;
  a.dec_max = kDecodeMaxRows;
  a.tile_n = q4_prefill_tile_n();
  a.x = (const __nv_bfloat16*)x;
  a.logits = logits;
  a.out = (__nv_bfloat16*)out;
  a.hdr = (int32_t*)(ws + o.hdr);
  a.ids = (int32_t*)(ws + o.ids);
  a.w = (float*)(ws + o.w);
  a.counts = (int32_t*)(ws + o.counts);
  a.offsets = (int32_t*)(ws + o.offsets);
  a.row_token = (int32_t*)(ws + o.row_token);
  a.inv = (int32_t*)(ws + o.inv);
  a.dec_list = (int32_t*)(ws + o.dec_list);
  a.pre_list = (int32_t*)(ws + o.pre_list);
  a.mid_list = (int32_t*)(ws + o.mid_list);
  // the wide kernel's weight tiles are 256 rows: layers whose I or H is not a
  // multiple of 256 keep every tensor-core expert on the swap-AB tiles
  const bool wide_ok = L->I % 256 == 0 && L->H % 256 == 0;
  a.wide_max = wide_ok ? q4_prefill_wide_max() : kDecodeMaxRows;
  a.tiles = (int32_t*)(ws + o.tiles);
  a.chunk_cnt = (int32_t*)(ws + o.chunk_cnt);
  a.chunk_base = (int32_t*)(ws + o.chunk_base);
  a.xg = o.xg ? (__nv_bfloat16*)(ws + o.xg) : nullptr;
  a.dk_counter = (int32_t*)(ws + o.dk_counter);
  a.dk_counter_n = (o.dk_units_gu + o.dk_units_dn) * kDkSlabs;
  a.h = (__nv_bfloat16*)(ws + o.h);
  a.h_lo = (__nv_bfloat16*)(ws + o.h_lo);
  a.y = (float*)(ws + o.y);
  a.out_f32 = out_f32;
  a.y_s = S ? (const float*)(ws + o.y_s) : nullptr;
  a.user_ids = topk_ids;
  a.user_w = topk_w;
  a.user_counts = counts;
  a.gate_w = L->gate_w;
  a.gate_s = L->gate_s;
  a.up_w = L->up_w;
  a.up_s = L->up_s;
  a.down_w = L->down_w;
  a.down_s = L->down_s;
  auto mark = [&](int i) {
    if (events && cudaEventRecord((cudaEvent_t)events[i], s) != cudaSuccess) return MOE_Q4_ECUDA;
    return MOE_Q4_OK;
  };
  // With T <= kDecodeMaxRows no expert can have more rows than the streaming
  // path takes, so the tensor-core kernels are not launched at all.
  const bool pre = uses_prefill(T);
  int rc = mark(0);
  if (rc == MOE_Q4_OK && router_w) {
    // the router gate in front: the logits land in `logits` (the caller's
    // buffer or the workspace's); the status word and the fused kernel's
    // ticket start at zero, and the routing leaves the status alone
    a.keep_status = 1;
    a.logits_in_forward = 1;
    if (cudaMemsetAsync(a.hdr, 0, 8 * sizeof(int32_t), s) != cudaSuccess) rc = MOE_Q4_ECUDA;
    if (rc == MOE_Q4_OK && q4_router_route_fused(T, L->H, k)) {
      rc = q4_launch_router_route(a, router_w, s);
    } else if (rc == MOE_Q4_OK) {
      rc = q4_launch_router(x, router_w, T, L->H, L->E, const_cast<float*>(logits), ws + o.router_partial,
                            a.hdr + kStatus, s);
      if (rc == MOE_Q4_OK) rc = q4_launch_route(a, s);
    }
  } else if (rc == MOE_Q4_OK) {
    rc = q4_launch_route(a, s);
  }
  if (rc == MOE_Q4_OK) rc = mark(1);
  const int grid = dk_grid();
  float* part_gu = (float*)(ws + o.dk_partial);
  float* part_dn = part_gu + (size_t)2 * kDkMaxGrid * 2 * o.n_max * 128;
  int32_t* cnt_gu = a.dk_counter;
  int32_t* cnt_dn = a.dk_counter + (size_t)o.dk_units_gu * kDkSlabs;
  // grouped activation rows feed the tensor-core path only (the small-M kernels
  // copy their rows from x themselves)
  if (rc == MOE_Q4_OK && pre) rc = q4_launch_gather(a, s);
  if (rc == MOE_Q4_OK) rc = mark(2);
  if (rc == MOE_Q4_OK && pre) rc = q4_launch_prefill(a, tp, true, wide_ok, s);
  if (rc == MOE_Q4_OK && pre && wide_ok) rc = q4_launch_prefill_wide(a, tp, true, s);
  if (rc == MOE_Q4_OK) rc = mark(3);
  if (rc == MOE_Q4_OK) rc = q4_launch_decode(a, tp, true, part_gu, cnt_gu, grid, s);
  if (rc == MOE_Q4_OK) rc = mark(4);
  if (rc == MOE_Q4_OK && pre) rc = q4_launch_prefill(a, tp, false, wide_ok, s);
  if (rc == MOE_Q4_OK && pre && wide_ok) rc = q4_launch_prefill_wide(a, tp, false, s);
  if (rc == MOE_Q4_OK) rc = mark(5);
  if (rc == MOE_Q4_OK) rc = q4_launch_decode(a, tp, false, part_dn, cnt_dn, grid, s);
  if (rc == MOE_Q4_OK && S) {
    // the shared expert: merged gate+up with the SwiGLU, then down (its time
    // falls between events 6 and 7, with the combine)
    __nv_bfloat16* h_s = (__nv_bfloat16*)(ws + o.h_s);
    float* y_s = (float*)(ws + o.y_s);
    float* part = (float*)(ws + o.sx_partial);
    rc = q4_launch_dense(S->gate_up, 2, S->I, S->I, L->H, x, T, h_s, nullptr, S->I, part, a.hdr + kStatus, s);
    if (rc == MOE_Q4_OK)
      rc = q4_launch_dense(S->down, 1, 0, L->H, S->I, h_s, T, nullptr, y_s, L->H, part, a.hdr + kStatus, s);
  }
  if (rc == MOE_Q4_OK) rc = mark(6);
  if (rc == MOE_Q4_OK) rc = q4_launch_combine(a, s);
  if (rc == MOE_Q4_OK) rc = mark(7);
  return rc;
}

}  // namespace

int q4_fill_tables(TableParams* tp, const float* tables, int n_tables, const uint8_t* table_id, int E) {
  if (!tables || !table_id || n_tables < 1 || n_tables > kMaxTables || E < 0 || E > kMaxExperts)
    return MOE_Q4_EINVAL;
  memset(tp, 0, sizeof *tp);
  tp->n = n_tables;
  for (int t = 0; t < n_tables; ++t) {
    float mx = 0.0f;
    for (int i = 0; i < 8; ++i) {
      const float v = tables[8 * t + i];
      if (!isfinite(v) || signbit(v)) return MOE_Q4_EINVAL;
      mx = v > mx ? v : mx;
      tp->t[t][i] = v;
    }
    if (!(mx > 0.0f)) return MOE_Q4_EINVAL;
  }
  for (int e = 0; e < E; ++e) {
    if (table_id[e] >= n_tables) return MOE_Q4_EINVAL;
    tp->id[e] = table_id[e];
  }
  return MOE_Q4_OK;
}

extern "C" int moe_q4_abi_version(void) { return MOE_Q4_ABI_VERSION; }

extern "C" const char* moe_q4_status_string(int status) {
  switch (status) {
    case MOE_Q4_OK: return "ok";
    case MOE_Q4_EINVAL: return "invalid argument";
    case MOE_Q4_ECUDA: return "CUDA error";
    case MOE_Q4_EWORKSPACE: return "workspace missing or too small";
    case MOE_Q4_ETIMEOUT: return "bounded device wait timed out";
    case MOE_Q4_EDEVICE: return "device detected invalid data (non-finite input)";
    case MOE_Q4_ENOTSUP: return "size not supported by this build";
    case MOE_Q4_EBOUNDS: return "device index check failed (debug build)";
    default: return "unknown status";
  }
}

extern "C" size_t moe_q4_forward_workspace(const moe_q4_layer* layer, int T, int top_k) {
  if (!shape_ok(layer, T, top_k)) return 0;
  return layout(layer, T, top_k).end;
}

extern "C" size_t moe_q4_forward_host_workspace(const moe_q4_layer* layer, int T, int top_k) {
  if (!shape_ok(layer, T, top_k)) return 0;
  return host_stage(layer, T, layout(layer, T, top_k).end).end;
}

extern "C" int moe_q4_forward(const moe_q4_layer* layer, const void* x, const float* logits, int T,
                              int top_k, void* out, float* out_f32, int32_t* topk_ids, float* topk_w,
                              int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  if (!shape_ok(layer, T, top_k)) return MOE_Q4_EINVAL;
  TableParams tp;
  int rc = q4_fill_tables(&tp, layer->tables, layer->n_tables, layer->table_id, layer->E);
  if (rc != MOE_Q4_OK) return rc;
  if (T == 0) return MOE_Q4_OK;
  if (!x || !logits || !out || ((uintptr_t)x & 15) || ((uintptr_t)out & 15) || ((uintptr_t)logits & 3) ||
      ((uintptr_t)out_f32 & 15))
    return MOE_Q4_EINVAL;
  if (!ws || ((uintptr_t)ws & (kAlign - 1)) || ws_bytes < layout(layer, T, top_k).end)
    return MOE_Q4_EWORKSPACE;
  return run_forward(layer, tp, x, logits, T, top_k, out, out_f32, topk_ids, topk_w, counts,
                     (char*)ws, (cudaStream_t)stream);
}

extern "C" size_t moe_q4_forward_ex_workspace(const moe_q4_layer* layer, const moe_q4_shared* shared, int T,
                                              int top_k) {
  if (!shape_ok(layer, T, top_k) || !shared_ok(layer, shared)) return 0;
  return layout(layer, T, top_k, shared).end;
}

extern "C" int moe_q4_forward_ex(const moe_q4_layer* layer, const moe_q4_shared* shared, const void* x,
                                 const float* logits, int T, int top_k, void* out, float* out_f32,
                                 int32_t* topk_ids, float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                                 void* stream) {
  if (!shared)
    return moe_q4_forward(layer, x, logits, T, top_k, out, out_f32, topk_ids, topk_w, counts, ws, ws_bytes, stream);
  if (!shape_ok(layer, T, top_k) || !shared_ok(layer, shared)) return MOE_Q4_EINVAL;
  TableParams tp;
  int rc = q4_fill_tables(&tp, layer->tables, layer->n_tables, layer->table_id, layer->E);
  if (rc != MOE_Q4_OK) return rc;
  if (T == 0) return MOE_Q4_OK;
  if (!x || !logits || !out || ((uintptr_t)x & 15) || ((uintptr_t)out & 15) || ((uintptr_t)logits & 3) ||
      ((uintptr_t)out_f32 & 15))
    return MOE_Q4_EINVAL;
  if (!ws || ((uintptr_t)ws & (kAlign - 1)) || ws_bytes < layout(layer, T, top_k, shared).end)
    return MOE_Q4_EWORKSPACE;
  return run_forward(layer, tp, x, logits, T, top_k, out, out_f32, topk_ids, topk_w, counts, (char*)ws,
                     (cudaStream_t)stream, nullptr, shared);
}

extern "C" size_t moe_q4_forward_gated_workspace(const moe_q4_layer* layer, const moe_q4_shared* shared, int T,
                                                 int top_k) {
  if (!shape_ok(layer, T, top_k) || !shared_ok(layer, shared)) return 0;
  return layout(layer, T, top_k, shared, true).end;
}

extern "C" int moe_q4_forward_gated(const moe_q4_layer* layer, const moe_q4_shared* shared, const void* router_w,
                                    const void* x, int T, int top_k, void* out, float* out_f32, float* logits,
                                    int32_t* topk_ids, float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                                    void* stream) {
  if (!shape_ok(layer, T, top_k) || !shared_ok(layer, shared)) return MOE_Q4_EINVAL;
  TableParams tp;
  int rc = q4_fill_tables(&tp, layer->tables, layer->n_tables, layer->table_id, layer->E);
  if (rc != MOE_Q4_OK) return rc;
  if (T == 0) return MOE_Q4_OK;
  if (!router_w || !x || !out || ((uintptr_t)router_w & 15) || ((uintptr_t)x & 15) || ((uintptr_t)out & 15) ||
      ((uintptr_t)out_f32 & 15) || ((uintptr_t)logits & 3))
    return MOE_Q4_EINVAL;
  const Layout o = layout(layer, T, top_k, shared, true);
  if (!ws || ((uintptr_t)ws & (kAlign - 1)) || ws_bytes < o.end) return MOE_Q4_EWORKSPACE;
  float* lg = logits ? logits : reinterpret_cast<float*>((char*)ws + o.logits);
  return run_forward(layer, tp, x, lg, T, top_k, out, out_f32, topk_ids, topk_w, counts, (char*)ws,
                     (cudaStream_t)stream, nullptr, shared, router_w);
}

extern "C" int moe_q4_forward_stages(const moe_q4_layer* layer, const void* x, const float* logits,
                                     int T, int top_k, void* out, void* ws, size_t ws_bytes,
                                     void* stream, void* const* events, int n_events) {
  if (!events || n_events < 8) return MOE_Q4_EINVAL;
  for (int i = 0; i < 8; ++i)
    if (!events[i]) return MOE_Q4_EINVAL;
  if (!shape_ok(layer, T, top_k)) return MOE_Q4_EINVAL;
  TableParams tp;
  int rc = q4_fill_tables(&tp, layer->tables, layer->n_tables, layer->table_id, layer->E);
  if (rc != MOE_Q4_OK) return rc;
  if (T == 0) return MOE_Q4_OK;
  if (!x || !logits || !out || ((uintptr_t)x & 15) || ((uintptr_t)out & 15) || ((uintptr_t)logits & 3))
    return MOE_Q4_EINVAL;
  if (!ws || ((uintptr_t)ws & (kAlign - 1)) || ws_bytes < layout(layer, T, top_k).end)
    return MOE_Q4_EWORKSPACE;
  return run_forward(layer, tp, x, logits, T, top_k, out, nullptr, nullptr, nullptr, nullptr,
                     (char*)ws, (cudaStream_t)stream, events);
}

static int read_device_int(const int32_t* p, cudaStream_t s, int32_t* v) {
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_Q4_ECUDA;
  if (cudaMemcpy(v, p, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_Q4_ECUDA;
  return MOE_Q4_OK;
}

extern "C" int moe_q4_forward_status(const void* ws, void* stream) {
  if (!ws) return MOE_Q4_EWORKSPACE;
  int32_t v = 0;
  const int rc = read_device_int((const int32_t*)ws + kStatus, (cudaStream_t)stream, &v);
  return rc != MOE_Q4_OK ? rc : (int)v;
}

extern "C" int moe_q4_read_status(const int32_t* status, void* stream) {
  if (!status) return MOE_Q4_EINVAL;
  int32_t v = 0;
  const int rc = read_device_int(status, (cudaStream_t)stream, &v);
  return rc != MOE_Q4_OK ? rc : (int)v;
}

extern "C" int moe_q4_forward_host_async(const moe_q4_layer* layer, const void* x_host,
                                         const float* logits_host, int T, int top_k, void* out_host, void* ws,
                                         size_t ws_bytes, void* stream) {
  if (!shape_ok(layer, T, top_k)) return MOE_Q4_EINVAL;
  TableParams tp;
  int rc = q4_fill_tables(&tp, layer->tables, layer->n_tables, layer->table_id, layer->E);
  if (rc != MOE_Q4_OK) return rc;
  if (T == 0) return MOE_Q4_OK;
  if (!x_host || !logits_host || !out_host) return MOE_Q4_EINVAL;
  const Layout o = layout(layer, T, top_k);
  const HostStage hs = host_stage(layer, T, o.end);
  if (!ws || ((uintptr_t)ws & (kAlign - 1)) || ws_bytes < hs.end) return MOE_Q4_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* w = (char*)ws;
  const size_t xb = sizeof(__nv_bfloat16) * (size_t)T * layer->H;
  const size_t lb = sizeof(float) * (size_t)T * layer->E;
  if (cudaMemcpyAsync(w + hs.x, x_host, xb, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_Q4_ECUDA;
  if (cudaMemcpyAsync(w + hs.logits, logits_host, lb, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_Q4_ECUDA;
  rc = run_forward(layer, tp, w + hs.x, (const float*)(w + hs.logits), T, top_k, w + hs.out, nullptr,
                   nullptr, nullptr, nullptr, w, s);
  if (rc != MOE_Q4_OK) return rc;
  if (cudaMemcpyAsync(out_host, w + hs.out, xb, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_Q4_ECUDA;
  return MOE_Q4_OK;
}

extern "C" int moe_q4_forward_host(const moe_q4_layer* layer, const void* x_host,
                                   const float* logits_host, int T, int top_k, void* out_host,
                                   void* ws, size_t ws_bytes, void* stream) {
  const int rc = moe_q4_forward_host_async(layer, x_host, logits_host, T, top_k, out_host, ws, ws_bytes, stream);
  if (rc != MOE_Q4_OK || T == 0) return rc;
  return moe_q4_forward_status(ws, stream);
}

// Routing-only workspace: header | dec_list[E] | pre_list[E] | with T > 256:
// chunk_cnt[chunks][E] | chunk_base[chunks][E].
static size_t route_chunk_bytes(int E, int T) {
  return align_up(sizeof(int32_t) * (size_t)q4_route_chunks(T) * E);
}

extern "C" size_t moe_q4_route_workspace(int E, int T, int top_k) {
  if (E < 1 || E > kMaxExperts || T < 0 || top_k < 1 || top_k > E || top_k > kMaxTopK) return 0;
  if ((long long)T * top_k > (1LL << 24)) return 0;
  return align_up(sizeof(int32_t) * kHeaderWords) + 2 * align_up(sizeof(int32_t) * E) +
         2 * route_chunk_bytes(E, T);
}

extern "C" int moe_q4_route(const float* logits, int T, int E, int top_k, int32_t* ids, float* w,
                            int32_t* counts, int32_t* offsets, int32_t* row_token, int32_t* inv,
                            void* ws, size_t ws_bytes, void* stream) {
  const size_t need = moe_q4_route_workspace(E, T, top_k);
  if (need == 0) return MOE_Q4_EINVAL;
  if (!counts || !offsets) return MOE_Q4_EINVAL;
  if (T > 0 && (!logits || !ids || !w || !row_token || !inv || ((uintptr_t)logits & 3)))
    return MOE_Q4_EINVAL;
  if (!ws || ((uintptr_t)ws & (kAlign - 1)) || ws_bytes < need) return MOE_Q4_EWORKSPACE;
  char* p = (char*)ws;
  FwdArgs a;
  memset(&a, 0, sizeof a);
  a.T = T;
  a.k = top_k;
  a.E = E;
  a.dec_max = INT_MAX;
  a.logits = logits;
  a.hdr = (int32_t*)p;
  a.dec_list = (int32_t*)(p + align_up(sizeof(int32_t) * kHeaderWords));
  a.pre_list = (int32_t*)(p + align_up(sizeof(int32_t) * kHeaderWords) + align_up(sizeof(int32_t) * E));
  const size_t chunks_at = align_up(sizeof(int32_t) * kHeaderWords) + 2 * align_up(sizeof(int32_t) * E);
  a.chunk_cnt = (int32_t*)(p + chunks_at);
  a.chunk_base = (int32_t*)(p + chunks_at + route_chunk_bytes(E, T));
  a.ids = ids;
  a.w = w;
  a.counts = counts;
  a.offsets = offsets;
  a.row_token = row_token;
  a.inv = inv;
  return q4_launch_route(a, (cudaStream_t)stream);
}

// Validation + launch of one forward into a workspace the caller already
// holds; used by the entry point that supplies its own static scratch.
int q4_forward_in_workspace(const moe_q4_layer* layer, const void* x, const float* logits, int T, int top_k,
                            void* out, float* out_f32, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return moe_q4_forward(layer, x, logits, T, top_k, out, out_f32, nullptr, nullptr, nullptr, ws, ws_bytes,
                        (void*)stream);
}
