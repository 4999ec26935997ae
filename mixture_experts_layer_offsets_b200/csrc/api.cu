// api.cu -- the extern "C" entry points declared in include/moe.h: argument
// validation on the host, workspace carving, and dispatch to the kernels.
// Nothing here computes on the host and nothing synchronises a stream (except
// the documented diagnostic moe_get_device_status).
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

namespace {
struct ProfState {
  void* const* events = nullptr;  // 2 * cap cudaEvent_t of the caller
  const char** names = nullptr;   // cap entries
  int cap = 0;
  int n = 0;
  bool on = false;
};
thread_local ProfState g_prof;
}  // namespace

ProfScope::ProfScope(const char* name, cudaStream_t st) : st_(st), slot_(-1) {
  if (!g_prof.on) return;
  const int i = g_prof.n++;
  if (i >= g_prof.cap) return;
  slot_ = i;
  g_prof.names[i] = name;
  cudaEventRecord(static_cast<cudaEvent_t>(g_prof.events[2 * i]), st);
}

ProfScope::~ProfScope() {
  if (slot_ >= 0) cudaEventRecord(static_cast<cudaEvent_t>(g_prof.events[2 * slot_ + 1]), st_);
}

}  // namespace moe

using namespace moe;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31) == 0; }

// All pointers non-null and 16-byte aligned.
template <typename... P>
inline bool ptrs_ok(P... ps) {
  const void* arr[] = {static_cast<const void*>(ps)...};
  for (const void* p : arr)
    if (!p || !aligned16(p)) return false;
  return true;
}

inline bool dtype_act_ok(int dtype) { return dtype == MOE_F32 || dtype == MOE_BF16; }

moe_status shape_ok(const moe_shape& s) {
  if (s.T < 0 || s.d_model <= 0 || s.E <= 0 || s.top_k <= 0 || s.d_ff <= 0) return MOE_ERR_INVALID_ARG;
  if (s.E > 1024 || s.top_k > s.E || s.top_k > 32) return MOE_ERR_INVALID_ARG;
  if (s.d_model % 8 || s.d_ff % 8) return MOE_ERR_INVALID_ARG;
  if ((int64_t)s.T * s.top_k >= (int64_t)1 << 31) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

inline int* status_word(void* ws) { return static_cast<int*>(ws); }
inline void* scratch(void* ws) { return static_cast<uint8_t*>(ws) + kStatusBytes; }

size_t ws_need(const moe_shape& s, int dtype, int64_t rows) {
  if (rows <= 0) rows = (int64_t)s.T * s.top_k;
  FfnShape fs{s.d_model, s.E, s.d_ff, rows};
  size_t need = route_ws_bytes(s.T, s.E, s.top_k);
  need = std::max(need, route_bwd_ws_bytes(s.T, s.d_model, s.E));
  need = std::max(need, ffn_bwd_ws_bytes(fs, dtype != MOE_F32));
  if (dtype == MOE_MXFP8) need = std::max(need, ffn_mx_ws_bytes(fs));
  return kStatusBytes + align256(need);
}

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// host copy of a moe_mx_weights: every pointer present and 16-byte aligned
moe_status mx_weights_ok(const void* mx, MxWeights& w) {
  if (!mx) return MOE_ERR_INVALID_ARG;
  moe_mx_weights m;
  memcpy(&m, mx, sizeof(m));
  w = MxWeights{m.w1_q, m.w1_s, m.w1t_q, m.w1t_s, m.w2_q, m.w2_s, m.w2t_q, m.w2t_s};
  const void* all[] = {m.w1_q, m.w1_s, m.w1t_q, m.w1t_s, m.w2_q, m.w2_s, m.w2t_q, m.w2t_s};
  for (const void* q : all)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

size_t moe_workspace_size(moe_shape shape, int dtype, int64_t rows) {
  if (shape_ok(shape) != MOE_OK) return 0;
  return ws_need(shape, dtype, rows);
}

moe_status moe_mx_workspace_layout(moe_shape s, int64_t rows, int64_t* offsets_out, int n) {
  if (shape_ok(s) != MOE_OK || !offsets_out || n < kMxRegions) return MOE_ERR_INVALID_ARG;
  if (s.d_model % 128 || s.d_ff % 128) return MOE_ERR_UNSUPPORTED;
  if (rows <= 0) rows = (int64_t)s.T * s.top_k;
  size_t r[kMxRegions];
  ffn_mx_ws_regions(FfnShape{s.d_model, s.E, s.d_ff, rows}, r);
  for (int i = 0; i < kMxRegions; ++i) offsets_out[i] = (int64_t)(kStatusBytes + r[i]);
  return MOE_OK;
}

int32_t moe_capacity(moe_shape s, int32_t cf_num, int32_t cf_den) {
  if (shape_ok(s) != MOE_OK || cf_num <= 0 || cf_den <= 0) return -1;
  // ceil(cf_num * T * k / (cf_den * E)) in exact integer arithmetic
  const __int128 num = (__int128)cf_num * s.T * s.top_k;
  const __int128 den = (__int128)cf_den * s.E;
  const __int128 c = (num + den - 1) / den;
  return c > INT32_MAX ? -1 : (int32_t)c;
}

moe_status moe_profile_begin(void* const* events, const char** names, int capacity) {
  if (!events || !names || capacity <= 0 || g_prof.on) return MOE_ERR_INVALID_ARG;
  g_prof = ProfState{events, names, capacity, 0, true};
  return MOE_OK;
}

moe_status moe_profile_end(int32_t* count) {
  if (!count || !g_prof.on) return MOE_ERR_INVALID_ARG;
  *count = g_prof.n;
  g_prof = ProfState{};
  return MOE_OK;
}

moe_status moe_get_device_status(void* ws, void* stream, int32_t* status_out) {
  if (!ws || !status_out) return MOE_ERR_INVALID_ARG;
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, as_stream(stream));
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(v), as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  *status_out = v;
  return MOE_OK;
}

moe_status moe_route(moe_shape s, int dtype, const void* x, const void* w_router, const float* bias,
                     float* logits, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                     int32_t* offsets, int32_t* slot_row, void* ws, size_t ws_bytes,
                     void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (!dtype_act_ok(dtype)) return dtype == MOE_MXFP8 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (!ptrs_ok(w_router, counts, offsets, ws)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && !ptrs_ok(x, logits, topk_idx, topk_gate, slot_row)) return MOE_ERR_INVALID_ARG;
  if (bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < kStatusBytes + route_ws_bytes(s.T, s.E, s.top_k)) return MOE_ERR_INVALID_ARG;
  RouteArgs a{x, w_router, bias, s.T, s.d_model, s.E, s.top_k, logits, topk_idx, topk_gate,
              counts, offsets, slot_row, scratch(ws), status_word(ws)};
  return cuda_status(route_launch(a, dtype == MOE_BF16, as_stream(stream)));
}

moe_status moe_permute(moe_shape s, int dtype, const void* x, const int32_t* slot_row,
                       void* x_perm, int32_t* perm_src, void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (!dtype_act_ok(dtype)) return dtype == MOE_MXFP8 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  if (!ptrs_ok(x, slot_row, x_perm, perm_src)) return MOE_ERR_INVALID_ARG;
  return cuda_status(permute_launch(dtype == MOE_BF16, x, slot_row, x_perm, perm_src, s.T,
                                    s.d_model, s.top_k, as_stream(stream)));
}

moe_status moe_permute_mx(moe_shape s, const void* x, const int32_t* slot_row,
                          const int32_t* offsets, int32_t* perm_src, void* ws, size_t ws_bytes,
                          void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (s.d_model % 128 || s.d_ff % 128) return MOE_ERR_UNSUPPORTED;
  if (!ptrs_ok(offsets, ws)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && !ptrs_ok(x, slot_row, perm_src)) return MOE_ERR_INVALID_ARG;
  FfnShape fs{s.d_model, s.E, s.d_ff, (int64_t)s.T * s.top_k};
  if (ws_bytes < kStatusBytes + ffn_mx_ws_bytes(fs)) return MOE_ERR_INVALID_ARG;
  cudaStream_t cs = as_stream(stream);
  cudaError_t e = perm_src_launch(slot_row, perm_src, s.T, s.top_k, cs);
  if (e == cudaSuccess) e = mx_dispatch(fs, x, perm_src, offsets, scratch(ws), cs);
  return cuda_status(e);
}

moe_status moe_grouped_ffn_fwd(moe_shape s, int dtype, int64_t rows, const void* x_perm,
                               const int32_t* offsets, const void* w1, const void* w2,
                               const void* mx, void* act_saved, void* y_perm, void* ws,
                               size_t ws_bytes, void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (rows < 0 || rows >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
  FfnShape fs{s.d_model, s.E, s.d_ff, rows};
  cudaStream_t cs = as_stream(stream);
  if (dtype == MOE_MXFP8) {
    MxWeights w;
    moe_status vs = mx_weights_ok(mx, w);
    if (vs != MOE_OK) return vs;
    if (s.d_model % 128 || s.d_ff % 128) return MOE_ERR_UNSUPPORTED;
    // the epilogues write h's MXFP8 copies into ws with 32-byte stores
    if (!ptrs_ok(offsets, ws) || !aligned32(ws)) return MOE_ERR_INVALID_ARG;
    // x_perm NULL: moe_permute_mx has put the quantised copies of x in ws
    if (rows > 0 && (!ptrs_ok(act_saved, y_perm) || (x_perm && !aligned16(x_perm))))
      return MOE_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes + ffn_mx_ws_bytes(fs)) return MOE_ERR_INVALID_ARG;
    return cuda_status(ffn_fwd_mx(fs, x_perm, offsets, w, act_saved, y_perm, scratch(ws),
                                  status_word(ws), cs));
  }
  if (mx) return MOE_ERR_INVALID_ARG;
  if (!dtype_act_ok(dtype)) return MOE_ERR_INVALID_ARG;
  if (!ptrs_ok(offsets, w1, w2, ws)) return MOE_ERR_INVALID_ARG;
  if (rows > 0 && !ptrs_ok(x_perm, act_saved, y_perm)) return MOE_ERR_INVALID_ARG;
  (void)ws_bytes;
  if (dtype == MOE_F32)
    return cuda_status(ffn_fwd_f32(fs, static_cast<const float*>(x_perm), offsets,
                                   static_cast<const float*>(w1), static_cast<const float*>(w2),
                                   static_cast<float*>(act_saved), static_cast<float*>(y_perm), cs));
  if (s.d_model % 256 || s.d_ff % 256) return MOE_ERR_UNSUPPORTED;
  return cuda_status(
      ffn_fwd_bf16(fs, x_perm, offsets, w1, w2, act_saved, y_perm, status_word(ws), cs));
}

moe_status moe_combine(moe_shape s, int dtype, const void* y_perm, const int32_t* slot_row,
                       const float* topk_gate, void* out, void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (!dtype_act_ok(dtype)) return dtype == MOE_MXFP8 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  if (!ptrs_ok(y_perm, slot_row, topk_gate, out)) return MOE_ERR_INVALID_ARG;
  return cuda_status(combine_launch(dtype == MOE_BF16, y_perm, slot_row, topk_gate, out, s.T,
                                    s.d_model, s.top_k, as_stream(stream)));
}

moe_status moe_combine_bwd(moe_shape s, int dtype, const void* dout, const void* y_perm,
                           const int32_t* slot_row, const float* topk_gate, void* dy_perm,
                           float* dgate, void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (!dtype_act_ok(dtype)) return dtype == MOE_MXFP8 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  if (!ptrs_ok(dout, y_perm, slot_row, topk_gate, dy_perm, dgate)) return MOE_ERR_INVALID_ARG;
  return cuda_status(combine_bwd_launch(dtype == MOE_BF16, dout, y_perm, slot_row, topk_gate,
                                        dy_perm, dgate, s.T, s.d_model, s.top_k,
                                        as_stream(stream)));
}

moe_status moe_combine_bwd_mx(moe_shape s, const void* dout, const void* y_perm,
                              const int32_t* slot_row, const float* topk_gate,
                              const int32_t* perm_src, float* dgate, void* ws, size_t ws_bytes,
                              void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (s.d_model % 128 || s.d_ff % 128) return MOE_ERR_UNSUPPORTED;
  if (!ptrs_ok(ws)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && !ptrs_ok(dout, y_perm, slot_row, topk_gate, perm_src, dgate))
    return MOE_ERR_INVALID_ARG;
  FfnShape fs{s.d_model, s.E, s.d_ff, (int64_t)s.T * s.top_k};
  if (ws_bytes < kStatusBytes + ffn_mx_ws_bytes(fs)) return MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  return cuda_status(mx_combine_bwd(fs, dout, y_perm, slot_row, topk_gate, perm_src, dgate, s.T,
                                    s.top_k, scratch(ws), as_stream(stream)));
}

}  // extern "C"

namespace {

// The grouped FFN backward; with `recompute` the call first refills act (a | u | h,
// and for MXFP8 the token-block copies of x and h in ws) from x_perm.
moe_status ffn_bwd_entry(moe_shape s, int dtype, int64_t rows, const void* dy_perm,
                         const void* x_perm, void* act, const int32_t* offsets, const void* w1,
                         const void* w2, const void* mx, void* dx_perm, void* dw1, void* dw2,
                         int dw_dtype, void* ws, size_t ws_bytes, void* stream, bool recompute) {
  const void* act_saved = act;
  const bool accumulate = (dw_dtype & MOE_DW_ACCUMULATE) != 0;
  dw_dtype &= ~MOE_DW_ACCUMULATE;
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (rows < 0 || rows >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
  if (dtype == MOE_MXFP8) {
    MxWeights w;
    moe_status vs = mx_weights_ok(mx, w);
    if (vs != MOE_OK) return vs;
    if (s.d_model % 128 || s.d_ff % 128) return MOE_ERR_UNSUPPORTED;
    if (dw_dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
    // the epilogues write [da | du]'s MXFP8 copies into ws with 32-byte stores
    if (!ptrs_ok(offsets, dw1, dw2, ws) || !aligned32(ws)) return MOE_ERR_INVALID_ARG;
    // x_perm is read only by the recompute (the backward uses the token-block copy);
    // dy_perm NULL: moe_combine_bwd_mx has put dy's copies in ws (not with the recompute,
    // whose forward half reuses that memory)
    if (rows > 0 && (!ptrs_ok(act_saved, dx_perm) || !aligned32(act_saved) ||
                     (recompute && !x_perm) ||
                     (x_perm && !aligned16(x_perm)) || (recompute && !dy_perm) ||
                     (dy_perm && !aligned16(dy_perm))))
      return MOE_ERR_INVALID_ARG;
    FfnShape fsm{s.d_model, s.E, s.d_ff, rows};
    if (ws_bytes < kStatusBytes + ffn_mx_ws_bytes(fsm)) return MOE_ERR_INVALID_ARG;
    if (recompute) {
      cudaError_t e = ffn_fwd_mx(fsm, x_perm, offsets, w, act, nullptr, scratch(ws),
                                 status_word(ws), as_stream(stream));
      if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    return cuda_status(ffn_bwd_mx(fsm, dy_perm, x_perm, act_saved, offsets, w, dx_perm,
                                  static_cast<float*>(dw1), static_cast<float*>(dw2), scratch(ws),
                                  status_word(ws), as_stream(stream), accumulate));
  }
  if (mx) return MOE_ERR_INVALID_ARG;
  if (!dtype_act_ok(dtype)) return MOE_ERR_INVALID_ARG;
  if (dw_dtype != MOE_F32 && dw_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (dtype == MOE_F32 && dw_dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (!ptrs_ok(offsets, w1, w2, dw1, dw2, ws)) return MOE_ERR_INVALID_ARG;
  if (rows > 0 && !ptrs_ok(dy_perm, x_perm, act_saved, dx_perm)) return MOE_ERR_INVALID_ARG;
  // the bf16 SwiGLU backward reads a and u in 32-byte pieces
  if (rows > 0 && dtype == MOE_BF16 && !aligned32(act_saved)) return MOE_ERR_INVALID_ARG;
  FfnShape fs{s.d_model, s.E, s.d_ff, rows};
  if (ws_bytes < kStatusBytes + ffn_bwd_ws_bytes(fs, dtype == MOE_BF16)) return MOE_ERR_INVALID_ARG;
  cudaStream_t cs = as_stream(stream);
  if (dtype == MOE_BF16 && (s.d_model % 256 || s.d_ff % 256)) return MOE_ERR_UNSUPPORTED;
  if (recompute) {
    cudaError_t e = dtype == MOE_F32
                        ? ffn_fwd_f32(fs, static_cast<const float*>(x_perm), offsets,
                                      static_cast<const float*>(w1), static_cast<const float*>(w2),
                                      static_cast<float*>(act), nullptr, cs)
                        : ffn_fwd_bf16(fs, x_perm, offsets, w1, w2, act, nullptr, status_word(ws), cs);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (dtype == MOE_F32)
    return cuda_status(ffn_bwd_f32(fs, static_cast<const float*>(dy_perm),
                                   static_cast<const float*>(x_perm),
                                   static_cast<const float*>(act_saved), offsets,
                                   static_cast<const float*>(w1), static_cast<const float*>(w2),
                                   static_cast<float*>(dx_perm), static_cast<float*>(dw1),
                                   static_cast<float*>(dw2), scratch(ws), cs, accumulate));
  return cuda_status(ffn_bwd_bf16(fs, dy_perm, x_perm, act_saved, offsets, w1, w2, dx_perm, dw1,
                                  dw2, dw_dtype == MOE_F32, scratch(ws), status_word(ws), cs,
                                  accumulate));
}

}  // namespace

extern "C" {

moe_status moe_grouped_ffn_bwd(moe_shape s, int dtype, int64_t rows, const void* dy_perm,
                               const void* x_perm, const void* act_saved,
                               const int32_t* offsets, const void* w1, const void* w2,
                               const void* mx, void* dx_perm, void* dw1, void* dw2,
                               int dw_dtype, void* ws, size_t ws_bytes, void* stream) {
  return ffn_bwd_entry(s, dtype, rows, dy_perm, x_perm, const_cast<void*>(act_saved), offsets, w1,
                       w2, mx, dx_perm, dw1, dw2, dw_dtype, ws, ws_bytes, stream, false);
}

moe_status moe_grouped_ffn_bwd_recompute(moe_shape s, int dtype, int64_t rows,
                                         const void* dy_perm, const void* x_perm,
                                         void* act_scratch, const int32_t* offsets,
                                         const void* w1, const void* w2, const void* mx,
                                         void* dx_perm, void* dw1, void* dw2, int dw_dtype,
                                         void* ws, size_t ws_bytes, void* stream) {
  return ffn_bwd_entry(s, dtype, rows, dy_perm, x_perm, act_scratch, offsets, w1, w2, mx, dx_perm,
                       dw1, dw2, dw_dtype, ws, ws_bytes, stream, true);
}

moe_status moe_route_bwd(moe_shape s, int dtype, const void* x, const void* w_router,
                         const float* logits, const int32_t* topk_idx, const float* dgate,
                         const void* dx_perm, const int32_t* slot_row, void* dx,
                         float* dw_router, void* ws, size_t ws_bytes, void* stream) {
  const bool accumulate = (dtype & MOE_DW_ACCUMULATE) != 0;
  dtype &= ~MOE_DW_ACCUMULATE;
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (!dtype_act_ok(dtype)) return dtype == MOE_MXFP8 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (!ptrs_ok(w_router, dw_router, ws)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && !ptrs_ok(x, logits, topk_idx, dgate, dx_perm, dx)) return MOE_ERR_INVALID_ARG;
  if (slot_row && !aligned16(slot_row)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < kStatusBytes + route_bwd_ws_bytes(s.T, s.d_model, s.E)) return MOE_ERR_INVALID_ARG;
  return cuda_status(route_bwd_launch(dtype == MOE_BF16, x, w_router, logits, topk_idx, dgate,
                                      dx_perm, slot_row, dx, dw_router, s.T, s.d_model, s.E,
                                      s.top_k, scratch(ws), status_word(ws), as_stream(stream),
                                      accumulate));
}

// ---- f2: expert parallelism across ranks
namespace {
// host array of n device pointers, all present and 16-byte aligned
bool peers_ok(const void* const* peers, int n, EpPeers& out) {
  if (!peers || n < 1 || n > kMaxRanks) return false;
  memset(&out, 0, sizeof(out));
  for (int i = 0; i < n; ++i) {
    if (!peers[i] || !aligned16(peers[i])) return false;
    out.p[i] = const_cast<void*>(peers[i]);
  }
  return true;
}
moe_status ep_args_ok(const moe_shape& s, int n_ranks) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (n_ranks < 1 || n_ranks > kMaxRanks || s.E % n_ranks) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}
}  // namespace

moe_status moe_ep_layout(moe_shape s, int n_ranks, int rank, const int32_t* counts_all,
                         int32_t* recv_offsets, int32_t* send_base, void* stream) {
  moe_status st = ep_args_ok(s, n_ranks);
  if (st != MOE_OK) return st;
  if (rank < 0 || rank >= n_ranks) return MOE_ERR_INVALID_ARG;
  if (!ptrs_ok(counts_all, recv_offsets, send_base)) return MOE_ERR_INVALID_ARG;
  return cuda_status(ep_layout_launch(counts_all, n_ranks, s.E, rank, recv_offsets, send_base,
                                      as_stream(stream)));
}

moe_status moe_ep_dispatch(moe_shape s, int dtype, int n_ranks, const void* x,
                           const int32_t* topk_idx, const int32_t* slot_row,
                           const int32_t* offsets, const int32_t* send_base,
                           void* const* peer_x, int32_t* ep_row, void* stream) {
  moe_status st = ep_args_ok(s, n_ranks);
  if (st != MOE_OK) return st;
  if (!dtype_act_ok(dtype)) return dtype == MOE_MXFP8 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  EpPeers peers;
  if (!peers_ok(peer_x, n_ranks, peers)) return MOE_ERR_INVALID_ARG;
  if (!ptrs_ok(x, topk_idx, slot_row, offsets, send_base, ep_row)) return MOE_ERR_INVALID_ARG;
  return cuda_status(ep_dispatch_launch(dtype == MOE_BF16, x, topk_idx, slot_row, offsets,
                                        send_base, peers, ep_row, s.T, s.d_model, s.top_k,
                                        s.E / n_ranks, n_ranks, as_stream(stream)));
}

moe_status moe_ep_combine(moe_shape s, int dtype, int n_ranks, const void* const* peer_y,
                          const int32_t* topk_idx, const int32_t* ep_row, const float* gate,
                          void* out, void* stream) {
  moe_status st = ep_args_ok(s, n_ranks);
  if (st != MOE_OK) return st;
  if (!dtype_act_ok(dtype)) return dtype == MOE_MXFP8 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  EpPeers peers;
  if (!peers_ok(peer_y, n_ranks, peers)) return MOE_ERR_INVALID_ARG;
  if (!ptrs_ok(topk_idx, ep_row, out)) return MOE_ERR_INVALID_ARG;
  if (gate && !aligned16(gate)) return MOE_ERR_INVALID_ARG;
  return cuda_status(ep_combine_launch(dtype == MOE_BF16, peers, topk_idx, ep_row, gate, out,
                                       s.T, s.d_model, s.top_k, s.E / n_ranks,
                                       as_stream(stream)));
}

moe_status moe_ep_combine_bwd(moe_shape s, int dtype, int n_ranks, const void* dout,
                              const void* const* peer_y, const int32_t* topk_idx,
                              const int32_t* ep_row, const float* gate, void* const* peer_dy,
                              float* dgate, void* stream) {
  moe_status st = ep_args_ok(s, n_ranks);
  if (st != MOE_OK) return st;
  if (!dtype_act_ok(dtype)) return dtype == MOE_MXFP8 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  EpPeers py, pdy;
  if (!peers_ok(peer_y, n_ranks, py) || !peers_ok(peer_dy, n_ranks, pdy)) return MOE_ERR_INVALID_ARG;
  if (!ptrs_ok(dout, topk_idx, ep_row, gate, dgate)) return MOE_ERR_INVALID_ARG;
  return cuda_status(ep_combine_bwd_launch(dtype == MOE_BF16, dout, py, pdy, topk_idx, ep_row,
                                           gate, dgate, s.T, s.d_model, s.top_k, s.E / n_ranks,
                                           as_stream(stream)));
}

moe_status moe_mx_quantize_weights(moe_shape s, const float* w1, const float* w2,
                                   const moe_mx_weights* out, void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  MxWeights w;
  moe_status vs = mx_weights_ok(out, w);
  if (vs != MOE_OK) return vs;
  if (s.d_model % 128 || s.d_ff % 128) return MOE_ERR_UNSUPPORTED;
  if (!ptrs_ok(w1, w2)) return MOE_ERR_INVALID_ARG;
  return cuda_status(mx_quantize_weights(s.E, s.d_model, s.d_ff, w1, w2, w, as_stream(stream)));
}

moe_status mxfp8_quantize(int64_t rows, int64_t K, int src_dtype, const void* src, int axis,
                          const int32_t* seg_offsets, int nseg, uint8_t* q, uint8_t* scale,
                          void* stream) {
  if (rows < 0 || K < 0 || (src_dtype != MOE_F32 && src_dtype != MOE_BF16)) return MOE_ERR_INVALID_ARG;
  if (axis == 0) {
    if (K % 32) return MOE_ERR_INVALID_ARG;
  } else if (axis == 1) {
    if (K % 16) return MOE_ERR_INVALID_ARG;
    if (seg_offsets && (nseg < 1 || nseg > 1024 || !aligned16(seg_offsets))) return MOE_ERR_INVALID_ARG;
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  if (rows == 0 || K == 0) return MOE_OK;
  if (!ptrs_ok(src, q, scale)) return MOE_ERR_INVALID_ARG;
  return cuda_status(mxfp8_launch(rows, K, src_dtype == MOE_BF16, src, axis, seg_offsets, nseg, q,
                                  scale, as_stream(stream)));
}

moe_status moe_padded_dispatch(moe_shape s, int dtype, int32_t capacity, const void* x,
                               const int32_t* topk_idx, const int32_t* slot_row,
                               const int32_t* offsets, void* x_pad, int32_t* pad_row,
                               int32_t* offsets_pad, void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (!dtype_act_ok(dtype)) return dtype == MOE_MXFP8 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (capacity <= 0 || (int64_t)capacity * s.E >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
  if (!ptrs_ok(offsets, x_pad, offsets_pad)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && !ptrs_ok(x, topk_idx, slot_row, pad_row)) return MOE_ERR_INVALID_ARG;
  return cuda_status(padded_dispatch_launch(dtype == MOE_BF16, capacity, x, topk_idx, slot_row,
                                            offsets, x_pad, pad_row, offsets_pad, s.T, s.d_model,
                                            s.E, s.top_k, as_stream(stream)));
}

moe_status moe_routing_stats(moe_shape s, const int32_t* counts, int32_t capacity, float* stats,
                             void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (capacity < 0 || !ptrs_ok(counts, stats)) return MOE_ERR_INVALID_ARG;
  return cuda_status(routing_stats_launch(counts, s.E, capacity, stats, as_stream(stream)));
}

moe_status moe_renorm_gates(moe_shape s, const float* topk_gate, float* gate_out, void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (s.T > 0 && !ptrs_ok(topk_gate, gate_out)) return MOE_ERR_INVALID_ARG;
  return cuda_status(renorm_gates_launch(topk_gate, gate_out, s.T, s.top_k, as_stream(stream)));
}

moe_status moe_renorm_gates_bwd(moe_shape s, const float* topk_gate, const float* dgate_out,
                                float* dgate, void* stream) {
  moe_status st = shape_ok(s);
  if (st != MOE_OK) return st;
  if (s.T > 0 && !ptrs_ok(topk_gate, dgate_out, dgate)) return MOE_ERR_INVALID_ARG;
  return cuda_status(renorm_gates_bwd_launch(topk_gate, dgate_out, dgate, s.T, s.top_k,
                                             as_stream(stream)));
}

}  // extern "C"
