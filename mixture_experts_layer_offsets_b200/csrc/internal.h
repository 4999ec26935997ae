// internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>

namespace moe {

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// ---------------------------------------------------------------- routing
struct RouteArgs {
  const void* x;
  const void* w_router;
  const float* bias;
  int T, d, E, k;
  float* logits;
  int32_t* topk_idx;
  float* topk_gate;
  int32_t* counts;
  int32_t* offsets;
  int32_t* slot_row;
  void* scratch;            // route_ws_bytes(T, E, k) bytes
  int* status = nullptr;    // workspace status word (bounded waits), may be null
  // filled in by route_launch
  int32_t* blockcounts = nullptr;
  int32_t* localrank = nullptr;
};
size_t route_ws_bytes(int T, int E, int k);
cudaError_t route_launch(const RouteArgs& a, bool bf16, cudaStream_t st);
// tensor-core router (bf16): logits GEMM with softmax/top-k/counts/ranks fused in
// the epilogue, one 128-token block per tile
bool route_tc_supported(int E, int k, int d);
cudaError_t route_tc_launch(const RouteArgs& a, int nb, cudaStream_t st);

// ---------------------------------------------------------- row movement
//   renorm_gates_launch / renorm_gates_bwd_launch: moe_renorm_gates and its backward (k <= 32)
cudaError_t renorm_gates_launch(const float* gate, float* out, int T, int k, cudaStream_t st);
cudaError_t renorm_gates_bwd_launch(const float* gate, const float* dgr, float* dgate, int T, int k,
                                    cudaStream_t st);
//   routing_stats_launch: the eight load statistics of moe_routing_stats (E <= 1024)
cudaError_t routing_stats_launch(const int32_t* counts, int E, int capacity, float* stats,
                                 cudaStream_t st);
cudaError_t permute_launch(bool bf16, const void* x, const int32_t* slot_row, void* x_perm,
                           int32_t* perm_src, int T, int d, int k, cudaStream_t st);
cudaError_t combine_launch(bool bf16, const void* y_perm, const int32_t* slot_row,
                           const float* gate, void* out, int T, int d, int k, cudaStream_t st,
                           const char* prof_name = "combine");
cudaError_t combine_bwd_launch(bool bf16, const void* dout, const void* y_perm,
                               const int32_t* slot_row, const float* gate, void* dy_perm,
                               float* dgate, int T, int d, int k, cudaStream_t st);
cudaError_t padded_dispatch_launch(bool bf16, int capacity, const void* x, const int32_t* topk_idx,
                                   const int32_t* slot_row, const int32_t* offsets, void* x_pad,
                                   int32_t* pad_row, int32_t* offsets_pad, int T, int d, int E,
                                   int k, cudaStream_t st);

// ------------------------------------------------------------ router bwd
size_t route_bwd_ws_bytes(int T, int d, int E);
// tensor-core router backward (bf16, E a multiple of 128): dx and per-split dW_r partials
bool route_bwd_tc_supported(int E, int k, int d);
cudaError_t route_bwd_tc_launch(const void* x, const void* w_router, const void* dl_bf16,
                                const void* dx_perm, const int32_t* slot_row, void* dx,
                                float* partial, int splits, int T, int d, int E, int k,
                                int* status, cudaStream_t st);
cudaError_t route_bwd_launch(bool bf16, const void* x, const void* w_router, const float* logits,
                             const int32_t* topk_idx, const float* dgate, const void* dx_perm,
                             const int32_t* slot_row, void* dx, float* dw_router, int T, int d,
                             int E, int k, void* scratch, int* status, cudaStream_t st,
                             bool accumulate = false);

// ----------------------------------------------------------------- MXFP8
cudaError_t mxfp8_launch(int64_t rows, int64_t K, bool src_bf16, const void* src, int axis,
                         const int32_t* seg_offsets, int nseg, uint8_t* q, uint8_t* scale,
                         cudaStream_t st);
// the same with a source row stride of `ld` elements (q and scale stay dense)
cudaError_t mxfp8_launch_ld(int64_t rows, int64_t K, int64_t ld, bool src_bf16, const void* src,
                            int axis, const int32_t* seg_offsets, int nseg, uint8_t* q,
                            uint8_t* scale, cudaStream_t st);

// Scale atoms of the block-scaled MMA (512 bytes: 128 rows x 4 blocks of 32 along K,
// byte (r % 32) * 16 + (r / 32) * 4 + kb), laid out in the order the grouped GEMM reads:
//   row_tile_launch: row -> tile * 128 + row in tile of the row-grouped GEMMs (-1 outside)
//   mxfp8_weights: FP32 [E][Rw][Kw] -> row-block and column-block copies (see mxfp8.cu)
cudaError_t row_tile_launch(const int32_t* offsets, int E, int64_t rows, int32_t* out, cudaStream_t st);
cudaError_t mxfp8_weights(const float* w, int E, int Rw, int Kw, uint8_t* q0, uint8_t* s0,
                          uint8_t* q1, uint8_t* s1, cudaStream_t st);
//   seg_blocks_launch: the 32-row token blocks of all segments (at most rows/32 + E) and
//     the first block of every 128-row stage (smap, at most rows/128 + E + 1 entries)
//   mxfp8_act: one pass over a bf16 activation writing its row copy (row-tile atoms) and its
//     token-block copy (stage atoms); with `gather`, operand row r is source row gather[r];
//     with `row_mul`, row r is first scaled by row_mul[r] and rounded to bf16
cudaError_t seg_blocks_launch(const int32_t* offsets, int E, int4* map, int32_t* count,
                              int32_t* smap, cudaStream_t st);
cudaError_t mxfp8_act(int64_t rows, int E, int64_t K, int64_t ld, const void* src_bf16,
                      const int4* map, const int32_t* count, const int32_t* smap,
                      const int32_t* row_tile, uint8_t* q_r, uint8_t* atoms_r, uint8_t* q_c,
                      uint8_t* atoms_c, cudaStream_t st, const int32_t* gather = nullptr,
                      const float* row_mul = nullptr);
//   perm_src_launch: perm_src[slot_row[t, j]] = t (the permute's source map, no row copy)
//   perm_gate_launch: gate_perm[slot_row[t, j]] = gate[t, j]
cudaError_t perm_gate_launch(const int32_t* slot_row, const float* gate, float* gate_perm, int T,
                             int k, cudaStream_t st);
cudaError_t perm_src_launch(const int32_t* slot_row, int32_t* perm_src, int T, int k,
                            cudaStream_t st);

// ------------------------------------------------------ expert parallelism
// Peer buffers of the ranks (device pointers valid on this device: peer mappings over
// NVLink, or this device's own memory), passed to the kernels by value.
constexpr int kMaxRanks = 64;
struct EpPeers {
  void* p[kMaxRanks];
};
cudaError_t ep_layout_launch(const int32_t* counts_all, int N, int E, int rank,
                             int32_t* recv_offsets, int32_t* send_base, cudaStream_t st);
cudaError_t ep_dispatch_launch(bool bf16, const void* x, const int32_t* topk_idx,
                               const int32_t* slot_row, const int32_t* offsets,
                               const int32_t* send_base, const EpPeers& peers, int32_t* ep_row,
                               int T, int d, int k, int El, int nranks, cudaStream_t st);
cudaError_t ep_combine_launch(bool bf16, const EpPeers& peers, const int32_t* topk_idx,
                              const int32_t* ep_row, const float* gate, void* out, int T, int d,
                              int k, int El, cudaStream_t st);
cudaError_t ep_combine_bwd_launch(bool bf16, const void* dout, const EpPeers& peers_y,
                                  const EpPeers& peers_dy, const int32_t* topk_idx,
                                  const int32_t* ep_row, const float* gate, float* dgate, int T,
                                  int d, int k, int El, cudaStream_t st);

// ---------------------------------------------------------- grouped FFN
struct FfnShape {
  int d, E, f;
  int64_t rows;
};
//   mx_dispatch: the fused MXFP8 dispatch: row maps and both quantised copies of x, gathered
//     through perm_src, into the workspace regions that ffn_fwd_mx reads
cudaError_t mx_dispatch(const FfnShape& s, const void* x, const int32_t* perm_src,
                        const int32_t* offsets, void* scratch, cudaStream_t st);
//   mx_combine_bwd: dgate as the combine backward computes it, and the two MXFP8 copies of
//     dy_perm (gate x dout rows, rounded to bf16) into the workspace regions that ffn_bwd_mx
//     reads when given no dy_perm; the block maps come from the forward
cudaError_t mx_combine_bwd(const FfnShape& s, const void* dout, const void* y_perm,
                           const int32_t* slot_row, const float* gate, const int32_t* perm_src,
                           float* dgate, int T, int k, void* scratch, cudaStream_t st);
size_t ffn_bwd_ws_bytes(const FfnShape& s, bool bf16);
// fp32 partial sums of weight-gradient groups cut into K ranges (tensor-core paths)
size_t wgrad_part_bytes(const FfnShape& s, bool fp8);
// fp32 path: CUDA-core grouped GEMMs
//   ffn_fwd_*: y_perm == nullptr runs the gate/up half only (the recompute of a | u | h)
cudaError_t ffn_fwd_f32(const FfnShape& s, const float* x_perm, const int32_t* offsets,
                        const float* w1, const float* w2, float* act, float* y_perm,
                        cudaStream_t st);
cudaError_t ffn_bwd_f32(const FfnShape& s, const float* dy_perm, const float* x_perm,
                        const float* act, const int32_t* offsets, const float* w1,
                        const float* w2, float* dx_perm, float* dw1, float* dw2, void* scratch,
                        cudaStream_t st, bool accumulate = false);
// bf16 path: tcgen05 tensor-core grouped GEMMs
cudaError_t ffn_fwd_bf16(const FfnShape& s, const void* x_perm, const int32_t* offsets,
                         const void* w1, const void* w2, void* act, void* y_perm, int* status,
                         cudaStream_t st);
cudaError_t ffn_bwd_bf16(const FfnShape& s, const void* dy_perm, const void* x_perm,
                         const void* act, const int32_t* offsets, const void* w1, const void* w2,
                         void* dx_perm, void* dw1, void* dw2, bool dw_f32, void* scratch,
                         int* status, cudaStream_t st, bool accumulate = false);

// MXFP8 path: E4M3 operands with E8M0 scales (see include/moe.h, moe_mx_weights)
struct MxWeights {
  const uint8_t *w1_q, *w1_s, *w1t_q, *w1t_s, *w2_q, *w2_s, *w2t_q, *w2t_s;
};
size_t ffn_mx_ws_bytes(const FfnShape& s);
// byte offsets (within the scratch part of the workspace) of the MXFP8 operand copies,
// in the order documented with moe_mx_workspace_layout
constexpr int kMxRegions = 20;
void ffn_mx_ws_regions(const FfnShape& s, size_t out[kMxRegions]);
cudaError_t mx_quantize_weights(int E, int d, int f, const float* w1, const float* w2,
                                const MxWeights& w, cudaStream_t st);
cudaError_t ffn_fwd_mx(const FfnShape& s, const void* x_perm, const int32_t* offsets,
                       const MxWeights& w, void* act, void* y_perm, void* scratch, int* status,
                       cudaStream_t st);
cudaError_t ffn_bwd_mx(const FfnShape& s, const void* dy_perm, const void* x_perm, const void* act,
                       const int32_t* offsets, const MxWeights& w, void* dx_perm, float* dw1,
                       float* dw2, void* scratch, int* status, cudaStream_t st,
                       bool accumulate = false);
// (accumulate: the weight gradients are added into dw1, dw2 instead of overwriting them)

int num_sms();

// Per-launch device timing for diagnostics (moe_profile_begin / moe_profile_end):
// a ProfScope built right before a kernel launch records the caller's start event
// on the launch stream, and its destructor, right after the launch, the end event.
// Inactive (no CUDA call at all) unless a profile is open on this host thread.
class ProfScope {
 public:
  ProfScope(const char* name, cudaStream_t st);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  cudaStream_t st_;
  int slot_;
};

}  // namespace moe
