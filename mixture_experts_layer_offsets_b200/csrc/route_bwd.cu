// route_bwd.cu -- unpermute-grad (sum of each token's k expert-row gradients)
// plus the router gradient through the softmax.
//
//   dl[t,:]   = p * (dp - <p, dp>),  p = softmax(logits[t,:]),  dp = dgate scattered
//   dx[t,:]   = sum_e dl[t,e] w_router[e,:] + sum_j dx_perm[slot_row[t,j],:]
//   dw_router = dl^T x
//
// Deterministic: every sum has a fixed order.  dw_router is reduced in two
// steps (per-split partial sums, then a fixed-order sum over splits), with
// no floating-point atomics.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kTT = 32;   // tokens per tile
constexpr int kEC = 32;   // experts per tile
constexpr int kCols = 256;

inline int route_bwd_splits(int T) { return std::max(1, std::min(32, T / 512)); }

// dl, one warp per token (fp32, written to the workspace).
__global__ void __launch_bounds__(256)
dlogit_kernel(const float* __restrict__ logits, const int32_t* __restrict__ topk_idx,
              const float* __restrict__ dgate, float* __restrict__ dl, int ntok, int E, int k) {
  const int lane = threadIdx.x & 31;
  for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < ntok; t += gridDim.x * 8) {
    const float* l = logits + (int64_t)t * E;
    const int32_t* idx = topk_idx + (int64_t)t * k;
    const float* dg = dgate + (int64_t)t * k;
    float m = -INFINITY;
    for (int e = lane; e < E; e += 32) m = fmaxf(m, l[e]);
    m = warp_max(m);
    float s = 0.f;
    for (int e = lane; e < E; e += 32) s += expf(l[e] - m);
    s = warp_sum(s);
    // <p, dp> only involves the k selected experts; sum them in slot order.
    float pdp = 0.f;
    for (int j = 0; j < k; ++j) pdp = fmaf(expf(l[__ldg(idx + j)] - m) / s, __ldg(dg + j), pdp);
    for (int e = lane; e < E; e += 32) {
      float dp = 0.f;
      for (int j = 0; j < k; ++j)
        if (__ldg(idx + j) == e) dp = __ldg(dg + j);
      dl[(int64_t)t * E + e] = (expf(l[e] - m) / s) * (dp - pdp);
    }
  }
}

// dx = dl w_router + sum_j dx_perm[slot_row[t,j]]; tile of kTT tokens x kCols columns.
template <typename T>
__global__ void __launch_bounds__(kCols)
dx_kernel(const float* __restrict__ dl, const T* __restrict__ w, const T* __restrict__ dx_perm,
          const int32_t* __restrict__ slot_row, T* __restrict__ dx, int ntok, int d, int E, int k) {
  __shared__ float dls[kTT][kEC + 1];
  __shared__ float ws[kEC][kCols];
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kTT;
  const int c = blockIdx.y * kCols + tid;
  float acc[kTT];
#pragma unroll
  for (int i = 0; i < kTT; ++i) acc[i] = 0.f;
  for (int e0 = 0; e0 < E; e0 += kEC) {
    for (int i = tid; i < kTT * kEC; i += kCols) {
      const int r = i / kEC, e = i % kEC;
      dls[r][e] = (t0 + r < ntok && e0 + e < E) ? dl[(int64_t)(t0 + r) * E + e0 + e] : 0.f;
    }
    for (int e = 0; e < kEC; ++e)
      ws[e][tid] = (e0 + e < E && c < d) ? to_f32(w[(int64_t)(e0 + e) * d + c]) : 0.f;
    __syncthreads();
#pragma unroll 4
    for (int e = 0; e < kEC; ++e) {
      const float wv = ws[e][tid];
#pragma unroll
      for (int i = 0; i < kTT; ++i) acc[i] = fmaf(dls[i][e], wv, acc[i]);
    }
    __syncthreads();
  }
  if (c >= d) return;
#pragma unroll 1
  for (int i = 0; i < kTT; ++i) {
    const int t = t0 + i;
    if (t >= ntok) break;
    float v = acc[i];
    for (int j = 0; j < k; ++j) {
      const int r = slot_row[(int64_t)t * k + j];
      if (r >= 0) v += to_f32(dx_perm[(int64_t)r * d + c]);
    }
    dx[(int64_t)t * d + c] = from_f32<T>(v);
  }
}

// partial[s][e][c] = sum over tokens of split s of dl[t,e] * x[t,c]
template <typename T>
__global__ void __launch_bounds__(kCols)
dwr_partial_kernel(const float* __restrict__ dl, const T* __restrict__ x,
                   float* __restrict__ partial, int ntok, int d, int E, int tok_per_split) {
  __shared__ float dls[kTT][kEC + 1];
  const int tid = threadIdx.x;
  const int c = blockIdx.x * kCols + tid;
  const int e0 = blockIdx.y * kEC;
  const int s = blockIdx.z;
  const int ta = s * tok_per_split, tb = min(ntok, ta + tok_per_split);
  float acc[kEC];
#pragma unroll
  for (int i = 0; i < kEC; ++i) acc[i] = 0.f;
  for (int t0 = ta; t0 < tb; t0 += kTT) {
    for (int i = tid; i < kTT * kEC; i += kCols) {
      const int r = i / kEC, e = i % kEC;
      dls[r][e] = (t0 + r < tb && e0 + e < E) ? dl[(int64_t)(t0 + r) * E + e0 + e] : 0.f;
    }
    __syncthreads();
    if (c < d) {
      const int n = min(kTT, tb - t0);
      for (int r = 0; r < n; ++r) {
        const float xv = to_f32(x[(int64_t)(t0 + r) * d + c]);
#pragma unroll
        for (int e = 0; e < kEC; ++e) acc[e] = fmaf(dls[r][e], xv, acc[e]);
      }
    }
    __syncthreads();
  }
  if (c >= d) return;
  for (int e = 0; e < kEC && e0 + e < E; ++e)
    partial[((int64_t)s * E + e0 + e) * d + c] = acc[e];
}

__global__ void dwr_reduce_kernel(const float* __restrict__ partial, float* __restrict__ dw,
                                  int64_t n, int splits) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += partial[(int64_t)s * n + i];
    dw[i] = v;
  }
}

template <typename T>
cudaError_t route_bwd_t(const void* x, const void* w_router, const float* logits,
                        const int32_t* topk_idx, const float* dgate, const void* dx_perm,
                        const int32_t* slot_row, void* dx, float* dw_router, int T_, int d, int E,
                        int k, void* scratch, cudaStream_t st) {
  const int splits = route_bwd_splits(T_);
  float* dl = static_cast<float*>(scratch);
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) +
                                            align256((size_t)T_ * E * 4));
  const int64_t n = (int64_t)E * d;
  if (T_ > 0) {
    dlogit_kernel<<<std::min((T_ + 7) / 8, num_sms() * 8), 256, 0, st>>>(logits, topk_idx, dgate,
                                                                         dl, T_, E, k);
    dim3 g1((T_ + kTT - 1) / kTT, (d + kCols - 1) / kCols);
    dx_kernel<T><<<g1, kCols, 0, st>>>(dl, static_cast<const T*>(w_router),
                                       static_cast<const T*>(dx_perm), slot_row,
                                       static_cast<T*>(dx), T_, d, E, k);
    const int tps = (T_ + splits - 1) / splits;
    dim3 g2((d + kCols - 1) / kCols, (E + kEC - 1) / kEC, splits);
    dwr_partial_kernel<T><<<g2, kCols, 0, st>>>(dl, static_cast<const T*>(x), partial, T_, d, E,
                                                tps);
    dwr_reduce_kernel<<<(int)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, st>>>(
        partial, dw_router, n, splits);
  } else {
    cudaMemsetAsync(dw_router, 0, n * sizeof(float), st);
  }
  return cudaGetLastError();
}

}  // namespace

size_t route_bwd_ws_bytes(int T, int d, int E) {
  return align256((size_t)T * E * 4) + align256((size_t)route_bwd_splits(T) * E * d * 4);
}

cudaError_t route_bwd_launch(bool bf16, const void* x, const void* w_router, const float* logits,
                             const int32_t* topk_idx, const float* dgate, const void* dx_perm,
                             const int32_t* slot_row, void* dx, float* dw_router, int T, int d,
                             int E, int k, void* scratch, cudaStream_t st) {
  if (bf16)
    return route_bwd_t<__nv_bfloat16>(x, w_router, logits, topk_idx, dgate, dx_perm, slot_row, dx,
                                      dw_router, T, d, E, k, scratch, st);
  return route_bwd_t<float>(x, w_router, logits, topk_idx, dgate, dx_perm, slot_row, dx,
                            dw_router, T, d, E, k, scratch, st);
}

}  // namespace moe
