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


// token splits of the CUDA-core dW_r partial sums (about 1024 tokens each)
inline int route_bwd_splits(int T) { return std::max(1, std::min(64, T / 1024)); }

// dl, one warp per token, written to the workspace in fp32 (CUDA-core path) or
// bf16 (tensor-core path, where dl is a GEMM operand).
__global__ void __launch_bounds__(256)
dlogit_kernel(const float* __restrict__ logits, const int32_t* __restrict__ topk_idx,
              const float* __restrict__ dgate, float* __restrict__ dl,
              __nv_bfloat16* __restrict__ dl_bf, int ntok, int E, int k) {
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
      const float v = (expf(l[e] - m) / s) * (dp - pdp);
      if (dl) dl[(int64_t)t * E + e] = v;
      if (dl_bf) dl_bf[(int64_t)t * E + e] = __float2bfloat16_rn(v);
    }
  }
}

// dx = dl w_router + sum_j dx_perm[slot_row[t,j]].  A warp takes 4 tokens and
// walks their rows in 16-byte chunks (one chunk per lane): the router term
// reuses each w_router chunk for the 4 tokens, dl comes from shared memory.
// The rows' indices sit in lanes (lane tt*k + j holds token tt's slot j) and
// all KMAX row chunks of a token are loaded before any is added.
template <typename T, int TPW, int KMAX>
__global__ void __launch_bounds__(256)
dx_kernel(const float* __restrict__ dl, const T* __restrict__ w, const T* __restrict__ dx_perm,
          const int32_t* __restrict__ slot_row, T* __restrict__ dx, int ntok, int d, int E, int k) {
  constexpr int V = Vec16<T>::N;
  // TPW * k <= 32: the row indices of a warp's tokens fit its lanes
  extern __shared__ float s_dl[];  // [8 warps][TPW][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = (blockIdx.x * 8 + warp) * TPW;
  float* my = s_dl + warp * TPW * E;
  for (int i = lane; i < TPW * E; i += 32) {
    const int t = t0 + i / E;
    my[i] = t < ntok ? dl[(int64_t)t * E + i % E] : 0.f;
  }
  int myrow = -1;
  if (lane < TPW * k) {
    const int t = t0 + lane / k;
    // without slot_row, dx_perm holds one row per token: the sum of its expert rows
    if (t < ntok) myrow = slot_row ? slot_row[(int64_t)t * k + lane % k] : (lane % k ? -1 : t);
  }
  __syncwarp();
  const int chunks = d / V;
  for (int c = lane; c < chunks; c += 32) {
    float acc[TPW][V];
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
      for (int i = 0; i < V; ++i) acc[tt][i] = 0.f;
    for (int e = 0; e < E; ++e) {
      Vec16<T> wv;
      wv.raw = ldg16(w + (int64_t)e * d + (int64_t)c * V);
#pragma unroll
      for (int tt = 0; tt < TPW; ++tt) {
        const float g = my[tt * E + e];
#pragma unroll
        for (int i = 0; i < V; ++i) acc[tt][i] = fmaf(g, wv.get(i), acc[tt][i]);
      }
    }
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
      for (int jb = 0; jb < k; jb += KMAX) {
        Vec16<T> v[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          const int r = __shfl_sync(0xffffffffu, myrow, (tt * k + jb + j) & 31);
          v[j].raw = (jb + j < k && r >= 0) ? ldg16(dx_perm + (int64_t)r * d + (int64_t)c * V)
                                            : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
#pragma unroll
          for (int i = 0; i < V; ++i) acc[tt][i] += v[j].get(i);
      }
      const int t = t0 + tt;
      if (t < ntok) {
        Vec16<T> o;
#pragma unroll
        for (int i = 0; i < V; ++i) o.set(i, acc[tt][i]);
        stg16(dx + (int64_t)t * d + (int64_t)c * V, o.raw);
      }
    }
  }
}

// partial[s][e][cols] = sum over the tokens of split s of dl[t,e] * x[t, cols] for a
// block of 8 column chunks (8 x V columns) and EB experts.  Thread (token lane tl,
// chunk cc) walks the split's tokens tl, tl + 32, ... with several 16-byte loads in
// flight; the 32 token lanes are then summed in a fixed order (warp shuffles, then
// shared memory), so the result does not depend on timing.
template <typename T, int EB>
__global__ void __launch_bounds__(256)
dwr_partial_kernel(const float* __restrict__ dl, const T* __restrict__ x,
                   float* __restrict__ partial, int ntok, int d, int E, int tok_per_split) {
  constexpr int V = Vec16<T>::N;
  constexpr int U = 4;                       // tokens in flight per thread
  __shared__ float s_red[8][8][EB * V];      // [warp][chunk][expert x element]
  const int cc = threadIdx.x & 7, tl = threadIdx.x >> 3;   // tl: 0 .. 31
  const int warp = threadIdx.x >> 5;
  const int c = blockIdx.x * 8 + cc;         // 16-byte column chunk
  const int e0 = blockIdx.z * EB;
  const int ta = blockIdx.y * tok_per_split, tb = min(ntok, ta + tok_per_split);
  const bool live = c < d / V;
  float acc[EB][V];
#pragma unroll
  for (int e = 0; e < EB; ++e)
#pragma unroll
    for (int i = 0; i < V; ++i) acc[e][i] = 0.f;
  if (live) {
    for (int t0 = ta + tl; t0 < tb; t0 += 32 * U) {
      Vec16<T> xv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + 32 * u;
        xv[u].raw = t < tb ? ldg16(x + (int64_t)t * d + (int64_t)c * V) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + 32 * u;
        if (t >= tb) break;
#pragma unroll
        for (int e = 0; e < EB; ++e) {
          const float g = e0 + e < E ? __ldg(dl + (int64_t)t * E + e0 + e) : 0.f;
#pragma unroll
          for (int i = 0; i < V; ++i) acc[e][i] = fmaf(g, xv[u].get(i), acc[e][i]);
        }
      }
    }
  }
  // token lanes tl and tl ^ 1, tl ^ 2 of a warp differ in lane bits 3 and 4
#pragma unroll
  for (int e = 0; e < EB; ++e)
#pragma unroll
    for (int i = 0; i < V; ++i) {
      float v = acc[e][i];
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      acc[e][i] = v;
    }
  if ((threadIdx.x & 31) < 8) {
#pragma unroll
    for (int e = 0; e < EB; ++e)
#pragma unroll
      for (int i = 0; i < V; ++i) s_red[warp][cc][e * V + i] = acc[e][i];
  }
  __syncthreads();
  // 8 chunks x EB x V sums over the 8 warps, in warp order
  for (int o = threadIdx.x; o < 8 * EB * V; o += blockDim.x) {
    const int ch = o / (EB * V), r = o % (EB * V), e = r / V, i = r % V;
    const int cg = blockIdx.x * 8 + ch;
    if (cg >= d / V || e0 + e >= E) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += s_red[w][ch][r];
    partial[((int64_t)blockIdx.y * E + e0 + e) * d + (int64_t)cg * V + i] = v;
  }
}

__global__ void dwr_reduce_kernel(const float* __restrict__ partial, float* __restrict__ dw,
                                  int64_t n, int splits, int accumulate) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += partial[(int64_t)s * n + i];
    dw[i] = accumulate ? dw[i] + v : v;  // the splits are summed first, then added
  }
}

template <typename T>
cudaError_t route_bwd_t(const void* x, const void* w_router, const float* logits,
                        const int32_t* topk_idx, const float* dgate, const void* dx_perm,
                        const int32_t* slot_row, void* dx, float* dw_router, int T_, int d, int E,
                        int k, void* scratch, int* status, cudaStream_t st, bool accumulate) {
  constexpr int V = Vec16<T>::N;
  constexpr int EB = 8;
  const int splits = route_bwd_splits(T_);
  float* dl = static_cast<float*>(scratch);
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) +
                                            align256((size_t)T_ * E * 4));
  const int64_t n = (int64_t)E * d;
  const int lgrid = std::min((T_ + 7) / 8, num_sms() * 8);
  if (T_ > 0 && sizeof(T) == 2 && route_bwd_tc_supported(E, k, d)) {
    // tensor cores: dl (bf16) is the A operand of both the dx and the dW_r GEMM
    __nv_bfloat16* dl_bf = static_cast<__nv_bfloat16*>(scratch);
    const int tsplits = std::max(1, std::min(32, T_ / 1024));
    {
      ProfScope prof("router_dlogit", st);
      dlogit_kernel<<<lgrid, 256, 0, st>>>(logits, topk_idx, dgate, nullptr, dl_bf, T_, E, k);
    }
    // the k expert rows of each token are summed first by the streaming row-sum (bf16
    // [T, d] in the workspace); the dx GEMM's epilogue then adds one contiguous row
    __nv_bfloat16* dxs = reinterpret_cast<__nv_bfloat16*>(
        reinterpret_cast<uint8_t*>(partial) + align256((size_t)route_bwd_splits(T_) * E * d * 4));
    // (without slot_row, dx_perm already holds each token's summed row)
    cudaError_t err = slot_row ? combine_launch(true, dx_perm, slot_row, nullptr, dxs, T_, d, k,
                                                st, "router_rowsum")
                               : cudaSuccess;
    if (err != cudaSuccess) return err;
    err = route_bwd_tc_launch(x, w_router, dl_bf, slot_row ? dxs : dx_perm, nullptr, dx, partial,
                              tsplits, T_, d, E, k, status, st);
    if (err != cudaSuccess) return err;
    {
      ProfScope prof("router_dw_reduce", st);
      dwr_reduce_kernel<<<(int)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, st>>>(
          partial, dw_router, n, tsplits, accumulate);
    }
    return cudaGetLastError();
  }
  if (T_ > 0) {
    {
      ProfScope prof("router_dlogit", st);
      dlogit_kernel<<<lgrid, 256, 0, st>>>(logits, topk_idx, dgate, dl, nullptr, T_, E, k);
    }
    const int tpw = k <= 8 ? 4 : 1;
    const size_t dl_smem = (size_t)8 * tpw * E * sizeof(float);
    auto dxk = k <= 4 ? dx_kernel<T, 4, 4> : (k <= 8 ? dx_kernel<T, 4, 8> : dx_kernel<T, 1, 8>);
    cudaError_t err = cudaFuncSetAttribute(dxk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)dl_smem);
    if (err != cudaSuccess) return err;
    {
      ProfScope prof("router_dx_simt", st);
      dxk<<<(T_ + 8 * tpw - 1) / (8 * tpw), 256, dl_smem, st>>>(dl, static_cast<const T*>(w_router),
                                                static_cast<const T*>(dx_perm), slot_row,
                                                static_cast<T*>(dx), T_, d, E, k);
    }
    const int tps = (T_ + splits - 1) / splits;
    dim3 g2((d / V + 7) / 8, splits, (E + EB - 1) / EB);
    {
      ProfScope prof("router_dw_simt", st);
      dwr_partial_kernel<T, EB><<<g2, 256, 0, st>>>(dl, static_cast<const T*>(x), partial, T_, d,
                                                    E, tps);
    }
    {
      ProfScope prof("router_dw_reduce", st);
      dwr_reduce_kernel<<<(int)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, st>>>(
          partial, dw_router, n, splits, accumulate);
    }
  } else if (!accumulate) {
    cudaMemsetAsync(dw_router, 0, n * sizeof(float), st);
  }
  return cudaGetLastError();
}

}  // namespace

size_t route_bwd_ws_bytes(int T, int d, int E) {
  // dl, the dW_r partial sums, and (tensor-core path) the bf16 row sums of dx_perm
  return align256((size_t)T * E * 4) + align256((size_t)route_bwd_splits(T) * E * d * 4) +
         align256((size_t)T * d * 2);
}

cudaError_t route_bwd_launch(bool bf16, const void* x, const void* w_router, const float* logits,
                             const int32_t* topk_idx, const float* dgate, const void* dx_perm,
                             const int32_t* slot_row, void* dx, float* dw_router, int T, int d,
                             int E, int k, void* scratch, int* status, cudaStream_t st,
                             bool accumulate) {
  if (bf16)
    return route_bwd_t<__nv_bfloat16>(x, w_router, logits, topk_idx, dgate, dx_perm, slot_row, dx,
                                      dw_router, T, d, E, k, scratch, status, st, accumulate);
  return route_bwd_t<float>(x, w_router, logits, topk_idx, dgate, dx_perm, slot_row, dx,
                            dw_router, T, d, E, k, scratch, status, st, accumulate);
}

}  // namespace moe
