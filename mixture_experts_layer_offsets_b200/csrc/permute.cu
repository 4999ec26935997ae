// permute.cu -- rowwise permute into the expert input buffers, gate-weighted
// combine and its backward, and the padded-capacity dispatch.
//
// Pages: "Olmo-core 3 mở rộng quy mô đào tạo mixture-of-experts ..." (bytechap.com),
// section "Cách thức hoạt động" (how it works): rowwise dispatch writes routed data
// straight into the experts' input buffers; "Ai2 Olmo-core 3：MoE训练吞吐量提升2.7倍
// 的秘诀" (kongchang.com), section 路由不只是模型问题，更是系统问题: comparison with
// padding every expert batch to a uniform capacity.
//
// All kernels here are HBM-bound row copies: one warp per token, 16-byte vector
// loads and stores (8 bf16 or 4 fp32 per lane per access), several loads in
// flight per lane, grids sized to a multiple of the SM count.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kBatch = 4;  // 16-byte chunks in flight per lane

inline int row_grid(int64_t warps_needed) {
  const int64_t blocks = (warps_needed + kWarpsPerBlock - 1) / kWarpsPerBlock;
  return (int)std::max<int64_t>(1, std::min<int64_t>(blocks, (int64_t)num_sms() * 16));
}

template <typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
permute_kernel(const T* __restrict__ x, const int32_t* __restrict__ slot_row, T* __restrict__ x_perm,
               int32_t* __restrict__ perm_src, int ntok, int d, int k) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int chunks = d / V;
  for (int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); t < ntok;
       t += gridDim.x * kWarpsPerBlock) {
    const int myrow = lane < k ? slot_row[(int64_t)t * k + lane] : -1;
    if (lane < k && myrow >= 0) perm_src[myrow] = t;
    const T* src = x + (int64_t)t * d;
    for (int c0 = 0; c0 < chunks; c0 += 32 * kBatch) {
      uint4 v[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int c = c0 + b * 32 + lane;
        if (c < chunks) v[b] = ldg16(src + c * V);
      }
      for (int j = 0; j < k; ++j) {
        const int r = __shfl_sync(0xffffffffu, myrow, j);
        if (r < 0) continue;
        T* dst = x_perm + (int64_t)r * d;
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int c = c0 + b * 32 + lane;
          if (c < chunks) stg16(dst + c * V, v[b]);
        }
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
combine_kernel(const T* __restrict__ y_perm, const int32_t* __restrict__ slot_row,
               const float* __restrict__ gate, T* __restrict__ out, int ntok, int d, int k) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int chunks = d / V;
  for (int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); t < ntok;
       t += gridDim.x * kWarpsPerBlock) {
    const int myrow = lane < k ? slot_row[(int64_t)t * k + lane] : -1;
    const float mygate = lane < k ? (gate ? gate[(int64_t)t * k + lane] : 1.f) : 0.f;  // no gate: sum
    for (int c0 = 0; c0 < chunks; c0 += 32 * kBatch) {
      float acc[kBatch][V];
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
#pragma unroll
        for (int i = 0; i < V; ++i) acc[b][i] = 0.f;
      for (int j = 0; j < k; ++j) {  // ascending j: fixed summation order
        const int r = __shfl_sync(0xffffffffu, myrow, j);
        const float g = __shfl_sync(0xffffffffu, mygate, j);
        if (r < 0) continue;
        const T* src = y_perm + (int64_t)r * d;
        Vec16<T> v[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int c = c0 + b * 32 + lane;
          if (c < chunks) v[b].raw = ldg16(src + c * V);
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b)
#pragma unroll
          for (int i = 0; i < V; ++i) acc[b][i] = fmaf(g, v[b].get(i), acc[b][i]);
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int c = c0 + b * 32 + lane;
        if (c < chunks) {
          Vec16<T> o;
#pragma unroll
          for (int i = 0; i < V; ++i) o.set(i, acc[b][i]);
          stg16(out + (int64_t)t * d + c * V, o.raw);
        }
      }
    }
  }
}

template <typename T, int KMAX>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
combine_bwd_kernel(const T* __restrict__ dout, const T* __restrict__ y_perm,
                   const int32_t* __restrict__ slot_row, const float* __restrict__ gate,
                   T* __restrict__ dy_perm, float* __restrict__ dgate, int ntok, int d, int k) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int chunks = d / V;
  for (int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); t < ntok;
       t += gridDim.x * kWarpsPerBlock) {
    const int myrow = lane < k ? slot_row[(int64_t)t * k + lane] : -1;
    const float mygate = lane < k ? gate[(int64_t)t * k + lane] : 0.f;
    float dot[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) dot[j] = 0.f;
    for (int c0 = 0; c0 < chunks; c0 += 32 * kBatch) {
      Vec16<T> g[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int c = c0 + b * 32 + lane;
        if (c < chunks) g[b].raw = ldg16(dout + (int64_t)t * d + c * V);
      }
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j >= k) break;
        const int r = __shfl_sync(0xffffffffu, myrow, j);
        const float gt = __shfl_sync(0xffffffffu, mygate, j);
        if (r < 0) continue;
        const T* ysrc = y_perm + (int64_t)r * d;
        T* dst = dy_perm ? dy_perm + (int64_t)r * d : nullptr;
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int c = c0 + b * 32 + lane;
          if (c < chunks) {
            Vec16<T> yv;
            yv.raw = ldg16(ysrc + c * V);
            Vec16<T> o;
#pragma unroll
            for (int i = 0; i < V; ++i) {
              dot[j] = fmaf(g[b].get(i), yv.get(i), dot[j]);
              o.set(i, gt * g[b].get(i));
            }
            if (dy_perm) stg16(dst + c * V, o.raw);  // null: dgate only
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= k) break;
      const float s = warp_sum(dot[j]);
      const int r = __shfl_sync(0xffffffffu, myrow, j);
      if (lane == 0) dgate[(int64_t)t * k + j] = r >= 0 ? s : 0.f;
    }
  }
}

// dgate alone (the combine backward of a layer that needs no dy_perm rows): every load of
// a chunk round, the output gradient's and all k expert rows', is issued before the first
// product, so the k rows' latencies overlap.  Each lane visits its chunks lane, lane + 32,
// ... in the same order as combine_bwd_kernel, whatever KB is, so the dot products, and
// dgate, are bit-identical to it.
template <typename T, int KMAX, int KB>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
dgate_kernel(const T* __restrict__ dout, const T* __restrict__ y_perm,
             const int32_t* __restrict__ slot_row, float* __restrict__ dgate, int ntok, int d,
             int k) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int chunks = d / V;
  for (int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); t < ntok;
       t += gridDim.x * kWarpsPerBlock) {
    const int myrow = lane < k ? slot_row[(int64_t)t * k + lane] : -1;
    int rows[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) rows[j] = __shfl_sync(0xffffffffu, myrow, j);
    float dot[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) dot[j] = 0.f;
    for (int c0 = 0; c0 < chunks; c0 += 32 * KB) {
      Vec16<T> g[KB], y[KMAX][KB];
#pragma unroll
      for (int b = 0; b < KB; ++b) {
        const int c = c0 + b * 32 + lane;
        g[b].raw = c < chunks ? ldg16(dout + (int64_t)t * d + c * V) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          y[j][b].raw = (j < k && rows[j] >= 0 && c < chunks)
                            ? ldg16(y_perm + (int64_t)rows[j] * d + c * V)
                            : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j >= k || rows[j] < 0) continue;
#pragma unroll
        for (int b = 0; b < KB; ++b) {
          if (c0 + b * 32 + lane >= chunks) continue;
#pragma unroll
          for (int i = 0; i < V; ++i) dot[j] = fmaf(g[b].get(i), y[j][b].get(i), dot[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= k) break;
      const float s = warp_sum(dot[j]);
      if (lane == 0) dgate[(int64_t)t * k + j] = rows[j] >= 0 ? s : 0.f;
    }
  }
}

// Zero the unused rows of x_pad (rank >= count) and write offsets_pad[e] = e * C.
template <typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
padded_zero_kernel(const int32_t* __restrict__ offsets, T* __restrict__ x_pad,
                   int32_t* __restrict__ offsets_pad, int E, int C, int d) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int gtid = blockIdx.x * blockDim.x + threadIdx.x;
  if (gtid <= E) offsets_pad[gtid] = gtid * C;
  const int64_t nrows = (int64_t)E * C;
  const int chunks = d / V;
  for (int64_t r = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); r < nrows;
       r += (int64_t)gridDim.x * kWarpsPerBlock) {
    const int e = (int)(r / C), q = (int)(r % C);
    if (q < offsets[e + 1] - offsets[e]) continue;
    for (int c = lane; c < chunks; c += 32) stg16(x_pad + r * d + c * V, make_uint4(0, 0, 0, 0));
  }
}

template <typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
padded_dispatch_kernel(const T* __restrict__ x, const int32_t* __restrict__ topk_idx,
                       const int32_t* __restrict__ slot_row, const int32_t* __restrict__ offsets,
                       T* __restrict__ x_pad, int32_t* __restrict__ pad_row, int ntok, int d,
                       int k, int C) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int chunks = d / V;
  for (int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); t < ntok;
       t += gridDim.x * kWarpsPerBlock) {
    int prow = -1;
    if (lane < k) {
      const int64_t i = (int64_t)t * k + lane;
      const int e = topk_idx[i];
      const int q = slot_row[i] - offsets[e];
      prow = q < C ? e * C + q : -1;
      pad_row[i] = prow;
    }
    const T* src = x + (int64_t)t * d;
    for (int j = 0; j < k; ++j) {
      const int r = __shfl_sync(0xffffffffu, prow, j);
      if (r < 0) continue;
      for (int c = lane; c < chunks; c += 32)
        stg16(x_pad + (int64_t)r * d + c * V, ldg16(src + c * V));
    }
  }
}

}  // namespace

namespace {
// gate_perm[slot_row[i]] = gate[i]: each routed row's gate, in the permuted row order
__global__ void __launch_bounds__(256) perm_gate_kernel(const int32_t* __restrict__ slot_row,
                                                        const float* __restrict__ gate,
                                                        float* __restrict__ gate_perm, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) gate_perm[slot_row[i]] = gate[i];
}

__global__ void __launch_bounds__(256) perm_src_kernel(const int32_t* __restrict__ slot_row,
                                                       int32_t* __restrict__ perm_src, int64_t n,
                                                       int k) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) perm_src[slot_row[i]] = (int32_t)(i / k);
}
}  // namespace

cudaError_t perm_src_launch(const int32_t* slot_row, int32_t* perm_src, int T, int k,
                            cudaStream_t st) {
  const int64_t n = (int64_t)T * k;
  if (n == 0) return cudaSuccess;
  {
    ProfScope prof("perm_src", st);
    perm_src_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(slot_row, perm_src, n, k);
  }
  return cudaGetLastError();
}

cudaError_t perm_gate_launch(const int32_t* slot_row, const float* gate, float* gate_perm, int T,
                             int k, cudaStream_t st) {
  const int64_t n = (int64_t)T * k;
  if (n == 0) return cudaSuccess;
  {
    ProfScope prof("perm_gate", st);
    perm_gate_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(slot_row, gate, gate_perm, n);
  }
  return cudaGetLastError();
}

cudaError_t permute_launch(bool bf16, const void* x, const int32_t* slot_row, void* x_perm,
                           int32_t* perm_src, int T, int d, int k, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int grid = row_grid(T);
  if (bf16) {
    ProfScope prof("permute", st);
    permute_kernel<__nv_bfloat16><<<grid, kWarpsPerBlock * 32, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), slot_row, static_cast<__nv_bfloat16*>(x_perm),
        perm_src, T, d, k);
  } else {
    ProfScope prof("permute", st);
    permute_kernel<float><<<grid, kWarpsPerBlock * 32, 0, st>>>(
        static_cast<const float*>(x), slot_row, static_cast<float*>(x_perm), perm_src, T, d, k);
  }
  return cudaGetLastError();
}

cudaError_t combine_launch(bool bf16, const void* y_perm, const int32_t* slot_row,
                           const float* gate, void* out, int T, int d, int k, cudaStream_t st,
                           const char* prof_name) {
  if (T == 0) return cudaSuccess;
  const int grid = row_grid(T);
  if (bf16) {
    ProfScope prof(prof_name, st);
    combine_kernel<__nv_bfloat16><<<grid, kWarpsPerBlock * 32, 0, st>>>(
        static_cast<const __nv_bfloat16*>(y_perm), slot_row, gate,
        static_cast<__nv_bfloat16*>(out), T, d, k);
  } else {
    ProfScope prof(prof_name, st);
    combine_kernel<float><<<grid, kWarpsPerBlock * 32, 0, st>>>(
        static_cast<const float*>(y_perm), slot_row, gate, static_cast<float*>(out), T, d, k);
  }
  return cudaGetLastError();
}

template <typename T>
static void combine_bwd_t(const void* dout, const void* y_perm, const int32_t* slot_row,
                          const float* gate, void* dy_perm, float* dgate, int ntok, int d, int k,
                          cudaStream_t st) {
  const int grid = row_grid(ntok);
  if (!dy_perm && k <= 8) {  // dgate only
    ProfScope prof("combine_bwd", st);
    if (k <= 4)
      dgate_kernel<T, 4, 4><<<grid, kWarpsPerBlock * 32, 0, st>>>(
          static_cast<const T*>(dout), static_cast<const T*>(y_perm), slot_row, dgate, ntok, d, k);
    else
      dgate_kernel<T, 8, 2><<<grid, kWarpsPerBlock * 32, 0, st>>>(
          static_cast<const T*>(dout), static_cast<const T*>(y_perm), slot_row, dgate, ntok, d, k);
    return;
  }
  if (k <= 8) {
    ProfScope prof("combine_bwd", st);
    combine_bwd_kernel<T, 8><<<grid, kWarpsPerBlock * 32, 0, st>>>(
        static_cast<const T*>(dout), static_cast<const T*>(y_perm), slot_row, gate,
        static_cast<T*>(dy_perm), dgate, ntok, d, k);
  } else {
    ProfScope prof("combine_bwd", st);
    combine_bwd_kernel<T, 32><<<grid, kWarpsPerBlock * 32, 0, st>>>(
        static_cast<const T*>(dout), static_cast<const T*>(y_perm), slot_row, gate,
        static_cast<T*>(dy_perm), dgate, ntok, d, k);
  }
}

cudaError_t combine_bwd_launch(bool bf16, const void* dout, const void* y_perm,
                               const int32_t* slot_row, const float* gate, void* dy_perm,
                               float* dgate, int T, int d, int k, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (bf16)
    combine_bwd_t<__nv_bfloat16>(dout, y_perm, slot_row, gate, dy_perm, dgate, T, d, k, st);
  else
    combine_bwd_t<float>(dout, y_perm, slot_row, gate, dy_perm, dgate, T, d, k, st);
  return cudaGetLastError();
}

template <typename T>
static void padded_t(int C, const void* x, const int32_t* topk_idx, const int32_t* slot_row,
                     const int32_t* offsets, void* x_pad, int32_t* pad_row, int32_t* offsets_pad,
                     int ntok, int d, int E, int k, cudaStream_t st) {
  const int64_t nrows = (int64_t)E * C;
  int grid = row_grid(nrows);
  grid = std::max(grid, (E + 1 + kWarpsPerBlock * 32 - 1) / (kWarpsPerBlock * 32));
  {
    ProfScope prof("padded_zero", st);
    padded_zero_kernel<T><<<grid, kWarpsPerBlock * 32, 0, st>>>(offsets, static_cast<T*>(x_pad),
                                                               offsets_pad, E, C, d);
  }
  if (ntok > 0) {
    ProfScope prof("padded_dispatch", st);
    padded_dispatch_kernel<T><<<row_grid(ntok), kWarpsPerBlock * 32, 0, st>>>(
        static_cast<const T*>(x), topk_idx, slot_row, offsets, static_cast<T*>(x_pad), pad_row,
        ntok, d, k, C);
  }
}

cudaError_t padded_dispatch_launch(bool bf16, int capacity, const void* x, const int32_t* topk_idx,
                                   const int32_t* slot_row, const int32_t* offsets, void* x_pad,
                                   int32_t* pad_row, int32_t* offsets_pad, int T, int d, int E,
                                   int k, cudaStream_t st) {
  if (bf16)
    padded_t<__nv_bfloat16>(capacity, x, topk_idx, slot_row, offsets, x_pad, pad_row, offsets_pad,
                            T, d, E, k, st);
  else
    padded_t<float>(capacity, x, topk_idx, slot_row, offsets, x_pad, pad_row, offsets_pad, T, d,
                    E, k, st);
  return cudaGetLastError();
}

}  // namespace moe
