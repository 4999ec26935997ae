// ep.cu -- expert parallelism across ranks: the layout of the row exchange, the dispatch
// that writes the selected token rows straight into the expert owners' buffers, and the
// combine steps that read the owners' rows back (plain loads and stores through peer
// pointers over NVLink; no TMA, no library kernel touches peer memory).
//
// Page: "Ai2 Olmo-core 3：MoE训练吞吐量提升2.7倍的秘诀" (kongchang.com), section 容量税:
// expert parallelism spreads the routed experts over the ranks and writes only the
// selected token rows directly into the target rank's buffer; section
// 路由不只是模型问题，更是系统问题: the exchange's split sizes stay on the GPU.
// "Olmo-core 3 mở rộng quy mô ..." (bytechap.com), "Cách thức hoạt động": each device
// holds a fraction of the experts; rowwise expert parallelism places routed rows directly
// in the experts' input buffers.
//
// Layout (rank o owns experts [o E_loc, (o + 1) E_loc), E_loc = E / N): an owner's
// buffer holds its experts' rows expert by expert, within an expert by source rank,
// within a source in token order -- the rows one device would permute from the ranks'
// concatenated batches, in the same order.  All sizes come from the gathered counts
// [N, E] on the device.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kWarps = 8;
constexpr int kBatch = 4;  // 16-byte chunks in flight per lane

inline int ep_grid(int64_t warps) {
  const int64_t blocks = (warps + kWarps - 1) / kWarps;
  return (int)std::max<int64_t>(1, std::min<int64_t>(blocks, (int64_t)num_sms() * 16));
}

// One block of up to 1024 threads, thread e = expert e.
__global__ void __launch_bounds__(1024)
ep_layout_kernel(const int32_t* __restrict__ counts_all, int N, int E, int rank,
                 int32_t* __restrict__ recv_offsets, int32_t* __restrict__ send_base) {
  __shared__ int32_t s_scan[1025];
  __shared__ int32_t s_warp[32];
  const int e = threadIdx.x, lane = e & 31, w = e >> 5;
  const int El = E / N;
  int tot = 0, before = 0;  // rows of expert e from all ranks, from the ranks before `rank`
  if (e < E)
    for (int s = 0; s < N; ++s) {
      const int c = counts_all[(int64_t)s * E + e];
      tot += c;
      if (s < rank) before += c;
    }
  // exclusive scan of tot over all experts
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) s_warp[w] = incl;
  __syncthreads();
  if (w == 0) {
    int v = lane < (int)((blockDim.x + 31) / 32) ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    s_warp[lane] = v;
  }
  __syncthreads();
  const int excl = incl - tot + (w > 0 ? s_warp[w - 1] : 0);
  if (e < E) s_scan[e] = excl;
  if (e == E - 1) s_scan[E] = excl + tot;
  __syncthreads();
  if (e < E) {
    const int o = e / El;  // owner of expert e
    send_base[e] = excl - s_scan[o * El] + before;
  }
  for (int i = e; i <= El; i += blockDim.x) recv_offsets[i] = s_scan[rank * El + i] - s_scan[rank * El];
}

// One warp per token: lanes < k compute their pair's owner and row, then the warp copies
// the token row to each owner's buffer with 16-byte stores (the row read once).
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
ep_dispatch_kernel(const T* __restrict__ x, const int32_t* __restrict__ topk_idx,
                   const int32_t* __restrict__ slot_row, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ send_base, EpPeers peers,
                   int32_t* __restrict__ ep_row, int ntok, int d, int k, int El, int nranks) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int chunks = d / V;
  for (int t = blockIdx.x * kWarps + (threadIdx.x >> 5); t < ntok; t += gridDim.x * kWarps) {
    int row = -1, own = 0;
    if (lane < k) {
      const int64_t i = (int64_t)t * k + lane;
      const int e = topk_idx[i], sr = slot_row[i];
      // (a routing pass that gave up a bounded wait can leave a pair unrouted: row -1)
      if ((unsigned)e < (unsigned)(El * nranks) && sr >= 0) {
        own = e / El;
        row = send_base[e] + (sr - offsets[e]);
      }
      ep_row[i] = row;
    }
    const T* src = x + (int64_t)t * d;
    for (int c0 = 0; c0 < chunks; c0 += 32 * kBatch) {
      uint4 v[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int c = c0 + b * 32 + lane;
        if (c < chunks) v[b] = ldg16(src + c * V);
      }
      for (int j = 0; j < k; ++j) {
        const int r = __shfl_sync(0xffffffffu, row, j);
        const int o = __shfl_sync(0xffffffffu, own, j);
        if (r < 0) continue;
        T* dst = static_cast<T*>(peers.p[o]) + (int64_t)r * d;
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int c = c0 + b * 32 + lane;
          if (c < chunks) stg16(dst + c * V, v[b]);
        }
      }
    }
  }
  // the rows written into other ranks' memory are ordered before anything this rank
  // issues after the kernel (the collective that tells the owners they may read)
  __threadfence_system();
}

// out[t] = sum_j gate[t, j] * y[owner][ep_row[t, j]] in fp32, ascending j, rounded once
// (gate == nullptr: the plain sum, for the input-gradient rows).
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
ep_combine_kernel(EpPeers peers, const int32_t* __restrict__ topk_idx,
                  const int32_t* __restrict__ ep_row, const float* __restrict__ gate,
                  T* __restrict__ out, int ntok, int d, int k, int El) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int chunks = d / V;
  for (int t = blockIdx.x * kWarps + (threadIdx.x >> 5); t < ntok; t += gridDim.x * kWarps) {
    int row = -1, own = 0;
    float g = 0.f;
    if (lane < k) {
      const int64_t i = (int64_t)t * k + lane;
      row = ep_row[i];
      own = row >= 0 ? topk_idx[i] / El : 0;
      g = gate ? gate[i] : 1.f;
    }
    for (int c0 = 0; c0 < chunks; c0 += 32 * kBatch) {
      float acc[kBatch][V];
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
#pragma unroll
        for (int i = 0; i < V; ++i) acc[b][i] = 0.f;
      for (int j = 0; j < k; ++j) {
        const int r = __shfl_sync(0xffffffffu, row, j);
        const int o = __shfl_sync(0xffffffffu, own, j);
        const float gj = __shfl_sync(0xffffffffu, g, j);
        if (r < 0) continue;
        const T* src = static_cast<const T*>(peers.p[o]) + (int64_t)r * d;
        Vec16<T> v[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int c = c0 + b * 32 + lane;
          if (c < chunks) v[b].raw = ldg16(src + c * V);
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b)
#pragma unroll
          for (int i = 0; i < V; ++i) acc[b][i] = fmaf(gj, v[b].get(i), acc[b][i]);
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

// dgate[t, j] = <dout[t], y[owner][row]>; dy[owner][row] = gate[t, j] * dout[t].
template <typename T, int KMAX>
__global__ void __launch_bounds__(kWarps * 32)
ep_combine_bwd_kernel(const T* __restrict__ dout, EpPeers peers_y, EpPeers peers_dy,
                      const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ ep_row,
                      const float* __restrict__ gate, float* __restrict__ dgate, int ntok, int d,
                      int k, int El) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int chunks = d / V;
  for (int t = blockIdx.x * kWarps + (threadIdx.x >> 5); t < ntok; t += gridDim.x * kWarps) {
    int row = -1, own = 0;
    float g = 0.f;
    if (lane < k) {
      const int64_t i = (int64_t)t * k + lane;
      row = ep_row[i];
      own = row >= 0 ? topk_idx[i] / El : 0;
      g = gate[i];
    }
    float dot[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) dot[j] = 0.f;
    for (int c0 = 0; c0 < chunks; c0 += 32 * kBatch) {
      Vec16<T> gv[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int c = c0 + b * 32 + lane;
        if (c < chunks) gv[b].raw = ldg16(dout + (int64_t)t * d + c * V);
      }
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j >= k) break;
        const int r = __shfl_sync(0xffffffffu, row, j);
        const int o = __shfl_sync(0xffffffffu, own, j);
        const float gj = __shfl_sync(0xffffffffu, g, j);
        if (r < 0) continue;
        const T* ysrc = static_cast<const T*>(peers_y.p[o]) + (int64_t)r * d;
        T* dst = static_cast<T*>(peers_dy.p[o]) + (int64_t)r * d;
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int c = c0 + b * 32 + lane;
          if (c < chunks) {
            Vec16<T> yv;
            yv.raw = ldg16(ysrc + c * V);
            Vec16<T> ov;
#pragma unroll
            for (int i = 0; i < V; ++i) {
              dot[j] = fmaf(gv[b].get(i), yv.get(i), dot[j]);
              ov.set(i, gj * gv[b].get(i));
            }
            stg16(dst + c * V, ov.raw);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= k) break;
      const float s = warp_sum(dot[j]);
      const int r = __shfl_sync(0xffffffffu, row, j);
      if (lane == 0) dgate[(int64_t)t * k + j] = r >= 0 ? s : 0.f;
    }
  }
  __threadfence_system();
}

}  // namespace

cudaError_t ep_layout_launch(const int32_t* counts_all, int N, int E, int rank,
                             int32_t* recv_offsets, int32_t* send_base, cudaStream_t st) {
  const int threads = std::max(32, ((E + 31) / 32) * 32);  // E <= 1024
  ProfScope prof("ep_layout", st);
  ep_layout_kernel<<<1, threads, 0, st>>>(counts_all, N, E, rank, recv_offsets, send_base);
  return cudaGetLastError();
}

cudaError_t ep_dispatch_launch(bool bf16, const void* x, const int32_t* topk_idx,
                               const int32_t* slot_row, const int32_t* offsets,
                               const int32_t* send_base, const EpPeers& peers, int32_t* ep_row,
                               int T, int d, int k, int El, int nranks, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  ProfScope prof("ep_dispatch", st);
  if (bf16)
    ep_dispatch_kernel<__nv_bfloat16><<<ep_grid(T), kWarps * 32, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), topk_idx, slot_row, offsets, send_base, peers,
        ep_row, T, d, k, El, nranks);
  else
    ep_dispatch_kernel<float><<<ep_grid(T), kWarps * 32, 0, st>>>(
        static_cast<const float*>(x), topk_idx, slot_row, offsets, send_base, peers, ep_row, T,
        d, k, El, nranks);
  return cudaGetLastError();
}

cudaError_t ep_combine_launch(bool bf16, const EpPeers& peers, const int32_t* topk_idx,
                              const int32_t* ep_row, const float* gate, void* out, int T, int d,
                              int k, int El, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  ProfScope prof(gate ? "ep_combine" : "ep_gather_grad", st);
  if (bf16)
    ep_combine_kernel<__nv_bfloat16><<<ep_grid(T), kWarps * 32, 0, st>>>(
        peers, topk_idx, ep_row, gate, static_cast<__nv_bfloat16*>(out), T, d, k, El);
  else
    ep_combine_kernel<float><<<ep_grid(T), kWarps * 32, 0, st>>>(
        peers, topk_idx, ep_row, gate, static_cast<float*>(out), T, d, k, El);
  return cudaGetLastError();
}

cudaError_t ep_combine_bwd_launch(bool bf16, const void* dout, const EpPeers& peers_y,
                                  const EpPeers& peers_dy, const int32_t* topk_idx,
                                  const int32_t* ep_row, const float* gate, float* dgate, int T,
                                  int d, int k, int El, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  ProfScope prof("ep_combine_bwd", st);
  const int grid = ep_grid(T);
  if (bf16) {
    if (k <= 8)
      ep_combine_bwd_kernel<__nv_bfloat16, 8><<<grid, kWarps * 32, 0, st>>>(
          static_cast<const __nv_bfloat16*>(dout), peers_y, peers_dy, topk_idx, ep_row, gate,
          dgate, T, d, k, El);
    else
      ep_combine_bwd_kernel<__nv_bfloat16, 32><<<grid, kWarps * 32, 0, st>>>(
          static_cast<const __nv_bfloat16*>(dout), peers_y, peers_dy, topk_idx, ep_row, gate,
          dgate, T, d, k, El);
  } else {
    if (k <= 8)
      ep_combine_bwd_kernel<float, 8><<<grid, kWarps * 32, 0, st>>>(
          static_cast<const float*>(dout), peers_y, peers_dy, topk_idx, ep_row, gate, dgate, T,
          d, k, El);
    else
      ep_combine_bwd_kernel<float, 32><<<grid, kWarps * 32, 0, st>>>(
          static_cast<const float*>(dout), peers_y, peers_dy, topk_idx, ep_row, gate, dgate, T,
          d, k, El);
  }
  return cudaGetLastError();
}

}  // namespace moe
