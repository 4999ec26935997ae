// route.cu -- router logits, fused softmax/top-k, on-device histogram and
// prefix scan of expert counts, and the slot row of every (token, slot) pair.
//
// Page: "Ai2 Olmo-core 3：MoE训练吞吐量提升2.7倍的秘诀" (kongchang.com), section
// 路由不只是模型问题，更是系统问题 (routing is a systems problem): routing metadata
// (split sizes, expert GEMM group sizes) stays on the GPU; section 容量税: each
// token activates a few of the experts through a route function.
//
// Three launches, no host round trip:
//   1. route_topk_kernel   -- per block of TB tokens: fp32 logits (CUDA-core dot
//      products; for E <= 32 each warp streams 4 token rows with 16-byte loads,
//      for larger E shared-memory tiles), softmax, top-k (warp argmax, lowest
//      index wins ties), the
//      block's per-expert counts and each pair's rank among the block's pairs
//      of the same expert;
//   2. block_scan_kernel    -- per expert: exclusive scan of the block counts in
//      block order (gives each block's base inside the expert) and the total;
//   3. slot_rows_kernel     -- offsets = exclusive scan of the totals;
//      slot_row = offsets[e] + block base + rank within the block.
// Rows inside an expert segment therefore follow token order, and every
// integer is deterministic.
#include "common.cuh"
#include "internal.h"

#include <stdlib.h>

namespace moe {

namespace {

constexpr int kRouteThreads = 256;
constexpr int kDC = 32;  // d-chunk staged in shared memory

// Tokens per block: keep the [TB, E] logit tile within 32 KB.
__host__ __device__ inline int route_tb(int E) { return E <= 256 ? 32 : (E <= 512 ? 16 : 8); }

// Logits of TB = 32 tokens for E <= EMAX experts: each warp takes 4 tokens,
// each lane 16-byte chunks of their rows (coalesced reads of x) and keeps
// 4 x EMAX partial dot products; the router rows come through L1.
template <typename T, int EMAX>
__device__ __forceinline__ void logits_narrow(const T* __restrict__ x, const T* __restrict__ w,
                                              const float* __restrict__ bias, int ntok, int d,
                                              int E, int t0, float* lg) {
  constexpr int V = Vec16<T>::N;
  constexpr int TPW = 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = warp * TPW;
  float acc[TPW][EMAX];
#pragma unroll
  for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[tt][e] = 0.f;
  const int chunks = d / V;
  for (int c = lane; c < chunks; c += 32) {
    Vec16<T> xv[TPW];
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
      const int t = t0 + r0 + tt;
      xv[tt].raw = t < ntok ? ldg16(x + (int64_t)t * d + (int64_t)c * V) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < E) {
        Vec16<T> wv;
        wv.raw = ldg16(w + (int64_t)e * d + (int64_t)c * V);
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
          for (int i = 0; i < V; ++i) acc[tt][e] = fmaf(xv[tt].get(i), wv.get(i), acc[tt][e]);
      }
    }
  }
#pragma unroll
  for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < E) {
        const float v = warp_sum(acc[tt][e]);
        if (lane == 0) lg[(r0 + tt) * E + e] = v + (bias ? bias[e] : 0.f);
      }
    }
}

// Softmax and top-k of a block's TB x E logit tile in shared memory (lg, with the bias
// already added), one warp per token: writes logits, topk_idx, topk_gate and the block's
// selection table sel (-1 for tokens past ntok).  The lowest index wins ties.
template <int TB>
__device__ void topk_tile(const float* lg, int t0, int ntok, int E, int k,
                          float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                          float* __restrict__ topk_gate, int32_t (*sel)[32]) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < TB; r += kRouteThreads / 32) {
    const int t = t0 + r;
    if (t >= ntok) {
      if (lane < k) sel[r][lane] = -1;
      continue;
    }
    const float* row = lg + r * E;
    float m = -INFINITY;
    for (int e = lane; e < E; e += 32) m = fmaxf(m, row[e]);
    m = warp_max(m);
    float s = 0.f;
    for (int e = lane; e < E; e += 32) {
      s += expf(row[e] - m);
      logits[(int64_t)t * E + e] = row[e];
    }
    s = warp_sum(s);
    uint32_t taken = 0;  // bit i <-> expert lane + 32 i
    for (int j = 0; j < k; ++j) {
      float bv = 0.f;
      int be = -1;
      for (int i = 0, e = lane; e < E; ++i, e += 32) {
        if (taken & (1u << i)) continue;
        const float v = row[e];
        if (be < 0 || v > bv) { bv = v; be = e; }  // ascending e: ties keep the lower index
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (oe >= 0 && (be < 0 || ov > bv || (ov == bv && oe < be))) { bv = ov; be = oe; }
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      if (lane == 0) {
        topk_idx[(int64_t)t * k + j] = be;
        topk_gate[(int64_t)t * k + j] = expf(bv - m) / s;
        sel[r][j] = be;
      }
    }
  }
  __syncthreads();
}

// The block's per-expert counts (blockcounts[e * nb + block]) and each pair's rank among
// the block's earlier pairs of the same expert (token order).
template <int TB>
__device__ void counts_ranks(const int32_t (*sel)[32], int t0, int ntok, int E, int k,
                             int32_t* __restrict__ blockcounts, int32_t* __restrict__ localrank,
                             int nb) {
  const int tid = threadIdx.x;
  for (int i = tid; i < TB * k; i += kRouteThreads) {
    const int r = i / k, j = i % k;
    const int t = t0 + r;
    if (t >= ntok) continue;
    const int e = sel[r][j];
    int rank = 0;
    for (int rr = 0; rr < r; ++rr)
      for (int jj = 0; jj < k; ++jj) rank += (sel[rr][jj] == e);
    localrank[(int64_t)t * k + j] = rank;
  }
  const int nvalid = min(TB, ntok - t0);
  for (int e = tid; e < E; e += kRouteThreads) {
    int c = 0;
    for (int r = 0; r < nvalid; ++r)
      for (int j = 0; j < k; ++j) c += (sel[r][j] == e);
    blockcounts[(int64_t)e * nb + blockIdx.x] = c;
  }
}

// EC experts per pass of the dot-product phase; EMAX > 0 selects the narrow
// (E <= EMAX, TB = 32) logit phase instead of the shared-memory tiles.
template <typename T, int TB, int EC, int EMAX>
__global__ void __launch_bounds__(kRouteThreads)
route_topk_kernel(const T* __restrict__ x, const T* __restrict__ w, const float* __restrict__ bias,
                  int ntok, int d, int E, int k, float* __restrict__ logits,
                  int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                  int32_t* __restrict__ blockcounts, int32_t* __restrict__ localrank, int nb) {
  constexpr int kPer = TB * EC / kRouteThreads;  // outputs per thread
  static_assert(kPer >= 1 && (TB * EC) % kRouteThreads == 0, "tile");
  static_assert(EMAX == 0 || TB == 32, "the narrow phase covers 8 warps x 4 tokens");
  __shared__ float xs[EMAX ? 1 : TB][kDC + 1];
  __shared__ float ws[EMAX ? 1 : EC][kDC + 1];
  __shared__ int32_t sel[TB][32];
  extern __shared__ float lg[];  // [TB][E]

  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * TB;
  const int col = tid % EC;
  const int row0 = tid / EC;
  constexpr int kRowStep = kRouteThreads / EC;

  if constexpr (EMAX > 0) logits_narrow<T, EMAX>(x, w, bias, ntok, d, E, t0, lg);
  else for (int e0 = 0; e0 < E; e0 += EC) {
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
    for (int c0 = 0; c0 < d; c0 += kDC) {
      for (int i = tid; i < TB * kDC; i += kRouteThreads) {
        const int r = i / kDC, c = i % kDC;
        const int t = t0 + r;
        xs[r][c] = (t < ntok && c0 + c < d) ? to_f32(x[(int64_t)t * d + c0 + c]) : 0.f;
      }
      for (int i = tid; i < EC * kDC; i += kRouteThreads) {
        const int r = i / kDC, c = i % kDC;
        const int e = e0 + r;
        ws[r][c] = (e < E && c0 + c < d) ? to_f32(w[(int64_t)e * d + c0 + c]) : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int c = 0; c < kDC; ++c) {
        const float wv = ws[col][c];
#pragma unroll
        for (int i = 0; i < kPer; ++i) acc[i] = fmaf(xs[row0 + i * kRowStep][c], wv, acc[i]);
      }
      __syncthreads();
    }
    const int e = e0 + col;
    if (e < E) {
      const float b = bias ? bias[e] : 0.f;
#pragma unroll
      for (int i = 0; i < kPer; ++i) lg[(row0 + i * kRowStep) * E + e] = acc[i] + b;
    }
  }
  __syncthreads();

  topk_tile<TB>(lg, t0, ntok, E, k, logits, topk_idx, topk_gate, sel);
  counts_ranks<TB>(sel, t0, ntok, E, k, blockcounts, localrank, nb);
}

// Exclusive scan of blockcounts[e][0..nb) for expert e = blockIdx.x.
__global__ void __launch_bounds__(256)
block_scan_kernel(const int32_t* __restrict__ blockcounts, int32_t* __restrict__ blockoffs, int nb,
                  int32_t* __restrict__ counts) {
  __shared__ int32_t warp_tot[8];
  __shared__ int32_t carry;
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* src = blockcounts + (int64_t)e * nb;
  int32_t* dst = blockoffs + (int64_t)e * nb;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < nb; base += 256) {
    const int i = base + tid;
    const int v = i < nb ? src[i] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int wbase = 0, total = 0;
    for (int w2 = 0; w2 < 8; ++w2) {
      if (w2 < warp) wbase += warp_tot[w2];
      total += warp_tot[w2];
    }
    const int c = carry;
    if (i < nb) dst[i] = c + wbase + incl - v;
    __syncthreads();
    if (tid == 0) carry = c + total;
    __syncthreads();
  }
  if (tid == 0) counts[e] = carry;
}

// Exclusive scan of counts[0..E) into s_off[0..E] by one block (E <= 1024).
__device__ void block_offsets(const int32_t* __restrict__ counts, int E, int32_t* s_off) {
  __shared__ int32_t lane_tot[32];
  const int tid = threadIdx.x;
  if (tid < 32) {
    const int lo = tid * 32, hi = min(lo + 32, E);
    int s = 0;
    for (int e = lo; e < hi; ++e) s += counts[e];
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += n;
    }
    int run = incl - s;
    for (int e = lo; e < hi; ++e) {
      s_off[e] = run;
      run += counts[e];
    }
    if (tid == 31) s_off[E] = incl;
    lane_tot[tid] = incl;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(256)
slot_rows_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ localrank,
                 const int32_t* __restrict__ blockoffs, const int32_t* __restrict__ counts,
                 int ntok, int E, int k, int tb, int nb, int32_t* __restrict__ offsets,
                 int32_t* __restrict__ slot_row, int* __restrict__ done_reset) {
  __shared__ int32_t s_off[1025];
  // every block of the routing pass has counted itself (stream order): ready for the next call
  if (done_reset && blockIdx.x == 0 && threadIdx.x == 0) *done_reset = 0;
  block_offsets(counts, E, s_off);
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = s_off[e];
  const int64_t n = (int64_t)ntok * k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / k);
    const int e = topk_idx[i];
    // A routing pass that gave up a bounded wait leaves some indices and ranks
    // unwritten: a pair whose expert or row falls outside its segment gets row -1
    // (which every later step skips), so no later launch indexes out of bounds.
    int r = -1;
    if ((unsigned)e < (unsigned)E) {
      r = s_off[e] + blockoffs[(int64_t)e * nb + t / tb] + localrank[i];
      if (r < s_off[e] || r >= s_off[e + 1]) r = -1;
    }
    slot_row[i] = r;
  }
}

template <typename T, int TB, int EC, int EMAX = 0>
cudaError_t launch_topk(const RouteArgs& a, int nb, cudaStream_t st) {
  const size_t lg_bytes = sizeof(float) * TB * a.E;
  auto kern = route_topk_kernel<T, TB, EC, EMAX>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)lg_bytes);
  if (err != cudaSuccess) return err;
  {
    ProfScope prof("router_simt", st);
    kern<<<nb, kRouteThreads, lg_bytes, st>>>(
        static_cast<const T*>(a.x), static_cast<const T*>(a.w_router), a.bias, a.T, a.d, a.E, a.k,
        a.logits, a.topk_idx, a.topk_gate, a.blockcounts, a.localrank, nb);
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_topk(const RouteArgs& a, int nb, cudaStream_t st) {
  const int tb = route_tb(a.E);
  if (tb == 32) {
    if (a.E <= 8) return launch_topk<T, 32, 8, 8>(a, nb, st);
    if (a.E <= 16) return launch_topk<T, 32, 8, 16>(a, nb, st);
    if (a.E <= 32) return launch_topk<T, 32, 8, 32>(a, nb, st);
    return launch_topk<T, 32, 64>(a, nb, st);
  }
  if (tb == 16) return launch_topk<T, 16, 64>(a, nb, st);
  return launch_topk<T, 8, 64>(a, nb, st);
}

// ---- router for a few experts (bf16, E <= 32): warp-level tensor-core MMA
// The logits are a skinny product (N = E), so the step is bound by reading x once.  Each
// block takes 32 tokens; its 8 warps split them into two 16-token groups and d into four
// quarters, so that the whole token range is spread evenly over every SM in one wave.  A
// warp accumulates its 16 x 8 x NT logit fragment with mma.sync m16n8k16 (bf16 in, fp32
// accumulate) while streaming its rows with 16-byte loads: inside each 32-column chunk,
// lane (g, q) loads columns 8q .. 8q+7 of rows g and g+8 and of expert row g, and the two
// K = 16 steps take elements 0-3 and 4-7 of those loads, so every column of the chunk is
// summed exactly once (the order of the K terms inside a chunk is a fixed permutation,
// the same for x and w_router).  The four quarters' sums are then added in quarter
// order in shared memory, with the bias, which keeps the logits deterministic.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NT>  // E <= 8 * NT
__global__ void __launch_bounds__(kRouteThreads, NT == 1 ? 4 : 2)
route_mma_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w,
                 const float* __restrict__ bias, int ntok, int d, int E, int k,
                 float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                 float* __restrict__ topk_gate, int32_t* __restrict__ blockcounts,
                 int32_t* __restrict__ blockoffs, int32_t* __restrict__ localrank,
                 int32_t* __restrict__ counts, int nb, int* __restrict__ done) {
  constexpr int TB = 32;
  constexpr int EP = 8 * NT + 1;  // padded row of the partial-sum tile
  __shared__ float part[4][TB][EP];
  __shared__ int32_t sel[TB][32];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * TB;
  const int grp = warp & 1, quarter = warp >> 1;
  const int g = lane >> 2, q = lane & 3;
  const int ra = t0 + 16 * grp + g, rb = ra + 8;
  const __nv_bfloat16* xa = x + (int64_t)min(ra, ntok - 1) * d + 8 * q;
  const __nv_bfloat16* xb = x + (int64_t)min(rb, ntok - 1) * d + 8 * q;
  const bool va = ra < ntok, vb = rb < ntok;
  const __nv_bfloat16* wr[NT];
  bool we[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int e = 8 * nt + g;
    we[nt] = e < E;
    wr[nt] = w + (int64_t)min(e, E - 1) * d + 8 * q;
  }
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  // 64-column chunks, dealt round robin to the four warps of a token group, so that at any
  // time the group's warps read neighbouring 128-byte pieces of the same rows; the next
  // chunk's loads are issued before this chunk's MMAs.
  struct Chunk { uint4 a[2], b[2], w[2][NT]; };
  auto load = [&](int c, Chunk& k_) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      k_.a[h] = va ? ldg16(xa + c + 32 * h) : zero;
      k_.b[h] = vb ? ldg16(xb + c + 32 * h) : zero;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) k_.w[h][nt] = we[nt] ? ldg16(wr[nt] + c + 32 * h) : zero;
    }
  };
  const int nchunk = d >> 6;  // d % 128 == 0
  Chunk cur, nxt;
  int ch = quarter;
  if (ch < nchunk) load(ch << 6, cur);
  for (; ch < nchunk; ch += 4) {
    if (ch + 4 < nchunk) load((ch + 4) << 6, nxt);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_bf16_16816(acc[nt], cur.a[h].x, cur.b[h].x, cur.a[h].y, cur.b[h].y, cur.w[h][nt].x,
                       cur.w[h][nt].y);
        mma_bf16_16816(acc[nt], cur.a[h].z, cur.b[h].z, cur.a[h].w, cur.b[h].w, cur.w[h][nt].z,
                       cur.w[h][nt].w);
      }
    cur = nxt;
  }
  // fragment: acc[nt][0..1] = (row g, experts 8nt + 2q, +1), acc[nt][2..3] = row g + 8
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int e = 8 * nt + 2 * q;
    float* p0 = &part[quarter][16 * grp + g][e];
    float* p1 = &part[quarter][16 * grp + g + 8][e];
    p0[0] = acc[nt][0];
    p0[1] = acc[nt][1];
    p1[0] = acc[nt][2];
    p1[1] = acc[nt][3];
  }
  __syncthreads();
  // Epilogue, warp 0, one lane per token with its E <= 32 logits in registers: the four
  // quarters' partial sums added in order (+ bias), softmax, top-k (experts in ascending
  // index, so equal logits keep the lower index), then the block's counts and each pair's
  // rank among the earlier tokens of the block, both from one ballot per expert.
  if (warp == 0) {
    const int t = t0 + lane;
    const bool valid = t < ntok;
    float l[8 * NT];
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < 8 * NT; ++e) {
      l[e] = -INFINITY;
      if (e < E) {
        l[e] = ((part[0][lane][e] + part[1][lane][e]) + part[2][lane][e]) + part[3][lane][e] +
               (bias ? bias[e] : 0.f);
        m = fmaxf(m, l[e]);
      }
    }
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < 8 * NT; ++e)
      if (e < E) sum += expf(l[e] - m);
    uint32_t taken = 0;  // bit e: expert e is one of this token's selection
    for (int j = 0; j < k; ++j) {
      int be = -1;
      float bv = -INFINITY;
#pragma unroll
      for (int e = 0; e < 8 * NT; ++e)
        if (e < E && !(taken >> e & 1u) && (be < 0 || l[e] > bv)) { bv = l[e]; be = e; }
      taken |= 1u << be;
      if (valid) {
        topk_idx[(int64_t)t * k + j] = be;
        topk_gate[(int64_t)t * k + j] = expf(bv - m) / sum;
      }
      sel[lane][j] = be;
    }
    if (valid) {
#pragma unroll
      for (int e4 = 0; e4 < 8 * NT; e4 += 4)
        if (e4 < E) {
          float* o = logits + (int64_t)t * E + e4;
          if ((E & 3) == 0) {
            *reinterpret_cast<float4*>(o) = make_float4(l[e4], l[e4 + 1], l[e4 + 2], l[e4 + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (e4 + i < E) o[i] = l[e4 + i];
          }
        }
    }
    if (!valid) taken = 0;
    const uint32_t below = (1u << lane) - 1u;
    for (int e = 0; e < E; ++e) {
      const uint32_t has = __ballot_sync(0xffffffffu, taken >> e & 1u);
      if (lane == 0) blockcounts[(int64_t)e * nb + blockIdx.x] = __popc(has);
      if (taken >> e & 1u) {
        const int rank = __popc(has & below);
        for (int j = 0; j < k; ++j)
          if (sel[lane][j] == e) localrank[(int64_t)t * k + j] = rank;
      }
    }
  }

  // The last block to finish scans every block's counts (no launch of its own): each
  // expert's exclusive prefix over the blocks, and its total.  `done` counts finished
  // blocks; the slot-row pass that follows resets it to zero.
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(done, 1) == nb - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // one warp per expert: the counts come in rounds of 32 blocks, up to 32 rounds loaded
  // at once (independent loads, one L2 latency), then scanned round by round
  for (int e = warp; e < E; e += kRouteThreads / 32) {
    const int32_t* src = blockcounts + (int64_t)e * nb;
    int32_t* dst = blockoffs + (int64_t)e * nb;
    int carry = 0;
    for (int base = 0; base < nb; base += 1024) {
      int v[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        const int b = base + 32 * r + lane;
        v[r] = b < nb ? __ldcg(src + b) : 0;
      }
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        if (base + 32 * r >= nb) break;
        int incl = v[r];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        const int b = base + 32 * r + lane;
        if (b < nb) dst[b] = carry + incl - v[r];
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    if (lane == 0) counts[e] = carry;
  }
}

template <int NT>
cudaError_t launch_route_mma(const RouteArgs& a, int32_t* blockoffs, int nb, cudaStream_t st) {
  ProfScope prof("router_mma", st);
  route_mma_kernel<NT><<<nb, kRouteThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(a.x), static_cast<const __nv_bfloat16*>(a.w_router),
      a.bias, a.T, a.d, a.E, a.k, a.logits, a.topk_idx, a.topk_gate, a.blockcounts, blockoffs,
      a.localrank, a.counts, nb, a.status + 1);
  return cudaGetLastError();
}

}  // namespace

bool route_mma_supported(int E, int k, int d) { return E <= 32 && k <= E && d % 128 == 0; }

size_t route_ws_bytes(int T, int E, int k) {
  const int tb = route_tb(E);
  const size_t nb = (size_t)((T + tb - 1) / tb);
  return align256(nb * E * 4) * 2 + align256((size_t)T * k * 4);
}

cudaError_t route_launch(const RouteArgs& a0, bool bf16, cudaStream_t st) {
  RouteArgs a = a0;
  // a few experts (bf16): the warp-level MMA router, which needs the workspace's block
  // counter next to its status word; up to 256 experts the tensor-core tile router.
  // MOE_B200_ROUTER=tile / warp selects one of the two where both apply (read per call).
  const char* force = getenv("MOE_B200_ROUTER");
  const bool no_warp = force && force[0] == 't';
  const bool mma = !no_warp && bf16 && a.T > 0 && a.status && route_mma_supported(a.E, a.k, a.d);
  const bool tc = !mma && bf16 && a.T > 0 && route_tc_supported(a.E, a.k, a.d);
  const int tb = tc ? 128 : route_tb(a.E);  // tokens per block of the count/rank pass
  const int nb = (a.T + tb - 1) / tb;
  uint8_t* ws = static_cast<uint8_t*>(a.scratch);
  a.blockcounts = reinterpret_cast<int32_t*>(ws);
  int32_t* blockoffs = reinterpret_cast<int32_t*>(ws + align256((size_t)nb * a.E * 4));
  a.localrank = reinterpret_cast<int32_t*>(ws + 2 * align256((size_t)nb * a.E * 4));
  cudaError_t err;
  if (mma) {
    // logits, top-k, block counts and (in its last block) the scan of the counts
    err = a.E <= 8 ? launch_route_mma<1>(a, blockoffs, nb, st)
                   : (a.E <= 16 ? launch_route_mma<2>(a, blockoffs, nb, st)
                                : launch_route_mma<4>(a, blockoffs, nb, st));
    if (err != cudaSuccess) return err;
  } else {
    if (nb > 0) {
      if (tc)
        err = route_tc_launch(a, nb, st);
      else
        err = bf16 ? dispatch_topk<__nv_bfloat16>(a, nb, st) : dispatch_topk<float>(a, nb, st);
      if (err != cudaSuccess) return err;
    }
    // With T == 0 the scan still writes zero counts and offsets.
    {
      ProfScope prof("route_block_scan", st);
      block_scan_kernel<<<a.E, 256, 0, st>>>(a.blockcounts, blockoffs, nb, a.counts);
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  const int64_t n = (int64_t)a.T * a.k;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 1184));
  {
    ProfScope prof("route_slot_rows", st);
    slot_rows_kernel<<<grid, 256, 0, st>>>(a.topk_idx, a.localrank, blockoffs, a.counts, a.T, a.E,
                                            a.k, tb, nb, a.offsets, a.slot_row,
                                            mma ? a.status + 1 : nullptr);
  }
  return cudaGetLastError();
}


// ---- load balance of a routing -------------------------------------------
// [kongchang] routing section: the load spread over the experts is what sets
// the grouped GEMM's throughput.  One block of 1024 threads, one expert per
// thread (E <= 1024); integer totals, then the squared deviations in double,
// both reduced in a fixed order so the result does not depend on timing.
namespace {

template <class T, class Op>
__device__ T block_reduce(T v, Op op, T* red) {
  for (int o = 16; o; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = red[l];
  for (int o = 16; o; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__global__ void __launch_bounds__(1024) routing_stats_kernel(const int32_t* __restrict__ counts,
                                                             int E, int capacity,
                                                             float* __restrict__ stats) {
  __shared__ long long red_i[32];
  __shared__ double red_d[32];
  const int e = threadIdx.x;
  const long long c = e < E ? counts[e] : 0;
  const long long big = 1ll << 62;
  auto add = [](long long a, long long b) { return a + b; };
  const long long R = block_reduce(c, add, red_i);
  const long long mx = block_reduce(e < E ? c : -big, [](long long a, long long b) { return a > b ? a : b; }, red_i);
  const long long mn = block_reduce(e < E ? c : big, [](long long a, long long b) { return a < b ? a : b; }, red_i);
  const long long empty = block_reduce((long long)(e < E && c == 0), add, red_i);
  const long long over = capacity > 0 ? (c > capacity ? c - capacity : 0) : 0;
  const long long dropped = block_reduce(over, add, red_i);
  const double mean = (double)R / E;
  const double dev = e < E ? ((double)c - mean) * ((double)c - mean) : 0.0;
  const double ss = block_reduce(dev, [](double a, double b) { return a + b; }, red_d);
  if (e == 0) {
    const bool any = R > 0;
    stats[0] = (float)R;
    stats[1] = (float)mean;
    stats[2] = any ? (float)(mx / mean) : 0.f;
    stats[3] = any ? (float)(mn / mean) : 0.f;
    stats[4] = any ? (float)(sqrt(ss / E) / mean) : 0.f;
    stats[5] = (float)empty;
    const bool cap = capacity > 0 && any;
    stats[6] = cap ? (float)((double)dropped / R) : 0.f;
    stats[7] = cap ? (float)((double)(R - dropped) / ((double)E * capacity)) : 0.f;
  }
}

}  // namespace

cudaError_t routing_stats_launch(const int32_t* counts, int E, int capacity, float* stats,
                                 cudaStream_t st) {
  {
    ProfScope prof("routing_stats", st);
    routing_stats_kernel<<<1, 1024, 0, st>>>(counts, E, capacity, stats);
  }
  return cudaGetLastError();
}


// ---- renormalised gates (optional gate rule) -----------------------------
// g'[t, j] = g[t, j] / S[t], S[t] = sum_j g[t, j]; backward
// dg[t, j] = (dg'[t, j] - sum_i g'[t, i] dg'[t, i]) / S[t].  One thread per
// token; the k gates of a token are summed in index order.
namespace {

__global__ void __launch_bounds__(256) renorm_gates_kernel(const float* __restrict__ gate,
                                                           float* __restrict__ out, int T, int k) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const float* g = gate + (int64_t)t * k;
  float S = 0.f;
  for (int j = 0; j < k; ++j) S += g[j];
  float v[32];
  for (int j = 0; j < k; ++j) v[j] = g[j] / S;
  float* o = out + (int64_t)t * k;
  for (int j = 0; j < k; ++j) o[j] = v[j];
}

__global__ void __launch_bounds__(256) renorm_gates_bwd_kernel(const float* __restrict__ gate,
                                                               const float* __restrict__ dgr,
                                                               float* __restrict__ dgate, int T,
                                                               int k) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const float* g = gate + (int64_t)t * k;
  const float* dg = dgr + (int64_t)t * k;
  float S = 0.f;
  for (int j = 0; j < k; ++j) S += g[j];
  float dot = 0.f;
  for (int j = 0; j < k; ++j) dot += (g[j] / S) * dg[j];
  float v[32];
  for (int j = 0; j < k; ++j) v[j] = (dg[j] - dot) / S;
  float* o = dgate + (int64_t)t * k;
  for (int j = 0; j < k; ++j) o[j] = v[j];
}

}  // namespace

cudaError_t renorm_gates_launch(const float* gate, float* out, int T, int k, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  {
    ProfScope prof("renorm_gates", st);
    renorm_gates_kernel<<<(T + 255) / 256, 256, 0, st>>>(gate, out, T, k);
  }
  return cudaGetLastError();
}

cudaError_t renorm_gates_bwd_launch(const float* gate, const float* dgr, float* dgate, int T, int k,
                                    cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  {
    ProfScope prof("renorm_gates_bwd", st);
    renorm_gates_bwd_kernel<<<(T + 255) / 256, 256, 0, st>>>(gate, dgr, dgate, T, k);
  }
  return cudaGetLastError();
}

}  // namespace moe

// ---------------------------------------------------------------------------
// moe_route_noalloc: the same routing step for callers that cannot allocate
// device memory (a plugin inside a framework that owns all device memory, a
// latency-critical path where cudaMalloc could synchronise the device, a
// deployment with a footprint fixed at start-up).  Its scratch is one fixed
// array of this library instead of a caller workspace.
namespace moe {

// Device scratch of moe_route_noalloc, shared by every call on a device: the first
// kNoallocStatusBytes hold the status word of the bounded waits, the rest the route
// scratch.  Zero at load; moe_route_noalloc_status reads and clears the status word.
constexpr size_t kNoallocStatusBytes = 256;
static __device__ __align__(256) uint8_t g_route_scratch[MOE_ROUTE_NOALLOC_MAX_SCRATCH];

namespace {

// In host code g_route_scratch names a host-side stand-in, not device memory: the
// kernels get the array's device address, looked up with the caller's device current.
// The lookup is repeated on every call (it allocates nothing and is cheap), so an
// address never outlives the context it was taken in.
cudaError_t noalloc_scratch(void** out) {
  void* p = nullptr;
  const cudaError_t err = cudaGetSymbolAddress(&p, g_route_scratch);
  if (err != cudaSuccess) return err;
  *out = p;
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace moe

extern "C" moe_status moe_route_noalloc(moe_shape s, int dtype, const void* x,
                                        const void* w_router, const float* bias, float* logits,
                                        int32_t* topk_idx, float* topk_gate, int32_t* counts,
                                        int32_t* offsets, int32_t* slot_row, void* stream) {
  using namespace moe;
  // the argument rules of moe_route
  if (s.T < 0 || s.d_model <= 0 || s.E <= 0 || s.top_k <= 0 || s.d_ff <= 0) return MOE_ERR_INVALID_ARG;
  if (s.E > 1024 || s.top_k > s.E || s.top_k > 32) return MOE_ERR_INVALID_ARG;
  if (s.d_model % 8 || s.d_ff % 8) return MOE_ERR_INVALID_ARG;
  if ((int64_t)s.T * s.top_k >= (int64_t)1 << 31) return MOE_ERR_INVALID_ARG;
  if (dtype == MOE_MXFP8) return MOE_ERR_UNSUPPORTED;
  if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  const void* always[] = {w_router, counts, offsets};
  for (const void* p : always)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0) {
    const void* per_token[] = {x, logits, topk_idx, topk_gate, slot_row};
    for (const void* p : per_token)
      if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  }
  if (bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  // the fixed scratch (after its status word) bounds the shapes this variant can take
  if (route_ws_bytes(s.T, s.E, s.top_k) > MOE_ROUTE_NOALLOC_MAX_SCRATCH - kNoallocStatusBytes)
    return MOE_ERR_UNSUPPORTED;
  void* base = nullptr;
  if (noalloc_scratch(&base) != cudaSuccess) return MOE_ERR_CUDA;
  uint8_t* b = static_cast<uint8_t*>(base);
  RouteArgs a{x, w_router, bias, s.T, s.d_model, s.E, s.top_k, logits, topk_idx, topk_gate,
              counts, offsets, slot_row, b + kNoallocStatusBytes, reinterpret_cast<int*>(b)};
  return route_launch(a, dtype == MOE_BF16, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

extern "C" moe_status moe_route_noalloc_status(void* stream, int32_t* status_out) {
  using namespace moe;
  if (!status_out) return MOE_ERR_INVALID_ARG;
  void* base = nullptr;
  if (noalloc_scratch(&base) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, base, sizeof(v), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(base, 0, sizeof(v), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  *status_out = v;
  return MOE_OK;
}
