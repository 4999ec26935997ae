// mxfp8.cu -- MXFP8 block quantisation: E4M3 elements, one E8M0 scale per
// 32 consecutive elements.
//
// Page: "Ai2 Olmo-core 3：MoE训练吞吐量提升2.7倍的秘诀" (kongchang.com), section
// 吞吐量数字的边界条件: MXFP8 is the OCP 8-bit microscaling format whose blocks of
// 32 elements share one scale; an FP32 master weight is kept.  Rule used (OCP MX
// conversion): e = floor(log2(amax)) - 8, clamped to [-127, 127] (amax 0 -> -127);
// scale byte e + 127; element = E4M3 round-to-nearest-even of v * 2^-e with
// saturation at 448; the sign bit follows v.
//
// floor(log2(amax)) comes straight from the fp32 exponent bits (exact, also for
// subnormal inputs); v * 2^-e is exact in fp32 (a power-of-two scaling whose
// result lies below 512); the element rounding is the hardware conversion
// cvt.rn.satfinite.e4m3x2.f32 applied to |v * 2^-e|, with the sign bit set
// from v afterwards.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

__device__ __forceinline__ int block_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int ex = (int)((bits >> 23) & 0xFF);
  int fl;
  if (ex == 0) {
    const uint32_t man = bits & 0x7FFFFF;
    if (man == 0) return -127;
    fl = -149 + (31 - __clz(man));
  } else {
    fl = ex - 127;
  }
  return min(max(fl - 8, -127), 127);
}

// 2^-e as an fp32 (e <= 119 for any finite fp32 amax, so 2^-e is normal).
__device__ __forceinline__ float pow2_neg(int e) { return __uint_as_float((uint32_t)(127 - e) << 23); }

__device__ __forceinline__ uint32_t e4m3_pair(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(fabsf(hi)), "f"(fabsf(lo)));
  uint32_t v = r;
  if (signbit(lo)) v |= 0x80u;
  if (signbit(hi)) v |= 0x8000u;
  return v;
}

// axis 0: a quad of lanes covers one 32-element block, 8 elements per lane.
template <typename T>
__global__ void __launch_bounds__(256)
mx_rows_kernel(const T* __restrict__ src, int64_t nblocks, int64_t kblocks, int64_t ld,
               uint8_t* __restrict__ q, uint8_t* __restrict__ scale) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t blk = g >> 2;
  const int part = (int)(g & 3);
  const bool live = blk < nblocks;
  float v[8];
  if (live) {
    const T* p = src + (blk / kblocks) * ld + (blk % kblocks) * 32 + part * 8;
    if constexpr (sizeof(T) == 2) {
      Vec16<T> a;
      a.raw = ldg16(p);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = a.get(i);
    } else {
      Vec16<T> a, b;
      a.raw = ldg16(p);
      b.raw = ldg16(p + 4);
#pragma unroll
      for (int i = 0; i < 4; ++i) { v[i] = a.get(i); v[4 + i] = b.get(i); }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  if (!live) return;
  const int e = block_exponent(amax);
  const float mul = pow2_neg(e);
  uint2 out;
  out.x = e4m3_pair(v[1] * mul, v[0] * mul) | (e4m3_pair(v[3] * mul, v[2] * mul) << 16);
  out.y = e4m3_pair(v[5] * mul, v[4] * mul) | (e4m3_pair(v[7] * mul, v[6] * mul) << 16);
  *reinterpret_cast<uint2*>(q + blk * 32 + part * 8) = out;
  if (part == 0) scale[blk] = (uint8_t)(e + 127);
}

// axis 1: one thread = one 32-row block x 8 columns; blocks restart at segments.
template <typename T>
__global__ void __launch_bounds__(128)
mx_cols_kernel(const T* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
               const int32_t* __restrict__ seg, int nseg, uint8_t* __restrict__ q,
               uint8_t* __restrict__ scale) {
  __shared__ int32_t s_pre[1026];   // block prefix per segment
  __shared__ int32_t s_seg[1026];
  const int tid = threadIdx.x;
  for (int g = tid; g <= nseg; g += blockDim.x) s_seg[g] = seg ? seg[g] : (g == 0 ? 0 : (int)rows);
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int g = 0; g < nseg; ++g) {
      s_pre[g] = acc;
      acc += (s_seg[g + 1] - s_seg[g] + 31) / 32;
    }
    s_pre[nseg] = acc;
  }
  __syncthreads();
  const int total = s_pre[nseg];
  const int64_t col = ((int64_t)blockIdx.x * blockDim.x + tid) * 8;
  if (col >= K) return;
  for (int rb = blockIdx.y; rb < total; rb += gridDim.y) {
    int lo = 0, hi = nseg - 1;  // last segment g with s_pre[g] <= rb and a non-empty range
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= rb) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int64_t r0 = s_seg[g] + (int64_t)(rb - s_pre[g]) * 32;
    const int64_t r1 = min((int64_t)s_seg[g + 1], r0 + 32);
    float amax[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) amax[i] = 0.f;
    for (int64_t r = r0; r < r1; ++r) {
      const T* p = src + r * ld + col;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax[i] = fmaxf(amax[i], fabsf(to_f32(p[i])));
    }
    int ex[8];
    float mul[8];
    uint32_t sb[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ex[i] = block_exponent(amax[i]);
      mul[i] = pow2_neg(ex[i]);
      sb[i >> 2] |= (uint32_t)(ex[i] + 127) << ((i & 3) * 8);
    }
    *reinterpret_cast<uint2*>(scale + (int64_t)rb * K + col) = make_uint2(sb[0], sb[1]);
    for (int64_t r = r0; r < r1; ++r) {
      const T* p = src + r * ld + col;
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = to_f32(p[i]) * mul[i];
      uint2 out;
      out.x = e4m3_pair(v[1], v[0]) | (e4m3_pair(v[3], v[2]) << 16);
      out.y = e4m3_pair(v[5], v[4]) | (e4m3_pair(v[7], v[6]) << 16);
      *reinterpret_cast<uint2*>(q + r * K + col) = out;
    }
  }
}

}  // namespace

cudaError_t mxfp8_launch_ld(int64_t rows, int64_t K, int64_t ld, bool src_bf16, const void* src,
                            int axis, const int32_t* seg_offsets, int nseg, uint8_t* q,
                            uint8_t* scale, cudaStream_t st) {
  if (rows == 0 || K == 0) return cudaSuccess;
  if (axis == 0) {
    const int64_t nblocks = rows * K / 32;
    const int64_t threads = nblocks * 4;
    const int grid = (int)((threads + 255) / 256);
    if (src_bf16)
      mx_rows_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src),
                                                          nblocks, K / 32, ld, q, scale);
    else
      mx_rows_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(src), nblocks, K / 32,
                                                  ld, q, scale);
    return cudaGetLastError();
  }
  const int nsegs = seg_offsets ? nseg : 1;
  dim3 grid((unsigned)((K / 8 + 127) / 128),
            (unsigned)std::min<int64_t>(rows / 32 + nsegs + 1, 65535));
  if (src_bf16)
    mx_cols_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(src),
                                                        rows, K, ld, seg_offsets, nsegs, q, scale);
  else
    mx_cols_kernel<float><<<grid, 128, 0, st>>>(static_cast<const float*>(src), rows, K, ld,
                                                seg_offsets, nsegs, q, scale);
  return cudaGetLastError();
}

cudaError_t mxfp8_launch(int64_t rows, int64_t K, bool src_bf16, const void* src, int axis,
                         const int32_t* seg_offsets, int nseg, uint8_t* q, uint8_t* scale,
                         cudaStream_t st) {
  return mxfp8_launch_ld(rows, K, K, src_bf16, src, axis, seg_offsets, nseg, q, scale, st);
}

}  // namespace moe
