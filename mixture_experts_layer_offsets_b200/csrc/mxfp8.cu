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
// cvt.rn.satfinite.e4m3x2.f32 applied to v * 2^-e (it carries the sign of v,
// signed zeros included).
#include "common.cuh"
#include "internal.h"
#include "mx_common.cuh"

namespace moe {

namespace {

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

// eight consecutive elements (16-byte aligned for bf16, 32-byte for fp32) as floats
template <typename T>
__device__ __forceinline__ void load8(const T* p, float* v) {
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
}

// Row -> (128-row tile, row in tile) of the row-grouped GEMMs: tile = number of 128-row
// tiles of the experts before the row's expert + (row - expert start) / 128.  Encoded
// as tile * 128 + row in tile; -1 for rows outside every expert segment.
__global__ void __launch_bounds__(256)
row_tile_kernel(const int32_t* __restrict__ offsets, int E, int64_t rows, int32_t* __restrict__ out) {
  __shared__ int s_off[1025];
  __shared__ int s_pre[1025];
  for (int g = threadIdx.x; g <= E; g += blockDim.x) s_off[g] = offsets[g];
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x, lo = lane * 32, hi = min(lo + 32, E);
    int sum = 0;
    for (int g = lo; g < hi; ++g) sum += (s_off[g + 1] - s_off[g] + 127) / 128;
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    int run = incl - sum;
    for (int g = lo; g < hi; ++g) {
      s_pre[g] = run;
      run += (s_off[g + 1] - s_off[g] + 127) / 128;
    }
  }
  __syncthreads();
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < rows;
       r += (int64_t)gridDim.x * blockDim.x) {
    int lo = 0, hi = E - 1;  // last expert whose start is <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int lr = (int)(r - s_off[lo]);
    out[r] = (r >= s_off[lo] && r < s_off[lo + 1]) ? (s_pre[lo] + lr / 128) * 128 + (lr & 127) : -1;
  }
}

// FP32 master weights -> both MXFP8 copies in one pass over a 64 x 128 half tile (rows
// 64 h .. of a 128 x 128 tile) of one expert's [Rw, Kw] matrix: q0 / s0 in blocks of 32
// along a row (K-major GEMM operand), q1 / s1 in blocks of 32 rows within a column
// (MN-major GEMM operand).
//   s0 atom ((e * Rw/128 + row tile) * Kw/128 + kq), kq the 128-column stage.
//   s1 atom ((e * Rw/128 + kq) * Kw/128 + column tile), kq the 128-row stage.
// The half tile is staged in shared memory with 36 floats per 32-column block (4 words of
// padding, so that the row pass writes and the column pass reads without bank conflicts);
// a half tile owns half of each of its two atoms' bytes.
constexpr int kWBlk = 36;              // floats per staged 32-column block
constexpr int kWPitch = 4 * kWBlk;     // floats per staged row
constexpr int kWSmem = 64 * kWPitch * 4 + 64 * 128 + 256 + 256;
__global__ void __launch_bounds__(128)
mx_weights_kernel(const float* __restrict__ w, int E, int Rw, int Kw, uint8_t* __restrict__ q0,
                  uint8_t* __restrict__ s0, uint8_t* __restrict__ q1, uint8_t* __restrict__ s1) {
  extern __shared__ float tile[];                                  // [64][kWPitch]
  uint8_t* qt = reinterpret_cast<uint8_t*>(tile + 64 * kWPitch);   // [64][128] q1 bytes
  uint8_t* sa0 = qt + 64 * 128;          // s0 bytes of rows 64 h .. 64 h + 63: [32][8]
  uint8_t* sa1 = sa0 + 256;              // s1 bytes of row blocks 2 h, 2 h + 1: [128][2]
  const int tid = threadIdx.x;
  // half tiles in (expert, 64-row half, 128-column tile) order; the CTA loops over them
  const int nct = Kw >> 7, nhalf = Rw >> 6;
  const int64_t ntiles = (int64_t)E * nhalf * nct;
  // pass 1 takes blocks along rows; a quad of lanes covers one 32-wide block.  The sixteen
  // 16-byte loads of a thread for the next half tile are issued as soon as the current one
  // sits in shared memory, so they are in flight during the column pass and the stores.
  float4 ld[16];
  auto load = [&](int64_t t) {
    const int ct = (int)(t % nct);
    const int64_t rest = t / nct;
    const int64_t row0 = (rest / nhalf) * Rw + (rest % nhalf) * 64;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int task = it * 128 + tid;          // 1024 = 64 rows x 4 blocks x 4 parts
      const int r = task >> 4, kb = (task >> 2) & 3, part = task & 3;
      const float* p = w + (row0 + r) * Kw + ct * 128 + kb * 32 + part * 8;
      ld[2 * it] = __ldg(reinterpret_cast<const float4*>(p));
      ld[2 * it + 1] = __ldg(reinterpret_cast<const float4*>(p + 4));
    }
  };
  if ((int64_t)blockIdx.x < ntiles) load(blockIdx.x);
  for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
    const int ct = (int)(t % nct);
    const int64_t rest = t / nct;
    const int e = (int)(rest / nhalf), hrow = (int)(rest % nhalf);
    const int rt = hrow >> 1, half = hrow & 1;
    const int64_t row0 = (int64_t)e * Rw + hrow * 64;
    const int col0 = ct * 128;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int task = it * 128 + tid;
      const int r = task >> 4, kb = (task >> 2) & 3, part = task & 3;
      const float4 a = ld[2 * it], b = ld[2 * it + 1];
      float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      float* tp = tile + r * kWPitch + kb * kWBlk + part * 8;
      *reinterpret_cast<float4*>(tp) = a;
      *reinterpret_cast<float4*>(tp + 4) = b;
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const int ex = block_exponent(amax);
      const float mul = pow2_neg(ex);
      uint2 out;
      out.x = e4m3_pair(v[1] * mul, v[0] * mul) | (e4m3_pair(v[3] * mul, v[2] * mul) << 16);
      out.y = e4m3_pair(v[5] * mul, v[4] * mul) | (e4m3_pair(v[7] * mul, v[6] * mul) << 16);
      *reinterpret_cast<uint2*>(q0 + (row0 + r) * Kw + col0 + kb * 32 + part * 8) = out;
      // atom row r % 32 holds groups (r / 32) of 4 bytes; this half owns groups 2 h, 2 h + 1
      if (part == 0) sa0[(r & 31) * 8 + (r >> 5) * 4 + kb] = (uint8_t)(ex + 127);
    }
    if (t + (int64_t)gridDim.x < ntiles) load(t + gridDim.x);
    __syncthreads();
    // pass 2: blocks of 32 rows within a column; a thread takes two adjacent columns of one
    // row block (64 column pairs x 2 row blocks)
    {
      const int cp = tid & 63, rb = tid >> 6;
      const int c = 2 * cp;
      const float* col = tile + (c >> 5) * kWBlk + (c & 31);
      float am0 = 0.f, am1 = 0.f;
#pragma unroll 8
      for (int i = 0; i < 32; ++i) {
        const float2 v = *reinterpret_cast<const float2*>(col + (rb * 32 + i) * kWPitch);
        am0 = fmaxf(am0, fabsf(v.x));
        am1 = fmaxf(am1, fabsf(v.y));
      }
      const int ex0 = block_exponent(am0), ex1 = block_exponent(am1);
      const float m0 = pow2_neg(ex0), m1 = pow2_neg(ex1);
#pragma unroll 8
      for (int i = 0; i < 32; ++i) {
        const float2 v = *reinterpret_cast<const float2*>(col + (rb * 32 + i) * kWPitch);
        *reinterpret_cast<uint16_t*>(qt + (rb * 32 + i) * 128 + c) = (uint16_t)e4m3_pair(v.y * m1, v.x * m0);
      }
      // atom bytes (c % 32) * 16 + (c / 32) * 4 + (2 h + rb): two bytes per column here
      sa1[c * 2 + rb] = (uint8_t)(ex0 + 127);
      sa1[(c + 1) * 2 + rb] = (uint8_t)(ex1 + 127);
    }
    __syncthreads();
    // write the q1 half tile (64 rows x 128 bytes), 16 bytes per store
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int idx = it * 128 + tid;            // 512 pieces of 16 bytes
      const int r = idx >> 3, c16 = idx & 7;
      *reinterpret_cast<uint4*>(q1 + (row0 + r) * Kw + col0 + c16 * 16) =
          *reinterpret_cast<const uint4*>(qt + r * 128 + c16 * 16);
    }
    uint8_t* a0 = s0 + (((int64_t)e * (Rw >> 7) + rt) * (Kw >> 7) + ct) * 512;
    uint8_t* a1 = s1 + (((int64_t)e * (Rw >> 7) + rt) * (Kw >> 7) + ct) * 512;
    if (tid < 32) {   // s0: 8 bytes per atom row
      *reinterpret_cast<uint2*>(a0 + tid * 16 + half * 8) = *reinterpret_cast<const uint2*>(sa0 + tid * 8);
    } else {          // s1: 2 bytes per column, at offset (c % 32) * 16 + (c / 32) * 4 + 2 h
      for (int c = tid - 32; c < 128; c += 96)
        *reinterpret_cast<uint16_t*>(a1 + (c & 31) * 16 + (c >> 5) * 4 + half * 2) =
            *reinterpret_cast<const uint16_t*>(sa1 + c * 2);
    }
    __syncthreads();  // the staging areas are rewritten by the next half tile
  }
}

// 32-row blocks of the token axis, restarting at every segment (expert): block b (in
// segment order) -> {first row, rows (1..32), 128-row stage over all segments, (position of
// the block in its stage) | 4 if it is its segment's last block}.  count[0] = number of
// blocks, count[1] = number of stages, smap[z] = first block of stage z (smap[count[1]] =
// count[0]).  One CTA of 1024 threads (E <= 1024): a scan of the per-segment block counts,
// then each thread writes its segment's entries.
__global__ void __launch_bounds__(1024)
seg_blocks_kernel(const int32_t* __restrict__ offsets, int E, int4* __restrict__ map,
                  int32_t* __restrict__ count, int32_t* __restrict__ smap) {
  const int g = threadIdx.x, lane = g & 31, w = g >> 5;
  const int r0 = g < E ? offsets[g] : 0, c = g < E ? offsets[g + 1] - r0 : 0;
  const int nb = (c + 31) / 32, ns = (c + 127) / 128;
  // inclusive scans of nb and ns over the threads (warp shuffles, then warp totals)
  int ib = nb, is = ns;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, ib, o), b = __shfl_up_sync(0xffffffffu, is, o);
    if (lane >= o) { ib += a; is += b; }
  }
  __shared__ int s_wb[32], s_ws[32];
  if (lane == 31) { s_wb[w] = ib; s_ws[w] = is; }
  __syncthreads();
  if (w == 0) {
    int vb = s_wb[lane], vs = s_ws[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, vb, o), b = __shfl_up_sync(0xffffffffu, vs, o);
      if (lane >= o) { vb += a; vs += b; }
    }
    s_wb[lane] = vb;
    s_ws[lane] = vs;
  }
  __syncthreads();
  const int b0 = ib - nb + (w > 0 ? s_wb[w - 1] : 0);
  const int st0 = is - ns + (w > 0 ? s_ws[w - 1] : 0);
  for (int lb = 0; lb < nb; ++lb)
    map[b0 + lb] = make_int4(r0 + 32 * lb, min(32, c - 32 * lb), st0 + lb / 4,
                             (lb & 3) | (lb == nb - 1 ? 4 : 0));
  for (int s2 = 0; s2 < ns; ++s2) smap[st0 + s2] = b0 + 4 * s2;  // first block of each stage
  if (g == 1023) {
    count[0] = b0 + nb;
    count[1] = st0 + ns;
    smap[st0 + ns] = b0 + nb;
  }
}

// One pass over a bf16 activation tile of one 32-row token block (of one segment) x 128
// columns, writing both MXFP8 copies: q_r / atoms_r in blocks of 32 along each row (row-tile
// atoms, tile and row from row_tile), and q_c / atoms_c in the block's 32 rows within each
// column (stage atoms; the blocks of a segment's last stage past its end get 2^0).  q_c is
// column-major over the stage-padded token axis: column c's code of the block's row i sits
// at q_c[c * Rp + 128 * stage + 32 * (block in stage) + i]; the rows past a segment's last
// token, up to the end of its last stage, get code 0.  A CTA takes whole stages (their
// blocks one after another) and writes each column's 128 codes of a stage as one line.
constexpr int kActPitch = 136;  // bf16 per staged row (16 bytes of padding)
constexpr int kQtPitch = 132;   // bytes per staged column of a stage's column copy
__global__ void __launch_bounds__(128, 8)
mx_act_kernel(const __nv_bfloat16* __restrict__ src, int64_t K, int64_t ld,
              const int4* __restrict__ map, const int32_t* __restrict__ count,
              const int32_t* __restrict__ smap, const int32_t* __restrict__ row_tile,
              uint8_t* __restrict__ q_r, uint8_t* __restrict__ atoms_r, uint8_t* __restrict__ q_c,
              uint8_t* __restrict__ atoms_c, const int32_t* __restrict__ gather, int64_t Rp,
              const float* __restrict__ row_mul) {
  __shared__ __align__(16) __nv_bfloat16 s_t[32 * kActPitch];
  __shared__ __align__(16) uint8_t s_q[128 * kQtPitch];
  const int tid = threadIdx.x, ct = blockIdx.x;
  const int64_t c0 = (int64_t)ct * 128;
  const int64_t kq = K >> 7;
  const int nstages = count[1];
  // n rows x 128 columns of block b: 16 pieces of 16 bytes per row, 4 per thread.  The next
  // block's pieces are loaded into registers while this block is quantised (nothing
  // consumes them before they are staged, so the loads stay in flight meanwhile).
  auto load = [&](int b, int4& m, uint4 (&v)[4], float (&g)[4]) {
    m = map[b];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = tid + 128 * j, row = i >> 4, p8 = i & 15;
      v[j] = make_uint4(0, 0, 0, 0);
      g[j] = 1.f;
      if (row < m.y) {
        // row r of the operand is source row gather[r] (the fused dispatch), else r; with
        // row_mul, its factor row_mul[r], applied when the row is staged
        const int64_t sr = gather ? (int64_t)__ldg(gather + m.x + row) : (int64_t)(m.x + row);
        v[j] = ldg16(src + sr * ld + c0 + p8 * 8);
        if (row_mul) g[j] = __ldg(row_mul + m.x + row);
      }
    }
  };
  // this CTA's blocks: stages blockIdx.y, + gridDim.y, ..., each stage's blocks in order
  int z = blockIdx.y;
  int b = z < nstages ? smap[z] : 0;
  int4 mnext;
  uint4 vnext[4];
  float gnext[4];
  if (z < nstages) load(b, mnext, vnext, gnext);
  while (z < nstages) {
    const int4 m = mnext;
    const int r0 = m.x, n = m.y;
    const int pos = m.w & 3;
    const bool stage_end = b + 1 == smap[z + 1];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = tid + 128 * j, row = i >> 4, p8 = i & 15;
      uint4 v = vnext[j];
      if (row_mul) {
        // the fused combine backward's rows: the bf16 of gate times output gradient,
        // rounded as the combine backward rounds dy_perm
        Vec16<__nv_bfloat16> a, o;
        a.raw = v;
#pragma unroll
        for (int e = 0; e < 8; ++e) o.set(e, gnext[j] * a.get(e));
        v = o.raw;
      }
      *reinterpret_cast<uint4*>(s_t + row * kActPitch + p8 * 8) = v;
    }
    __syncthreads();
    int zn = z, bn = b + 1;
    if (stage_end) {
      zn = z + gridDim.y;
      bn = zn < nstages ? smap[zn] : 0;
    }
    if (zn < nstages) load(bn, mnext, vnext, gnext);
    // rows: thread = (row, 32-column block)
    {
      const int row = tid >> 2, kb = tid & 3;
      if (row < n) {
        float v[32];
        const __nv_bfloat16* t = s_t + row * kActPitch + kb * 32;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          Vec16<__nv_bfloat16> a;
          a.raw = *reinterpret_cast<const uint4*>(t + 8 * i);
#pragma unroll
          for (int e = 0; e < 8; ++e) v[8 * i + e] = a.get(e);
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
        const int ex = block_exponent(amax);
        const float mul = pow2_neg(ex);
        uint32_t w8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          w8[i] = e4m3_pair(v[4 * i + 1] * mul, v[4 * i] * mul) |
                  (e4m3_pair(v[4 * i + 3] * mul, v[4 * i + 2] * mul) << 16);
        uint8_t* dq = q_r + (int64_t)(r0 + row) * K + c0 + kb * 32;
        *reinterpret_cast<uint4*>(dq) = make_uint4(w8[0], w8[1], w8[2], w8[3]);
        *reinterpret_cast<uint4*>(dq + 16) = make_uint4(w8[4], w8[5], w8[6], w8[7]);
        const int rt = row_tile[r0 + row];
        if (rt >= 0) atoms_r[((int64_t)(rt >> 7) * kq + ct) * 512 + atom_byte(rt & 127, kb)] = (uint8_t)(ex + 127);
      }
    }
    // columns: thread = (pair of adjacent columns, half of the 32 rows); the two halves of
    // a pair are neighbouring lanes.  The rows a lane pair reads in one step are 4 apart
    // (rows 0-3, 8-11, .. for one half, 4-7, 12-15, .. for the other), which puts the two
    // halves 16 banks apart.  Rows past n are zero in s_t, so they do not change the
    // maximum and their codes are 0.
    {
      const int cp = tid >> 1, rh = tid & 1;
      uint32_t w[16];
      __nv_bfloat162 am = __float2bfloat162_rn(0.f);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = (i & 3) + ((i >> 2) << 3) + 4 * rh;
        w[i] = *reinterpret_cast<const uint32_t*>(s_t + r * kActPitch + 2 * cp);
        am = __hmax2(am, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[i])));
      }
      uint32_t amw = *reinterpret_cast<uint32_t*>(&am);
      const uint32_t oth = __shfl_xor_sync(0xffffffffu, amw, 1);
      am = __hmax2(am, *reinterpret_cast<const __nv_bfloat162*>(&oth));
      const int ex0 = block_exponent(__low2float(am)), ex1 = block_exponent(__high2float(am));
      const float m0 = pow2_neg(ex0), m1 = pow2_neg(ex1);
      // rows 8 g + 4 rh .. + 3 of the two columns, four codes per 32-bit store into the
      // stage's column-major staging (132-byte pitch: no bank conflicts)
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t wl = 0, wh = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t v = w[4 * g + i];
          const uint32_t pr = e4m3_pair(__uint_as_float(v & 0xFFFF0000u) * m1,
                                        __uint_as_float(v << 16) * m0);
          wl |= (pr & 0xFFu) << (8 * i);
          wh |= (pr >> 8) << (8 * i);
        }
        *reinterpret_cast<uint32_t*>(s_q + (2 * cp) * kQtPitch + 32 * pos + 8 * g + 4 * rh) = wl;
        *reinterpret_cast<uint32_t*>(s_q + (2 * cp + 1) * kQtPitch + 32 * pos + 8 * g + 4 * rh) = wh;
      }
      // each of the pair's two threads writes the scale byte of one of its columns
      const int col = 2 * cp + rh;
      const int ex = rh ? ex1 : ex0;
      uint8_t* at = atoms_c + ((int64_t)m.z * kq + ct) * 512;
      at[atom_byte(col, pos)] = (uint8_t)(ex + 127);
      if (m.w & 4)
        for (int kb = pos + 1; kb < 4; ++kb) at[atom_byte(col, kb)] = 0x7F;
    }
    if (stage_end) {
      // the stage's column copy: each column's 128 codes as one 128-byte line, eight
      // lanes per line (16 bytes each), so that one warp store writes four whole lines;
      // the blocks the stage does not have (past its segment's end) are zero.  The
      // lanes of one load touch 32 distinct banks (pitch 33 words).
      __syncthreads();
      const int p16 = tid & 7;
      const bool have = p16 < 2 * (pos + 1);  // 32 bytes per block present
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = 16 * j + (tid >> 3);
        const uint32_t* sc = reinterpret_cast<const uint32_t*>(s_q + col * kQtPitch + 16 * p16);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (have) v = make_uint4(sc[0], sc[1], sc[2], sc[3]);
        *reinterpret_cast<uint4*>(q_c + (c0 + col) * Rp + 128 * (int64_t)m.z + 16 * p16) = v;
      }
    }
    __syncthreads();
    z = zn;
    b = bn;
  }
}

}  // namespace

cudaError_t row_tile_launch(const int32_t* offsets, int E, int64_t rows, int32_t* out, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>((rows + 255) / 256, 1184);
  {
    ProfScope prof("mx_row_tile", st);
    row_tile_kernel<<<grid, 256, 0, st>>>(offsets, E, rows, out);
  }
  return cudaGetLastError();
}

cudaError_t seg_blocks_launch(const int32_t* offsets, int E, int4* map, int32_t* count,
                              int32_t* smap, cudaStream_t st) {
  {
    ProfScope prof("mx_seg_blocks", st);
    seg_blocks_kernel<<<1, 1024, 0, st>>>(offsets, E, map, count, smap);
  }
  return cudaGetLastError();
}

cudaError_t mxfp8_act(int64_t rows, int E, int64_t K, int64_t ld, const void* src_bf16,
                      const int4* map, const int32_t* count, const int32_t* smap,
                      const int32_t* row_tile, uint8_t* q_r, uint8_t* atoms_r, uint8_t* q_c,
                      uint8_t* atoms_c, cudaStream_t st, const int32_t* gather,
                      const float* row_mul) {
  if (rows == 0) return cudaSuccess;
  const int64_t Rp = (rows / 128 + E) * 128;  // padded token axis of the column copy
  // about 8 blocks of 128 threads per SM at a time, each looping over several stages
  const int64_t want = std::max<int64_t>(1, (int64_t)num_sms() * 8 / (K / 128));
  dim3 grid((unsigned)(K / 128), (unsigned)std::min<int64_t>({rows / 128 + E, want, 65535}));
  {
    ProfScope prof("mx_act", st);
    mx_act_kernel<<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(src_bf16), K, ld, map,
                                         count, smap, row_tile, q_r, atoms_r, q_c, atoms_c, gather,
                                         Rp, row_mul);
  }
  return cudaGetLastError();
}

cudaError_t mxfp8_weights(const float* w, int E, int Rw, int Kw, uint8_t* q0, uint8_t* s0,
                          uint8_t* q1, uint8_t* s1, cudaStream_t st) {
  if (E == 0) return cudaSuccess;
  cudaError_t err = cudaFuncSetAttribute(mx_weights_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kWSmem);
  if (err != cudaSuccess) return err;
  // persistent: exactly as many CTAs as are resident at once (registers allow three per SM),
  // so that every CTA runs from the start and they all finish together
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mx_weights_kernel, 128, kWSmem);
  if (err != cudaSuccess) return err;
  const int64_t ntiles = (int64_t)E * (Rw / 64) * (Kw / 128);
  const int grid = (int)std::min<int64_t>(ntiles, (int64_t)num_sms() * std::max(per_sm, 1));
  {
    ProfScope prof("mx_weights", st);
    mx_weights_kernel<<<grid, 128, kWSmem, st>>>(w, E, Rw, Kw, q0, s0, q1, s1);
  }
  return cudaGetLastError();
}

cudaError_t mxfp8_launch_ld(int64_t rows, int64_t K, int64_t ld, bool src_bf16, const void* src,
                            int axis, const int32_t* seg_offsets, int nseg, uint8_t* q,
                            uint8_t* scale, cudaStream_t st) {
  if (rows == 0 || K == 0) return cudaSuccess;
  if (axis == 0) {
    const int64_t nblocks = rows * K / 32;
    const int64_t threads = nblocks * 4;
    const int grid = (int)((threads + 255) / 256);
    if (src_bf16) {
      ProfScope prof("mx_rows", st);
      mx_rows_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src),
                                                          nblocks, K / 32, ld, q, scale);
    } else {
      ProfScope prof("mx_rows", st);
      mx_rows_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(src), nblocks, K / 32,
                                                  ld, q, scale);
    }
    return cudaGetLastError();
  }
  const int nsegs = seg_offsets ? nseg : 1;
  dim3 grid((unsigned)((K / 8 + 127) / 128),
            (unsigned)std::min<int64_t>(rows / 32 + nsegs + 1, 65535));
  if (src_bf16) {
    ProfScope prof("mx_cols", st);
    mx_cols_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(src),
                                                        rows, K, ld, seg_offsets, nsegs, q, scale);
  } else {
    ProfScope prof("mx_cols", st);
    mx_cols_kernel<float><<<grid, 128, 0, st>>>(static_cast<const float*>(src), rows, K, ld,
                                                seg_offsets, nsegs, q, scale);
  }
  return cudaGetLastError();
}

cudaError_t mxfp8_launch(int64_t rows, int64_t K, bool src_bf16, const void* src, int axis,
                         const int32_t* seg_offsets, int nseg, uint8_t* q, uint8_t* scale,
                         cudaStream_t st) {
  return mxfp8_launch_ld(rows, K, K, src_bf16, src, axis, seg_offsets, nseg, q, scale, st);
}

}  // namespace moe
