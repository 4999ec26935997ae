// ffn_f32.cu -- grouped SwiGLU expert FFN, forward and backward, in fp32 on
// CUDA cores (the fp32 workload needs fp32 products: tcgen05 has no fp32
// operand kind, and tf32 would miss a 1e-5 relative tolerance).
//
// One generic grouped GEMM C = A B^T with strided operand access and a
// device-side tile scheduler that reads the expert offsets from device memory:
//   GROUP_M: expert g owns rows [off[g], off[g+1]) of A and C, and B_g;
//   GROUP_K: expert g owns the K range [off[g], off[g+1]) and output C_g
//            (weight gradients; an empty expert writes zeros).
// SwiGLU and its derivative run as separate elementwise kernels here.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kTM = 64, kTN = 64, kTK = 16;

struct SimtGemm {
  const float* A;
  int64_t a_sm, a_sk;      // A(m,k) = A[m*a_sm + k*a_sk]
  const float* B;
  int64_t b_sn, b_sk;      // B(n,k) = B[n*b_sn + k*b_sk]
  int64_t b_group;         // GROUP_M: B_g = B + g*b_group
  float* C;
  int64_t c_sm;            // C(m,n) = C[m*c_sm + n]
  int64_t c_group;         // GROUP_K: C_g = C + g*c_group
  const int32_t* offsets;
  int E;
  int group_k;
  int M, N, K;             // M fixed for GROUP_K, K fixed for GROUP_M
  int accumulate = 0;      // C += A B^T instead of C = A B^T
};

__global__ void __launch_bounds__(256) simt_grouped_gemm(const SimtGemm p) {
  __shared__ float As[kTK][kTM + 4];
  __shared__ float Bs[kTK][kTN + 4];
  __shared__ int32_t s_off[1025];
  __shared__ int32_t s_pre[1025];
  const int tid = threadIdx.x;
  for (int g = tid; g <= p.E; g += blockDim.x) s_off[g] = p.offsets[g];
  __syncthreads();
  const int ntn = (p.N + kTN - 1) / kTN;
  if (tid == 0) {
    int acc = 0;
    for (int g = 0; g < p.E; ++g) {
      s_pre[g] = acc;
      const int mg = p.group_k ? p.M : s_off[g + 1] - s_off[g];
      acc += ((mg + kTM - 1) / kTM) * ntn;
    }
    s_pre[p.E] = acc;
  }
  __syncthreads();
  const int total = s_pre[p.E];
  const int tx = tid % 16, ty = tid / 16;
  for (int t = blockIdx.x; t < total; t += gridDim.x) {
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int local = t - s_pre[g];
    const int m0 = (local / ntn) * kTM, n0 = (local % ntn) * kTN;
    int64_t row_base, k_lo, k_hi;
    int mg;
    const float* B = p.B;
    float* C = p.C;
    if (p.group_k) {
      row_base = 0; mg = p.M; k_lo = s_off[g]; k_hi = s_off[g + 1];
      C += g * p.c_group;
    } else {
      row_base = s_off[g]; mg = s_off[g + 1] - s_off[g]; k_lo = 0; k_hi = p.K;
      B += g * p.b_group;
    }
    float acc[4][4] = {};
    for (int64_t k0 = k_lo; k0 < k_hi; k0 += kTK) {
      for (int i = tid; i < kTK * kTM; i += 256) {
        const int kk = i / kTM, mm = i % kTM;
        const int64_t k = k0 + kk;
        const int m = m0 + mm;
        As[kk][mm] = (k < k_hi && m < mg) ? p.A[(row_base + m) * p.a_sm + k * p.a_sk] : 0.f;
        const int n = n0 + mm;
        Bs[kk][mm] = (k < k_hi && n < p.N) ? B[n * p.b_sn + k * p.b_sk] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kTK; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty + 16 * i]; b[i] = Bs[kk][tx + 16 * i]; }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = m0 + ty + 16 * i;
      if (m >= mg) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx + 16 * j;
        if (n < p.N) {
          float* c = C + (row_base + m) * p.c_sm + n;
          *c = p.accumulate ? *c + acc[i][j] : acc[i][j];
        }
      }
    }
  }
}

cudaError_t run(const SimtGemm& p, int64_t max_tiles, cudaStream_t st) {
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(max_tiles, (int64_t)num_sms() * 8));
  {
    ProfScope prof("gemm_simt_f32", st);
    simt_grouped_gemm<<<grid, 256, 0, st>>>(p);
  }
  return cudaGetLastError();
}

int64_t bound_tiles_m(int64_t rows, int E, int N) {
  return (rows / kTM + E) * ((N + kTN - 1) / kTN);
}

// act[r, 2f + c] = silu(act[r, c]) * act[r, f + c] for rows inside expert segments.
__global__ void swiglu_fwd_kernel(float* act, const int32_t* offsets, int E, int64_t rows, int f) {
  const int64_t n = rows * f;
  const int64_t used = offsets[E];
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / f;
    if (r >= used) break;
    const int c = (int)(i % f);
    float* row = act + r * 3 * f;
    const float a = row[c], u = row[f + c];
    row[2 * f + c] = a / (1.f + expf(-a)) * u;
  }
}

// dadu[r, c] <- dh * u * silu'(a);  dadu[r, f + c] <- dh * silu(a), with dh = dadu[r, c].
__global__ void swiglu_bwd_kernel(float* dadu, const float* act, const int32_t* offsets, int E,
                                  int64_t rows, int f) {
  const int64_t n = rows * f;
  const int64_t used = offsets[E];
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / f;
    if (r >= used) break;
    const int c = (int)(i % f);
    const float a = act[r * 3 * f + c], u = act[r * 3 * f + f + c];
    float* row = dadu + r * 2 * f;
    const float dh = row[c];
    const float s = 1.f / (1.f + expf(-a));
    row[c] = dh * u * s * (1.f + a * (1.f - s));
    row[f + c] = dh * a * s;
  }
}

int elem_grid(int64_t n) {
  return (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, (int64_t)num_sms() * 16));
}

}  // namespace

cudaError_t ffn_fwd_f32(const FfnShape& s, const float* x_perm, const int32_t* offsets,
                        const float* w1, const float* w2, float* act, float* y_perm,
                        cudaStream_t st) {
  if (s.rows == 0) return cudaSuccess;
  const int d = s.d, f = s.f;
  cudaError_t err;
  SimtGemm g1{x_perm, d, 1, w1, d, 1, (int64_t)2 * f * d, act, 3 * f, 0, offsets, s.E, 0,
              0, 2 * f, d};
  if ((err = run(g1, bound_tiles_m(s.rows, s.E, 2 * f), st)) != cudaSuccess) return err;
  {
    ProfScope prof("swiglu_fwd_f32", st);
    swiglu_fwd_kernel<<<elem_grid(s.rows * f), 256, 0, st>>>(act, offsets, s.E, s.rows, f);
  }
  if (!y_perm) return cudaGetLastError();  // recompute of a | u | h only
  SimtGemm g2{act + 2 * f, 3 * f, 1, w2, f, 1, (int64_t)d * f, y_perm, d, 0, offsets, s.E, 0,
              0, d, f};
  return run(g2, bound_tiles_m(s.rows, s.E, d), st);
}

cudaError_t ffn_bwd_f32(const FfnShape& s, const float* dy_perm, const float* x_perm,
                        const float* act, const int32_t* offsets, const float* w1,
                        const float* w2, float* dx_perm, float* dw1, float* dw2, void* scratch,
                        cudaStream_t st, bool accumulate) {
  const int d = s.d, f = s.f, E = s.E;
  float* dadu = static_cast<float*>(scratch);
  cudaError_t err;
  if (s.rows > 0) {
    // dh = dy W2[e]  (B(n=c of f, k=row of d) = W2[k][n])
    SimtGemm g1{dy_perm, d, 1, w2, 1, f, (int64_t)d * f, dadu, 2 * f, 0, offsets, E, 0, 0, f, d};
    if ((err = run(g1, bound_tiles_m(s.rows, E, f), st)) != cudaSuccess) return err;
    {
      ProfScope prof("swiglu_bwd_f32", st);
      swiglu_bwd_kernel<<<elem_grid(s.rows * f), 256, 0, st>>>(dadu, act, offsets, E, s.rows, f);
    }
    // dx = [da|du] W1[e]  (B(n=c of d, k=row of 2f) = W1[k][n])
    SimtGemm g2{dadu, 2 * f, 1, w1, 1, d, (int64_t)2 * f * d, dx_perm, d, 0, offsets, E, 0,
                0, d, 2 * f};
    if ((err = run(g2, bound_tiles_m(s.rows, E, d), st)) != cudaSuccess) return err;
  }
  // dW2[e] = dy^T h:  A(m=c of d, k=row) = dy[k][m];  B(n=c of f, k=row) = h[k][n]
  SimtGemm g3{dy_perm, 1, d, act + 2 * f, 1, 3 * f, 0, dw2, f, (int64_t)d * f, offsets, E, 1,
              d, f, 0, accumulate};
  if ((err = run(g3, (int64_t)E * ((d + 63) / 64) * ((f + 63) / 64), st)) != cudaSuccess) return err;
  // dW1[e] = [da|du]^T x:  A(m=c of 2f, k=row) = dadu[k][m];  B(n=c of d, k=row) = x[k][n]
  SimtGemm g4{dadu, 1, 2 * f, x_perm, 1, d, 0, dw1, d, (int64_t)2 * f * d, offsets, E, 1,
              2 * f, d, 0, accumulate};
  return run(g4, (int64_t)E * ((2 * f + 63) / 64) * ((d + 63) / 64), st);
}

size_t ffn_bwd_ws_bytes(const FfnShape& s, bool bf16) {
  // [da | du], then (tensor-core path) the split weight-gradient partial sums
  return align256((size_t)s.rows * 2 * s.f * (bf16 ? 2 : 4)) + (bf16 ? wgrad_part_bytes(s, false) : 0);
}

}  // namespace moe
