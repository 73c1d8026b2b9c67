// FP32 grouped GEMM on the CUDA cores, for the FP32 layer (the tensor cores'
// TF32 path cannot hold a 1e-4 relative error bound).  64 x 64 output tile per
// CTA, 16-deep K slices staged in shared memory, 4 x 4 outputs per thread.
// Groups follow the same two layouts as the tensor-core kernel: expert
// segments along the rows (forward / input gradients) or along K (weight
// gradients).
#include "common.cuh"
#include "kernels.h"

namespace pfmoe {

namespace {
constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtGemm g) {
  const int grp = blockIdx.z;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const float* A = g.A;
  const float* B = g.B;
  float* D = g.D;
  int M, K;
  if (g.mode == 0) {
    const int r0 = g.seg ? g.seg[grp] : 0;
    const int r1 = g.seg ? g.seg[grp + 1] : g.M;
    M = r1 - r0;
    K = g.K;
    A += static_cast<long long>(r0) * g.sam;
    D += static_cast<long long>(r0) * g.sdm;
    B += static_cast<long long>(grp) * g.b_gstride;
  } else {
    const int k0 = g.seg ? g.seg[grp] : 0;
    const int k1 = g.seg ? g.seg[grp + 1] : g.K;
    K = k1 - k0;
    M = g.M;
    A += static_cast<long long>(k0) * g.sak;
    B += static_cast<long long>(k0) * g.sbk;
    D += static_cast<long long>(grp) * g.d_gstride;
  }
  if (m0 >= M || n0 >= g.N) return;

  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int kt = 0; kt < K; kt += TK) {
    for (int i = threadIdx.x; i < TK * TM; i += 256) {
      const int kk = i / TM, mm = i % TM;
      const int m = m0 + mm, k = kt + kk;
      As[kk][mm] = (m < M && k < K) ? A[m * g.sam + k * g.sak] : 0.f;
      const int n = n0 + mm;
      Bs[kk][mm] = (n < g.N && k < K) ? B[n * g.sbn + k * g.sbk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      float v = acc[i][j];
      if (g.bias) v += g.bias[n];
      float* dp = D + static_cast<long long>(m) * g.sdm + n;
      *dp = g.beta == 0.f ? v : v + g.beta * *dp;
    }
  }
}

__global__ void swiglu_fwd_kernel(const float* h1, const float* h3, float* a, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    a[i] = silu_f(h1[i]) * h3[i];
}

__global__ void swiglu_bwd_kernel(const float* da, const float* h1, const float* h3, float* dh1, float* dh3,
                                  long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float u = h1[i], s = 1.0f / (1.0f + expf(-u));
    dh1[i] = da[i] * h3[i] * s * (1.0f + u * (1.0f - s));
    dh3[i] = da[i] * u * s;
  }
}

int grid_1d(long long n) {
  long long b = (n + 255) / 256;
  const long long cap = static_cast<long long>(num_sms()) * 16;
  if (b > cap) b = cap;
  return static_cast<int>(b < 1 ? 1 : b);
}
}  // namespace

int simt_gemm_f32(const SimtGemm& g, int32_t* /*err*/, cudaStream_t s, const char* name) {
  // Rows per group are on the device for mode 0; g.M bounds them (total rows).
  const int gy = (g.M + TM - 1) / TM, gx = (g.N + TN - 1) / TN;
  if (gx == 0 || gy == 0 || g.G == 0) return PFMOE_OK;
  dim3 grid(gx, gy, g.G);
  PFMOE_LAUNCH(name, s, simt_gemm_kernel<<<grid, 256, 0, s>>>(g));
  return PFMOE_OK;
}

int simt_swiglu_fwd_f32(const float* h1, const float* h3, float* a, long long n, cudaStream_t s) {
  if (n <= 0) return PFMOE_OK;
  PFMOE_LAUNCH("swiglu_fwd_f32", s, swiglu_fwd_kernel<<<grid_1d(n), 256, 0, s>>>(h1, h3, a, n));
  return PFMOE_OK;
}

int simt_swiglu_bwd_f32(const float* da, const float* h1, const float* h3, float* dh1, float* dh3, long long n,
                        cudaStream_t s) {
  if (n <= 0) return PFMOE_OK;
  PFMOE_LAUNCH("swiglu_bwd_f32", s, swiglu_bwd_kernel<<<grid_1d(n), 256, 0, s>>>(da, h1, h3, dh1, dh3, n));
  return PFMOE_OK;
}

}  // namespace pfmoe
